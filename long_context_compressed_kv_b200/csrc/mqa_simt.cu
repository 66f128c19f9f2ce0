// Shared-KV MQA over compressed entries + window tokens with an attention
// sink: CUDA-core split-K kernel (any d <= 512, any entry format) and the
// split-K combine / epilogue shared with the tensor-core kernels.
//
// Method: "DeepSeek-V4 深读" (ricardokevins.github.io), model-spec table
// (64 / 128 query heads of dim 512 over one shared KV head) and section
// "其他稳定性细节" (RMSNorm of queries, RoPE on the last 64 dims with the
// output rotated back by the query position, a learnable per-head sink that
// lets the weights sum to less than one); "拆解 DeepSeekv4", section "细节"
// (the sink adds exp(z'_h) to the softmax denominator; 128-token window).
//
// Split-K (flash-decoding): the key list of a query (selected or visible
// entries, then its window tokens) is cut into fixed chunks of split_keys
// keys; every chunk yields an unnormalised partial (O, running max, running
// sum); the combine merges them in a fixed order, adds the sink to the
// denominator, normalises and applies the inverse RoPE.  Chunk boundaries
// depend only on the key count, so results do not depend on the batch.
#include "common.cuh"
#include "kernels.h"

namespace v4a {

constexpr int kHG = 8;    // heads per CTA (one warp per head for the query prep)
constexpr int kTK = 16;   // keys per tile
constexpr int kMaxPairs = 8;  // d / 64 pairs per lane, d <= 512

// Query prep shared by every MQA kernel: [RMSNorm] -> RoPE at p -> FP8 coding
// of the non-RoPE dims (power-of-two scale per head) when the KV is FP8.
// One warp per head; writes d floats to `dst`.
__device__ void prep_query_warp(const MqaParams& P, int q, int h, int64_t p, float* dst) {
  const int lane = threadIdx.x & 31;
  const int npair = P.d / 2;
  float x0[kMaxPairs], x1[kMaxPairs];
  const int64_t base = ((int64_t)q * P.H + h) * P.d;
#pragma unroll
  for (int t = 0; t < kMaxPairs; ++t) {
    const int pr = lane + 32 * t;
    x0[t] = x1[t] = 0.f;
    if (pr < npair) {
      x0[t] = load_in(P.Q, P.q_dtype, base + 2 * pr);
      x1[t] = load_in(P.Q, P.q_dtype, base + 2 * pr + 1);
    }
  }
  if (P.q_rmsnorm) {
    float ss = 0.f;
#pragma unroll
    for (int t = 0; t < kMaxPairs; ++t) ss += x0[t] * x0[t] + x1[t] * x1[t];
    ss = warp_sum(ss);
    const float inv = 1.0f / sqrtf(ss / (float)P.d + P.eps);
#pragma unroll
    for (int t = 0; t < kMaxPairs; ++t) {
      x0[t] *= inv;
      x1[t] *= inv;
    }
  }
  const int rope0 = (P.d - P.d_rope) / 2;
#pragma unroll
  for (int t = 0; t < kMaxPairs; ++t) {
    const int pr = lane + 32 * t;
    if (pr < npair && pr >= rope0) {
      float cs, sn;
      rope_cs(p, pr - rope0, P.d_rope, P.theta, cs, sn);
      const float r0 = x0[t] * cs - x1[t] * sn;
      const float r1 = x0[t] * sn + x1[t] * cs;
      x0[t] = r0;
      x1[t] = r1;
    }
  }
  if (P.kv_dtype == V4A_E4M3_BF16ROPE) {
    float am = 0.f;
#pragma unroll
    for (int t = 0; t < kMaxPairs; ++t) {
      const int pr = lane + 32 * t;
      if (pr < rope0) am = fmaxf(am, fmaxf(fabsf(x0[t]), fabsf(x1[t])));
    }
    am = warp_max(am);
    const int se = e4m3_scale_exp(am);
    const float s = exp2i(se);
#pragma unroll
    for (int t = 0; t < kMaxPairs; ++t) {
      const int pr = lane + 32 * t;
      if (pr < npair) {
        if (pr < rope0) {
          x0[t] = e4m3_to_f32(f32_to_e4m3(scale_pow2(x0[t], se))) * s;
          x1[t] = e4m3_to_f32(f32_to_e4m3(scale_pow2(x1[t], se))) * s;
        } else {
          x0[t] = bf16_bits_to_f32(f32_to_bf16_bits(x0[t]));
          x1[t] = bf16_bits_to_f32(f32_to_bf16_bits(x1[t]));
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kMaxPairs; ++t) {
    const int pr = lane + 32 * t;
    if (pr < npair) {
      dst[2 * pr] = x0[t];
      dst[2 * pr + 1] = x1[t];
    }
  }
}

// Resolve virtual key j of query (b, p): entries first, then window tokens.
// Returns 0 (no key), 1 (entry row) or 2 (window row); `row` is the global row.
__device__ __forceinline__ int resolve_key(const MqaParams& P, int q, int b, int64_t p,
                                           int64_t n_vis, int64_t n_main, int n_swa, int64_t j,
                                           int64_t& row) {
  if (j < n_main) {
    int64_t e = j;
    if (P.idx) {
      e = P.idx[(int64_t)q * P.n_sel + j];
      if (e < 0) return 0;
      if (e >= n_vis || e >= P.kv_rows) {
        flag(P.status, ST_BAD_INDEX);
        return 0;
      }
    }
    row = (int64_t)b * P.kv_rows + e;
    return 1;
  }
  const int64_t w = j - n_main;
  if (w < n_swa) {
    const int64_t t = p - n_swa + 1 + w;
    row = (int64_t)b * P.swa_rows + (t % P.swa_rows);
    return 2;
  }
  return 0;
}

__device__ __forceinline__ void query_geometry(const MqaParams& P, int q, int& b, int64_t& p,
                                               int64_t& n_vis, int64_t& n_main, int& n_swa) {
  b = P.q_seq ? P.q_seq[q] : P.q_base + q;
  p = P.q_pos[q];
  n_vis = (p + 1) / P.m;
  if (b < 0 || b >= P.B) {
    if (threadIdx.x == 0) flag(P.status, ST_BAD_SEQ);
    b = 0;
    n_vis = 0;
    p = -1;
  }
  if (n_vis > P.kv_rows) {
    if (threadIdx.x == 0) flag(P.status, ST_BAD_POSITION);
    n_vis = P.kv_rows;
  }
  if (P.idx) {
    n_main = P.n_sel;
  } else {
    n_main = n_vis;
    if (n_main > P.max_vis) {
      if (threadIdx.x == 0) flag(P.status, ST_BAD_POSITION);
      n_main = P.max_vis;
    }
  }
  n_swa = (int)min((int64_t)P.n_win, p + 1);
  if (n_swa < 0) n_swa = 0;
}

__global__ void __launch_bounds__(256) mqa_simt_kernel(MqaParams P) {
  extern __shared__ float sm[];
  float* qs = sm;                        // [kHG][d]
  float* ks = qs + kHG * P.d;            // [kTK][d]
  float* ps = ks + kTK * P.d;            // [kHG][kTK]
  __shared__ float alpha_s[kHG];
  __shared__ int64_t key_row[kTK];
  __shared__ int key_src[kTK];
  const int split = blockIdx.x, q = blockIdx.y, h0 = blockIdx.z * kHG;
  const int nh = min(kHG, P.H - h0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int b, n_swa;
  int64_t p, n_vis, n_main;
  query_geometry(P, q, b, p, n_vis, n_main, n_swa);
  const int64_t n_keys = n_main + n_swa;
  const int64_t j0 = (int64_t)split * P.split_keys;
  const int64_t j1 = min(n_keys, j0 + P.split_keys);

  if (warp < nh) prep_query_warp(P, q, h0 + warp, p, qs + warp * P.d);
  float m_run = -INFINITY, l_run = 0.f;   // lane 0 of warp h keeps head h's state
  constexpr int kMaxO = kHG * 512 / 256;
  float o[kMaxO];
#pragma unroll
  for (int t = 0; t < kMaxO; ++t) o[t] = 0.f;
  const int rb = (int)row_bytes(P.kv_dtype, P.d, P.d_rope);
  __syncthreads();

  for (int64_t jt = j0; jt < j1; jt += kTK) {
    if (threadIdx.x < kTK) {
      int64_t row = 0;
      const int64_t j = jt + threadIdx.x;
      const int src = (j < j1) ? resolve_key(P, q, b, p, n_vis, n_main, n_swa, j, row) : 0;
      key_src[threadIdx.x] = src;
      key_row[threadIdx.x] = row;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < kTK * P.d; e += blockDim.x) {
      const int jj = e / P.d, dim = e % P.d;
      const int src = key_src[jj];
      float v = 0.f;
      if (src) {
        const uint8_t* base = (src == 1) ? P.kv : P.swa;
        const float* sc = (src == 1) ? P.kv_scale : P.swa_scale;
        const int64_t row = key_row[jj];
        const float scale = (P.kv_dtype == V4A_E4M3_BF16ROPE) ? sc[row] : 1.f;
        v = kv_elem(base + row * rb, P.kv_dtype, scale, dim, P.d, P.d_rope);
      }
      ks[e] = v;
    }
    __syncthreads();
    if (warp < nh) {
      const float* qh = qs + warp * P.d;
      float sv[kTK];
#pragma unroll
      for (int jj = 0; jj < kTK; ++jj) {
        float acc = 0.f;
        for (int dim = lane; dim < P.d; dim += 32) acc = fmaf(qh[dim], ks[jj * P.d + dim], acc);
        acc = warp_sum(acc);
        sv[jj] = key_src[jj] ? acc * P.scale : -INFINITY;
      }
      if (lane == 0) {
        float mt = m_run;
#pragma unroll
        for (int jj = 0; jj < kTK; ++jj) mt = fmaxf(mt, sv[jj]);
        float alpha = 1.f, lsum = 0.f;
        if (mt != -INFINITY) {
          alpha = __expf(m_run - mt);
#pragma unroll
          for (int jj = 0; jj < kTK; ++jj) {
            const float pj = __expf(sv[jj] - mt);
            ps[warp * kTK + jj] = pj;
            lsum += pj;
          }
          m_run = mt;
        } else {
#pragma unroll
          for (int jj = 0; jj < kTK; ++jj) ps[warp * kTK + jj] = 0.f;
        }
        l_run = l_run * alpha + lsum;
        alpha_s[warp] = alpha;
      }
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < kMaxO; ++t) {
      const int e = threadIdx.x + t * 256;
      if (e < nh * P.d) {
        const int h = e / P.d, dim = e % P.d;
        float acc = o[t] * alpha_s[h];
#pragma unroll
        for (int jj = 0; jj < kTK; ++jj) acc = fmaf(ps[h * kTK + jj], ks[jj * P.d + dim], acc);
        o[t] = acc;
      }
    }
    __syncthreads();
  }
  // partials
  const int64_t pbase = ((int64_t)q * P.n_split + split) * P.H;
#pragma unroll
  for (int t = 0; t < kMaxO; ++t) {
    const int e = threadIdx.x + t * 256;
    if (e < nh * P.d) {
      const int h = e / P.d, dim = e % P.d;
      P.part_o[(pbase + h0 + h) * P.d + dim] = o[t];
    }
  }
  if (warp < nh && lane == 0) {
    P.part_ml[(pbase + h0 + warp) * 2 + 0] = m_run;
    P.part_ml[(pbase + h0 + warp) * 2 + 1] = l_run;
  }
}

cudaError_t launch_mqa_simt(const MqaParams& P, cudaStream_t st) {
  dim3 grid(P.n_split, P.n_q, (P.H + kHG - 1) / kHG);
  const size_t smem = (size_t)(kHG * P.d + kTK * P.d + kHG * kTK) * sizeof(float);
  // the shared-memory limit is a per-device function attribute: set it (to the
  // largest size any call needs) once per device
  static unsigned long long configured = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !(configured & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(mqa_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (kHG * 512 + kTK * 512 + kHG * kTK) * (int)sizeof(float));
    if (e != cudaSuccess) return e;
    configured |= 1ull << dev;
  }
  mqa_simt_kernel<<<grid, 256, smem, st>>>(P);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- combine
// One CTA per (head, query); thread k owns the output pair (2k, 2k+1).
// One CTA per (head, query): merge the split partials with their running
// maxima, add the sink to the denominator, rotate the RoPE dims back by -p,
// cast.  The splits' (m, l) pairs are read into shared memory in parallel and
// the partial rows with 8 independent loads in flight per thread.
__global__ void mqa_combine_kernel(MqaParams P) {
  extern __shared__ float wgt[];                       // [n_split]
  __shared__ float red[32];
  const int h = blockIdx.x, q = blockIdx.y;
  const int k = threadIdx.x;
  const int64_t p = P.q_pos[q];
  const int64_t pbase = (int64_t)q * P.n_split * P.H;
  const int S = P.n_split;
  // splits' maxima -> M
  float mloc = -INFINITY;
  for (int s = k; s < S; s += blockDim.x) {
    const float ms = P.part_ml[((pbase + (int64_t)s * P.H) + h) * 2];
    wgt[s] = ms;
    mloc = fmaxf(mloc, ms);
  }
  const float z = P.sink ? P.sink[h] : -INFINITY;
  float M = block_max(mloc, red);
  M = fmaxf(M, z);
  // weights exp(m_s - M) and the denominator
  float dloc = 0.f;
  for (int s = k; s < S; s += blockDim.x) {
    const float ms = wgt[s];
    const float w = (ms == -INFINITY || M == -INFINITY) ? 0.f : __expf(ms - M);
    wgt[s] = w;
    dloc += w * P.part_ml[((pbase + (int64_t)s * P.H) + h) * 2 + 1];
  }
  float den = block_sum(dloc, red);
  if (P.sink && M != -INFINITY) den += __expf(z - M);
  float o0 = 0.f, o1 = 0.f;
  if (2 * k < P.d && M != -INFINITY) {
    const float2* base = reinterpret_cast<const float2*>(P.part_o + (pbase + h) * P.d) + k;
    const int64_t step = (int64_t)P.H * P.d / 2;           // float2 between splits
    int s = 0;
    for (; s + 8 <= S; s += 8) {
      float2 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = wgt[s + u] != 0.f ? base[(s + u) * step] : make_float2(0.f, 0.f);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        o0 = fmaf(v[u].x, wgt[s + u], o0);
        o1 = fmaf(v[u].y, wgt[s + u], o1);
      }
    }
    for (; s < S; ++s)
      if (wgt[s] != 0.f) {
        const float2 v = base[s * step];
        o0 = fmaf(v.x, wgt[s], o0);
        o1 = fmaf(v.y, wgt[s], o1);
      }
  }
  const float inv = den > 0.f ? 1.0f / den : 0.f;
  o0 *= inv;
  o1 *= inv;
  const int rope0 = (P.d - P.d_rope) / 2;
  if (2 * k < P.d && k >= rope0 && p >= 0) {
    float cs, sn;
    rope_cs(p, k - rope0, P.d_rope, P.theta, cs, sn);   // rotate by -p
    const float r0 = o0 * cs + o1 * sn;
    const float r1 = -o0 * sn + o1 * cs;
    o0 = r0;
    o1 = r1;
  }
  if (2 * k < P.d) {
    const int64_t ob = ((int64_t)q * P.H + h) * P.d;
    if (P.out_dtype == V4A_F32) {
      reinterpret_cast<float2*>(reinterpret_cast<float*>(P.out) + ob)[k] = make_float2(o0, o1);
    } else {
      __nv_bfloat162 v = __floats2bfloat162_rn(o0, o1);
      reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<__nv_bfloat16*>(P.out) + ob)[k] = v;
    }
  }
  if (P.lse && k == 0) P.lse[(int64_t)q * P.H + h] = (den > 0.f) ? M + logf(den) : -INFINITY;
}

cudaError_t launch_mqa_combine(const MqaParams& P, cudaStream_t st) {
  int threads = ((P.d / 2 + 31) / 32) * 32;
  dim3 grid(P.H, P.n_q);
  const size_t smem = (size_t)P.n_split * sizeof(float);
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(mqa_combine_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  mqa_combine_kernel<<<grid, threads, smem, st>>>(P);
  return cudaGetLastError();
}

}  // namespace v4a
