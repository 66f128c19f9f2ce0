// Softmax-gated KV pooling with the RMSNorm / RoPE / quantising epilogue.
//
// Method: "DeepSeek-V4 深读" (ricardokevins.github.io), section
// "CSA：4× 压缩之后再 top-k", equation C_i^comp (two branches of m tokens,
// per-channel softmax weights, 2m-token window at stride m); section
// "HCA：128× 压缩后保留 dense 全局视野" (m' = 128, no overlap); section
// "其他稳定性细节" (RMSNorm of compressed KV, RoPE on the last 64 dims, FP8
// non-RoPE dims + BF16 RoPE dims); "AI深一度 第15期|DeepSeek V4", section
// "一、CSA与HCA" (softmax gate with a learnable position bias).
//
// A cluster of CH CTAs computes one entry of one sequence, CTA r owning the
// channels [r*c/CH, (r+1)*c/CH) (whole 32-channel scale blocks), so that the
// window's rows are read by CH SMs at once.  Thread k of a row slice owns the
// channel pair (2k, 2k+1) of its chunk, which is also a RoPE pair; the
// window's rows are split over up to 8 row slices of the CTA.  Each slice runs an online
// (running-max) softmax per channel over its rows, 8 rows per batch with the
// batch's loads issued before its arithmetic, and the slices' (max, sum,
// weighted sum) triples are merged through shared memory.  The RMSNorm sum
// of squares and the E4M3 amax (taken on the pooled values; RMSNorm scales it
// by the same positive factor, and rounding is monotone) are added / maxed
// over the cluster through distributed shared memory.  Rows are read
// coalesced (consecutive threads, consecutive channels).  The step moves
// 2-4 x c values per window token and is HBM / latency bound.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace v4a {

namespace {
constexpr int kRowBatch = 8;

__device__ __forceinline__ float2 load_pair(const void* p, int dtype, int64_t i) {
  if (dtype == V4A_F32) return *reinterpret_cast<const float2*>(reinterpret_cast<const float*>(p) + i);
  const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(
      reinterpret_cast<const __nv_bfloat16*>(p) + i);
  return make_float2(__bfloat162float(v.x), __bfloat162float(v.y));
}

// fold a batch of (value, logit) pairs into the running (max, sum, acc) of one channel
__device__ __forceinline__ void fold(float& mx, float& sm, float& acc, const float* z,
                                     const float* v) {
  float m = mx;
#pragma unroll
  for (int u = 0; u < kRowBatch; ++u) m = fmaxf(m, z[u]);
  if (m == -INFINITY) return;
  const float al = __expf(mx - m);        // 0 when mx is still -inf
  acc *= al;
  sm *= al;
#pragma unroll
  for (int u = 0; u < kRowBatch; ++u) {
    const float e = __expf(z[u] - m);     // 0 for the -inf fillers
    acc += e * v[u];
    sm += e;
  }
  mx = m;
}
}  // namespace

__device__ void compress_entry(const CompressParams& P, int b, int64_t i, float* red, float* mrg,
                               float* part, int PT, int RS, int CH, int chunk) {
  const int64_t p_new = P.new_pos ? P.new_pos[b] : -1;
  const int64_t L = P.seq_len ? P.seq_len[b] : p_new + 1;
  const int m = P.m;
  const int c = P.c;
  // uniform early exits (whole CTA)
  if (i < 0 || (int64_t)m * i >= L) return;
  if (P.complete_only && (int64_t)m * (i + 1) > L) return;

  const int CW = c / CH;                       // channels of this CTA's chunk
  const int k = threadIdx.x % PT, slice = threadIdx.x / PT;
  const int c0 = chunk * CW + 2 * k;           // first channel of this thread's pair
  const bool active = chunk < CH && 2 * k < CW;   // ranks past the chunks only keep the cluster barriers
  const bool owner = active && slice == 0;
  const int R = P.overlap ? 2 * m : m;
  const int per = (R + RS - 1) / RS;
  const int r_lo = min(R, slice * per), r_hi = min(R, r_lo + per);
  const int64_t jbase = P.overlap ? (int64_t)m * (i - 1) : (int64_t)m * i;
  const int64_t seq_off = (int64_t)b * P.in_seq_stride;

  float mx0 = -INFINITY, mx1 = -INFINITY, s0 = 0.f, s1 = 0.f, a0 = 0.f, a1 = 0.f;
  if (active) {
    // input row of token j = jbase + r is j mod in_rows, kept incrementally
    // (one 64-bit modulo per thread instead of one per row)
    const int64_t nr = P.in_rows;
    int64_t jm = (jbase + r_lo) % nr;
    if (jm < 0) jm += nr;
    for (int r0 = r_lo; r0 < r_hi; r0 += kRowBatch) {
      float v0[kRowBatch], v1[kRowBatch], z0[kRowBatch], z1[kRowBatch];
#pragma unroll
      for (int u = 0; u < kRowBatch; ++u) {
        const int r = r0 + u;
        const int64_t j = jbase + r;
        v0[u] = v1[u] = 0.f;
        z0[u] = z1[u] = -INFINITY;
        const int64_t row = jm;
        if (++jm == nr) jm = 0;
        if (r < r_hi && j >= 0 && j < L) {
          const bool br_a = !P.overlap || r >= m;
          const bool fresh = j == p_new;          // the decode step's new token
          const void* Cp = fresh ? (br_a ? P.Ca_new : P.Cb_new) : (br_a ? P.Ca : P.Cb);
          const void* Zp = fresh ? (br_a ? P.Za_new : P.Zb_new) : (br_a ? P.Za : P.Zb);
          const int64_t off = fresh ? (int64_t)b * P.new_seq_stride + c0
                                    : seq_off + row * P.in_row_stride + c0;
          const float2 v = load_pair(Cp, P.in_dtype, off);
          float2 z = Zp ? load_pair(Zp, P.in_dtype, off) : make_float2(0.f, 0.f);
          if (P.bias) {
            const float2 bb = *reinterpret_cast<const float2*>(P.bias + (int64_t)r * c + c0);
            z.x += bb.x;
            z.y += bb.y;
          }
          v0[u] = v.x;
          v1[u] = v.y;
          z0[u] = z.x;
          z1[u] = z.y;
        }
      }
      fold(mx0, s0, a0, z0, v0);
      fold(mx1, s1, a1, z1, v1);
    }
  }
  if (RS > 1) {
    // merge the row slices into slice 0
    float* my = mrg + (size_t)threadIdx.x * 6;
    my[0] = mx0; my[1] = s0; my[2] = a0; my[3] = mx1; my[4] = s1; my[5] = a1;
    __syncthreads();
    if (slice == 0 && active) {
      float M0 = -INFINITY, M1 = -INFINITY;
      for (int q = 0; q < RS; ++q) {
        M0 = fmaxf(M0, mrg[(size_t)(q * PT + k) * 6]);
        M1 = fmaxf(M1, mrg[(size_t)(q * PT + k) * 6 + 3]);
      }
      s0 = a0 = s1 = a1 = 0.f;
      for (int q = 0; q < RS; ++q) {
        const float* o = mrg + (size_t)(q * PT + k) * 6;
        if (o[0] != -INFINITY) {
          const float f = __expf(o[0] - M0);
          s0 += f * o[1];
          a0 += f * o[2];
        }
        if (o[3] != -INFINITY) {
          const float f = __expf(o[3] - M1);
          s1 += f * o[4];
          a1 += f * o[5];
        }
      }
    }
  }
  float e0 = owner ? a0 / s0 : 0.f;
  float e1 = owner ? a1 / s1 : 0.f;

  // row-wide sum of squares (RMSNorm) and amax of the non-RoPE channels (E4M3)
  const bool e4m3 = P.out_dtype == V4A_E4M3_BF16ROPE;
  const int dn = c - P.d_rope;
  float ss = 0.f, amax = 0.f;
  if (P.apply_rmsnorm) ss = block_sum(e0 * e0 + e1 * e1, red);
  if (e4m3) amax = block_max((owner && c0 < dn) ? fmaxf(fabsf(e0), fabsf(e1)) : 0.f, red);
  if (CH > 1 && (P.apply_rmsnorm || e4m3)) {
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    if (threadIdx.x == 0) {
      part[0] = ss;
      part[1] = amax;
    }
    cl.sync();                                   // every chunk's partials are published
    if (threadIdx.x < 32) {
      float s2 = 0.f, a2 = 0.f;
      if ((int)threadIdx.x < CH) {
        const float* rp = cl.map_shared_rank(part, (unsigned)threadIdx.x);
        s2 = rp[0];
        a2 = rp[1];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        a2 = fmaxf(a2, __shfl_xor_sync(0xffffffffu, a2, o));
      }
      if (threadIdx.x == 0) {
        red[0] = s2;
        red[1] = a2;
      }
    }
    __syncthreads();
    ss = red[0];
    amax = red[1];
    cl.sync();                                   // no chunk rewrites its partials while read
  }
  if (P.apply_rmsnorm) {
    const float inv = 1.0f / sqrtf(ss / (float)c + P.eps);
    e0 *= inv;
    e1 *= inv;
    amax *= inv;                                 // == the amax of the normalised values
  }
  if (P.apply_rope && owner && c0 >= c - P.d_rope) {
    float cs, sn;
    rope_cs((int64_t)m * i, (c0 - (c - P.d_rope)) / 2, P.d_rope, P.theta, cs, sn);
    const float r0 = e0 * cs - e1 * sn;
    const float r1 = e0 * sn + e1 * cs;
    e0 = r0;
    e1 = r1;
  }

  const int64_t row = i % P.out_rows;
  const int64_t rb = row_bytes(P.out_dtype, c, P.d_rope);
  uint8_t* out = reinterpret_cast<uint8_t*>(P.out) + ((int64_t)b * P.out_rows + row) * rb;
  if (P.out_dtype == V4A_F32) {
    if (owner) reinterpret_cast<float2*>(out)[c0 >> 1] = make_float2(e0, e1);
  } else if (e4m3) {
    const int se = e4m3_scale_exp(amax);
    if (owner) {
      if (c0 < dn) {
        const uint16_t pr = (uint16_t)f32_to_e4m3(scale_pow2(e0, se)) |
                            ((uint16_t)f32_to_e4m3(scale_pow2(e1, se)) << 8);
        reinterpret_cast<uint16_t*>(out)[c0 >> 1] = pr;
      } else {
        const uint32_t pr = (uint32_t)f32_to_bf16_bits(e0) | ((uint32_t)f32_to_bf16_bits(e1) << 16);
        reinterpret_cast<uint32_t*>(out + dn)[(c0 - dn) / 2] = pr;
      }
    }
    if (threadIdx.x == 0 && chunk == 0)
      reinterpret_cast<float*>(P.out_scale)[(int64_t)b * P.out_rows + row] = exp2i(se);
  } else {  // V4A_MXFP4: 16 threads (32 channels) per scale block
    float am = owner ? fmaxf(fabsf(e0), fabsf(e1)) : 0.f;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    const int X = mx_scale_exp(am);
    if (owner) {
      const uint8_t lo = f32_to_e2m1(scale_pow2(e0, X));
      const uint8_t hi = f32_to_e2m1(scale_pow2(e1, X));
      out[c0 >> 1] = (uint8_t)(lo | (hi << 4));
      if ((c0 & 31) == 0)
        reinterpret_cast<uint8_t*>(P.out_scale)[((int64_t)b * P.out_rows + row) * (c / 32) +
                                                c0 / 32] = (uint8_t)(X + 127);
    }
  }
}

// Grid-stride over the entries of sequence blockIdx.y; the CH CTAs of a
// cluster (consecutive blockIdx.x) share an entry.
__global__ void __launch_bounds__(512) compress_kernel(CompressParams P, int n_entries, int PT, int RS,
                                                       int CH) {
  __shared__ float red[32];
  __shared__ float part[2];
  extern __shared__ float mrg[];
  const int b = blockIdx.y;
  const int chunk = (int)(blockIdx.x % CH);
  const int64_t e0 = P.entry_begin[b];
  for (int e = (int)(blockIdx.x / CH); e < n_entries; e += (int)(gridDim.x / CH)) {
    compress_entry(P, b, e0 + e, red, mrg, part, PT, RS, CH, chunk);
    __syncthreads();
  }
}

cudaError_t launch_compress(const CompressParams& P, int B, int n_entries, cudaStream_t st) {
  // chunks: whole 32-channel blocks of at least 64 channels each, up to 8
  int CH = 8;
  while (CH > 1 && (P.c % (32 * CH) != 0 || P.c / CH < 64)) CH >>= 1;
  const int CW = P.c / CH;
  int PT = ((CW / 2 + 31) / 32) * 32;      // threads per row slice
  if (PT < 32) PT = 32;
  const int R = P.overlap ? 2 * P.m : P.m;
  int RS = R / (2 * kRowBatch);            // row slices: at least 2 batches each
  RS = RS < 1 ? 1 : (RS > 8 ? 8 : RS);
  while (RS > 1 && PT * RS > 512) --RS;
  const size_t smem = RS > 1 ? (size_t)PT * RS * 6 * sizeof(float) : 0;
  const int per_b = n_entries < 4096 ? n_entries : 4096;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(per_b * CH), (unsigned)B, 1);
  cfg.blockDim = dim3((unsigned)(PT * RS), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)CH;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, compress_kernel, P, n_entries, PT, RS, CH);
}

}  // namespace v4a
