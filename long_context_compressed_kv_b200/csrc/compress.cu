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
#include "mqa_qimage.cuh"

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

// One decode step's appends for every sequence b, in one launch: job (b, t)
// is one cluster of kAppendCluster CTAs; t = 0 codes the new token's window
// KV (and copies its raw inputs into the main tail ring), t = 1 pools the
// entry its block completes, t = 2 (CSA) pools the indexer key (and copies
// the indexer inputs into the indexer tail ring).  The pooling jobs read the
// new token from its input row, so the ring copies run concurrently with them.
constexpr int kAppendCluster = 8;
constexpr int kAppendThreads = 256;

__device__ __forceinline__ int chunks_for(int c) {
  int CH = kAppendCluster;
  while (CH > 1 && (c % (32 * CH) != 0 || c / CH < 64)) CH >>= 1;
  return CH;
}

__device__ __forceinline__ void copy_share(uint8_t* dst, const uint8_t* src, int64_t n, int rank) {
  // rank's share of an n-byte copy, 16 bytes at a time where both ends allow it
  const int64_t per = (n / kAppendCluster + 15) / 16 * 16;
  const int64_t lo = min(n, per * rank), hi = min(n, lo + per);
  if ((((uintptr_t)(dst + lo)) | ((uintptr_t)(src + lo)) | (uintptr_t)(hi - lo)) % 16 == 0) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src + lo);
    uint4* d4 = reinterpret_cast<uint4*>(dst + lo);
    for (int64_t e = threadIdx.x; e < (hi - lo) / 16; e += blockDim.x) d4[e] = s4[e];
  } else {
    for (int64_t e = lo + threadIdx.x; e < hi; e += blockDim.x) dst[e] = src[e];
  }
}

__global__ void __launch_bounds__(kAppendThreads, 2) decode_append_kernel(AppendParams A) {
  __shared__ float red[32];
  __shared__ float part[2];
  __shared__ float mrg[kAppendThreads * 6];
  const int nbase = A.csa ? 3 : 2;
  const int nj = nbase + (A.qimg ? 1 : 0);
  const int job = blockIdx.x / kAppendCluster, rank = blockIdx.x % kAppendCluster;
  const int b = job / nj, t = job % nj;
  if (t == nbase) {
    // the tensor-core MQA's query image: CTA `rank` codes head rows 16*rank .. +15
    __shared__ float qcs[32], qsn[32];
    qimage_code_rows(reinterpret_cast<const __nv_bfloat16*>(A.Q) + (int64_t)b * A.H * 512, A.H,
                     A.pos[b], A.theta, A.qimg + (int64_t)b * kMqaQImageStride, rank, qcs, qsn);
    return;
  }
  const int elt = A.in_dtype == V4A_F32 ? 4 : 2;
  const int64_t p = A.pos[b];
  const int64_t nb = (int64_t)A.n_arr * A.d * elt;         // bytes of one main input row
  const uint8_t* xm = reinterpret_cast<const uint8_t*>(A.x_main);
  const uint8_t* tl = reinterpret_cast<const uint8_t*>(A.tail);
  CompressParams P;
  P.in_dtype = A.in_dtype;
  P.d_rope = A.d_rope;
  P.theta = A.theta;
  P.eps = A.eps;
  P.seq_len = nullptr;
  P.entry_begin = nullptr;
  P.new_pos = A.pos;
  int64_t i;
  if (t == 0) {
    if (p >= 0)
      copy_share(reinterpret_cast<uint8_t*>(A.tail) + ((int64_t)b * A.ring + p % A.ring) * nb,
                 xm + b * nb, nb, rank);
    P.m = 1;
    P.overlap = 0;
    P.c = A.d;
    P.Ca = A.x_main;
    P.Za = P.Cb = P.Zb = nullptr;
    P.Ca_new = A.x_main;
    P.in_seq_stride = P.in_row_stride = P.new_seq_stride = (int64_t)A.n_arr * A.d;
    P.in_rows = 1;
    P.bias = nullptr;
    P.complete_only = 0;
    P.apply_rmsnorm = 1;
    P.apply_rope = 1;
    P.out_dtype = A.kv_dtype;
    P.out = A.swa;
    P.out_scale = A.swa_scale;
    P.out_rows = A.swa_rows;
    i = p;
  } else if (t == 1) {
    const int64_t da = (int64_t)A.d * elt;
    P.m = A.m;
    P.overlap = A.csa;
    P.c = A.d;
    P.Ca = tl;
    P.Za = tl + da;
    P.Cb = A.csa ? tl + 2 * da : nullptr;
    P.Zb = A.csa ? tl + 3 * da : nullptr;
    P.Ca_new = xm;
    P.Za_new = xm + da;
    P.Cb_new = A.csa ? xm + 2 * da : nullptr;
    P.Zb_new = A.csa ? xm + 3 * da : nullptr;
    P.in_seq_stride = (int64_t)A.ring * A.n_arr * A.d;
    P.in_row_stride = P.new_seq_stride = (int64_t)A.n_arr * A.d;
    P.in_rows = A.ring;
    P.bias = A.bias;
    P.complete_only = 1;
    P.apply_rmsnorm = 1;
    P.apply_rope = 1;
    P.out_dtype = A.kv_dtype;
    P.out = A.kv;
    P.out_scale = A.kv_scale;
    P.out_rows = A.kv_rows;
    i = p / A.m;
  } else {
    const int64_t ni = (int64_t)4 * A.dI * elt;
    const uint8_t* xi = reinterpret_cast<const uint8_t*>(A.x_idx);
    const uint8_t* it = reinterpret_cast<const uint8_t*>(A.itail);
    if (p >= 0)
      copy_share(reinterpret_cast<uint8_t*>(A.itail) + ((int64_t)b * A.ring + p % A.ring) * ni,
                 xi + b * ni, ni, rank);
    const int64_t da = (int64_t)A.dI * elt;
    P.m = A.m;
    P.overlap = 1;
    P.c = A.dI;
    P.Ca = it;
    P.Za = it + da;
    P.Cb = it + 2 * da;
    P.Zb = it + 3 * da;
    P.Ca_new = xi;
    P.Za_new = xi + da;
    P.Cb_new = xi + 2 * da;
    P.Zb_new = xi + 3 * da;
    P.in_seq_stride = (int64_t)A.ring * 4 * A.dI;
    P.in_row_stride = P.new_seq_stride = (int64_t)4 * A.dI;
    P.in_rows = A.ring;
    P.bias = A.ibias;
    P.complete_only = 1;
    P.apply_rmsnorm = 0;
    P.apply_rope = 0;
    P.out_dtype = A.idx_dtype;
    P.out = A.keys;
    P.out_scale = A.keys_sf;
    P.out_rows = A.key_rows;
    i = p / A.m;
  }
  const int CH = chunks_for(P.c);
  int PT = ((P.c / CH / 2 + 31) / 32) * 32;
  if (PT < 32) PT = 32;
  compress_entry(P, b, i, red, mrg, part, PT, kAppendThreads / PT, CH, rank);
}

cudaError_t launch_decode_append(const AppendParams& A, cudaStream_t st) {
  static_assert(kAppendCluster == 8 && kAppendThreads >= 64, "query image: 8 CTAs of 16 head rows");
  const int nj = (A.csa ? 3 : 2) + (A.qimg ? 1 : 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(A.B * nj * kAppendCluster), 1, 1);
  cfg.blockDim = dim3(kAppendThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kAppendCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_append_kernel, A);
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
