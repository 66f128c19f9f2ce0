// One decode step's appends for every sequence of a layer, in one launch.
//
// Method: "DeepSeek-V4 深读" (ricardokevins.github.io), section "CSA：4× 压缩之后再
// top-k" (equation C_i^comp: softmax-gated pooling of a 2m-token window at
// stride m), "HCA：128× 压缩后保留 dense 全局视野" (m' = 128, no overlap),
// "其他稳定性细节" (RMSNorm, RoPE on the last 64 dims, E4M3 + bf16 storage, MXFP4
// indexer keys) and "异构 KV cache 与磁盘前缀复用" (the fixed-size state: the
// window of raw-token KV and the uncompressed tail of the current block).
//
// Jobs of sequence b (each a cluster of 8 CTAs of 256 threads):
//   W  rank 0: the new token's window KV (RMSNorm, RoPE at p, stored format)
//      into the window ring; ranks 1..7: the new token's raw compressor inputs
//      (and, for CSA, its indexer inputs) into the tail rings;
//   E  when the token completes a block: its entry, pooled over the block's
//      window (the new token read from its input row, the others from the
//      tail ring), then RMSNorm, RoPE at m*i, stored format; channels split
//      over the 8 CTAs, the RMS and amax reduced over the cluster;
//   K  (CSA) when the token completes a block: its indexer key (same pooling,
//      no RMSNorm / RoPE, MXFP4), 32 channels per CTA;
//   Q  (optional) the tensor-core MQA's query image, 16 head rows per CTA.
// The pooling issues the loads of every window row a thread needs (the biases
// by asynchronous copies) before it computes, so a job waits for memory once,
// and computes its RoPE angles while they are in flight; the row slices of
// each channel are merged by shuffles.  Only E synchronises its cluster (once).
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "mqa_qimage.cuh"
#include "tc_common.cuh"

namespace v4a {

namespace {
constexpr int kCl = 8;           // CTAs per job (cluster)
constexpr int kThr = 256;        // threads per CTA
constexpr int kMaxRps = 8;       // window rows per thread, at most (R <= 128, >= 16 slices)

// four consecutive channels starting at element `off` (16-byte / 8-byte aligned)
__device__ __forceinline__ float4 ld4(const void* base, int dtype, int64_t off) {
  if (dtype == V4A_F32) return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + off);
  const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(base) + off);
  return make_float4(bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y));
}

__device__ __forceinline__ float f4(const float4& v, int k) {
  return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
}

// Sum and max over the CTA (all threads call; `red` holds >= 64 floats).
__device__ __forceinline__ float2 cta_sum_max(float s, float m, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  s = warp_sum(s);
  m = warp_max(m);
  __syncthreads();
  if (lane == 0) {
    red[wid] = s;
    red[32 + wid] = m;
  }
  __syncthreads();
  float ts = lane < kThr / 32 ? red[lane] : 0.f, tm = lane < kThr / 32 ? red[32 + lane] : 0.f;
  ts = warp_sum(ts);
  tm = warp_max(tm);
  return make_float2(ts, tm);
}

struct PoolArgs {
  const void* tail;       // ring rows of this sequence: [ring][n_arr][d_row]
  const void* xnew;       // the new token's row: [n_arr][d_row]
  int dtype, ring, n_arr, d_row;
  int ia, iz, ib, izb;    // array index of C^a, Z^a, C^b, Z^b in a row
  int m, R;               // stride, window rows (2m overlapped, m otherwise; R <= ring)
  bool overlap;
  const float* bias;      // [R][d_row]
  int64_t p, i;           // the new token's position, the entry index
};

// RoPE angles a job needs (pair k of a vector at position pos), or none
struct RopeReq {
  bool on;
  int64_t pos;
  int k, d_rope;
  float theta;
};

// Softmax-gated pooling of channels [c_lo, c_lo + CW) of entry i (CW a
// multiple of 4, CW / 4 threads per row): e[c - c_lo] in shared memory.  Each
// thread issues the loads of all its rows (the biases by asynchronous copies
// into its own slots of `bsm`) before any arithmetic, computes the RoPE angle
// `rq` asks for while they are in flight (into rc / rs), then pools; the
// slices of each channel are merged by kThr / CW adjacent threads, four
// slices each.
__device__ void pool_channels(const PoolArgs& a, int c_lo, int CW, float* e, float* part,
                              float4* bsm, const RopeReq& rq, float& rc, float& rs) {
  const int PT = CW / 4, NS = kThr / PT;
  const int t = threadIdx.x, cg = t % PT, sl = t / PT;
  const int c0 = c_lo + 4 * cg;
  const int64_t j0 = a.overlap ? (int64_t)a.m * (a.i - 1) : (int64_t)a.m * a.i;
  const int64_t row_el = (int64_t)a.n_arr * a.d_row;
  // ring slot of window row 0; row r sits r slots later (R <= ring: one wrap at most)
  const int s0 = (int)(((j0 % a.ring) + a.ring) % a.ring);
  bool ok[kMaxRps];
#pragma unroll
  for (int k = 0; k < kMaxRps; ++k) {
    const int r = sl + k * NS;
    const int64_t j = j0 + r;
    ok[k] = r < a.R && j >= 0 && j <= a.p;
    if (a.bias)
      cp_async16(&bsm[k * kThr + t], a.bias + (ok[k] ? (int64_t)r * a.d_row + c0 : 0), ok[k]);
  }
  cp_async_commit();
  float4 cv[kMaxRps], zv[kMaxRps];
#pragma unroll
  for (int k = 0; k < kMaxRps; ++k) {
    cv[k] = zv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (ok[k]) {
      const int r = sl + k * NS;
      const bool br_a = !a.overlap || r >= a.m;
      const int ic = br_a ? a.ia : a.ib, iz = br_a ? a.iz : a.izb;
      const bool is_new = j0 + r == a.p;
      int slot = s0 + r;
      slot -= slot >= a.ring ? a.ring : 0;
      const void* src = is_new ? a.xnew : a.tail;
      const int64_t rb = is_new ? 0 : (int64_t)slot * row_el;
      cv[k] = ld4(src, a.dtype, rb + (int64_t)ic * a.d_row + c0);
      zv[k] = ld4(src, a.dtype, rb + (int64_t)iz * a.d_row + c0);
    }
  }
  rc = 1.f;
  rs = 0.f;
  if (rq.on) rope_cs(rq.pos, rq.k, rq.d_rope, rq.theta, rc, rs);
  cp_async_wait<0>();                                // this thread's own bias copies
  if (a.bias) {
#pragma unroll
    for (int k = 0; k < kMaxRps; ++k) {
      const float4 bb = bsm[k * kThr + t];
      zv[k].x += bb.x;
      zv[k].y += bb.y;
      zv[k].z += bb.z;
      zv[k].w += bb.w;
    }
  }
  // this slice's (max, sum, weighted sum) of each of its 4 channels
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float m = -INFINITY;
#pragma unroll
    for (int k = 0; k < kMaxRps; ++k)
      if (ok[k]) m = fmaxf(m, f4(zv[k], c));
    float sm = 0.f, acc = 0.f;
    if (m != -INFINITY) {
#pragma unroll
      for (int k = 0; k < kMaxRps; ++k)
        if (ok[k]) {
          const float w = __expf(f4(zv[k], c) - m);
          sm += w;
          acc = fmaf(w, f4(cv[k], c), acc);
        }
    }
    float* q = part + ((int64_t)sl * CW + 4 * cg + c) * 3;   // part[slice][channel][3]
    q[0] = m;
    q[1] = sm;
    q[2] = acc;
  }
  __syncthreads();
  // merge: channel t / TPC, slices 4 (t % TPC) .. + 3, then across the TPC lanes
  const int TPC = kThr / CW, ch = t / TPC, sub = t % TPC;
  float ms[4], ss[4], as[4];
  float M = -INFINITY;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const float* q = part + ((int64_t)(4 * sub + u) * CW + ch) * 3;
    ms[u] = q[0];
    ss[u] = q[1];
    as[u] = q[2];
    M = fmaxf(M, ms[u]);
  }
  for (int o = 1; o < TPC; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float S = 0.f, A = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (ms[u] != -INFINITY) {
        const float f = __expf(ms[u] - M);
        S = fmaf(f, ss[u], S);
        A = fmaf(f, as[u], A);
      }
  }
  for (int o = 1; o < TPC; o <<= 1) {
    S += __shfl_xor_sync(0xffffffffu, S, o);
    A += __shfl_xor_sync(0xffffffffu, A, o);
  }
  if (sub == 0) e[ch] = S > 0.f ? A / S : 0.f;
  __syncthreads();
}

// RMSNorm (over all d channels of the vector, CH CTAs of CW each), RoPE on the
// last d_rope channels with this thread's pair angle (rc, rs), and the stored
// format of channels [c_lo, c_lo + CW) of one row: E4M3 + bf16 (scale written
// by the CTA holding channel 0) or fp32.  All threads call; with CH > 1 the
// CTAs of the cluster call it together and meet at one cluster barrier (each
// pushes its partial sum / amax into every CTA's xch[2 rank ..]).
__device__ void finish_main(const float* e, int c_lo, int CW, int d, int d_rope, bool norm,
                            bool rope, float rc, float rs, float eps, int out_dtype,
                            uint8_t* out_row, float* out_scale, int CH, float* red, float* xch) {
  namespace cg = cooperative_groups;
  const int t = threadIdx.x;
  const bool act = 2 * t < CW;
  const int c = c_lo + 2 * t;
  float e0 = act ? e[2 * t] : 0.f, e1 = act ? e[2 * t + 1] : 0.f;
  const int dn = d - d_rope;
  const bool e4 = out_dtype == V4A_E4M3_BF16ROPE;
  float2 sa = cta_sum_max(e0 * e0 + e1 * e1,
                          (act && c < dn) ? fmaxf(fabsf(e0), fabsf(e1)) : 0.f, red);
  if (CH > 1) {
    cg::cluster_group cl = cg::this_cluster();
    const unsigned rank = cl.block_rank();
    if (t < CH) {
      float* rp = cl.map_shared_rank(xch, (unsigned)t);
      rp[2 * rank] = sa.x;
      rp[2 * rank + 1] = sa.y;
    }
    cl.sync();                                       // every CTA's partial in every xch
    float s2 = 0.f, a2 = 0.f;
    for (int r = 0; r < CH; ++r) {                   // the same order in every CTA
      s2 += xch[2 * r];
      a2 = fmaxf(a2, xch[2 * r + 1]);
    }
    sa = make_float2(s2, a2);
  }
  float amax = sa.y;
  if (norm) {
    const float inv = 1.0f / sqrtf(sa.x / (float)d + eps);
    e0 *= inv;
    e1 *= inv;
    amax *= inv;                                     // == the amax of the normalised values
  }
  if (act && rope && c >= dn) {
    const float r0 = e0 * rc - e1 * rs, r1 = e0 * rs + e1 * rc;
    e0 = r0;
    e1 = r1;
  }
  if (!act) return;
  if (out_dtype == V4A_F32) {
    reinterpret_cast<float2*>(out_row)[c >> 1] = make_float2(e0, e1);
  } else if (e4) {
    const int se = e4m3_scale_exp(amax);
    if (c < dn) {
      const uint16_t pr = (uint16_t)f32_to_e4m3(scale_pow2(e0, se)) |
                          ((uint16_t)f32_to_e4m3(scale_pow2(e1, se)) << 8);
      reinterpret_cast<uint16_t*>(out_row)[c >> 1] = pr;
    } else {
      const uint32_t pr = (uint32_t)f32_to_bf16_bits(e0) | ((uint32_t)f32_to_bf16_bits(e1) << 16);
      reinterpret_cast<uint32_t*>(out_row + dn)[(c - dn) / 2] = pr;
    }
    if (c == 0) *out_scale = exp2i(se);
  }
}

// MXFP4 coding of channels [c_lo, c_lo + 32) (one E8M0 block) of one row.
__device__ void finish_mxfp4(const float* e, int c_lo, uint8_t* out_row, uint8_t* out_sf) {
  const int t = threadIdx.x;
  if (t >= 16) return;                               // 16 threads, a channel pair each
  const float e0 = e[2 * t], e1 = e[2 * t + 1];
  float am = fmaxf(fabsf(e0), fabsf(e1));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0x0000ffffu, am, o));
  const int X = mx_scale_exp(am);
  const int c = c_lo + 2 * t;
  out_row[c >> 1] = (uint8_t)(f32_to_e2m1(scale_pow2(e0, X)) | (f32_to_e2m1(scale_pow2(e1, X)) << 4));
  if (t == 0) out_sf[c_lo / 32] = (uint8_t)(X + 127);
}

// rank's share of an n-byte copy, 16 bytes at a time where both ends allow it
__device__ __forceinline__ void copy_share(uint8_t* dst, const uint8_t* src, int64_t n, int rank,
                                           int parts) {
  const int64_t per = (n / parts + 15) / 16 * 16;
  const int64_t lo = min(n, per * rank), hi = min(n, lo + per);
  if ((((uintptr_t)(dst + lo)) | ((uintptr_t)(src + lo)) | (uintptr_t)(hi - lo)) % 16 == 0) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src + lo);
    uint4* d4 = reinterpret_cast<uint4*>(dst + lo);
    for (int64_t k = threadIdx.x; k < (hi - lo) / 16; k += blockDim.x) d4[k] = s4[k];
  } else {
    for (int64_t k = lo + threadIdx.x; k < hi; k += blockDim.x) dst[k] = src[k];
  }
}
}  // namespace

// PAGED: the entry and the indexer key go to their block's slot in the pools
// (A.kv_pages / A.key_pages); a compile-time switch, so that the per-sequence
// kernel carries none of it
template <bool PAGED>
__global__ void __launch_bounds__(kThr, 2) decode_append_kernel(AppendParams A) {
  __shared__ float red[72];
  __shared__ float xch[2 * kCl];
  __shared__ __align__(16) float ebuf[512];
  __shared__ float part[kThr * 4 * 3];               // slices x channels x (max, sum, acc)
  __shared__ float4 bsm[kMaxRps * kThr];             // each thread's pooling biases
  const int nbase = A.csa ? 3 : 2;
  const int nj = nbase + (A.qimg ? 1 : 0);
  const int job = blockIdx.x / kCl, rank = blockIdx.x % kCl;
  const int b = job / nj, t = job % nj;
  const int64_t p = A.pos[b];
  const int elt = A.in_dtype == V4A_F32 ? 4 : 2;
  if (t == nbase) {
    // Q: the tensor-core MQA's query image, head rows 16*rank .. +15
    __shared__ float qcs[32], qsn[32];
    qimage_code_rows(reinterpret_cast<const __nv_bfloat16*>(A.Q) + (int64_t)b * A.H * 512, A.H, p,
                     A.theta, A.qimg + (int64_t)b * kMqaQImageStride, rank, qcs, qsn);
    return;
  }
  if (p < 0) return;                                 // uniform for the whole cluster
  const int64_t nb = (int64_t)A.n_arr * A.d * elt;   // bytes of one main input row
  const uint8_t* xm = reinterpret_cast<const uint8_t*>(A.x_main) + b * nb;
  if (t == 0) {
    if (rank == 0) {
      // W: the new token's window KV = RMSNorm(C^a_p) with RoPE at p (d <= 4 kThr)
      const int c4 = threadIdx.x * 4, c2 = threadIdx.x * 2, dn = A.d - A.d_rope;
      const float4 v = c4 < A.d ? ld4(xm, A.in_dtype, c4) : make_float4(0.f, 0.f, 0.f, 0.f);
      float rc = 1.f, rs = 0.f;                      // this thread's pair in finish_main
      if (c2 >= dn && c2 < A.d) rope_cs(p, (c2 - dn) / 2, A.d_rope, A.theta, rc, rs);
      if (c4 < A.d) *reinterpret_cast<float4*>(&ebuf[c4]) = v;
      __syncthreads();
      const int64_t rb = row_bytes(A.kv_dtype, A.d, A.d_rope);
      const int64_t row = (int64_t)b * A.swa_rows + p % A.swa_rows;
      finish_main(ebuf, 0, A.d, A.d, A.d_rope, true, true, rc, rs, A.eps, A.kv_dtype,
                  reinterpret_cast<uint8_t*>(A.swa) + row * rb,
                  A.swa_scale ? reinterpret_cast<float*>(A.swa_scale) + row : nullptr, 1, red, xch);
    } else {
      // the new token's raw inputs into the tail rings (ranks 1..7)
      copy_share(reinterpret_cast<uint8_t*>(A.tail) + ((int64_t)b * A.ring + p % A.ring) * nb, xm,
                 nb, rank - 1, kCl - 1);
      if (A.csa) {
        const int64_t ni = (int64_t)4 * A.dI * elt;
        copy_share(reinterpret_cast<uint8_t*>(A.itail) + ((int64_t)b * A.ring + p % A.ring) * ni,
                   reinterpret_cast<const uint8_t*>(A.x_idx) + b * ni, ni, rank - 1, kCl - 1);
      }
    }
    return;
  }
  if ((p + 1) % A.m != 0) return;                    // no block completes: uniform per cluster
  const int64_t i = p / A.m;
  PoolArgs a;
  a.dtype = A.in_dtype;
  a.ring = A.ring;
  a.m = A.m;
  a.overlap = A.csa != 0;
  a.R = A.csa ? 2 * A.m : A.m;
  a.p = p;
  a.i = i;
  a.n_arr = 4;                                        // (Ca, Za, Cb, Zb) / CSA; HCA below
  a.ia = 0;
  a.iz = 1;
  a.ib = 2;
  a.izb = 3;
  if (t == 1) {
    // E: the entry this token completes; 8 CTAs of d / 8 channels
    a.tail = reinterpret_cast<const uint8_t*>(A.tail) + (int64_t)b * A.ring * nb;
    a.xnew = xm;
    a.n_arr = A.n_arr;
    a.d_row = A.d;
    a.bias = A.bias;
    const int CW = A.d / kCl, c_lo = rank * CW;
    // the RoPE angle of this thread's pair in finish_main (entry position m i)
    const int c2 = c_lo + 2 * (int)threadIdx.x, dn = A.d - A.d_rope;
    RopeReq rq{2 * (int)threadIdx.x < CW && c2 >= dn, (int64_t)A.m * i, (c2 - dn) / 2, A.d_rope,
               A.theta};
    float rc, rs;
    pool_channels(a, c_lo, CW, ebuf, part, bsm, rq, rc, rs);
    const int64_t rb = row_bytes(A.kv_dtype, A.d, A.d_rope);
    // the entry's row: its block's slot in the pool, or this sequence's row
    // (the same for every CTA of the cluster, so all of them return together)
    const int64_t row = PAGED ? page_row(A.kv_pages, b, i) : (int64_t)b * A.kv_rows + i % A.kv_rows;
    if (PAGED && row < 0) {
      if (rank == 0 && threadIdx.x == 0) flag(A.status, ST_BAD_INDEX);
      return;
    }
    uint8_t* orow = reinterpret_cast<uint8_t*>(A.kv) + row * rb;
    // this CTA's channels, offset so that finish_main writes them in place
    finish_main(ebuf, c_lo, CW, A.d, A.d_rope, true, true, rc, rs, A.eps, A.kv_dtype, orow,
                A.kv_scale ? reinterpret_cast<float*>(A.kv_scale) + row : nullptr, kCl, red, xch);
    return;
  }
  // K (CSA): the indexer key this token completes; 32 channels per CTA
  const int CW = 32, c_lo = rank * CW;
  if (c_lo >= A.dI) return;                          // no cluster barrier on this job
  const int64_t ni = (int64_t)4 * A.dI * elt;
  a.tail = reinterpret_cast<const uint8_t*>(A.itail) + (int64_t)b * A.ring * ni;
  a.xnew = reinterpret_cast<const uint8_t*>(A.x_idx) + b * ni;
  a.d_row = A.dI;
  a.bias = A.ibias;
  RopeReq none{false, 0, 0, 0, 0.f};
  float rc, rs;
  pool_channels(a, c_lo, CW, ebuf, part, bsm, none, rc, rs);
  const int64_t row =
      PAGED ? page_row(A.key_pages, b, i) : (int64_t)b * A.key_rows + i % A.key_rows;
  if (PAGED && row < 0) {                            // after the pooling: no barrier follows
    if (rank == 0 && threadIdx.x == 0) flag(A.status, ST_BAD_INDEX);
    return;
  }
  if (A.idx_dtype == V4A_MXFP4) {
    finish_mxfp4(ebuf, c_lo, reinterpret_cast<uint8_t*>(A.keys) + row * (A.dI / 2),
                 reinterpret_cast<uint8_t*>(A.keys_sf) + row * (A.dI / 32));
  } else if (threadIdx.x < CW) {
    reinterpret_cast<float*>(A.keys)[row * A.dI + c_lo + threadIdx.x] = ebuf[threadIdx.x];
  }
}

cudaError_t launch_decode_append(const AppendParams& A, cudaStream_t st) {
  static_assert(kCl == 8 && kThr >= 64, "query image: 8 CTAs of 16 head rows");
  const int nj = (A.csa ? 3 : 2) + (A.qimg ? 1 : 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(A.B * nj * kCl), 1, 1);
  cfg.blockDim = dim3(kThr, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCl;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return A.kv_pages.bt ? cudaLaunchKernelEx(&cfg, decode_append_kernel<true>, A)
                       : cudaLaunchKernelEx(&cfg, decode_append_kernel<false>, A);
}

}  // namespace v4a
