// Per-query top-k selection by one thread-block cluster per query.
//
// Method: "DeepSeek-V4 深读" (ricardokevins.github.io), section
// "CSA：4× 压缩之后再 top-k" (the k highest-scoring compressed entries per
// query; Flash k = 512, Pro k = 1024).  Ties go to the lower index and the
// selection is written in ascending index order, -1 padded.
//
// The CTAs of a cluster (16 for a few queries, fewer for many: the largest
// power of two whose clusters for all the call's queries fit on the GPU at
// once, down to one CTA a query) split the query's visible scores into slices and
// keep their slice in shared memory (as order-preserving uint32 keys).  A
// cluster-wide min / max first finds the key bits that every visible score
// shares; an exact radix select then resolves the remaining bits 8 at a time.
// Every pass builds a 256-bin histogram of the keys that match the bits
// resolved so far, one sub-histogram per warp (plain shared atomics: the
// leading bits of scores crowd into few bins, and warps never contend with
// each other), sums the warps' columns, and adds the CTA's non-empty bins into
// rank 0's totals with atomics on distributed shared memory; after a cluster
// barrier every CTA copies the 256 totals with vector loads and one warp
// finds the bin holding the k-th largest key.  When
// that bin is taken whole the select stops early and keys are compared on the
// resolved bits only.  The emission needs two block scans: each thread owns a
// contiguous run of its slice, counts the keys above the threshold and equal
// to it, and the CTA- and cluster-level prefix sums give every thread its
// first output position and its first tie rank, so indices are written in
// ascending order with no sort.  Cluster barriers are hardware barriers
// between co-scheduled CTAs that all take the same path.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace v4a {

namespace {
constexpr int TPB = 512;          // threads per CTA
constexpr int CACHE = 32768;      // keys a CTA keeps in shared memory (+1/64 padding)
constexpr int PAD_CACHE = CACHE + CACHE / 64;
constexpr int NB = 256;           // histogram bins (8 key bits per pass)
constexpr int MAXPASS = 4;        // 32 key bits
constexpr int NW = TPB / 32;      // warps = sub-histograms
constexpr size_t SMEM_WORDS = PAD_CACHE + NW * NB + NB + MAXPASS * NB;

__device__ __forceinline__ int padi(int i) { return i + (i >> 6); }   // bank-conflict-free runs

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

// Exclusive block scan of one int per thread (TPB threads); returns the prefix.
__device__ __forceinline__ int block_scan(int v, int* wsum, int& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) wsum[wid] = x;
  __syncthreads();
  if (wid == 0) {
    const int t = (lane < TPB / 32) ? wsum[lane] : 0;
    int s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    wsum[lane] = s - t;
    if (lane == 31) wsum[32] = s;
  }
  __syncthreads();
  total = wsum[32];
  return wsum[wid] + x - v;
}

__device__ __forceinline__ uint32_t high_mask(int bits) {   // the top `bits` bits set
  return bits <= 0 ? 0u : (bits >= 32 ? 0xFFFFFFFFu : ~(0xFFFFFFFFu >> bits));
}
}  // namespace

__global__ void __launch_bounds__(TPB, 1) topk_cluster_kernel(TopkParams P) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint32_t dyn[];
  uint32_t* keys = dyn;                         // PAD_CACHE entries
  uint32_t* whist = dyn + PAD_CACHE;            // [NW][NB] per-warp histograms
  uint32_t* hist = whist + NW * NB;             // [NB] this CTA's histogram
  uint32_t* tot = hist + NB;                    // [MAXPASS][NB] cluster totals (used in rank 0)
  __shared__ __align__(16) uint32_t tl[NB];     // this pass's totals, copied from rank 0
  __shared__ int wsum[33];
  __shared__ uint32_t sh_prefix, sh_mask, sh_bin;
  __shared__ int sh_rem, sh_bits, sh_done;
  __shared__ int sh_before[2];                  // (#gt, #eq) of the CTAs before this one
  __shared__ uint32_t mm[2];                    // this CTA's (min, max) key, read by the cluster
  __shared__ int cnt[2];                        // this CTA's (#gt, #eq), read by the cluster
  const uint32_t rank = cluster_rank();
  const int CL = (int)cluster.num_blocks();
  const int q = blockIdx.x / CL;
  const int lane = threadIdx.x & 31;
  int64_t nv64 = (P.q_pos[q] + 1) / P.m;
  if (nv64 > P.max_vis) nv64 = P.max_vis;
  const int nv = (int)nv64;
  const int kk = min(P.k, nv);
  int32_t* out = P.idx_out + (int64_t)q * P.k;
  if (rank == 0)
    for (int j = kk + threadIdx.x; j < P.k; j += TPB) out[j] = -1;
  if (kk == 0) return;                          // uniform for the whole cluster
  const int lo = (int)((int64_t)nv * rank / CL), hi = (int)((int64_t)nv * (rank + 1) / CL);
  const int len = hi - lo;
  if (nv <= P.k) {                              // every visible entry is selected
    for (int i = threadIdx.x; i < len; i += TPB) out[lo + i] = lo + i;
    return;                                     // uniform: no cluster barrier follows
  }
  const bool cached = len <= CACHE;
  // this CTA's slice of the row (fp32, or bf16 halves of 32-bit words)
  const int sbf = P.score_bf16;
  const float* src = sbf ? reinterpret_cast<const float*>(
                               reinterpret_cast<const uint16_t*>(P.scores) + (int64_t)q * P.scores_ld + lo)
                         : P.scores + (int64_t)q * P.scores_ld + lo;
  if (rank == 0)
    for (int t = threadIdx.x; t < MAXPASS * NB; t += TPB) tot[t] = 0;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  // bf16 rows: 16-bit order-preserving keys, so that at most two radix
  // passes resolve them
  auto take_key = [&](int i, float x) {
    const uint32_t k = sbf ? float_key(x) >> 16 : float_key(x);
    if (cached) keys[padi(i)] = k;
    kmin = min(kmin, k);
    kmax = max(kmax, k);
  };
  // scalar head up to a 16-byte boundary, then 16-byte loads, 8 in flight per
  // thread (bf16 rows: 8 loads of one score in flight, coalesced across the warp)
  const int head = sbf ? len : min(len, (int)((16 - (reinterpret_cast<uintptr_t>(src) & 15)) & 15) / 4);
  if (sbf) {
    // scalar head up to an 8-byte boundary, then 8-byte loads (4 scores), 8 in flight
    const uint16_t* s16 = reinterpret_cast<const uint16_t*>(src);
    auto bf = [](uint32_t b) { return __uint_as_float(b << 16); };
    const int hb = min(len, (int)((8 - (reinterpret_cast<uintptr_t>(s16) & 7)) & 7) / 2);
    if ((int)threadIdx.x < hb) take_key(threadIdx.x, bf(s16[threadIdx.x]));
    const uint2* s8 = reinterpret_cast<const uint2*>(s16 + hb);
    const int n8 = (len - hb) / 4;
    for (int j0 = 0; j0 < n8; j0 += 8 * TPB) {
      uint2 v8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * TPB + threadIdx.x;
        v8[u] = (j < n8) ? s8[j] : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int j = j0 + u * TPB + threadIdx.x;
        if (j < n8) {
          const int i = hb + 4 * j;
          take_key(i, bf(v8[u].x & 0xFFFFu));
          take_key(i + 1, bf(v8[u].x >> 16));
          take_key(i + 2, bf(v8[u].y & 0xFFFFu));
          take_key(i + 3, bf(v8[u].y >> 16));
        }
      }
    }
    for (int i = hb + 4 * n8 + threadIdx.x; i < len; i += TPB) take_key(i, bf(s16[i]));
  } else if ((int)threadIdx.x < head) {
    take_key(threadIdx.x, src[threadIdx.x]);
  }
  const float4* src4 = reinterpret_cast<const float4*>(src + (sbf ? 0 : head));
  const int n4 = sbf ? 0 : (len - head) / 4;
  for (int j0 = 0; j0 < n4; j0 += 8 * TPB) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * TPB + threadIdx.x;
      v[u] = (j < n4) ? src4[j] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * TPB + threadIdx.x;
      if (j < n4) {
        const int i = head + 4 * j;
        take_key(i, v[u].x);
        take_key(i + 1, v[u].y);
        take_key(i + 2, v[u].z);
        take_key(i + 3, v[u].w);
      }
    }
  }
  if (!sbf)
    for (int i = head + 4 * n4 + threadIdx.x; i < len; i += TPB) take_key(i, src[i]);
  auto key_at = [&](int i) -> uint32_t {
    return cached ? keys[padi(i)]
                  : (sbf ? float_key(get_score(src, i, 1)) >> 16 : float_key(src[i]));
  };
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (threadIdx.x == 0) {
    mm[0] = 0xFFFFFFFFu;
    mm[1] = 0u;
  }
  __syncthreads();
  if (lane == 0) {
    atomicMin(&mm[0], kmin);
    atomicMax(&mm[1], kmax);
  }
  cluster_sync_all();                           // every CTA's (min, max) and rank 0's zeroed totals
  if (threadIdx.x < 32) {
    // lanes 0..CL-1 read one CTA's (min, max) each
    uint32_t gmin = 0xFFFFFFFFu, gmax = 0u;
    if ((int)threadIdx.x < CL) {
      const uint32_t* rm = cluster.map_shared_rank(mm, (unsigned)threadIdx.x);
      gmin = rm[0];
      gmax = rm[1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gmin = min(gmin, __shfl_xor_sync(0xffffffffu, gmin, o));
      gmax = max(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
    }
    if (threadIdx.x == 0) {
      const int common = (gmin == gmax) ? 32 : __clz(gmin ^ gmax);
      sh_mask = high_mask(common);
      sh_prefix = gmin & sh_mask;
      sh_bits = 32 - common;                    // key bits still to resolve
      sh_rem = kk;
      sh_done = 0;
    }
  }
  __syncthreads();

  const uint32_t* tot0 = cluster.map_shared_rank(tot, 0u);   // rank 0's totals
  for (int pass = 0; sh_bits > 0 && !sh_done; ++pass) {
    const int bits = sh_bits;
    const int w = bits < 8 ? bits : 8;
    const int shift = bits - w;
    const uint32_t dmask = (1u << w) - 1u;
    uint32_t* wh = whist + (threadIdx.x >> 5) * NB;
    for (int t = threadIdx.x; t < NW * NB; t += TPB) whist[t] = 0;
    __syncthreads();
    const uint32_t prefix = sh_prefix, mask = sh_mask;
    auto count = [&](uint32_t key) {
      if ((key & mask) == prefix) atomicAdd(&wh[(key >> shift) & dmask], 1u);
    };
    if (cached) {
      // 8 independent shared loads per step
      int i0 = 0;
      for (; i0 + 8 * TPB <= len; i0 += 8 * TPB) {
        uint32_t k8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) k8[u] = keys[padi(i0 + u * TPB + threadIdx.x)];
#pragma unroll
        for (int u = 0; u < 8; ++u) count(k8[u]);
      }
      for (int i = i0 + threadIdx.x; i < len; i += TPB) count(keys[padi(i)]);
    } else {
      for (int i = threadIdx.x; i < len; i += TPB) count(key_at(i));
    }
    __syncthreads();
    // sum the warps' columns; add this CTA's non-empty bins into rank 0's totals
    if (threadIdx.x < NB) {
      uint32_t v = 0;
#pragma unroll
      for (int k = 0; k < NW; ++k) v += whist[k * NB + threadIdx.x];
      if (v) atomicAdd(const_cast<uint32_t*>(tot0) + pass * NB + threadIdx.x, v);
    }
    cluster_sync_all();                         // the pass's totals are complete
    if (threadIdx.x < NB / 4)
      reinterpret_cast<uint4*>(tl)[threadIdx.x] =
          reinterpret_cast<const uint4*>(tot0 + pass * NB)[threadIdx.x];
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns bins 255-8l-7 .. 255-8l (lane 0 the highest)
      const int b_lo = NB - 8 * (lane + 1);
      int own = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) own += (int)tl[b_lo + j];
      int x = own;                              // inclusive scan from lane 0 up
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      const int above = x - own;
      const int rem = sh_rem;
      if (above < rem && above + own >= rem) {
        int cum = above;
#pragma unroll
        for (int j = 7; j >= 0; --j) {
          const int h = (int)tl[b_lo + j];
          if (cum < rem && cum + h >= rem) {
            sh_bin = (uint32_t)(b_lo + j);
            sh_rem = rem - cum;
            sh_done = (h == rem - cum);         // the bin is taken whole
          }
          cum += h;
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      sh_prefix = prefix | (sh_bin << shift);
      sh_mask = mask | (dmask << shift);
      sh_bits = shift;
    }
    __syncthreads();
  }
  const uint32_t T = sh_prefix, M = sh_mask;
  const int need_eq = sh_rem;

  // ordered emission: thread t owns the contiguous run [r0, r1) of the slice;
  // keys are compared on the resolved bits M only
  const int per = (len + TPB - 1) / TPB;
  const int r0 = min(len, (int)threadIdx.x * per), r1 = min(len, r0 + per);
  int gt = 0, eq = 0;
  {
    int i = r0;
    if (cached)
      for (; i + 8 <= r1; i += 8) {
        uint32_t k8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) k8[u] = keys[padi(i + u)] & M;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          gt += k8[u] > T;
          eq += k8[u] == T;
        }
      }
    for (; i < r1; ++i) {
      const uint32_t key = key_at(i) & M;
      gt += key > T;
      eq += key == T;
    }
  }
  int tot_gt, tot_eq, gt_before_t, eq_before_t;
  if (len < 65536) {
    // both counts in one scan: 16 bits each, no carry while the slice is shorter
    int tot;
    const int pre = block_scan(gt | (eq << 16), wsum, tot);
    gt_before_t = pre & 0xFFFF;
    eq_before_t = pre >> 16;
    tot_gt = tot & 0xFFFF;
    tot_eq = tot >> 16;
  } else {
    gt_before_t = block_scan(gt, wsum, tot_gt);
    eq_before_t = block_scan(eq, wsum, tot_eq);
  }
  if (threadIdx.x == 0) {
    cnt[0] = tot_gt;
    cnt[1] = tot_eq;
  }
  cluster_sync_all();                           // every CTA's counts are published
  if (threadIdx.x < 32) {
    // lanes 0..rank-1 read one earlier CTA's counts each
    int g = 0, e = 0;
    if ((uint32_t)threadIdx.x < rank) {
      const int* rc = cluster.map_shared_rank(cnt, (unsigned)threadIdx.x);
      g = rc[0];
      e = rc[1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, o);
      e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    if (threadIdx.x == 0) {
      sh_before[0] = g;
      sh_before[1] = e;
    }
  }
  __syncthreads();
  const int gt_before_c = sh_before[0], eq_before_c = sh_before[1];
  // ties taken before this thread's run, and output slots before it
  int eq_rank = eq_before_c + eq_before_t;
  int pos = gt_before_c + min(eq_before_c, need_eq) + gt_before_t +
            max(0, min(eq_before_c + eq_before_t, need_eq) - min(eq_before_c, need_eq));
  auto emit = [&](int i, uint32_t key) {
    bool take = key > T;
    if (key == T) {
      take = eq_rank < need_eq;
      ++eq_rank;
    }
    if (take) out[pos++] = lo + i;
  };
  if (gt + eq > 0) {                            // runs with nothing to take write nothing
    int i = r0;
    if (cached)
      for (; i + 8 <= r1; i += 8) {
        uint32_t k8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) k8[u] = keys[padi(i + u)] & M;
#pragma unroll
        for (int u = 0; u < 8; ++u) emit(i + u, k8[u]);
      }
    for (; i < r1; ++i) emit(i, key_at(i) & M);
  }
  cluster_sync_all();                           // no CTA leaves while others read its counts
}

bool topk_cluster_supported(const TopkParams& P) { return P.n_q <= (1 << 20); }

cudaError_t launch_topk_cluster(const TopkParams& P, cudaStream_t st) {
  const size_t smem = SMEM_WORDS * sizeof(uint32_t);
  // per device: how many clusters of 1, 2, 4, 8, 16 CTAs can be resident at once
  static int max_active[64][5];
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed,
                             1) != cudaSuccess)
      cudaGetLastError();                            // 16-CTA clusters then report 0 below
    for (int k = 0; k < 5; ++k) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1u << k, 1, 1);
      cfg.blockDim = dim3(TPB, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 1u << k;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, topk_cluster_kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
      max_active[dev][k] = n;
    }
    configured[dev] = true;
  }
  // CTAs per query: the largest power of two <= 16 whose clusters for all the
  // queries are resident at once (few queries: wide clusters over long score
  // rows; many queries, as in prefill: one CTA each)
  int k = 4;
  while (k > 0 && max_active[dev][k] < P.n_q) --k;
  const int CL = 1 << k;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(P.n_q * CL), 1, 1);
  cfg.blockDim = dim3(TPB, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel, P);
}

}  // namespace v4a
