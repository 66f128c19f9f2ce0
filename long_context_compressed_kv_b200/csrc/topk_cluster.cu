// Per-query top-k selection by one thread-block cluster per query.
//
// Method: "DeepSeek-V4 深读" (ricardokevins.github.io), section
// "CSA：4× 压缩之后再 top-k" (the k highest-scoring compressed entries per
// query; Flash k = 512, Pro k = 1024).  Ties go to the lower index and the
// selection is written in ascending index order, -1 padded.
//
// The 8 CTAs of a cluster split the query's visible scores into slices and
// keep their slice in shared memory (as order-preserving uint32 keys).  An
// exact 4-pass radix select (8 bits per pass) finds the k-th largest key T:
// every pass builds a 256-bin histogram per CTA (warp-aggregated shared
// atomics), the CTAs read each other's histograms through distributed shared
// memory after a cluster barrier, and every CTA picks the same bin.  The
// emission then needs only two block scans: each thread owns a contiguous run
// of its slice, counts the keys above T and equal to T, and the CTA- and
// cluster-level prefix sums (again through distributed shared memory) give
// every thread its first output position and its first tie rank, so indices
// are written in ascending order with no sort.  Cluster barriers are
// hardware barriers between co-scheduled CTAs that all take the same path.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace v4a {

namespace {
constexpr int CL = 8;             // CTAs per cluster = slices per query
constexpr int TPB = 512;          // threads per CTA
constexpr int CACHE = 32768;      // keys a CTA keeps in shared memory (+1/64 padding)
constexpr int PAD_CACHE = CACHE + CACHE / 64;

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
__device__ __forceinline__ uint32_t dsmem_ld(const void* local, uint32_t rank) {
  uint32_t ra, v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(ra) : "memory");
  return v;
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
}  // namespace

__global__ void __cluster_dims__(CL, 1, 1) __launch_bounds__(TPB, 1)
    topk_cluster_kernel(TopkParams P) {
  extern __shared__ uint32_t keys[];            // PAD_CACHE entries
  __shared__ uint32_t hist[2][256];
  __shared__ uint32_t tot[256];
  __shared__ int wsum[33];
  __shared__ uint32_t sh_prefix, sh_mask;
  __shared__ int sh_rem;
  __shared__ int cnt[2];                        // this CTA's (#gt, #eq), read by the cluster
  const uint32_t rank = cluster_rank();
  const int q = blockIdx.x / CL;
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
  const bool cached = len <= CACHE;
  const float* src = P.scores + (int64_t)q * P.scores_ld + lo;
  if (cached)
    for (int i = threadIdx.x; i < len; i += TPB) keys[padi(i)] = float_key(src[i]);
  auto key_at = [&](int i) -> uint32_t { return cached ? keys[padi(i)] : float_key(src[i]); };

  if (threadIdx.x == 0) {
    sh_prefix = 0;
    sh_mask = 0;
    sh_rem = kk;
  }
  const int lane = threadIdx.x & 31;
  for (int pass = 0; pass < 4; ++pass) {
    const int buf = pass & 1, shift = 24 - 8 * pass;
    for (int t = threadIdx.x; t < 256; t += TPB) hist[buf][t] = 0;
    __syncthreads();
    const uint32_t prefix = sh_prefix, mask = sh_mask;
    const int n_iter = (len + TPB - 1) / TPB;
    for (int it = 0; it < n_iter; ++it) {
      const int i = it * TPB + threadIdx.x;
      uint32_t bin = 0xFFFFFFFFu;
      if (i < len) {
        const uint32_t key = key_at(i);
        if ((key & mask) == prefix) bin = (key >> shift) & 255u;
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (bin != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&hist[buf][bin], __popc(peers));
    }
    cluster_sync_all();                         // every CTA's hist[buf] is complete
    for (int t = threadIdx.x; t < 256; t += TPB) {
      uint32_t s = 0;
      for (uint32_t r = 0; r < CL; ++r) s += dsmem_ld(&hist[buf][t], r);
      tot[t] = s;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      const int rem = sh_rem;
      int cum = 0, sel = 0;
      for (int bin = 255; bin >= 0; --bin) {
        const int h = (int)tot[bin];
        if (cum + h >= rem) {
          sel = bin;
          break;
        }
        cum += h;
      }
      sh_rem = rem - cum;
      sh_prefix = prefix | ((uint32_t)sel << shift);
      sh_mask = mask | (255u << shift);
    }
    __syncthreads();
  }
  const uint32_t T = sh_prefix;
  const int need_eq = sh_rem;

  // ordered emission: thread t owns the contiguous run [r0, r1) of the slice
  const int per = (len + TPB - 1) / TPB;
  const int r0 = min(len, (int)threadIdx.x * per), r1 = min(len, r0 + per);
  int gt = 0, eq = 0;
  for (int i = r0; i < r1; ++i) {
    const uint32_t key = key_at(i);
    gt += key > T;
    eq += key == T;
  }
  int tot_gt, tot_eq;
  const int gt_before_t = block_scan(gt, wsum, tot_gt);
  const int eq_before_t = block_scan(eq, wsum, tot_eq);
  if (threadIdx.x == 0) {
    cnt[0] = tot_gt;
    cnt[1] = tot_eq;
  }
  cluster_sync_all();                           // every CTA's counts are published
  int gt_before_c = 0, eq_before_c = 0;
  for (uint32_t r = 0; r < rank; ++r) {
    gt_before_c += (int)dsmem_ld(&cnt[0], r);
    eq_before_c += (int)dsmem_ld(&cnt[1], r);
  }
  // ties taken before this thread's run, and output slots before it
  int eq_rank = eq_before_c + eq_before_t;
  int pos = gt_before_c + min(eq_before_c, need_eq) + gt_before_t +
            max(0, min(eq_before_c + eq_before_t, need_eq) - min(eq_before_c, need_eq));
  for (int i = r0; i < r1; ++i) {
    const uint32_t key = key_at(i);
    bool take = key > T;
    if (key == T) {
      take = eq_rank < need_eq;
      ++eq_rank;
    }
    if (take) out[pos++] = lo + i;
  }
  cluster_sync_all();                           // no CTA leaves while others read its counts
}

bool topk_cluster_supported(const TopkParams& P) { return P.n_q <= (1 << 20); }

cudaError_t launch_topk_cluster(const TopkParams& P, cudaStream_t st) {
  const size_t smem = (size_t)PAD_CACHE * sizeof(uint32_t);
  static unsigned long long configured = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !(configured & (1ull << dev))) {
    cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured |= 1ull << dev;
  }
  topk_cluster_kernel<<<P.n_q * CL, TPB, smem, st>>>(P);
  return cudaGetLastError();
}

}  // namespace v4a
