// Lightning-indexer scores (CUDA-core path) and per-query top-k selection.
//
// Method: "DeepSeek-V4 深读" (ricardokevins.github.io), section
// "CSA：4× 压缩之后再 top-k": 64 indexer heads score every compressed key
// through ReLU(q_h . k), the heads summed with input-dependent weights; Flash
// keeps 512 entries, Pro 1024 (model-spec table).  Section "FP4 QAT、可恢复
// rollout 与百万 Token RL": the indexer QK path is MXFP4.
//
// Scores are kept in fp32 (the selection tolerance is 1e-3 relative, below a
// bf16 step).  The selection is an exact radix select on the order-preserving
// uint32 image of the score followed by one ordered pass that emits, in
// ascending index order, every key above the threshold and the lowest-index
// keys equal to it.
#include "common.cuh"
#include "kernels.h"

namespace v4a {

__device__ __forceinline__ float mx_elem(const uint8_t* packed, const uint8_t* sf, int dim) {
  const uint8_t byte = packed[dim >> 1];
  const uint8_t code = (dim & 1) ? (byte >> 4) : (byte & 0xF);
  return e2m1_to_f32(code) * ldexpf(1.0f, (int)sf[dim >> 5] - 127);
}

// One thread per key; the query (dequantised) and head weights sit in shared
// memory and are read as warp-wide broadcasts.
template <int DI>
__global__ void __launch_bounds__(128) index_scores_simt(IndexParams P) {
  extern __shared__ float sm[];
  float* qs = sm;
  float* ws = sm + P.H_I * DI;
  const int q = blockIdx.y;
  int b = P.q_seq ? P.q_seq[q] : P.q_base + q;
  const int64_t p = P.q_pos[q];
  int64_t nv = (p + 1) / P.m;
  if (b < 0 || b >= P.B) {
    if (threadIdx.x == 0 && blockIdx.x == 0) flag(P.status, ST_BAD_SEQ);
    nv = 0;
    b = 0;
  }
  if (nv > P.key_rows || nv > P.max_vis) {
    if (threadIdx.x == 0 && blockIdx.x == 0) flag(P.status, ST_BAD_POSITION);
    nv = min(P.key_rows, P.max_vis);
  }
  for (int e = threadIdx.x; e < P.H_I * DI; e += blockDim.x) {
    const int h = e / DI, dd = e % DI;
    float v;
    if (P.idx_dtype == V4A_MXFP4) {
      const uint8_t* qp = reinterpret_cast<const uint8_t*>(P.qI) + ((int64_t)q * P.H_I + h) * (DI / 2);
      v = mx_elem(qp, P.qI_sf + ((int64_t)q * P.H_I + h) * (DI / 32), dd);
    } else {
      v = reinterpret_cast<const float*>(P.qI)[((int64_t)q * P.H_I + h) * DI + dd];
    }
    qs[e] = v;
  }
  for (int h = threadIdx.x; h < P.H_I; h += blockDim.x) ws[h] = P.w[(int64_t)q * P.H_I + h];
  __syncthreads();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= P.max_vis) return;
  float score = -INFINITY;
  if (i < nv) {
    float k[DI];
    if (P.idx_dtype == V4A_MXFP4) {
      const int64_t row = (int64_t)b * P.key_rows + i;
      const uint8_t* kp = reinterpret_cast<const uint8_t*>(P.keys) + row * (DI / 2);
      const uint8_t* ks = P.keys_sf + row * (DI / 32);
#pragma unroll
      for (int dd = 0; dd < DI; ++dd) k[dd] = mx_elem(kp, ks, dd);
    } else {
      const float* kp = reinterpret_cast<const float*>(P.keys) + ((int64_t)b * P.key_rows + i) * DI;
#pragma unroll
      for (int dd = 0; dd < DI; ++dd) k[dd] = kp[dd];
    }
    score = 0.f;
    for (int h = 0; h < P.H_I; ++h) {
      const float* qh = qs + h * DI;
      float acc = 0.f;
#pragma unroll
      for (int dd = 0; dd < DI; ++dd) acc = fmaf(qh[dd], k[dd], acc);
      score = fmaf(ws[h], fmaxf(acc, 0.f), score);
    }
  }
  put_score(P.scores, (int64_t)q * P.scores_ld + i, score, P.score_bf16);
}

cudaError_t launch_index_scores(const IndexParams& P, cudaStream_t st) {
  dim3 grid((unsigned)((P.max_vis + 127) / 128), P.n_q);
  const size_t smem = (size_t)(P.H_I * P.d_I + P.H_I) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaSuccess;
    switch (P.d_I) {
      case 64: e = cudaFuncSetAttribute(index_scores_simt<64>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); break;
      case 128: e = cudaFuncSetAttribute(index_scores_simt<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); break;
      default: break;
    }
    if (e != cudaSuccess) return e;
  }
  switch (P.d_I) {
    case 32: index_scores_simt<32><<<grid, 128, smem, st>>>(P); break;
    case 64: index_scores_simt<64><<<grid, 128, smem, st>>>(P); break;
    case 128: index_scores_simt<128><<<grid, 128, smem, st>>>(P); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- top-k
constexpr int kTopkThreads = 1024;

// Exclusive block scan of 0/1 flags; returns the prefix and writes the total.
__device__ __forceinline__ int block_excl_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) warp_tot[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int t = (lane < (int)(blockDim.x >> 5)) ? warp_tot[lane] : 0;
    int s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_tot[lane] = s - t;       // exclusive prefix of warp totals
    if (lane == 31) warp_tot[32] = s;
  }
  __syncthreads();
  total = warp_tot[32];
  return warp_tot[wid] + x - v;
}

__global__ void __launch_bounds__(kTopkThreads) topk_select(TopkParams P) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sh_prefix, sh_mask;
  __shared__ int sh_remaining;
  __shared__ int warp_tot[33];
  const int q = blockIdx.x;
  const int64_t p = P.q_pos[q];
  int64_t nv64 = (p + 1) / P.m;
  if (nv64 > P.max_vis) nv64 = P.max_vis;
  const int nv = (int)nv64;
  const int kk = min(P.k, nv);
  const float* s = P.scores + (int64_t)q * P.scores_ld;
  int32_t* out = P.idx_out + (int64_t)q * P.k;
  for (int j = kk + threadIdx.x; j < P.k; j += blockDim.x) out[j] = -1;
  if (kk == 0) return;
  if (threadIdx.x == 0) {
    sh_prefix = 0;
    sh_mask = 0;
    sh_remaining = kk;
  }
  __syncthreads();
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int t = threadIdx.x; t < 256; t += blockDim.x) hist[t] = 0;
    __syncthreads();
    const uint32_t prefix = sh_prefix, mask = sh_mask;
    for (int i = threadIdx.x; i < nv; i += blockDim.x) {
      const uint32_t key = float_key(get_score(s, i, P.score_bf16));
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int rem = sh_remaining;
      int cum = 0;
      int sel = 0;
      for (int bin = 255; bin >= 0; --bin) {
        const int h = (int)hist[bin];
        if (cum + h >= rem) {
          sel = bin;
          break;
        }
        cum += h;
      }
      sh_remaining = rem - cum;
      sh_prefix = prefix | ((uint32_t)sel << shift);
      sh_mask = mask | (255u << shift);
    }
    __syncthreads();
  }
  const uint32_t T = sh_prefix;
  const int need_eq = sh_remaining;
  int base_sel = 0, base_eq = 0;
  for (int c0 = 0; c0 < nv; c0 += blockDim.x) {
    const int i = c0 + threadIdx.x;
    const uint32_t key = (i < nv) ? float_key(get_score(s, i, P.score_bf16)) : 0u;
    const int gt = (i < nv) && key > T;
    const int eq = (i < nv) && key == T;
    int tot_eq, tot_sel;
    const int eq_rank = base_eq + block_excl_scan(eq, warp_tot, tot_eq);
    const int take = gt || (eq && eq_rank < need_eq);
    const int pos = base_sel + block_excl_scan(take, warp_tot, tot_sel);
    if (take) out[pos] = i;
    base_eq += tot_eq;
    base_sel += tot_sel;
  }
}

cudaError_t launch_topk(const TopkParams& P, cudaStream_t st) {
  topk_select<<<P.n_q, kTopkThreads, 0, st>>>(P);
  return cudaGetLastError();
}

}  // namespace v4a
