// Projection Y = X . W on the 5th-generation tensor cores (tcgen05 kind::f16,
// bf16 x bf16, fp32 accumulate): the linear maps that produce the compressor
// inputs C, Z of every token from its raw activations ("DeepSeek-V4 深读"
// (ricardokevins.github.io), section "CSA 与 HCA": per-channel learned gating
// of token KV), in the prefill form where they are a dense GEMM.
//
// Persistent kernel, one CTA per SM, 128 x 256 output tiles walked row-major
// (consecutive CTAs share the same 128-row stripe of X, and all of W stays in
// L2).  Roles: warp 0 loads (TMA: an X box of 128 rows x 64 k, K-major with a
// 128-byte swizzle; four W boxes of 64 k-rows x 64 columns, N-major with a
// 128-byte swizzle), warp 1 issues the MMAs (M = 128, N = 256, K = 16, four
// per 64-wide k step; X is the K-major A operand, W the N-major B operand),
// warps 2..5 drain the accumulator (TMEM lane quadrant = warp % 4, one output
// row per thread) into Y.  A 4-stage shared-memory ring (48 KB a stage) feeds
// the MMAs; two 256-column TMEM accumulators let the epilogue of one tile run
// under the main loop of the next.  Out-of-range rows, columns and k are read
// as zero by TMA and never stored.  Every wait is bounded; a wait that runs
// out stops all roles (through a shared abort word) and the CTA returns.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "tc_kernels.h"

namespace v4a {

namespace {
constexpr int BM = 128, BN = 256, BK = 64;
constexpr int PSTAGES = 4;
constexpr int A_STAGE = BM * BK * 2;            // 16 KB
constexpr int B_STAGE = BK * BN * 2;            // 32 KB: four [64 k-rows x 128 B] blocks
constexpr int PTHREADS = 192;

struct PSmem {
  alignas(1024) uint8_t a[PSTAGES][A_STAGE];
  alignas(1024) uint8_t b[PSTAGES][B_STAGE];
  uint64_t full[PSTAGES], empty[PSTAGES], accfull[2], accempty[2], done;
  uint32_t tmem_base;
  uint32_t abort_word;
};
}  // namespace

__global__ void __launch_bounds__(PTHREADS, 1)
    project_tc_kernel(ProjectParams P, const __grid_constant__ CUtensorMap tm_x,
                      const __grid_constant__ CUtensorMap tm_w) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  PSmem& s = *reinterpret_cast<PSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_mt = (int)((P.M + BM - 1) / BM), n_nt = (int)((P.N + BN - 1) / BN);
  const int tiles = n_mt * n_nt;
  const int k_iters = (int)((P.K + BK - 1) / BK);
  uint32_t* abortw = &s.abort_word;
  if (threadIdx.x == 0) {
    s.abort_word = 0;
    for (int i = 0; i < PSTAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.accfull[i], 1);
      mbar_init(&s.accempty[i], 4);
    }
    mbar_init(&s.done, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&s.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      prefetch_tmap(&tm_x);
      prefetch_tmap(&tm_w);
    }
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
      const int m0 = (t / n_nt) * BM, n0 = (t % n_nt) * BN;
      for (int k = 0; k < k_iters; ++k, ++it) {
        const int st = it % PSTAGES, u = it / PSTAGES;
        if (u >= 1 && !mbar_wait_warp(&s.empty[st], (u - 1) & 1, abortw, 0)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&s.full[st], A_STAGE + B_STAGE);
          tma_load_2d(s.a[st], &tm_x, &s.full[st], k * BK, m0);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tma_load_2d(s.b[st] + j * (B_STAGE / 4), &tm_w, &s.full[st], n0 + 64 * j, k * BK);
        }
        __syncwarp();
      }
    }
    // no load may still be landing when the CTA exits
    if (lane == 0)
      for (int k = 0; k < PSTAGES && k < it; ++k) {
        const int i2 = it - 1 - k;
        mbar_wait(&s.full[i2 % PSTAGES], (i2 / PSTAGES) & 1);   // time bound only
      }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    const uint64_t a_bits = smem_desc_bits(16, 1024, 2);          // K-major, 128B swizzle
    const uint64_t b_bits = smem_desc_bits(B_STAGE / 4, 1024, 2); // N-major, 128B swizzle
    const uint32_t id = idesc_f(1, 1, BM, BN, false, true);       // bf16 x bf16 -> f32
    int it = 0, lt = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++lt) {
      const int acc = lt & 1, ua = lt >> 1;
      if (ua >= 1 && !mbar_wait_warp(&s.accempty[acc], (ua - 1) & 1, abortw, 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem + acc * BN;
      for (int k = 0; k < k_iters; ++k, ++it) {
        const int st = it % PSTAGES;
        if (!mbar_wait_warp(&s.full[st], (it / PSTAGES) & 1, abortw, 2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint64_t da = smem_desc(s.a[st], a_bits), db = smem_desc(s.b[st], b_bits);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)   // A: +32 B per 16 k; B: +16 k-rows x 128 B
            mma_f16(d, da + 2 * kk, db + 128 * kk, id, (k | kk) != 0);
          tc_commit(&s.empty[st]);
          if (k == k_iters - 1) tc_commit(&s.accfull[acc]);
        }
        __syncwarp();
      }
    }
    if (lane == 0) {
      tc_commit(&s.done);
      mbar_wait(&s.done, 0);                      // time bound only
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int r = quad * 32 + lane;               // output row of this thread within a tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const bool f32_out = P.y_dtype == V4A_F32;
    const size_t esz = f32_out ? 4 : 2;
    int lt = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++lt) {
      const int acc = lt & 1;
      if (!mbar_wait_warp(&s.accfull[acc], (lt >> 1) & 1, abortw, 3)) break;
      tc_fence_after();
      const int64_t m = (int64_t)(t / n_nt) * BM + r;
      const int64_t n0 = (int64_t)(t % n_nt) * BN;
      uint8_t* yrow = reinterpret_cast<uint8_t*>(P.Y) + (m * P.ldy + n0) * (int64_t)esz;
      const bool row_in = m < P.M;
      // vector stores when the whole 32-column chunk is in range and aligned
      const bool vec_ok = ((reinterpret_cast<uintptr_t>(yrow) | (uintptr_t)(P.ldy * esz)) & 15) == 0;
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t v[128];
#pragma unroll
        for (int c = 0; c < 128; c += 32)
          tmem_ld32_nowait(tmem + lane_off + acc * BN + half * 128 + c, v + c);
        tmem_ld_wait();
        if (half == 1) {                          // accumulator fully read: release it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.accempty[acc]);
        }
        if (!row_in) continue;
#pragma unroll
        for (int c = 0; c < 128; c += 32) {
          const int64_t col = half * 128 + c;
          if (n0 + col + 32 <= P.N && vec_ok) {
            if (f32_out) {
              uint4* dst = reinterpret_cast<uint4*>(yrow + col * 4);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                dst[q] = make_uint4(v[c + 4 * q], v[c + 4 * q + 1], v[c + 4 * q + 2], v[c + 4 * q + 3]);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(yrow + col * 2);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  w4[e] = (uint32_t)f32_to_bf16_bits(__uint_as_float(v[c + 8 * q + 2 * e])) |
                          ((uint32_t)f32_to_bf16_bits(__uint_as_float(v[c + 8 * q + 2 * e + 1])) << 16);
                dst[q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
              }
            }
          } else {
            for (int e = 0; e < 32; ++e) {
              if (n0 + col + e >= P.N) break;
              const float x = __uint_as_float(v[c + e]);
              if (f32_out)
                reinterpret_cast<float*>(yrow)[col + e] = x;
              else
                reinterpret_cast<uint16_t*>(yrow)[col + e] = f32_to_bf16_bits(x);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- host side

int project_tc_check(const ProjectParams& P) {
  if (P.x_dtype != V4A_BF16 || P.K < 1 || P.M < 1 || P.N < 1) return 2;
  if (P.M > (1ll << 31) || P.N > (1ll << 31) || P.K > (1ll << 31)) return 2;
  // TMA: 16-byte aligned bases and row strides
  if (((uintptr_t)P.X & 15) || ((uintptr_t)P.W & 15) || ((P.ldx * 2) & 15) || ((P.ldw * 2) & 15))
    return 1;
  return tensor_map_encoder() != nullptr ? 0 : 2;
}

cudaError_t launch_project_tc(const ProjectParams& P, cudaStream_t st) {
  auto enc = reinterpret_cast<CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                           const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                           const cuuint32_t*, CUtensorMapInterleave,
                                           CUtensorMapSwizzle, CUtensorMapL2promotion,
                                           CUtensorMapFloatOOBfill)>(tensor_map_encoder());
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tx, tw;
  {
    cuuint64_t dims[2] = {(cuuint64_t)P.K, (cuuint64_t)P.M};
    cuuint64_t strides[1] = {(cuuint64_t)P.ldx * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)BM};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(P.X), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)P.N, (cuuint64_t)P.K};
    cuuint64_t strides[1] = {(cuuint64_t)P.ldw * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)BK};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(P.W), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t smem = sizeof(PSmem) + 1024;
  static unsigned long long configured = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !(configured & (1ull << dev))) {
    const cudaError_t e = cudaFuncSetAttribute(project_tc_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
    if (e != cudaSuccess) return e;
    configured |= 1ull << dev;
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = ((P.M + BM - 1) / BM) * ((P.N + BN - 1) / BN);
  const int grid = (int)(tiles < sms ? tiles : sms);
  project_tc_kernel<<<grid, PTHREADS, smem, st>>>(P, tx, tw);
  return cudaGetLastError();
}

}  // namespace v4a
