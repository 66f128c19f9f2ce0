// Projection Y = X . W (fp32 accumulation): the linear maps producing the
// compressor inputs C, Z (and, in the small fp32 layer, the queries) from raw
// tokens - "DeepSeek-V4 深读" (ricardokevins.github.io), section "CSA 与 HCA"
// (token KV and per-channel learned gating).
//
// CUDA-core tiled kernel: 64x64 output tile per CTA, K-step 16, 4x4 outputs
// per thread, operands staged through shared memory as fp32.
#include "common.cuh"
#include "kernels.h"

namespace v4a {

constexpr int kBM = 64, kBN = 64, kBK = 16;

__global__ void __launch_bounds__(256) project_simt(ProjectParams P) {
  __shared__ float xs[kBK][kBM + 4];
  __shared__ float wsm[kBK][kBN + 4];
  const int64_t m0 = (int64_t)blockIdx.y * kBM, n0 = (int64_t)blockIdx.x * kBN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < P.K; k0 += kBK) {
    for (int e = threadIdx.x; e < kBM * kBK; e += 256) {
      const int r = e / kBK, kk = e % kBK;
      const int64_t gm = m0 + r, gk = k0 + kk;
      xs[kk][r] = (gm < P.M && gk < P.K) ? load_in(P.X, P.x_dtype, gm * P.ldx + gk) : 0.f;
    }
    for (int e = threadIdx.x; e < kBK * kBN; e += 256) {
      const int kk = e / kBN, c = e % kBN;
      const int64_t gk = k0 + kk, gn = n0 + c;
      wsm[kk][c] = (gk < P.K && gn < P.N) ? load_in(P.W, P.x_dtype, gk * P.ldw + gn) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = wsm[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t gm = m0 + ty * 4 + i;
    if (gm >= P.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t gn = n0 + tx * 4 + j;
      if (gn >= P.N) continue;
      if (P.y_dtype == V4A_F32)
        reinterpret_cast<float*>(P.Y)[gm * P.ldy + gn] = acc[i][j];
      else
        reinterpret_cast<__nv_bfloat16*>(P.Y)[gm * P.ldy + gn] = __float2bfloat16_rn(acc[i][j]);
    }
  }
}

cudaError_t launch_project(const ProjectParams& P, cudaStream_t st) {
  dim3 grid((unsigned)((P.N + kBN - 1) / kBN), (unsigned)((P.M + kBM - 1) / kBM));
  project_simt<<<grid, 256, 0, st>>>(P);
  return cudaGetLastError();
}

}  // namespace v4a
