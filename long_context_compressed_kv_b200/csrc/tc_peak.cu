// Tensor-core throughput probe: the dense MMA rate of the three tcgen05 kinds
// this library's kernels use, measured on this GPU so that rooflines can be
// stated against a measured peak for each number format.
//
//   kind 0: kind::f16, bf16 x bf16 (K = 16 per instruction)
//   kind 1: kind::f8f6f4, E4M3 x E4M3 (K = 32)
//   kind 2: kind::mxf4 block-scaled, E2M1 x E2M1 with an E8M0 scale per 32
//           elements (K = 64)
//
// One CTA per SM; one thread issues n_iter x 4 back-to-back MMAs of
// M = 128 x N (N = 64, 128 or 256; fp32 accumulate in TMEM) over operands
// that stay in shared memory (zero-filled), so no memory traffic limits the
// rate.  Smaller N shows the per-instruction cost of narrow MMAs.  The
// accumulator and scale values are meaningless; only the time matters.  One
// commit at the end, a bounded wait for it, then the TMEM is released.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace v4a {

namespace {
constexpr int PM = 128, PN = 256;
constexpr int A_BYTES = PM * 128, B_BYTES = PN * 128;   // 128-byte K-major rows, 128B swizzle
}  // namespace

template <int KIND, int N>
__global__ void __launch_bounds__(128, 1) tc_peak_kernel(int n_iter, uint32_t* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* A = base;
  uint8_t* B = base + A_BYTES;
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  for (int i = threadIdx.x; i < (A_BYTES + B_BYTES) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(base)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();          // generic-proxy stores -> async-proxy (MMA) reads
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (threadIdx.x < 32) tmem_alloc(&tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  if (threadIdx.x == 0) {
    const uint64_t bits = smem_desc_bits(16, 1024, 2);    // K-major, 128B swizzle, 8-row groups
    const uint64_t da = smem_desc(A, bits), db = smem_desc(B, bits);
    const uint32_t id = KIND == 0 ? idesc_f(1, 1, PM, N, false, false)
                      : KIND == 1 ? idesc_f(0, 0, PM, N, false, false)
                                  : idesc_mxf4(PM, N, 0, 0);
    for (int it = 0; it < n_iter; ++it) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {          // 32 bytes of K per instruction
        const uint32_t acc = (it | k) != 0;
        if (KIND == 2)
          mma_mxf4(tmem, da + 2 * k, db + 2 * k, id, tmem + 256, tmem + 264, acc);
        else if (KIND == 1)
          mma_f8f6f4(tmem, da + 2 * k, db + 2 * k, id, acc);
        else
          mma_f16(tmem, da + 2 * k, db + 2 * k, id, acc);
      }
    }
    tc_commit(&bar);
    if (!mbar_wait(&bar, 0)) flag(status, ST_TIMEOUT);   // time bound only
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int KIND, int N>
static cudaError_t launch_one(int n_iter, uint32_t* status, size_t smem, int sms, cudaStream_t st,
                              int dev) {
  static unsigned long long configured = 0;
  if (dev < 64 && !(configured & (1ull << dev))) {
    const cudaError_t e = cudaFuncSetAttribute(tc_peak_kernel<KIND, N>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
    if (e != cudaSuccess) return e;
    configured |= 1ull << dev;
  }
  tc_peak_kernel<KIND, N><<<sms, 128, smem, st>>>(n_iter, status);
  return cudaGetLastError();
}

template <int KIND>
static cudaError_t launch_kind(int n, int n_iter, uint32_t* status, size_t smem, int sms,
                               cudaStream_t st, int dev) {
  switch (n) {
    case 64: return launch_one<KIND, 64>(n_iter, status, smem, sms, st, dev);
    case 128: return launch_one<KIND, 128>(n_iter, status, smem, sms, st, dev);
    case 256: return launch_one<KIND, 256>(n_iter, status, smem, sms, st, dev);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_tc_peak(int kind, int n, int n_iter, uint32_t* status, cudaStream_t st) {
  // more shared memory than two CTAs can share, so that every CTA has an SM
  // (and its tensor memory) to itself
  const size_t smem = 120 * 1024;
  static_assert(A_BYTES + B_BYTES + 1024 <= 120 * 1024, "operands fit");
  int dev = 0;
  cudaGetDevice(&dev);
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  switch (kind) {
    case 0: return launch_kind<0>(n, n_iter, status, smem, sms, st, dev);
    case 1: return launch_kind<1>(n, n_iter, status, smem, sms, st, dev);
    case 2: return launch_kind<2>(n, n_iter, status, smem, sms, st, dev);
  }
  return cudaErrorInvalidValue;
}

}  // namespace v4a

extern "C" v4attn_status v4attn_tc_peak_probe(int32_t kind, int32_t n_cols, int32_t n_iter,
                                              int32_t* n_ctas, double* flops, void* ws,
                                              cudaStream_t stream) {
  if (kind < 0 || kind > 2 || n_iter < 1 || n_iter > (1 << 24)) return V4A_ERR_INVALID_ARG;
  if (n_cols != 64 && n_cols != 128 && n_cols != 256) return V4A_ERR_INVALID_ARG;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return V4A_ERR_CUDA;
  const double kk = kind == 0 ? 16.0 : (kind == 1 ? 32.0 : 64.0);
  if (n_ctas) *n_ctas = sms;
  if (flops) *flops = 2.0 * v4a::PM * n_cols * kk * 4.0 * n_iter * sms;
  return v4a::launch_tc_peak(kind, n_cols, n_iter, reinterpret_cast<uint32_t*>(ws), stream) ==
                 cudaSuccess
             ? V4A_OK
             : V4A_ERR_CUDA;
}
