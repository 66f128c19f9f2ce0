// Shared device helpers of the v4attn CUDA library (sm_100a).
//
// Number formats (OCP OFP8 rev 1.0 E4M3; OCP MX v1.0 E2M1 + E8M0; bf16) are
// produced with CUDA's conversion intrinsics (cuda_fp8.h, cuda_fp4.h,
// cuda_bf16.h); the scale rules are the integer exponent arithmetic below.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_fp4.h>
#include <stdint.h>

#include "../../include/v4attn.h"

namespace v4a {

// ---------------------------------------------------------------- status word
// Bits set (atomicOr) by kernels in the first word of the workspace.
enum : uint32_t {
  ST_BAD_POSITION = 1u << 0,   // a position / visible count exceeds a cache
  ST_BAD_INDEX = 1u << 1,      // a selected index is outside the visible range
  ST_BAD_SEQ = 1u << 2,        // a query's sequence index is out of range
  ST_TIMEOUT = 1u << 8,        // a bounded wait ran out
};

struct WsHeader {
  uint32_t status;
  // the tensor-core MQA's grid barrier (arrivals, generation): zero after
  // workspace init, the count back at zero after every completed barrier
  uint32_t bar_count, bar_gen;
  uint32_t pad[61];
};
static_assert(sizeof(WsHeader) == 256, "workspace header");

__device__ __forceinline__ void flag(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

// ---------------------------------------------------------------- conversions
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  return (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
  return __half2float(*reinterpret_cast<__half*>(&h));
}
// E2M1 code (low nibble) of x; |x| is clamped to 6 first (saturation).
__device__ __forceinline__ uint8_t f32_to_e2m1(float x) {
  x = fminf(fmaxf(x, -6.0f), 6.0f);
  return (uint8_t)(__nv_cvt_float_to_fp4(x, __NV_E2M1, cudaRoundNearest) & 0xF);
}
__device__ __forceinline__ float e2m1_to_f32(uint8_t c) {
  const float mag[8] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f};
  float v = mag[c & 7];
  return (c & 8) ? -v : v;
}
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}
// element i of a score row held as fp32, or as bf16 (round to nearest even)
__device__ __forceinline__ void put_score(float* row, int64_t i, float v, int bf16) {
  if (bf16)
    reinterpret_cast<uint16_t*>(row)[i] = f32_to_bf16_bits(v);
  else
    row[i] = v;
}
__device__ __forceinline__ float get_score(const float* row, int64_t i, int bf16) {
  return bf16 ? __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(row)[i] << 16) : row[i];
}
__device__ __forceinline__ float exp2i(int e) {   // 2^e for e in the normal range
  return __int_as_float((e + 127) << 23);
}

// Exponent e of the smallest power of two 2^e with amax / 2^e <= 448
// (0 when amax == 0): amax = f * 2^E, f in [0.5, 1); 448 = 0.875 * 2^9.
__device__ __forceinline__ int e4m3_scale_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  int E;
  float f = frexpf(amax, &E);
  return (f <= 0.875f) ? (E - 9) : (E - 8);
}
// MX shared exponent X = floor(log2 amax) - 2 clamped to [-127, 127]; -127 for 0.
__device__ __forceinline__ int mx_scale_exp(float amax) {
  if (!(amax > 0.f)) return -127;
  int E;
  frexpf(amax, &E);
  int X = (E - 1) - 2;
  return X < -127 ? -127 : (X > 127 ? 127 : X);
}
// x * 2^-e exactly for any e in [-254, 254] (two steps avoid overflow of the factor).
__device__ __forceinline__ float scale_pow2(float x, int e) {
  int e1 = -e / 2, e2 = -e - e1;
  return x * exp2i(e1) * exp2i(e2);
}

// ---------------------------------------------------------------- RoPE
// Angle (cos, sin) of pair k at position pos, a = pos * theta^(-2k/d_rope),
// computed in double so that positions up to 2^20 and beyond keep full
// accuracy.  The frequency is exp2(-(2k/d_rope) * log2(theta)); the angle
// (up to ~2^31 rad) is first brought into [-pi, pi] by Cody-Waite reduction
// with 2*pi split into two doubles (W. J. Cody and W. Waite, "Software Manual
// for the Elementary Functions", 1980), so that sincos always sees a small
// argument.  n < 2^31 and the product n * 2pi_hi is exact in the fma, so the
// reduced angle is accurate to about 2^-52 absolute.
__device__ __forceinline__ void rope_cs(int64_t pos, int k, int d_rope, float theta, float& c,
                                        float& s) {
  constexpr double kTwoPiHi = 6.283185307179586232;       // 2*pi rounded to double
  constexpr double kTwoPiLo = 2.4492935982947064e-16;     // 2*pi - kTwoPiHi
  constexpr double kInvTwoPi = 0.15915494309189533577;
  const double w = exp2(-(2.0 * k / (double)d_rope) * log2((double)theta));
  const double a = (double)pos * w;
  const double n = rint(a * kInvTwoPi);
  double r = fma(-n, kTwoPiHi, a);
  r = fma(-n, kTwoPiLo, r);
  double sd, cd;
  sincos(r, &sd, &cd);
  c = (float)cd;
  s = (float)sd;
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// Block-wide sum / max; `red` must hold >= 32 floats; all threads get the result.
__device__ __forceinline__ float block_sum(float v, float* red) {
  int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = (threadIdx.x < nw) ? red[threadIdx.x] : 0.f;
  if (wid == 0) t = warp_sum(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  return red[0];
}
__device__ __forceinline__ float block_max(float v, float* red) {
  int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = (threadIdx.x < nw) ? red[threadIdx.x] : -INFINITY;
  if (wid == 0) t = warp_max(t);
  if (threadIdx.x == 0) red[0] = t;
  __syncthreads();
  return red[0];
}

// Order-preserving map of a float to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- entry rows
// Bytes of one stored row.
__host__ __device__ __forceinline__ int64_t row_bytes(int dtype, int c, int d_rope) {
  if (dtype == V4A_F32) return 4 * (int64_t)c;
  if (dtype == V4A_E4M3_BF16ROPE) return (int64_t)(c - d_rope) + 2 * (int64_t)d_rope;
  if (dtype == V4A_MXFP4) return (int64_t)c / 2;
  return 0;
}

// Load dims [d0, d0+n) of a stored KV row as floats (scale applied).
__device__ __forceinline__ float kv_elem(const uint8_t* row, int dtype, float scale, int dim, int d,
                                         int d_rope) {
  if (dtype == V4A_F32) return reinterpret_cast<const float*>(row)[dim];
  int dn = d - d_rope;
  if (dim < dn) return e4m3_to_f32(row[dim]) * scale;
  return bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(row + dn)[dim - dn]);
}

__device__ __forceinline__ float load_in(const void* p, int dtype, int64_t i) {
  if (dtype == V4A_F32) return reinterpret_cast<const float*>(p)[i];
  return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}

// ---------------------------------------------------------------- split policy
// Fixed key-chunk length of the split-K MQA: split boundaries depend only on
// the key count, never on the batch or the SM count (batch invariance).
constexpr int kSimtSplitKeys = 128;

}  // namespace v4a
