// Query image of the tensor-core MQA: one query's H <= 128 head rows coded
// once into the swizzled shared-memory layout its MMAs read, so that every CTA
// of the query brings it in with one bulk copy.
//
// Method: "DeepSeek-V4 深读" (ricardokevins.github.io), section "其他稳定性细节"
// (dims 0..447 in FP8, dims 448..511 the BF16 RoPE part, RoPE applied at the
// query's position).
//
// Image layout (kMqaQImageStride bytes a query): Q nope bytes 0..383 as three
// K-major 128-byte-swizzled blocks of 128 rows, bytes 384..447 as one K-major
// 64-byte-swizzled block, the RoPE dims (bf16) as one K-major 128-byte-swizzled
// block, then the 128 per-row E4M3 scales (fp32 powers of two).  Rows >= H are
// zero.
#pragma once
#include "common.cuh"

namespace v4a {

constexpr int kQImgNope3 = 3 * 16384;                // offset of the SW64 nope block
constexpr int kQImgRope = kQImgNope3 + 8192;         // offset of the RoPE block
constexpr int kQImgTile = kQImgRope + 16384;         // offset of the row scales
constexpr int kQImgBytes = kQImgTile + 128 * 4;

// byte offset of (row, byte c) in a K-major tile of 128-byte rows, 128B swizzle
__device__ __forceinline__ int sw128(int row, int c) {
  return (row >> 3) * 1024 + (row & 7) * 128 + ((((c >> 4) ^ (row & 7)) & 7) << 4) + (c & 15);
}
// ... of 64-byte rows, 64B swizzle
__device__ __forceinline__ int sw64(int row, int c) {
  return (row >> 3) * 512 + (row & 7) * 64 + ((((c >> 4) ^ ((row & 7) >> 1)) & 3) << 4) + (c & 15);
}
// two floats -> two E4M3 codes (saturating, round to nearest even), low byte = a
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Codes head rows 16*hblk .. 16*hblk+15 of one query (bf16 rows of 512 dims,
// `Qrow0` = its head 0, H heads) at position p into `img`, after a per-head
// RMSNorm (unit weight, epsilon eps) when `rmsnorm` is set.  Threads 0..63 of
// the block work, four per head row (7 of the 28 E4M3 chunks and 2 of the 8
// RoPE chunks each), and issue all of their loads before the RoPE angles are
// computed; every thread of the block must call this (one __syncthreads).
// cs / sn: 32 floats of shared memory each.
// Image row h holds head h - row0 of Qrow0 (rows outside [row0, row0 + H) are
// zero): row0 = 64 puts a second query's heads in rows 64.. of a shared image.
__device__ __forceinline__ void qimage_code_rows(const __nv_bfloat16* Qrow0, int H, int64_t p,
                                                 float theta, uint8_t* img, int hblk,
                                                 float* cs, float* sn, bool rmsnorm = false,
                                                 float eps = 0.f, int row0 = 0) {
  const int tid = threadIdx.x;
  const bool worker = tid < 64;
  const int h = hblk * 16 + ((tid & 63) >> 2), part = tid & 3;
  const int hs = h - row0;
  const bool live = worker && hs >= 0 && hs < H;
  const uint4* src = reinterpret_cast<const uint4*>(Qrow0 + (int64_t)(live ? hs : 0) * 512);
  uint4 nope[14], rope[2];
#pragma unroll
  for (int i = 0; i < 14; ++i) nope[i] = live ? src[part * 14 + i] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
  for (int i = 0; i < 2; ++i) rope[i] = live ? src[56 + part * 2 + i] : make_uint4(0u, 0u, 0u, 0u);
  if (tid < 32) {
    float c = 1.f, sv = 0.f;
    if (p >= 0) rope_cs(p, tid, 64, theta, c, sv);
    cs[tid] = c;
    sn[tid] = sv;
  }
  // RMSNorm factor of the row (the four threads of a row are adjacent lanes)
  float inv = 1.f;
  if (rmsnorm) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint4 u = i < 14 ? nope[i] : rope[i - 14];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float a = bf16lo(w[k]), b = bf16hi(w[k]);
        ss = fmaf(a, a, fmaf(b, b, ss));
      }
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    const float den = ss / 512.f + eps;
    inv = den > 0.f ? 1.0f / sqrtf(den) : 0.f;     // an all-zero row stays zero
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 14; ++i) {
    const uint32_t w[4] = {nope[i].x, nope[i].y, nope[i].z, nope[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      amax = fmaxf(amax, fmaxf(fabsf(bf16lo(w[k]) * inv), fabsf(bf16hi(w[k]) * inv)));
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  const int se = e4m3_scale_exp(amax);
  if (worker) {
    // dims 0..447: 16 E4M3 codes per 16-byte chunk (chunks part*7 .. part*7+6)
#pragma unroll
    for (int j = 0; j < 7; ++j) {
      const uint4 a = nope[2 * j], b = nope[2 * j + 1];
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint32_t pk[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t lo = e4m3x2(scale_pow2(bf16lo(w[2 * k]) * inv, se),
                                   scale_pow2(bf16hi(w[2 * k]) * inv, se));
        const uint32_t hi = e4m3x2(scale_pow2(bf16lo(w[2 * k + 1]) * inv, se),
                                   scale_pow2(bf16hi(w[2 * k + 1]) * inv, se));
        pk[k] = lo | (hi << 16);
      }
      const int c = (part * 7 + j) * 16;
      uint8_t* dst = (c < 384) ? img + (c >> 7) * 16384 + sw128(h, c & 127)
                               : img + kQImgNope3 + sw64(h, c - 384);
      *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
  __syncthreads();                          // RoPE angles
  if (worker) {
    // dims 448..511: RoPE at the query position, kept in bf16
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int c16 = part * 2 + j;
      const uint32_t w[4] = {rope[j].x, rope[j].y, rope[j].z, rope[j].w};
      uint32_t pk[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int pr = c16 * 4 + k;
        const float x0 = bf16lo(w[k]) * inv, x1 = bf16hi(w[k]) * inv;
        const float r0 = x0 * cs[pr] - x1 * sn[pr], r1 = x0 * sn[pr] + x1 * cs[pr];
        pk[k] = (uint32_t)f32_to_bf16_bits(r0) | ((uint32_t)f32_to_bf16_bits(r1) << 16);
      }
      *reinterpret_cast<uint4*>(img + kQImgRope + sw128(h, c16 * 16)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
    if (part == 0) reinterpret_cast<float*>(img + kQImgTile)[h] = exp2i(se);
  }
}

}  // namespace v4a
