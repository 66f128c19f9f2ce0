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
// One CTA computes one entry of one sequence; thread k owns the channel pair
// (2k, 2k+1), which is also a RoPE pair.  The softmax over the window is an
// online (running-max) softmax per channel, so the window is read once; rows
// are read coalesced (consecutive threads, consecutive channels).  This step
// moves 2-4 x c values per token and is HBM / latency bound.
#include "common.cuh"
#include "kernels.h"

namespace v4a {

__device__ void compress_entry(const CompressParams& P, int b, int64_t i, float* red) {
  const int64_t L = P.seq_len[b];
  const int m = P.m;
  const int c = P.c;
  // uniform early exits (whole CTA)
  if (i < 0 || (int64_t)m * i >= L) return;
  if (P.complete_only && (int64_t)m * (i + 1) > L) return;

  const int k = threadIdx.x;
  const int c0 = 2 * k;
  const bool active = c0 < c;
  const int R = P.overlap ? 2 * m : m;
  const int64_t jbase = P.overlap ? (int64_t)m * (i - 1) : (int64_t)m * i;
  const int64_t seq_off = (int64_t)b * P.in_seq_stride;

  float mx0 = -INFINITY, mx1 = -INFINITY, s0 = 0.f, s1 = 0.f, a0 = 0.f, a1 = 0.f;
  if (active) {
    for (int r = 0; r < R; ++r) {
      const int64_t j = jbase + r;
      if (j < 0 || j >= L) continue;
      const bool br_a = !P.overlap || r >= m;
      const void* Cp = br_a ? P.Ca : P.Cb;
      const void* Zp = br_a ? P.Za : P.Zb;
      const int64_t off = seq_off + (j % P.in_rows) * P.in_row_stride + c0;
      const float v0 = load_in(Cp, P.in_dtype, off);
      const float v1 = load_in(Cp, P.in_dtype, off + 1);
      float z0 = Zp ? load_in(Zp, P.in_dtype, off) : 0.f;
      float z1 = Zp ? load_in(Zp, P.in_dtype, off + 1) : 0.f;
      if (P.bias) {
        z0 += P.bias[(int64_t)r * c + c0];
        z1 += P.bias[(int64_t)r * c + c0 + 1];
      }
      // running-max softmax accumulation (channel 0 of the pair)
      if (z0 > mx0) {
        const float al = __expf(mx0 - z0);
        a0 = a0 * al + v0;
        s0 = s0 * al + 1.f;
        mx0 = z0;
      } else {
        const float e = __expf(z0 - mx0);
        a0 += e * v0;
        s0 += e;
      }
      if (z1 > mx1) {
        const float al = __expf(mx1 - z1);
        a1 = a1 * al + v1;
        s1 = s1 * al + 1.f;
        mx1 = z1;
      } else {
        const float e = __expf(z1 - mx1);
        a1 += e * v1;
        s1 += e;
      }
    }
  }
  float e0 = active ? a0 / s0 : 0.f;
  float e1 = active ? a1 / s1 : 0.f;

  if (P.apply_rmsnorm) {
    const float ss = block_sum(e0 * e0 + e1 * e1, red);
    const float inv = 1.0f / sqrtf(ss / (float)c + P.eps);
    e0 *= inv;
    e1 *= inv;
  }
  if (P.apply_rope && active && c0 >= c - P.d_rope) {
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
    if (active) reinterpret_cast<float2*>(out)[k] = make_float2(e0, e1);
  } else if (P.out_dtype == V4A_E4M3_BF16ROPE) {
    const int dn = c - P.d_rope;
    const float am = (active && c0 < dn) ? fmaxf(fabsf(e0), fabsf(e1)) : 0.f;
    const float amax = block_max(am, red);
    const int se = e4m3_scale_exp(amax);
    if (active) {
      if (c0 < dn) {
        const uint16_t pr = (uint16_t)f32_to_e4m3(scale_pow2(e0, se)) |
                            ((uint16_t)f32_to_e4m3(scale_pow2(e1, se)) << 8);
        reinterpret_cast<uint16_t*>(out)[k] = pr;
      } else {
        const uint32_t pr = (uint32_t)f32_to_bf16_bits(e0) | ((uint32_t)f32_to_bf16_bits(e1) << 16);
        reinterpret_cast<uint32_t*>(out + dn)[(c0 - dn) / 2] = pr;
      }
    }
    if (threadIdx.x == 0)
      reinterpret_cast<float*>(P.out_scale)[(int64_t)b * P.out_rows + row] = exp2i(se);
  } else {  // V4A_MXFP4: 16 threads (32 channels) per scale block
    float am = active ? fmaxf(fabsf(e0), fabsf(e1)) : 0.f;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    const int X = mx_scale_exp(am);
    if (active) {
      const uint8_t lo = f32_to_e2m1(scale_pow2(e0, X));
      const uint8_t hi = f32_to_e2m1(scale_pow2(e1, X));
      out[k] = (uint8_t)(lo | (hi << 4));
      if ((k & 15) == 0)
        reinterpret_cast<uint8_t*>(P.out_scale)[((int64_t)b * P.out_rows + row) * (c / 32) +
                                                c0 / 32] = (uint8_t)(X + 127);
    }
  }
}

// Grid-stride over the entries of sequence blockIdx.y.
__global__ void compress_kernel(CompressParams P, int n_entries) {
  __shared__ float red[32];
  const int b = blockIdx.y;
  const int64_t e0 = P.entry_begin[b];
  for (int e = blockIdx.x; e < n_entries; e += gridDim.x) {
    compress_entry(P, b, e0 + e, red);
    __syncthreads();
  }
}

cudaError_t launch_compress(const CompressParams& P, int B, int n_entries, cudaStream_t st) {
  int threads = ((P.c / 2 + 31) / 32) * 32;
  if (threads < 32) threads = 32;
  dim3 grid(n_entries < 8192 ? n_entries : 8192, B);
  compress_kernel<<<grid, threads, 0, st>>>(P, n_entries);
  return cudaGetLastError();
}

}  // namespace v4a
