// Kernel parameter blocks and launchers of the v4attn library (internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace v4a {

// Paged compressed caches (see "Paged caches" in v4attn.h): entry e of
// sequence b at row bt[b * bps + e / epb] * epb + e % epb of a pool of
// n_blocks * epb rows; bt == nullptr: per-sequence caches.
struct PageMap {
  const int32_t* bt = nullptr;
  int32_t bps = 0;        // blocks per sequence (columns of the table)
  int32_t epb = 1;        // entries per block: 128 / m
  int64_t n_blocks = 0;   // blocks in the pool
};

#if defined(__CUDACC__)
// Pool row of entry e of sequence b, or -1 when the table holds no valid
// block for it (a table entry outside [0, n_blocks) or e past the table).
__device__ __forceinline__ int64_t page_row(const PageMap& pm, int b, int64_t e) {
  const int64_t lb = e / pm.epb;
  if (e < 0 || lb >= pm.bps) return -1;
  const int32_t pb = __ldg(pm.bt + (int64_t)b * pm.bps + lb);
  if (pb < 0 || (int64_t)pb >= pm.n_blocks) return -1;
  return (int64_t)pb * pm.epb + (e - lb * pm.epb);
}
#endif

struct CompressParams {
  int m, overlap, c;
  const void *Ca, *Za, *Cb, *Zb;
  int in_dtype;
  int64_t in_seq_stride, in_row_stride, in_rows;
  const float* bias;
  const int64_t* seq_len;
  const int64_t* entry_begin;
  int complete_only, apply_rmsnorm, apply_rope;
  int out_dtype;
  void* out;
  void* out_scale;
  int64_t out_rows;
  int d_rope;
  float theta, eps;
  // decode: the token at position new_pos[b] is read from the *_new arrays
  // (row b at new_seq_stride) instead of the input ring; seq_len / entry_begin
  // may instead be derived from new_pos (L = p + 1; entry p for m = 1, p / m
  // otherwise) when the pointers are null
  const int64_t* new_pos = nullptr;
  const void *Ca_new = nullptr, *Za_new = nullptr, *Cb_new = nullptr, *Zb_new = nullptr;
  int64_t new_seq_stride = 0;
};

// One decode step's appends (see decode_append_kernel).
struct AppendParams {
  int B, csa;
  const int64_t* pos;
  int in_dtype;                               // of x_main / tail / x_idx / itail
  const void* x_main;                         // [B][n_arr][d]
  void* tail;                                 // [B][ring][n_arr][d]
  int m, ring, n_arr, d;
  const float* bias;
  const void* x_idx;                          // CSA: [B][4][dI]
  void* itail;                                // CSA: [B][ring][4][dI]
  int dI;
  const float* ibias;
  int kv_dtype, idx_dtype, d_rope;
  float theta, eps;
  void *swa, *swa_scale;
  int64_t swa_rows;
  void *kv, *kv_scale;
  int64_t kv_rows;
  void *keys, *keys_sf;
  int64_t key_rows;
  // optional: code each sequence's bf16 query (H heads of 512 dims, RoPE at
  // pos[b]) into the tensor-core MQA's query image at qimg + b * kMqaQImageStride
  const void* Q = nullptr;
  int H = 0;
  uint8_t* qimg = nullptr;
  // paged caches: the entry's and the indexer key's rows come from the block
  // table (a bad table entry sets ST_BAD_INDEX in *status and skips the write)
  PageMap kv_pages, key_pages;
  uint32_t* status = nullptr;
};

struct IndexParams {
  int n_q, B, m, H_I, d_I, idx_dtype;
  const void* qI;
  const uint8_t* qI_sf;
  const float* w;
  const int32_t* q_seq;
  int q_base = 0;       // without q_seq, query q belongs to sequence q_base + q
  const int64_t* q_pos;
  const void* keys;
  const uint8_t* keys_sf;
  int64_t key_rows, max_vis;
  float* scores;        // [n_q][max_vis] fp32, or bf16 when score_bf16
  int64_t scores_ld;
  int score_bf16 = 0;
  uint32_t* status;
  uint32_t wait_ns = 0; // bound of the tensor-core kernel's waits (0: the default, 1 s)
  int stall = 0;        // debug: the tensor-core kernel's MMA warp waits on a barrier
                        // nothing completes, so that its bounded wait runs out
  PageMap pages;        // paged keys (tensor-core kernel): key_rows = pool rows
};

struct TopkParams {
  int n_q, m, k;
  const float* scores;  // fp32, or bf16 when score_bf16
  int64_t scores_ld, max_vis;
  int score_bf16 = 0;
  const int64_t* q_pos;
  int32_t* idx_out;
};

// Bytes per query of the tensor-core MQA's coded query image (73728 bytes of
// swizzled E4M3 / bf16 tiles + 512 bytes of per-head scales, 1024-aligned).
constexpr int64_t kMqaQImageStride = 74752;
// The tensor-core MQA's split-K partials (launches of a few queries split each
// (query, half) over several resident CTAs): at most kMqaTcMaxCtas CTAs, each
// 128 x 256 fp32 of O and 2 x 128 row statistics.
constexpr int kMqaTcMaxCtas = 160;
constexpr size_t kMqaTcPartFloats = (size_t)kMqaTcMaxCtas * 128 * 256;
constexpr size_t kMqaTcPartBytes = (kMqaTcPartFloats + (size_t)kMqaTcMaxCtas * 256) * sizeof(float);

struct MqaParams {
  int n_q, B, H, d, d_rope, n_win, m;
  float theta, scale, eps;
  const void* Q;
  int q_dtype, q_rmsnorm;
  const int32_t* q_seq;
  int q_base = 0;       // without q_seq, query q belongs to sequence q_base + q
  const int64_t* q_pos;
  int kv_dtype;
  const uint8_t* kv;
  const float* kv_scale;
  int64_t kv_rows;
  const uint8_t* swa;
  const float* swa_scale;
  int64_t swa_rows;
  const int32_t* idx;   // sparse: [n_q][n_sel]; dense: nullptr
  int n_sel;
  int64_t max_vis;
  const float* sink;
  int n_split;          // splits per query
  int split_keys;       // keys per split
  float* part_o;        // [n_q][n_split][H][d]; tensor-core path: [CTA][128][256]
  float* part_ml;       // [n_q][n_split][H][2]; tensor-core path: [CTA][2][128]
  uint32_t* grid_bar = nullptr;   // tensor-core path: [count, generation] in the workspace header
  uint8_t* qbuf;        // tensor-core path: [n_q] coded query images (kMqaQImageStride bytes)
  int q_ready = 0;      // the images in qbuf are already coded (decode: by the append kernel)
  int pair = 0;         // tensor-core path: two consecutive queries of one sequence per CTA
                        // (H <= 64: head rows 0..63 the first, 64..127 the second)
  void* out;
  int out_dtype;
  float* lse;
  uint32_t* status;
  PageMap pages;        // paged entries (tensor-core kernel): kv_rows = pool rows
};

struct ProjectParams {
  int64_t M, N, K;
  const void* X;
  int x_dtype;
  int64_t ldx;
  const void* W;
  int64_t ldw;
  void* Y;
  int y_dtype;
  int64_t ldy;
};

cudaError_t launch_compress(const CompressParams& P, int B, int n_entries, cudaStream_t st);
cudaError_t launch_decode_append(const AppendParams& A, cudaStream_t st);
cudaError_t launch_index_scores(const IndexParams& P, cudaStream_t st);
cudaError_t launch_topk(const TopkParams& P, cudaStream_t st);
cudaError_t launch_mqa_simt(const MqaParams& P, cudaStream_t st);
cudaError_t launch_mqa_combine(const MqaParams& P, cudaStream_t st);
cudaError_t launch_project(const ProjectParams& P, cudaStream_t st);

}  // namespace v4a
