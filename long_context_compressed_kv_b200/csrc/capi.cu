// C-ABI entry points of the v4attn library: argument validation, workspace
// layout, kernel selection and the decode-step orchestration.
//
// Every entry point validates its arguments on the host and returns before
// launching anything when they are wrong; device-side checks (positions past a
// cache, indices out of range) skip the access and set a bit of the status
// word at the start of the workspace, read by v4attn_device_status().
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_kernels.h"

using namespace v4a;

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Workspace: [status header | decode scratch | query images | body].  The
// query images are the tensor-core MQA's coded queries of one query chunk (none
// for other KV formats); in a decode step the append kernel writes them before
// the indexer runs, so they sit outside the body.  The body holds either the
// indexer scores of an index_topk call or the split-K partials of an MQA call;
// the two never live at the same time (stream order), so they overlap.  A
// stand-alone index_topk call, which leaves the images alone, starts its body
// at the images' offset.
size_t dec_bytes(int32_t n_q) { return align_up((size_t)n_q * 3 * sizeof(int64_t)); }
size_t qimg_off(int32_t n_q) { return align_up(sizeof(WsHeader)) + dec_bytes(n_q); }
// index_topk and the MQA calls walk their queries in chunks of kQChunk; the
// scores / split-K partials of one chunk live in the workspace body, reused
// by the next chunk in stream order.
constexpr int32_t kQChunk = 1024;
constexpr int32_t kMaxQueries = 1 << 20;   // queries per index_topk / MQA call
inline int32_t q_chunk(int32_t n_q) { return std::min(n_q, kQChunk); }
size_t index_need(int32_t n_q, int64_t max_vis) {
  return align_up((size_t)q_chunk(n_q) * (size_t)std::max<int64_t>(max_vis, 1) * sizeof(float));
}
size_t mqa_part_o_bytes(const v4attn_layer_desc* d, int32_t n_q, int n_split) {
  return align_up((size_t)n_q * n_split * d->H * d->d * sizeof(float));
}
// partials for at most n_main_max entries per query (selected or visible)
size_t mqa_part_ml_bytes(const v4attn_layer_desc* d, int32_t n_q, int n_split) {
  return align_up((size_t)n_q * n_split * d->H * 2 * sizeof(float));
}
size_t mqa_qbuf_bytes(const v4attn_layer_desc* d, int32_t n_q) {
  return d->kv_dtype == V4A_E4M3_BF16ROPE ? align_up((size_t)q_chunk(n_q) * kMqaQImageStride) : 0;
}
// body offset of MQA calls and of every call of a decode step
size_t body_mqa(const v4attn_layer_desc* d, int32_t n_q) { return qimg_off(n_q) + mqa_qbuf_bytes(d, n_q); }
size_t mqa_need(const v4attn_layer_desc* d, int32_t n_q, int64_t n_main_max) {
  // the tensor-core MQA (E4M3 caches) splits a (query, half) over several
  // CTAs only when at least two CTAs per (query, half) fit kMqaTcMaxCtas
  if (d->kv_dtype == V4A_E4M3_BF16ROPE)
    return 4 * (int64_t)q_chunk(n_q) <= kMqaTcMaxCtas ? align_up(kMqaTcPartBytes) : 0;
  const int S = mqa_num_splits(d, n_main_max);
  const int32_t c = q_chunk(n_q);
  return mqa_part_o_bytes(d, c, S) + mqa_part_ml_bytes(d, c, S);
}
size_t total_need(const v4attn_layer_desc* d, int32_t n_q, int64_t max_vis) {
  size_t body = mqa_need(d, n_q, max_vis);
  if (d->kind == V4A_CSA) {
    body = std::max(body, index_need(n_q, max_vis));
    body = std::max(body, mqa_need(d, n_q, (int64_t)d->top_k));
  }
  return body_mqa(d, n_q) + body;
}

v4attn_status check_desc(const v4attn_layer_desc* d) {
  if (!d) return V4A_ERR_INVALID_ARG;
  if (d->kind != V4A_CSA && d->kind != V4A_HCA) return V4A_ERR_INVALID_ARG;
  if (d->m < 1 || d->m > 128) return V4A_ERR_INVALID_ARG;
  if (d->n_win < 0 || d->n_win > 1024) return V4A_ERR_INVALID_ARG;
  if (d->H < 1 || d->H > 128) return V4A_ERR_UNSUPPORTED;
  if (d->d < 32 || d->d > 512 || d->d % 32) return V4A_ERR_UNSUPPORTED;
  if (d->d_rope < 0 || d->d_rope > d->d || d->d_rope % 2) return V4A_ERR_INVALID_ARG;
  if (!(d->rope_theta > 0.f)) return V4A_ERR_INVALID_ARG;
  if (!(d->rms_eps >= 0.f)) return V4A_ERR_INVALID_ARG;
  if (d->kv_dtype != V4A_F32 && d->kv_dtype != V4A_E4M3_BF16ROPE) return V4A_ERR_UNSUPPORTED;
  if (d->kv_dtype == V4A_E4M3_BF16ROPE && (d->d != 512 || d->d_rope != 64))
    return V4A_ERR_UNSUPPORTED;
  if (d->kind == V4A_CSA) {
    if (d->idx_dtype != V4A_F32 && d->idx_dtype != V4A_MXFP4) return V4A_ERR_UNSUPPORTED;
    if (d->d_I != 32 && d->d_I != 64 && d->d_I != 128) return V4A_ERR_UNSUPPORTED;
    if (d->H_I < 1 || d->H_I > 128) return V4A_ERR_UNSUPPORTED;
    if (d->top_k < 1 || d->top_k > 2048) return V4A_ERR_UNSUPPORTED;
  }
  return V4A_OK;
}

float softmax_scale(const v4attn_layer_desc* d) {
  return d->softmax_scale > 0.f ? d->softmax_scale : 1.0f / sqrtf((float)d->d);
}

// the last CUDA error an entry point met on this host thread (v4attn_last_cuda_error)
thread_local cudaError_t t_last_cuda = cudaSuccess;
v4attn_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return V4A_OK;
  t_last_cuda = e;
  return V4A_ERR_CUDA;
}

v4attn_status run_compress(const v4attn_layer_desc* d, const v4attn_compress_args* a,
                           cudaStream_t st) {
  if (!a) return V4A_ERR_INVALID_ARG;
  if (a->m < 1 || a->m > 128 || a->c < 32 || a->c > 1024 || a->c % 2 || a->B < 1)
    return V4A_ERR_INVALID_ARG;
  if (a->n_entries < 0 || a->B > 65535) return V4A_ERR_INVALID_ARG;
  if (!a->Ca || (!a->Za && a->m != 1) || !a->seq_len || !a->entry_begin || !a->out)
    return V4A_ERR_INVALID_ARG;
  if (a->overlap && (!a->Cb || !a->Zb)) return V4A_ERR_INVALID_ARG;
  if (a->in_dtype != V4A_F32 && a->in_dtype != V4A_BF16) return V4A_ERR_UNSUPPORTED;
  if (a->in_rows < 1 || a->in_row_stride < a->c || a->out_rows < 1) return V4A_ERR_INVALID_ARG;
  {
    // channel pairs are read as one 2-element load: even strides, bases aligned to 2 elements
    const uintptr_t al = a->in_dtype == V4A_F32 ? 8 : 4;
    if ((a->in_row_stride | a->in_seq_stride) & 1) return V4A_ERR_INVALID_ARG;
    for (const void* p : {a->Ca, a->Za, a->Cb, a->Zb})
      if (p && (reinterpret_cast<uintptr_t>(p) % al)) return V4A_ERR_INVALID_ARG;
    if (a->bias && (reinterpret_cast<uintptr_t>(a->bias) % 8)) return V4A_ERR_INVALID_ARG;
  }
  if (a->out_dtype == V4A_E4M3_BF16ROPE) {
    if (a->c != 512 || d->d_rope != 64 || !a->out_scale) return V4A_ERR_UNSUPPORTED;
  } else if (a->out_dtype == V4A_MXFP4) {
    if (a->c % 32 || !a->out_scale) return V4A_ERR_UNSUPPORTED;
  } else if (a->out_dtype != V4A_F32) {
    return V4A_ERR_UNSUPPORTED;
  }
  if (a->apply_rope && d->d_rope > a->c) return V4A_ERR_INVALID_ARG;
  if (a->n_entries == 0) return V4A_OK;
  CompressParams P;
  P.m = a->m;
  P.overlap = a->overlap ? 1 : 0;
  P.c = a->c;
  P.Ca = a->Ca;
  P.Za = a->Za;
  P.Cb = a->Cb;
  P.Zb = a->Zb;
  P.in_dtype = a->in_dtype;
  P.in_seq_stride = a->in_seq_stride;
  P.in_row_stride = a->in_row_stride;
  P.in_rows = a->in_rows;
  P.bias = a->bias;
  P.seq_len = a->seq_len;
  P.entry_begin = a->entry_begin;
  P.complete_only = a->complete_only;
  P.apply_rmsnorm = a->apply_rmsnorm;
  P.apply_rope = a->apply_rope;
  P.out_dtype = a->out_dtype;
  P.out = a->out;
  P.out_scale = a->out_scale;
  P.out_rows = a->out_rows;
  P.d_rope = d->d_rope;   // stored-format split; rotation only when apply_rope
  P.theta = d->rope_theta;
  P.eps = d->rms_eps;
  return cuda_status(launch_compress(P, a->B, a->n_entries, st));
}

// Checks of the tensor-core paths, taken on the host before anything is
// launched: an E4M3 / MXFP4 call either runs on its tcgen05 kernel or is
// refused (there is no slower fallback for these formats).
v4attn_status tc_status(int code) {
  return code == 0 ? V4A_OK : (code == 1 ? V4A_ERR_INVALID_ARG : V4A_ERR_UNSUPPORTED);
}

// Paged caches (see "Paged caches" in v4attn.h): a block table needs at least
// one block per sequence, 128 % m == 0 (blocks of 128 raw tokens), the
// tensor-core formats and a pool of whole blocks.
static v4attn_status check_pages(const v4attn_layer_desc* d, const int32_t* bt, int32_t bps,
                                 int64_t rows, bool tc_format) {
  if (!bt) return V4A_OK;
  if (bps < 1 || rows < 1 || (reinterpret_cast<uintptr_t>(bt) & 3)) return V4A_ERR_INVALID_ARG;
  if (128 % d->m != 0 || !tc_format) return V4A_ERR_UNSUPPORTED;
  if (rows % (128 / d->m) != 0) return V4A_ERR_INVALID_ARG;
  return V4A_OK;
}
static PageMap page_map(const v4attn_layer_desc* d, const int32_t* bt, int32_t bps, int64_t rows) {
  PageMap pm;
  if (!bt) return pm;
  pm.bt = bt;
  pm.bps = bps;
  pm.epb = 128 / d->m;
  pm.n_blocks = rows / pm.epb;
  return pm;
}
// Entries a sequence can hold: its part of the cache, or its blocks of the pool.
static int64_t seq_cap(const v4attn_layer_desc* d, const int32_t* bt, int32_t bps, int64_t rows) {
  return bt ? (int64_t)bps * (128 / d->m) : rows;
}

// `dry`: validate and return without launching.  `wait_ns` / `stall`: the
// failure-detection test hook (see v4attn_debug_index_stall).
v4attn_status run_index_topk(const v4attn_layer_desc* d, const v4attn_index_args* a, void* ws,
                             size_t ws_bytes, cudaStream_t st, size_t body_off, bool dry = false,
                             uint32_t wait_ns = 0, int stall = 0) {
  if (d->kind != V4A_CSA) return V4A_ERR_INVALID_ARG;
  if (!a || a->n_q < 1 || a->n_q > kMaxQueries || a->B < 1) return V4A_ERR_INVALID_ARG;
  if (!a->qI || !a->w || !a->q_pos || !a->keys || (!a->idx_out && !a->scores_out))
    return V4A_ERR_INVALID_ARG;
  if (d->idx_dtype == V4A_MXFP4 && (!a->qI_sf || !a->keys_sf)) return V4A_ERR_INVALID_ARG;
  if (a->score_dtype != V4A_F32 && a->score_dtype != V4A_BF16) return V4A_ERR_INVALID_ARG;
  const int sbf = a->score_dtype == V4A_BF16 ? 1 : 0;
  const size_t s_esz = sbf ? 2 : 4;
  if (const v4attn_status sp = check_pages(d, a->block_table, a->blocks_per_seq, a->key_rows,
                                           d->idx_dtype == V4A_MXFP4))
    return sp;
  const PageMap pages = page_map(d, a->block_table, a->blocks_per_seq, a->key_rows);
  if (a->key_rows < 1 || a->max_vis < 0 ||
      a->max_vis > seq_cap(d, a->block_table, a->blocks_per_seq, a->key_rows))
    return V4A_ERR_INVALID_ARG;
  if (!ws) return V4A_ERR_WORKSPACE;
  if (ws_bytes < body_off + index_need(a->n_q, a->max_vis)) return V4A_ERR_WORKSPACE;
  uint8_t* w8 = reinterpret_cast<uint8_t*>(ws);
  const int64_t ld = std::max<int64_t>(a->max_vis, 1);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  const bool fp4 = d->idx_dtype == V4A_MXFP4;
  const size_t qrow = fp4 ? (size_t)d->d_I / 2 : (size_t)d->d_I * sizeof(float);
  if (fp4) {
    // the first chunk's pointers stand for every chunk: chunk offsets are
    // multiples of 64-byte query rows, H_I scale rows and H_I weights
    IndexParams P;
    P.n_q = std::min(kQChunk, a->n_q);
    P.B = a->B;
    P.m = d->m;
    P.H_I = d->H_I;
    P.d_I = d->d_I;
    P.idx_dtype = d->idx_dtype;
    P.qI = a->qI;
    P.qI_sf = a->qI_sf;
    P.w = a->w;
    P.keys = a->keys;
    P.keys_sf = a->keys_sf;
    P.key_rows = a->key_rows;
    P.max_vis = a->max_vis;
    P.pages = pages;
    const v4attn_status s = tc_status(index_tc_check(P));
    if (s != V4A_OK) return s;
  }
  if (dry) return V4A_OK;
  for (int32_t q0 = 0; q0 < a->n_q; q0 += kQChunk) {
    const int32_t cn = std::min(kQChunk, a->n_q - q0);
    float* scores = a->scores_out
                        ? reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a->scores_out) +
                                                   (size_t)q0 * ld * s_esz)
                        : reinterpret_cast<float*>(w8 + body_off);
    if (a->max_vis > 0) {
      IndexParams P;
      P.n_q = cn;
      P.B = a->B;
      P.m = d->m;
      P.H_I = d->H_I;
      P.d_I = d->d_I;
      P.idx_dtype = d->idx_dtype;
      P.qI = reinterpret_cast<const uint8_t*>(a->qI) + (size_t)q0 * d->H_I * qrow;
      P.qI_sf = fp4 ? a->qI_sf + (size_t)q0 * d->H_I * (d->d_I / 32) : nullptr;
      P.w = a->w + (size_t)q0 * d->H_I;
      P.q_seq = a->q_seq ? a->q_seq + q0 : nullptr;
      P.q_base = q0;
      P.q_pos = a->q_pos + q0;
      P.keys = a->keys;
      P.keys_sf = a->keys_sf;
      P.key_rows = a->key_rows;
      P.max_vis = a->max_vis;
      P.scores = scores;
      P.scores_ld = ld;
      P.score_bf16 = sbf;
      P.status = status;
      P.pages = pages;
      P.wait_ns = wait_ns;
      P.stall = stall;
      if (const cudaError_t e = index_scores_dispatch(P, st)) return cuda_status(e);
    }
    if (!a->idx_out) continue;   // scores-only call
    TopkParams T;
    T.n_q = cn;
    T.m = d->m;
    T.k = d->top_k;
    T.scores = scores;
    T.scores_ld = ld;
    T.score_bf16 = sbf;
    T.max_vis = a->max_vis;
    T.q_pos = a->q_pos + q0;
    T.idx_out = a->idx_out + (int64_t)q0 * d->top_k;
    if (const cudaError_t e = topk_dispatch(T, st)) return cuda_status(e);
  }
  return V4A_OK;
}

v4attn_status run_mqa(const v4attn_layer_desc* d, const v4attn_mqa_args* a, void* ws,
                      size_t ws_bytes, cudaStream_t st, bool sparse, bool q_ready = false,
                      bool dry = false) {
  if (!a || a->n_q < 1 || a->n_q > kMaxQueries || a->B < 1) return V4A_ERR_INVALID_ARG;
  if (!a->Q || !a->q_pos || !a->kv || !a->out) return V4A_ERR_INVALID_ARG;
  if (d->n_win > 0 && (!a->swa || a->swa_rows < d->n_win)) return V4A_ERR_INVALID_ARG;
  if (d->kv_dtype == V4A_E4M3_BF16ROPE && (!a->kv_scale || (d->n_win > 0 && !a->swa_scale)))
    return V4A_ERR_INVALID_ARG;
  if (a->q_dtype != V4A_F32 && a->q_dtype != V4A_BF16) return V4A_ERR_UNSUPPORTED;
  if (a->out_dtype != V4A_F32 && a->out_dtype != V4A_BF16) return V4A_ERR_UNSUPPORTED;
  if (a->kv_rows < 1) return V4A_ERR_INVALID_ARG;
  if (sparse && (!a->idx || a->n_sel < 1 || a->n_sel > 4096)) return V4A_ERR_INVALID_ARG;
  if (const v4attn_status sp = check_pages(d, a->block_table, a->blocks_per_seq, a->kv_rows,
                                           d->kv_dtype == V4A_E4M3_BF16ROPE))
    return sp;
  if (!sparse && (a->max_vis < 0 ||
                  a->max_vis > seq_cap(d, a->block_table, a->blocks_per_seq, a->kv_rows)))
    return V4A_ERR_INVALID_ARG;
  if (!aligned16(a->kv) || (a->swa && !aligned16(a->swa)) || !aligned16(a->out))
    return V4A_ERR_INVALID_ARG;
  if (!ws) return V4A_ERR_WORKSPACE;
  const int64_t n_main_max = sparse ? (int64_t)a->n_sel : a->max_vis;
  const size_t b0 = body_mqa(d, a->n_q);
  if (ws_bytes < b0 + mqa_need(d, a->n_q, n_main_max)) return V4A_ERR_WORKSPACE;
  uint8_t* w8 = reinterpret_cast<uint8_t*>(ws);
  const int32_t c = q_chunk(a->n_q);
  const size_t qb = (size_t)d->H * d->d * (a->q_dtype == V4A_BF16 ? 2 : 4);
  const size_t ob = (size_t)d->H * d->d * (a->out_dtype == V4A_BF16 ? 2 : 4);
  for (int32_t q0 = 0; q0 < a->n_q; q0 += kQChunk) {
    if (dry && q0 > 0) break;
    MqaParams P;
    P.n_q = std::min(kQChunk, a->n_q - q0);
    P.B = a->B;
    P.H = d->H;
    P.d = d->d;
    P.d_rope = d->d_rope;
    P.n_win = d->n_win;
    P.m = d->m;
    P.theta = d->rope_theta;
    P.scale = softmax_scale(d);
    P.eps = d->rms_eps;
    P.Q = reinterpret_cast<const uint8_t*>(a->Q) + (size_t)q0 * qb;
    P.q_dtype = a->q_dtype;
    P.q_rmsnorm = a->q_rmsnorm;
    P.q_seq = a->q_seq ? a->q_seq + q0 : nullptr;
    P.q_base = q0;
    P.q_pos = a->q_pos + q0;
    P.kv_dtype = d->kv_dtype;
    P.kv = reinterpret_cast<const uint8_t*>(a->kv);
    P.kv_scale = a->kv_scale;
    P.kv_rows = a->kv_rows;
    P.swa = reinterpret_cast<const uint8_t*>(a->swa);
    P.swa_scale = a->swa_scale;
    P.swa_rows = a->swa_rows > 0 ? a->swa_rows : 1;
    P.idx = sparse ? a->idx + (int64_t)q0 * a->n_sel : nullptr;
    P.n_sel = sparse ? a->n_sel : 0;
    P.max_vis = sparse ? a->kv_rows : a->max_vis;
    P.sink = a->sink;
    P.split_keys = mqa_split_keys(d);
    P.n_split = mqa_num_splits(d, n_main_max);
    P.part_o = reinterpret_cast<float*>(w8 + b0);
    P.part_ml = d->kv_dtype == V4A_E4M3_BF16ROPE
                    ? P.part_o + kMqaTcPartFloats
                    : reinterpret_cast<float*>(w8 + b0 + mqa_part_o_bytes(d, c, P.n_split));
    P.grid_bar = &reinterpret_cast<WsHeader*>(ws)->bar_count;
    P.qbuf = mqa_qbuf_bytes(d, c) ? w8 + qimg_off(a->n_q) : nullptr;
    P.q_ready = q_ready ? 1 : 0;
    P.out = reinterpret_cast<uint8_t*>(a->out) + (size_t)q0 * ob;
    P.out_dtype = a->out_dtype;
    P.lse = a->lse ? a->lse + (int64_t)q0 * d->H : nullptr;
    P.status = reinterpret_cast<uint32_t*>(ws);
    P.pages = page_map(d, a->block_table, a->blocks_per_seq, a->kv_rows);
    if (q0 == 0 && d->kv_dtype == V4A_E4M3_BF16ROPE) {
      const v4attn_status s = tc_status(mqa_tc_check(P));
      if (s != V4A_OK) return s;
    }
    if (dry) return V4A_OK;
    if (const cudaError_t e = mqa_dispatch(P, st)) return cuda_status(e);
    if (d->kv_dtype != V4A_E4M3_BF16ROPE)
      if (const cudaError_t e = launch_mqa_combine(P, st)) return cuda_status(e);
  }
  return V4A_OK;
}


}  // namespace

extern "C" {

size_t v4attn_workspace_size(const v4attn_layer_desc* desc, int32_t n_q, int64_t max_vis) {
  if (check_desc(desc) != V4A_OK || n_q < 1 || max_vis < 0) return 0;
  return total_need(desc, n_q, max_vis);
}

v4attn_status v4attn_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (!ws || ws_bytes < sizeof(WsHeader)) return V4A_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, sizeof(WsHeader), stream));
}

v4attn_status v4attn_compress(const v4attn_layer_desc* desc, const v4attn_compress_args* args,
                              void* ws, size_t ws_bytes, cudaStream_t stream) {
  (void)ws;
  (void)ws_bytes;
  if (!desc || desc->d_rope < 0 || desc->d_rope % 2 || !(desc->rope_theta > 0.f))
    return V4A_ERR_INVALID_ARG;
  return run_compress(desc, args, stream);
}

v4attn_status v4attn_index_topk(const v4attn_layer_desc* desc, const v4attn_index_args* args,
                                void* ws, size_t ws_bytes, cudaStream_t stream) {
  v4attn_status s = check_desc(desc);
  if (s != V4A_OK) return s;
  return run_index_topk(desc, args, ws, ws_bytes, stream, args ? qimg_off(args->n_q) : 0);
}

v4attn_status v4attn_sparse_mqa(const v4attn_layer_desc* desc, const v4attn_mqa_args* args,
                                void* ws, size_t ws_bytes, cudaStream_t stream) {
  v4attn_status s = check_desc(desc);
  if (s != V4A_OK) return s;
  return run_mqa(desc, args, ws, ws_bytes, stream, true);
}

v4attn_status v4attn_dense_mqa(const v4attn_layer_desc* desc, const v4attn_mqa_args* args,
                               void* ws, size_t ws_bytes, cudaStream_t stream) {
  v4attn_status s = check_desc(desc);
  if (s != V4A_OK) return s;
  return run_mqa(desc, args, ws, ws_bytes, stream, false);
}

v4attn_status v4attn_decode(const v4attn_layer_desc* desc, const v4attn_decode_args* a, void* ws,
                            size_t ws_bytes, cudaStream_t stream) {
  v4attn_status s = check_desc(desc);
  if (s != V4A_OK) return s;
  if (!a || a->B < 1 || a->B > 65535 || !a->pos || !a->x_main || !a->tail || !a->kv || !a->swa ||
      !a->Q || !a->out)
    return V4A_ERR_INVALID_ARG;
  const bool csa = desc->kind == V4A_CSA;
  if (csa && (!a->x_idx || !a->itail || !a->keys || !a->qI || !a->w || !a->idx_out))
    return V4A_ERR_INVALID_ARG;
  if (a->in_dtype != V4A_F32 && a->in_dtype != V4A_BF16) return V4A_ERR_UNSUPPORTED;
  if (const v4attn_status sp = check_pages(desc, a->block_table, a->blocks_per_seq, a->kv_rows,
                                           desc->kv_dtype == V4A_E4M3_BF16ROPE &&
                                               (!csa || desc->idx_dtype == V4A_MXFP4)))
    return sp;
  if (csa && a->block_table && a->key_rows % (128 / desc->m) != 0) return V4A_ERR_INVALID_ARG;
  if (a->max_vis < 0 || a->max_vis > seq_cap(desc, a->block_table, a->blocks_per_seq, a->kv_rows) ||
      (csa && a->max_vis > seq_cap(desc, a->block_table, a->blocks_per_seq, a->key_rows)))
    return V4A_ERR_INVALID_ARG;
  if (!ws) return V4A_ERR_WORKSPACE;
  if (ws_bytes < total_need(desc, a->B, a->max_vis)) return V4A_ERR_WORKSPACE;
  const int m = desc->m;
  const int ring = csa ? 2 * m : m;
  const int n_arr = csa ? 4 : 2;
  const int d = desc->d;
  const int elt = a->in_dtype == V4A_F32 ? 4 : 2;
  {
    // the append kernel reads four channels per load: bases aligned to 4 elements,
    // biases to 16 bytes
    const uintptr_t al = 4 * (uintptr_t)elt;
    for (const void* p : {a->x_main, (const void*)a->tail, a->x_idx, (const void*)a->itail})
      if (p && (reinterpret_cast<uintptr_t>(p) % al)) return V4A_ERR_INVALID_ARG;
    for (const void* p : {(const void*)a->bias, (const void*)a->ibias})
      if (p && (reinterpret_cast<uintptr_t>(p) % 16)) return V4A_ERR_INVALID_ARG;
    // a pooling window of at most 65536 / d rows per entry (8 rows per thread
    // over the d / 8 channels of each of the job's 8 CTAs, whose row slices
    // are merged by 2048 / d adjacent lanes)
    if ((int64_t)ring * d > 65536) return V4A_ERR_UNSUPPORTED;
    if (d != 64 && d != 128 && d != 256 && d != 512) return V4A_ERR_UNSUPPORTED;
  }
  // 1.-2. tail rings, the new token's window KV (RMSNorm, RoPE at p), the
  // entry (and indexer key) its block completes: one launch
  AppendParams A;
  A.B = a->B;
  A.csa = csa ? 1 : 0;
  A.pos = a->pos;
  A.in_dtype = a->in_dtype;
  A.x_main = a->x_main;
  A.tail = a->tail;
  A.m = m;
  A.ring = ring;
  A.n_arr = n_arr;
  A.d = d;
  A.bias = a->bias;
  A.x_idx = csa ? a->x_idx : nullptr;
  A.itail = csa ? a->itail : nullptr;
  A.dI = desc->d_I;
  A.ibias = a->ibias;
  A.kv_dtype = desc->kv_dtype;
  A.idx_dtype = desc->idx_dtype;
  A.d_rope = desc->d_rope;
  A.theta = desc->rope_theta;
  A.eps = desc->rms_eps;
  A.swa = a->swa;
  A.swa_scale = a->swa_scale;
  A.swa_rows = a->swa_rows;
  A.kv = a->kv;
  A.kv_scale = a->kv_scale;
  A.kv_rows = a->kv_rows;
  A.keys = csa ? a->keys : nullptr;
  A.keys_sf = csa ? a->keys_sf : nullptr;
  A.key_rows = csa ? a->key_rows : 0;
  A.kv_pages = page_map(desc, a->block_table, a->blocks_per_seq, a->kv_rows);
  if (csa) A.key_pages = page_map(desc, a->block_table, a->blocks_per_seq, a->key_rows);
  A.status = reinterpret_cast<uint32_t*>(ws);
  // the tensor-core MQA's query images, coded in the same launch when its
  // format applies and the step's queries fit one query chunk
  const bool fuse_q = desc->kv_dtype == V4A_E4M3_BF16ROPE && a->q_dtype == V4A_BF16 &&
                      d == 512 && desc->d_rope == 64 && desc->H <= 128 && a->B <= kQChunk &&
                      aligned16(a->Q);
  if (fuse_q) {
    A.Q = a->Q;
    A.H = desc->H;
    A.qimg = reinterpret_cast<uint8_t*>(ws) + qimg_off(a->B);
  }
  // 3. indexer + top-k, 4. MQA: arguments built and validated before the
  // first launch, so that a refused step leaves the caches untouched
  v4attn_index_args ix{};
  v4attn_mqa_args q{};
  if (csa) {
    ix.n_q = a->B;
    ix.B = a->B;
    ix.qI = a->qI;
    ix.qI_sf = a->qI_sf;
    ix.w = a->w;
    ix.q_seq = nullptr;
    ix.q_pos = a->pos;
    ix.keys = a->keys;
    ix.keys_sf = a->keys_sf;
    ix.key_rows = a->key_rows;
    ix.max_vis = a->max_vis;
    ix.idx_out = a->idx_out;
    ix.block_table = a->block_table;
    ix.blocks_per_seq = a->blocks_per_seq;
    s = run_index_topk(desc, &ix, ws, ws_bytes, stream, body_mqa(desc, a->B), true);
    if (s != V4A_OK) return s;
  }
  q.n_q = a->B;
  q.B = a->B;
  q.Q = a->Q;
  q.q_dtype = a->q_dtype;
  q.q_rmsnorm = 0;
  q.q_seq = nullptr;
  q.q_pos = a->pos;
  q.kv = a->kv;
  q.kv_scale = a->kv_scale;
  q.kv_rows = a->kv_rows;
  q.swa = a->swa;
  q.swa_scale = a->swa_scale;
  q.swa_rows = a->swa_rows;
  q.idx = csa ? a->idx_out : nullptr;
  q.n_sel = csa ? desc->top_k : 0;
  q.max_vis = a->max_vis;
  q.sink = a->sink;
  q.out = a->out;
  q.out_dtype = a->out_dtype;
  q.lse = a->lse;
  q.block_table = a->block_table;
  q.blocks_per_seq = a->blocks_per_seq;
  s = run_mqa(desc, &q, ws, ws_bytes, stream, csa, fuse_q, true);
  if (s != V4A_OK) return s;
  if (const cudaError_t e = launch_decode_append(A, stream)) return cuda_status(e);
  if (csa) {
    s = run_index_topk(desc, &ix, ws, ws_bytes, stream, body_mqa(desc, a->B));
    if (s != V4A_OK) return s;
  }
  // 4. MQA
  return run_mqa(desc, &q, ws, ws_bytes, stream, csa, fuse_q);
}

v4attn_status v4attn_project(const v4attn_project_args* a, cudaStream_t stream) {
  if (!a || a->M < 0 || a->N < 0 || a->K < 0 || !a->X || !a->W || !a->Y) return V4A_ERR_INVALID_ARG;
  if ((a->x_dtype != V4A_F32 && a->x_dtype != V4A_BF16) || a->w_dtype != a->x_dtype)
    return V4A_ERR_UNSUPPORTED;
  if (a->y_dtype != V4A_F32 && a->y_dtype != V4A_BF16) return V4A_ERR_UNSUPPORTED;
  if (a->ldx < a->K || a->ldw < a->N || a->ldy < a->N) return V4A_ERR_INVALID_ARG;
  if (a->M == 0 || a->N == 0) return V4A_OK;
  if (a->M > 65535LL * 64) return V4A_ERR_UNSUPPORTED;
  if ((int64_t)a->K < 1) return V4A_ERR_INVALID_ARG;
  ProjectParams P;
  P.M = a->M;
  P.N = a->N;
  P.K = a->K;
  P.X = a->X;
  P.x_dtype = a->x_dtype;
  P.ldx = a->ldx;
  P.W = a->W;
  P.ldw = a->ldw;
  P.Y = a->Y;
  P.y_dtype = a->y_dtype;
  P.ldy = a->ldy;
  if (P.x_dtype == V4A_BF16) {
    const v4attn_status s = tc_status(project_tc_check(P));
    if (s != V4A_OK) return s;
  }
  return cuda_status(project_dispatch(P, stream));
}

v4attn_status v4attn_device_status(const void* ws, cudaStream_t stream, uint32_t* bits) {
  if (!ws) return V4A_ERR_WORKSPACE;
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(uint32_t), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return V4A_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return V4A_ERR_CUDA;
  if (bits) *bits = word;
  if (word & ST_TIMEOUT) return V4A_ERR_TIMEOUT;
  if (word) return V4A_ERR_DEVICE_CHECK;
  return V4A_OK;
}

const char* v4attn_status_string(v4attn_status s) {
  switch (s) {
    case V4A_OK: return "ok";
    case V4A_ERR_INVALID_ARG: return "invalid argument";
    case V4A_ERR_UNSUPPORTED: return "unsupported shape or format";
    case V4A_ERR_WORKSPACE: return "workspace missing or too small";
    case V4A_ERR_CUDA: return "CUDA launch error";
    case V4A_ERR_TIMEOUT: return "a bounded device wait ran out";
    case V4A_ERR_DEVICE_CHECK: return "a device-side argument check failed";
  }
  return "unknown status";
}

const char* v4attn_build_info(void) { return build_info_string(); }

const char* v4attn_last_cuda_error(void) { return cudaGetErrorString(t_last_cuda); }

v4attn_status v4attn_debug_index_stall(const v4attn_layer_desc* desc,
                                       const v4attn_index_args* args, void* ws, size_t ws_bytes,
                                       uint32_t wait_ns, cudaStream_t stream) {
  v4attn_status s = check_desc(desc);
  if (s != V4A_OK) return s;
  if (desc->idx_dtype != V4A_MXFP4) return V4A_ERR_UNSUPPORTED;   // the tcgen05 kernel only
  if (wait_ns < 100000u || wait_ns > 1000000000u) return V4A_ERR_INVALID_ARG;
  return run_index_topk(desc, args, ws, ws_bytes, stream, args ? qimg_off(args->n_q) : 0, false,
                        wait_ns, 1);
}

}  // extern "C"

// ---------------------------------------------------------------- no-allocation variant
// Scratch of v4attn_index_topk_noalloc, for callers that cannot allocate
// device memory: status header, decode region and the fp32 scores of up to
// V4A_NOALLOC_MAX_SCORES (query, key) pairs.  It is a file-scope device array,
// so every GPU that loads this library holds it (about 8.4 MB) until the
// process exits.  In host code the symbol is only a host-side stand-in, never
// a device address: the device address comes from cudaGetSymbolAddress, looked
// up once per device with that device current, on the first call there.
namespace {
constexpr size_t kNoallocBytes = 256 + 32768 + (size_t)V4A_NOALLOC_MAX_SCORES * sizeof(float);
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocBytes];
void* g_noalloc_ptr[64] = {nullptr};
}  // namespace

// The array's device address on the current device (looked up on first use).
static v4attn_status noalloc_scratch(void** ws) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return V4A_ERR_CUDA;
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return V4A_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *ws = g_noalloc_ptr[dev];
  return V4A_OK;
}

extern "C" v4attn_status v4attn_index_topk_noalloc(const v4attn_layer_desc* desc,
                                                   const v4attn_index_args* args,
                                                   cudaStream_t stream) {
  v4attn_status s = check_desc(desc);
  if (s != V4A_OK) return s;
  if (!args || args->n_q < 1 || args->max_vis < 0) return V4A_ERR_INVALID_ARG;
  // both limits of the header, checked as stated (the byte check follows from them)
  if (args->n_q > V4A_NOALLOC_MAX_QUERIES ||
      (int64_t)args->n_q * std::max<int64_t>(args->max_vis, 1) > V4A_NOALLOC_MAX_SCORES ||
      qimg_off(args->n_q) + index_need(args->n_q, args->max_vis) > kNoallocBytes)
    return V4A_ERR_UNSUPPORTED;
  void* ws = nullptr;
  s = noalloc_scratch(&ws);
  if (s != V4A_OK) return s;
  // the status word must start at zero; the scores are fully rewritten by the call
  if (cudaMemsetAsync(ws, 0, sizeof(WsHeader), stream) != cudaSuccess) return V4A_ERR_CUDA;
  return run_index_topk(desc, args, ws, kNoallocBytes, stream, qimg_off(args->n_q));
}

extern "C" v4attn_status v4attn_noalloc_device_status(cudaStream_t stream, uint32_t* bits) {
  void* ws = nullptr;
  const v4attn_status s = noalloc_scratch(&ws);
  if (s != V4A_OK) return s;
  return v4attn_device_status(ws, stream, bits);
}
