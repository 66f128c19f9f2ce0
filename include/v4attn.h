/*
 * v4attn.h - C ABI of the DeepSeek-V4 hybrid compressed attention hot path
 * (CSA / HCA) on NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and section:
 *   [deep-read] "DeepSeek-V4 深读：百万 Token 不是窗口数字，而是一整套系统契约"
 *               (ricardokevins.github.io): "CSA：4× 压缩之后再 top-k" (equation
 *               C_i^comp, lightning indexer, top-k), "HCA：128× 压缩后保留 dense
 *               全局视野", "其他稳定性细节" (RMSNorm, partial RoPE, inverse output
 *               rotation, sink, FP8/BF16 KV, FP4 indexer), the model-spec table
 *               "模型规格", "异构 KV cache 与磁盘前缀复用" (state vs block cache).
 *   [news]      "AI深一度 第15期|DeepSeek V4" (yeyulingfeng.com), "一、CSA与HCA":
 *               softmax gate with a learnable position bias.
 *   [notes]     "拆解 DeepSeekv4" (daixd5520.github.io), "CSA" (half-overlapping
 *               windows) and "细节" (sink exp(z'_h) in the denominator).
 *
 * Conventions shared by every entry point
 *   - Ownership: the caller allocates and owns every buffer (inputs, caches,
 *     outputs, workspace).  The library never allocates, frees or
 *     synchronises the device, keeps no global state and is thread-safe per
 *     stream.
 *   - Pointers: "device" pointers must be device memory of the current
 *     device; every device pointer must be 16-byte aligned and every row
 *     stride a multiple of 16 bytes unless stated otherwise.
 *   - Ordering: all work is enqueued on `stream`; argument errors are
 *     returned synchronously, before anything is launched.
 *   - Errors: V4A_ERR_INVALID_ARG / _UNSUPPORTED for bad or unsupported
 *     arguments, V4A_ERR_WORKSPACE when ws_bytes is too small,
 *     V4A_ERR_CUDA when a launch fails.  Checks that need device data
 *     (positions beyond a cache, indices out of range) are made by the
 *     kernels, which then skip the access and set a bit in the workspace's
 *     status word; v4attn_device_status() reads it (and synchronises).
 *   - Positions are 0-based absolute token positions.  Entry i of a layer
 *     with ratio m is visible to the query at p iff m*(i+1)-1 <= p, so
 *     n_vis(p) = floor((p+1)/m); a query sees the visible entries plus the
 *     raw tokens max(0, p-n_win+1) .. p of its sliding window.
 *   - Stored entry formats (one row per entry or window token):
 *       V4A_F32            d floats (4*d bytes), no scale;
 *       V4A_E4M3_BF16ROPE  d-d_rope E4M3 codes, then d_rope bf16 values
 *                          (d - d_rope + 2*d_rope bytes; 576 for d=512),
 *                          plus one float scale per row in a separate array
 *                          (a power of two: the smallest s with
 *                          max|x_nope|/s <= 448; 1 when all are zero);
 *       V4A_MXFP4          c/2 bytes of E2M1 pairs (element 2j in the low
 *                          nibble) plus c/32 E8M0 scale bytes in a separate
 *                          array (OCP MX v1.0: X = floor(log2 amax) - 2).
 *   - Paged caches ([deep-read] "异构 KV cache 与磁盘前缀复用": a classical
 *     block cache over blocks of lcm(4, 128) = 128 raw tokens, next to the
 *     per-sequence state cache of window and uncompressed tail).  With
 *     block_table == NULL the compressed caches are per sequence: entry e of
 *     sequence b at row b * rows + e.  With a block table (device int32
 *     [B][blocks_per_seq]) they are pools shared by all sequences, `rows`
 *     rows in all: one block holds epb = 128 / m consecutive entries (32 CSA
 *     entries and 32 indexer keys, or 1 HCA entry), and entry e of sequence
 *     b is at row block_table[b * blocks_per_seq + e / epb] * epb + e % epb.
 *     rows must be a multiple of epb, a sequence sees at most
 *     blocks_per_seq * epb entries, and a table entry outside
 *     [0, rows / epb) is caught by the kernels (status bit, the access
 *     skipped).  The window and tail rings stay per sequence.  Paged caches
 *     need the tensor-core formats (E4M3 entries, MXFP4 keys; else
 *     V4A_ERR_UNSUPPORTED).
 */
#ifndef V4ATTN_H
#define V4ATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  V4A_OK = 0,
  V4A_ERR_INVALID_ARG = 1,
  V4A_ERR_UNSUPPORTED = 2,
  V4A_ERR_WORKSPACE = 3,
  V4A_ERR_CUDA = 4,
  V4A_ERR_TIMEOUT = 5,
  V4A_ERR_DEVICE_CHECK = 6
} v4attn_status;

typedef enum { V4A_F32 = 0, V4A_BF16 = 1, V4A_E4M3_BF16ROPE = 2, V4A_MXFP4 = 3 } v4attn_dtype;

typedef enum { V4A_CSA = 0, V4A_HCA = 1 } v4attn_kind;

/* Shape of one attention layer ([deep-read] model-spec table: 64 / 128 query
 * heads of dim 512, one shared KV head, 64 RoPE dims, RoPE theta 160000,
 * CSA m = 4 with top-k 512 / 1024, HCA m' = 128, window 128; 64 indexer heads). */
typedef struct {
  int32_t kind;          /* V4A_CSA (windows of 2m at stride m) or V4A_HCA (windows of m) */
  int32_t m;             /* compression ratio */
  int32_t n_win;         /* sliding-window tokens (0..128) */
  int32_t H;             /* query heads (1..128) */
  int32_t d;             /* head / entry dim: 32..512, multiple of 32 */
  int32_t d_rope;        /* RoPE dims at the end of d: even, <= d */
  float rope_theta;      /* RoPE base */
  float softmax_scale;   /* <= 0 selects 1/sqrt(d) */
  int32_t H_I;           /* indexer heads (CSA) */
  int32_t d_I;           /* indexer dim (CSA), multiple of 32 */
  int32_t top_k;         /* selected entries per query (CSA), 1..2048 */
  int32_t kv_dtype;      /* V4A_F32 or V4A_E4M3_BF16ROPE (then d = 512, d_rope = 64) */
  int32_t idx_dtype;     /* V4A_F32 or V4A_MXFP4 */
  float rms_eps;         /* RMSNorm epsilon (1e-6) */
} v4attn_layer_desc;

/* ---------------------------------------------------------------- compress
 * Softmax-gated pooling ([deep-read] "CSA：4× 压缩之后再 top-k", equation
 * C_i^comp; [news] "一、CSA与HCA"; [deep-read] "HCA：128× 压缩后保留 dense
 * 全局视野").  For entry i and channel c:
 *   overlap (CSA): window token j = m*(i-1) + r, r in [0, 2m); r <  m reads
 *                  (Cb, Zb), r >= m reads (Ca, Za);
 *   no overlap:    j = m*i + r, r in [0, m), reads (Ca, Za);
 *   e_i[c] = sum_r softmax_r(Z_j[c] + bias[r][c]) * C_j[c], the softmax
 *   taken jointly over the window tokens with 0 <= j < seq_len[b].
 * Then optionally RMSNorm over the c channels (unit weight) and RoPE at
 * position m*i on the last d_rope channels (adjacent pairs, frequency
 * theta^(-2k/d_rope)); then the entry is stored in out_dtype.
 * With m = 1 and no overlap the window is the token itself (Z may be NULL):
 * this stores a raw token's KV, e.g. for the sliding window.  */
typedef struct {
  int32_t m;                  /* window stride (1..128) */
  int32_t overlap;            /* 1: CSA windows of 2m, 0: windows of m */
  int32_t c;                  /* channels: 32..1024, even; multiple of 32 for MXFP4 */
  int32_t B;                  /* sequences */
  const void* Ca;             /* device [B] x [in_rows] x [c] values, token j at row (j mod in_rows) */
  const void* Za;             /* device, same layout: gate logits (NULL allowed iff m == 1) */
  const void* Cb;             /* device, branch-b values (overlap only) */
  const void* Zb;             /* device, branch-b logits (overlap only) */
  int32_t in_dtype;           /* V4A_F32 or V4A_BF16 */
  int64_t in_seq_stride;      /* elements between sequences (even) */
  int64_t in_row_stride;      /* elements between token rows (>= c, even); Ca/Za/Cb/Zb aligned
                                 to 2 elements, bias to 8 bytes, else V4A_ERR_INVALID_ARG */
  int64_t in_rows;            /* rows per sequence in the input arrays */
  const float* bias;          /* device [2m or m][c] position bias; NULL = 0 */
  const int64_t* seq_len;     /* device [B] tokens present (window tokens >= it are left out) */
  const int64_t* entry_begin; /* device [B] first entry to compute */
  int32_t n_entries;          /* entries per sequence (entry_begin .. entry_begin+n_entries-1) */
  int32_t complete_only;      /* 1: skip entries whose block has m*(i+1) > seq_len */
  int32_t apply_rmsnorm;
  int32_t apply_rope;
  int32_t out_dtype;          /* V4A_F32, V4A_E4M3_BF16ROPE (c = 512, d_rope = 64) or V4A_MXFP4 */
  void* out;                  /* device [B] x [out_rows] x [row bytes]; entry i at row (i mod out_rows) */
  void* out_scale;            /* E4M3: float [B][out_rows]; MXFP4: uint8 [B][out_rows][c/32]; else NULL */
  int64_t out_rows;
} v4attn_compress_args;

/* ---------------------------------------------------------------- index_topk
 * Lightning indexer and top-k ([deep-read] "CSA：4× 压缩之后再 top-k";
 * "FP4 QAT、可恢复 rollout 与百万 Token RL" for the MXFP4 QK path):
 *   s_i = sum_h w_h * max(0, q_h . k_i)   for i < n_vis(p)
 * then the top_k largest s_i (exact ties to the lower index), written in
 * ascending index order, -1 padded when n_vis < top_k.
 * Formats: V4A_F32 (d_I 32, 64 or 128, any H_I <= 128) runs on CUDA cores;
 * V4A_MXFP4 runs on the tcgen05 block-scaled tensor-core kernel only and needs
 * d_I = 128, H_I in {32, 64, 128} and key_rows % 4 == 0 (else
 * V4A_ERR_UNSUPPORTED), with qI, qI_sf, w, keys, keys_sf 16-byte aligned
 * (else V4A_ERR_INVALID_ARG).
 * score_dtype V4A_BF16 ([deep-read] "FP4 QAT、可恢复 rollout 与百万 Token RL":
 * the selector on BF16 scores) rounds every score to bf16 (nearest even)
 * before the top-k, which then selects exactly among those bf16 values (ties
 * to the lower index); scores_out, if given, receives them as bf16.  */
typedef struct {
  int32_t n_q;                /* queries, 1 .. 2^20 */
  int32_t B;                  /* sequences */
  const void* qI;             /* device MXFP4: uint8 [n_q][H_I][d_I/2]; F32: float [n_q][H_I][d_I] */
  const uint8_t* qI_sf;       /* device MXFP4: E8M0 [n_q][H_I][d_I/32]; else NULL */
  const float* w;             /* device [n_q][H_I] head weights */
  const int32_t* q_seq;       /* device [n_q] sequence of each query; NULL = query q in sequence q */
  const int64_t* q_pos;       /* device [n_q] position p of each query */
  const void* keys;           /* device MXFP4: uint8 [B][key_rows][d_I/2]; F32: float [B][key_rows][d_I] */
  const uint8_t* keys_sf;     /* device MXFP4: E8M0 [B][key_rows][d_I/32]; else NULL */
  int64_t key_rows;           /* rows per sequence; n_vis(p) must not exceed it */
  int64_t max_vis;            /* upper bound of n_vis over the queries (<= key_rows) */
  int32_t* idx_out;           /* device [n_q][top_k]; NULL = scores only (scores_out required) */
  void* scores_out;           /* device [n_q][max_vis] float (bf16 with score_dtype V4A_BF16)
                                 or NULL; entries >= n_vis are -inf */
  int32_t score_dtype;        /* V4A_F32 (0) or V4A_BF16 */
  const int32_t* block_table; /* device [B][blocks_per_seq], or NULL: keys / keys_sf per
                                 sequence (see "Paged caches"; key_rows = pool rows) */
  int32_t blocks_per_seq;
} v4attn_index_args;

/* ---------------------------------------------------------------- MQA
 * Shared-KV MQA with window and sink ([deep-read] model-spec table and
 * "其他稳定性细节"; [notes] "细节"):
 *   q_h   = RoPE_p( [RMSNorm] Q_h ); with FP8 KV its d-d_rope dims are coded
 *           E4M3 with one power-of-two scale per (query, head), its RoPE
 *           dims bf16;
 *   s_hj  = softmax_scale * q_h . k_j over the key set
 *           sparse: entries idx[q][0..n_sel) (-1 skipped) + window tokens,
 *           dense:  entries 0..n_vis(p)-1 + window tokens;
 *   o_h   = sum_j exp(s_hj) k_j / (exp(sink_h) + sum_j exp(s_hj))   (V = K)
 *   out   = o_h with its RoPE dims rotated by -p;  lse_h = log of the denominator.
 * Formats: V4A_F32 caches run on CUDA cores; V4A_E4M3_BF16ROPE caches run on
 * the tcgen05 tensor-core kernel only and need a bf16 Q (else
 * V4A_ERR_UNSUPPORTED), 16-byte aligned Q, kv, swa and out (else
 * V4A_ERR_INVALID_ARG), and B * kv_rows, B * swa_rows < 2^31.  That kernel
 * takes P V in f16: stored values (entry scale x code, RoPE dims) must lie
 * below 65504 in magnitude (values below 2^-14 lose bits; an RMSNorm'ed row
 * is at most sqrt(d) = 22.6), and the softmax weights carry 11 significant
 * bits.  */
typedef struct {
  int32_t n_q;                /* queries, 1 .. 2^20 */
  int32_t B;
  const void* Q;              /* device [n_q][H][d] */
  int32_t q_dtype;            /* V4A_F32 or V4A_BF16 */
  int32_t q_rmsnorm;          /* 1: per-head RMSNorm of Q before RoPE */
  const int32_t* q_seq;       /* device [n_q] or NULL (query q in sequence q) */
  const int64_t* q_pos;       /* device [n_q] */
  const void* kv;             /* device entries [B][kv_rows][row bytes] in kv_dtype */
  const float* kv_scale;      /* device [B][kv_rows] (E4M3 format) or NULL */
  int64_t kv_rows;            /* entry i at row i (n_vis and indices must stay below kv_rows) */
  const void* swa;            /* device window tokens [B][swa_rows][row bytes]; token t at row (t mod swa_rows) */
  const float* swa_scale;     /* device [B][swa_rows] (E4M3 format) or NULL */
  int64_t swa_rows;           /* >= n_win */
  const int32_t* idx;         /* sparse: device [n_q][n_sel]; dense: NULL */
  int32_t n_sel;              /* sparse: columns of idx (top_k) */
  int64_t max_vis;            /* dense: upper bound of n_vis over the queries */
  const float* sink;          /* device [H] sink logits or NULL (no sink) */
  void* out;                  /* device [n_q][H][d] */
  int32_t out_dtype;          /* V4A_F32 or V4A_BF16 */
  float* lse;                 /* device [n_q][H] or NULL */
  const int32_t* block_table; /* device [B][blocks_per_seq], or NULL: kv / kv_scale per
                                 sequence (see "Paged caches"; kv_rows = pool rows) */
  int32_t blocks_per_seq;
} v4attn_mqa_args;

/* ---------------------------------------------------------------- decode
 * One decode step of one layer for B sequences, one new token each
 * ([deep-read] "CSA：4× 压缩之后再 top-k" / "HCA：128× 压缩后保留 dense 全局视野"
 * call order; "异构 KV cache 与磁盘前缀复用" for the split into a fixed-size
 * state cache (window + uncompressed tail) and the compressed caches):
 *   1. the new token's raw compressor inputs go to the tail ring, its window
 *      KV (RMSNorm, RoPE at p, stored format) to the window ring;
 *   2. if (p+1) % m == 0 the completed block is pooled into entry (p+1)/m-1
 *      of the main cache (and, for CSA, of the indexer-key cache);
 *   3. CSA: indexer + top-k over the visible keys;
 *   4. MQA over the selected (CSA) or all visible (HCA) entries + window.
 * x_main, tail, x_idx, itail must be aligned to 4 elements and bias, ibias
 * to 16 bytes (else V4A_ERR_INVALID_ARG); d must be 64, 128, 256 or 512 and
 * the pooling window (ring rows) times d must not exceed 65536 (else
 * V4A_ERR_UNSUPPORTED).  */
typedef struct {
  int32_t B;
  const int64_t* pos;         /* device [B] position p of each sequence's new token */
  int32_t in_dtype;           /* V4A_F32 or V4A_BF16 for the raw inputs and tails */
  const void* x_main;         /* device [B][n_arr][d]: the new token's (Ca, Za, Cb, Zb) (CSA) or (C, Z) (HCA) */
  void* tail;                 /* device [B][ring][n_arr][d] tail ring, token t in slot t mod ring;
                                 ring = 2m (CSA) or m (HCA); n_arr = 4 (CSA) or 2 (HCA) */
  const float* bias;          /* device [2m or m][d] */
  const void* x_idx;          /* CSA: device [B][4][d_I] the new token's indexer-compressor inputs */
  void* itail;                /* CSA: device [B][2m][4][d_I] indexer tail ring */
  const float* ibias;         /* CSA: device [2m][d_I] */
  void* kv; float* kv_scale; int64_t kv_rows;          /* main compressed cache (entry i at row i) */
  void* keys; uint8_t* keys_sf; int64_t key_rows;      /* CSA indexer keys (MXFP4 or F32) */
  void* swa; float* swa_scale; int64_t swa_rows;       /* window ring, token t at row t mod swa_rows */
  const void* Q; int32_t q_dtype;                      /* [B][H][d] */
  const void* qI; const uint8_t* qI_sf; const float* w; /* CSA indexer query [B][H_I][...] and weights */
  const float* sink;                                   /* [H] or NULL */
  void* out; int32_t out_dtype; float* lse;            /* [B][H][d], [B][H] or NULL */
  int32_t* idx_out;                                    /* CSA: [B][top_k] selected entries (required) */
  int64_t max_vis;                                     /* upper bound of n_vis after the step */
  const int32_t* block_table;  /* device [B][blocks_per_seq] or NULL: the main cache and the
                                  indexer keys as pools (see "Paged caches"); the new entry
                                  goes to its block's row, the window and tails stay per sequence */
  int32_t blocks_per_seq;
} v4attn_decode_args;

/* ---------------------------------------------------------------- projection
 * Y[M][N] = X[M][K] . W[K][N] with fp32 accumulation: the linear maps that
 * produce the compressor inputs C, Z from raw tokens ([deep-read] "CSA 与 HCA":
 * per-channel learned gating of token KV) and, in the small fp32 layer, the
 * queries.  X, W, Y row-major with the given leading dimensions (elements).
 * bf16 X and W run on the tcgen05 tensor-core GEMM only (X, W 16-byte aligned
 * with ldx, ldw multiples of 8 elements, else V4A_ERR_INVALID_ARG); fp32 X and
 * W run on CUDA cores.  K >= 1 (V4A_ERR_INVALID_ARG otherwise). */
typedef struct {
  int64_t M, N, K;
  const void* X; int32_t x_dtype; int64_t ldx;   /* V4A_F32 or V4A_BF16 */
  const void* W; int32_t w_dtype; int64_t ldw;   /* same dtype as X */
  void* Y; int32_t y_dtype; int64_t ldy;         /* V4A_F32 or V4A_BF16 */
} v4attn_project_args;

/* Bytes of workspace the calls below need for this layer, n_q queries and at
 * most max_vis visible entries per query (>= 256; includes the status word).
 * index_topk and the MQA calls process their queries in chunks of 1024 (up to
 * 2^20 queries per call), so the body of the workspace holds the scores or
 * split-K partials of one chunk; for a V4A_E4M3_BF16ROPE layer it also holds
 * the coded queries of one chunk (74,752 bytes a query) that the tensor-core
 * MQA reads, and, when n_q <= 40, room for that MQA's split-K partials
 * (160 CTAs x 129 KiB: a call of few queries spreads each (query, half of the
 * output dims) over up to 64 resident CTAs that meet at one grid barrier).
 * The size grows with n_q only by 24 bytes per query beyond 1024.
 * Its layout is internal to the library; one workspace serves one stream. */
size_t v4attn_workspace_size(const v4attn_layer_desc* desc, int32_t n_q, int64_t max_vis);

/* Zero the workspace's header: the status word and the tensor-core MQA's grid
 * barrier state (stream-ordered).  Call it once before the first call and
 * again after a call has reported V4A_ERR_TIMEOUT. */
v4attn_status v4attn_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream);

v4attn_status v4attn_compress(const v4attn_layer_desc* desc, const v4attn_compress_args* args,
                              void* ws, size_t ws_bytes, cudaStream_t stream);
v4attn_status v4attn_index_topk(const v4attn_layer_desc* desc, const v4attn_index_args* args,
                                void* ws, size_t ws_bytes, cudaStream_t stream);
v4attn_status v4attn_sparse_mqa(const v4attn_layer_desc* desc, const v4attn_mqa_args* args,
                                void* ws, size_t ws_bytes, cudaStream_t stream);
v4attn_status v4attn_dense_mqa(const v4attn_layer_desc* desc, const v4attn_mqa_args* args,
                               void* ws, size_t ws_bytes, cudaStream_t stream);
v4attn_status v4attn_decode(const v4attn_layer_desc* desc, const v4attn_decode_args* args,
                            void* ws, size_t ws_bytes, cudaStream_t stream);
v4attn_status v4attn_project(const v4attn_project_args* args, cudaStream_t stream);

/* ---------------------------------------------------------------- no-allocation variant
 * The paper has no counterpart to this call; it is a convenience of this
 * library.  It is v4attn_index_topk without a caller-supplied workspace, for
 * callers that cannot call cudaMalloc: code that runs inside a host framework
 * which owns the device allocator and exposes none of it, or a serving loop
 * that is not allowed to allocate device memory once it has started.
 *   - The scratch it needs (a status word and the fp32 scores) is one array
 *     compiled into the library, so every GPU that loads libv4attn holds it
 *     (about 8.4 MB) until the process exits.
 *   - Limits: n_q * max(max_vis, 1) <= V4A_NOALLOC_MAX_SCORES and
 *     n_q <= V4A_NOALLOC_MAX_QUERIES; a larger call returns
 *     V4A_ERR_UNSUPPORTED before launching anything.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 *   - Every call shares the one array, which keeps the last call's contents:
 *     the call clears the status word and rewrites every score it reads, but
 *     two calls whose work overlaps on the GPU (unordered streams, or several
 *     host threads) race on the array; the caller must order them.
 *   - Device-side check bits (out-of-range positions, which are skipped as in
 *     v4attn_index_topk, and a bounded wait that ran out, after which the
 *     selection is not valid) land in the array's status word; each call
 *     clears it first.  v4attn_noalloc_device_status reads it.
 * Arguments and results are those of v4attn_index_topk (scores_out may be
 * given; idx_out may be NULL only when scores_out is given). */
#define V4A_NOALLOC_MAX_SCORES 2097152
#define V4A_NOALLOC_MAX_QUERIES 1365
v4attn_status v4attn_index_topk_noalloc(const v4attn_layer_desc* desc,
                                        const v4attn_index_args* args, cudaStream_t stream);
/* Status word of the last v4attn_index_topk_noalloc call on the current
 * device, read and mapped as v4attn_device_status does (it synchronises
 * `stream`; order it after the call). */
v4attn_status v4attn_noalloc_device_status(cudaStream_t stream, uint32_t* bits);

/* Failure-detection test hook (no counterpart in the pages): v4attn_index_topk
 * on the MXFP4 tensor-core indexer with one of its waits made to run out.  The
 * kernel's MMA-issuing warp first waits on a barrier that nothing ever
 * completes, with every bounded wait of the launch limited to `wait_ns`
 * (1e5 .. 1e9 ns).  That wait gives up before any MMA is issued, records
 * V4A_ERR_TIMEOUT (status bit 8, and bit 16 + 12 for this wait site) in the
 * workspace's status word, and the kernel's other warps stop at their next
 * wait; the launch returns with no copy in flight and its tensor memory
 * released.  Read the result with v4attn_device_status; clear the word with
 * v4attn_workspace_init before the next call.  Arguments as v4attn_index_topk
 * (scores written by the stalled launch are undefined).  Returns
 * V4A_ERR_UNSUPPORTED for a layer whose indexer is not MXFP4. */
v4attn_status v4attn_debug_index_stall(const v4attn_layer_desc* desc,
                                       const v4attn_index_args* args, void* ws, size_t ws_bytes,
                                       uint32_t wait_ns, cudaStream_t stream);

/* Tensor-core throughput probe (measurement support; no counterpart in the
 * pages).  Launches one CTA per SM, each issuing n_iter x 4 back-to-back
 * tcgen05 MMAs of M = 128 x N = n_cols (64, 128 or 256) with operands
 * resident in shared memory
 * and fp32 accumulators in tensor memory, of kind
 *   0: kind::f16 bf16 x bf16 (K = 16),  1: kind::f8f6f4 E4M3 x E4M3 (K = 32),
 *   2: kind::mxf4 block-scaled E2M1 x E2M1, E8M0 per 32 elements (K = 64).
 * Time the launch on `stream` (e.g. with CUDA events) and divide *flops (the
 * dense FLOPs the launch performs, 2*M*N*K per MMA) by it for the GPU's MMA
 * rate of that format.  *n_ctas receives the CTA count.  `ws`: a workspace
 * whose status word receives V4A_ERR_TIMEOUT's bit if the final wait runs
 * out, or NULL.  Nothing is read or written in global memory otherwise.
 * n_iter in 1 .. 2^24 and n_cols in {64, 128, 256}, else V4A_ERR_INVALID_ARG. */
v4attn_status v4attn_tc_peak_probe(int32_t kind, int32_t n_cols, int32_t n_iter, int32_t* n_ctas,
                                   double* flops, void* ws, cudaStream_t stream);

/* Synchronise `stream`, read the status word the kernels left in `ws` and
 * map it: 0 -> V4A_OK, a bounds / argument check -> V4A_ERR_DEVICE_CHECK,
 * a bounded wait that ran out -> V4A_ERR_TIMEOUT.  *bits (if not NULL)
 * receives the raw word.  The word is not cleared. */
v4attn_status v4attn_device_status(const void* ws, cudaStream_t stream, uint32_t* bits);

const char* v4attn_status_string(v4attn_status s);

/* The description of the last CUDA error behind a V4A_ERR_CUDA return on the
 * calling host thread ("no error" when there was none). */
const char* v4attn_last_cuda_error(void);

/* Library build identification (kernel variants compiled in). */
const char* v4attn_build_info(void);

#ifdef __cplusplus
}
#endif
#endif /* V4ATTN_H */
