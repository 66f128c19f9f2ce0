// Shared-KV MQA on the 5th-generation tensor cores (tcgen05): each query's H
// heads against its selected (CSA) or visible (HCA) compressed entries and its
// window tokens, softmax with a per-head sink, inverse RoPE on the output.
//
// Method: "DeepSeek-V4 深读" (ricardokevins.github.io), model-spec table (64 /
// 128 query heads of dim 512 over one shared KV head) and section
// "其他稳定性细节" (448 FP8 + 64 BF16 RoPE dims, sink, inverse RoPE on the
// output); "拆解 DeepSeekv4", section "细节".
//
// Layout of the work.  Each query is coded once (RoPE at its position on dims
// 448..511, E4M3 with a power-of-two scale on dims 0..447) straight into the
// swizzled shared-memory image the MMAs read, by a small pre-kernel or, in the
// decode step, by the append kernel that runs before it; every CTA of the
// query copies that image in with bulk copies.  A CTA owns (query, one of C
// key splits, half of the 512 output dims).  Output dims are split because
// fp32 O for 128 heads x 512 dims is all of TMEM (512 columns x 128 lanes):
// each CTA keeps O[128 x 256] in TMEM columns 256..511 and S for two 64-key
// tiles in columns 0..255, and recomputes S = Q K^T (the two halves of a split
// run on neighbouring CTAs, so the second read of its rows comes from L2).
// With few queries C > 1 key splits per (query, half) keep every SM busy; the
// launch is then cooperative and the splits merge through L2 after one grid
// barrier.
//
// Per 64-key tile:
//   S_nope = Q_nope(E4M3) . K_nope(E4M3)^T   14 x tcgen05.mma kind::f8f6f4, K=32
//   S_rope = Q_rope(BF16) . K_rope(BF16)^T    4 x tcgen05.mma kind::f16,   K=16
//   s_j    = scale * (q_scale * k_scale_j * S_nope + S_rope)       (log2 units)
//   P_j    = exp2(s_j - M_s)                                        (f16, in TMEM)
//   V_j    = k_scale_j * code_j (dims < 448), bf16 RoPE dims        (f16, in smem)
//   O     += P V                                 4 x tcgen05.mma kind::f16, K=16, N=256
// M_s is the row's running score maximum, moved only when a tile beats it by
// more than tau = 4, so P <= 2^tau; O is rescaled in TMEM only when M_s moves.
// V in f16 is exact for stored values of magnitude 2^-14 .. 65504 (an entry
// scale times an E4M3 code has four significant bits); P in f16 carries 11
// significant bits, and the row sum is taken over those f16 values.
//
// Rows arrive by TMA: tile mode for contiguous HCA entries, tile::gather4 (4
// rows per instruction) for selected entries and window tokens; the entry
// scales by 4-byte cp.async.  Roles: warp 0 loads, warp 1 issues the
// MMAs (one lane), warps 2..17 run the softmax, the conversion of V to f16
// and the epilogue: four warps per TMEM lane quarter, one per 16-key group of
// each tile, exchanging row maxima through shared memory.  Every cross-warp
// hand-off is an mbarrier with a bounded, warp-uniform wait, and the grid
// barrier is bounded too, so a stalled kernel ends with a status bit.
#include <algorithm>
#include <cstddef>

#include "common.cuh"
#include "kernels.h"
#include "mqa_qimage.cuh"
#include "tc_common.cuh"
#include "tc_kernels.h"

namespace v4a {

namespace {

constexpr int NK = 64;          // keys per tile
constexpr int KST = 3;          // tile stages in flight
constexpr int KG = 4;           // key groups per tile = softmax warps per TMEM lane quarter
constexpr int KPG = 64 / KG;    // keys per group
constexpr int NSM = 4 * KG;     // softmax / epilogue warps
constexpr int NTHR = 64 + 32 * NSM;
constexpr int ROWB = 576;       // stored row: 448 E4M3 + 64 bf16
constexpr int TILE_BYTES = NK * (4 * 128 + 64);
constexpr float kTau = 4.f;     // lazy-rescale margin of the running score maximum (log2 units)
// query image (layout in mqa_qimage.cuh)
constexpr int Q_NOPE3 = kQImgNope3, Q_ROPE = kQImgRope, QTILE = kQImgTile;
constexpr int QIMG = kQImgBytes;
static_assert(kQImgBytes <= kMqaQImageStride, "query image stride");
constexpr int QCHUNK = QIMG / 4;
static_assert(QCHUNK % 16 == 0, "bulk copies move multiples of 16 bytes");

struct Smem {
  alignas(1024) uint8_t q[QTILE];
  float qsc[128];                             // contiguous with q: one image
  alignas(1024) uint8_t kv[KST][4][NK * 128]; // nope blocks 0..2 and the rope block, SW128
  alignas(1024) uint8_t kv3[KST][NK * 64];    // nope bytes 384..447, SW64
  // V of the tile in f16 (values = code x entry scale; RoPE dims converted
  // from bf16) for this CTA's 256 output dims: four MN-major SW128 blocks of
  // 64 dims x NK keys, the B operand of P V
  alignas(1024) uint8_t v16[4][NK * 128];
  alignas(16) float kscale[KST][NK];
  union {
    float xmax[2][KG][128];                   // tile loop: [tile parity][key group][row]
    struct {                                  // merge (the loop is over for every warp):
      float rms[128], rl[128];                // this split's row max (log2), row sum
      float fself[128], invl[128];            // merge factor of this split, 1 / denominator
    } mg;
  };
  float rcs[2][32], rsn[2][32];               // RoPE angles of the query positions (dh = 1)
  int bar_ok;                                 // the grid barrier's outcome, for the whole CTA
  float xl[KG - 1][128];                      // the other groups' row sums, for the epilogue
  uint64_t full[KST], empty[KST], sfull[2], pfull[2], pdone[2], xbar[4][2];
  uint64_t qready, ofinal, done, lbar;
  uint32_t tmem_base;
};

static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory per CTA");
static_assert(offsetof(Smem, qsc) == QTILE, "the query image is one contiguous copy");
// the merge stages this split's O / l (f16, 128 rows of SSTB bytes) over the
// query image and the key stages, which are free once the last P.V has completed
constexpr int SSTB = 528;                    // staged f16 row stride (bytes): conflict-free 16-byte rows
constexpr int kMaxSplit = 64;                // key splits per (query, half), at most
constexpr int kMinSplitTiles = 3;            // dense calls: key tiles per split, at least
constexpr int kWinCost = 2;                  // a gathered window tile costs about two contiguous ones
constexpr int kFastSplits = 24;              // merges of at most this many splits load in one flight
static_assert(offsetof(Smem, kscale) >= 128 * SSTB, "merge stage fits");
static_assert(offsetof(Smem, kscale) >= 2 * kMaxSplit * 128 * 4, "merge factors fit");
// TMEM column of P (f16, two keys a column, 32 columns) inside a tile's
// 128-column S buffer, written after the buffer's S has been read
constexpr uint32_t PC_F16 = 0;

struct Maps {
  CUtensorMap kv128, kv64;      // tile mode, boxes {128 B | 64 B} x NK rows
  CUtensorMap kvg128, kvg64;    // tile::gather4 over entry rows, boxes one row high
  CUtensorMap swg128, swg64;    // tile::gather4 over window rows
};

// Four rows (r0..r3, 4 x the box width) into consecutive rows of a swizzled
// tile.  The swizzle follows the absolute shared-memory address, so a group
// may start in the middle of an 8-row swizzle atom (rows 4..7 at +512 bytes
// for 128-byte rows, checked on B200).
__device__ __forceinline__ void gather4(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                        int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(r0), "r"(r1),
      "r"(r2), "r"(r3)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// 32 lanes x 8 consecutive columns from registers
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                   taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}
// MMA whose A operand is read from tensor memory (M = 128 rows at lanes
// 0..127, K along the columns: two 16-bit elements a column)
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// two E4M3 codes (low byte first) -> f16x2, exact, times the f16x2 scale
__device__ __forceinline__ uint32_t e4m3x2_f16x2_scaled(uint32_t c, __half2 sc) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(c & 0xFFFFu), __NV_E4M3);
  const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&h), sc);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// two bf16 (low half first) -> f16x2 (round to nearest even)
__device__ __forceinline__ uint32_t bf16x2_f16x2(uint32_t w) {
  const __half2 v = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  return *reinterpret_cast<const uint32_t*>(&v);
}
// 16 E4M3 codes (one 16-byte chunk) -> 16 f16 values scaled by sc, as 2 x 16 bytes
__device__ __forceinline__ void e4m3x16_f16(const uint4 c, __half2 sc, uint4& lo, uint4& hi) {
  lo.x = e4m3x2_f16x2_scaled(c.x, sc);
  lo.y = e4m3x2_f16x2_scaled(c.x >> 16, sc);
  lo.z = e4m3x2_f16x2_scaled(c.y, sc);
  lo.w = e4m3x2_f16x2_scaled(c.y >> 16, sc);
  hi.x = e4m3x2_f16x2_scaled(c.z, sc);
  hi.y = e4m3x2_f16x2_scaled(c.z >> 16, sc);
  hi.z = e4m3x2_f16x2_scaled(c.w, sc);
  hi.w = e4m3x2_f16x2_scaled(c.w >> 16, sc);
}
// 2^x by the SFU (ex2.approx, flush to zero; 2^-inf = 0)
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// V of the tile in stage st into s.v16 for this CTA's 256 output dims
// (dh * 256 ..), by the 512 softmax threads (ctid = 0..511), one 16-byte
// source chunk (16 E4M3 codes or 8 bf16 of one key) at a time.  The E4M3 codes
// are scaled by the entry's scale (a power of two; zero for an empty slot).
template <typename SmemT>
__device__ __forceinline__ void convert_v(SmemT& s, int st, int dh, int ctid) {
  if (dh == 0) {
    // dims 0..255: blocks 0 and 1 of the stage, 16 chunks a key
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int u = ctid + 512 * i;
      const int k = u >> 4, c16 = u & 15;
      const uint4 c = *reinterpret_cast<const uint4*>(s.kv[st][c16 >> 3] + sw128(k, (c16 & 7) * 16));
      const __half2 sc = __float2half2_rn(s.kscale[st][k]);
      uint4 lo, hi;
      e4m3x16_f16(c, sc, lo, hi);
      uint8_t* blk = s.v16[c16 >> 2];            // output dims 16 c16 .. + 15
      const int nb = (c16 & 3) * 32;
      *reinterpret_cast<uint4*>(blk + sw128(k, nb)) = lo;
      *reinterpret_cast<uint4*>(blk + sw128(k, nb + 16)) = hi;
    }
  } else {
    // dims 256..383 (block 2), 384..447 (the SW64 block), RoPE 448..511
    // (block 3, bf16): 20 chunks a key
    for (int u = ctid; u < NK * 20; u += 512) {
      const int k = u / 20, w = u - k * 20;
      if (w < 12) {
        const uint4 c = w < 8 ? *reinterpret_cast<const uint4*>(s.kv[st][2] + sw128(k, w * 16))
                              : *reinterpret_cast<const uint4*>(s.kv3[st] + sw64(k, (w - 8) * 16));
        const __half2 sc = __float2half2_rn(s.kscale[st][k]);
        uint4 lo, hi;
        e4m3x16_f16(c, sc, lo, hi);
        uint8_t* blk = s.v16[w >> 2];            // output dims 16 w .. + 15
        const int nb = (w & 3) * 32;
        *reinterpret_cast<uint4*>(blk + sw128(k, nb)) = lo;
        *reinterpret_cast<uint4*>(blk + sw128(k, nb + 16)) = hi;
      } else {
        const int r = w - 12;                    // dims 448 + 8 r .. + 7
        const uint4 b = *reinterpret_cast<const uint4*>(s.kv[st][3] + sw128(k, r * 16));
        const uint4 o = make_uint4(bf16x2_f16x2(b.x), bf16x2_f16x2(b.y), bf16x2_f16x2(b.z),
                                   bf16x2_f16x2(b.w));
        *reinterpret_cast<uint4*>(s.v16[3] + sw128(k, r * 16)) = o;
      }
    }
  }
}

struct Geo {
  int b;
  int64_t p, n_vis;
  int n_main, n_swa, nmp, total, s0, T;
  // pairs: the two queries' positions and visible entries (rows 0..63 / 64..127)
  int64_t pq[2], nq[2];
};

// Position and visible entries of query q, checked against the call's bounds
// (PAGED: a sequence holds at most its table's blocks of entries).
template <bool PAGED>
__device__ __forceinline__ void query_span(const MqaParams& P, int q, int& b, int64_t& p,
                                           int64_t& nv) {
  b = P.q_seq ? P.q_seq[q] : P.q_base + q;
  p = P.q_pos[q];
  nv = (p + 1) / P.m;
  if (b < 0 || b >= P.B) {
    if (threadIdx.x == 0) flag(P.status, ST_BAD_SEQ);
    b = 0;
    nv = 0;
    p = -1;
  }
  const int64_t cap = PAGED ? (int64_t)P.pages.bps * P.pages.epb : P.kv_rows;
  if (nv > cap) {
    if (threadIdx.x == 0) flag(P.status, ST_BAD_POSITION);
    nv = cap;
  }
  if (!P.idx && nv > P.max_vis) {
    if (threadIdx.x == 0) flag(P.status, ST_BAD_POSITION);
    nv = P.max_vis;
  }
}

// q: the query, or with P.pair the pair (queries 2q, 2q + 1 of one sequence:
// the union of their visible entries and of their windows, each row masked to
// its own query's in the softmax)
template <bool PAIR, bool PAGED>
__device__ __forceinline__ Geo geometry(const MqaParams& P, int q, int split) {
  Geo g;
  if (PAIR) {
    int b1;
    query_span<PAGED>(P, 2 * q, g.b, g.pq[0], g.nq[0]);
    query_span<PAGED>(P, 2 * q + 1, b1, g.pq[1], g.nq[1]);
    if (b1 != g.b) {
      if (threadIdx.x == 0) flag(P.status, ST_BAD_SEQ);
      g.nq[1] = 0;
      g.pq[1] = -1;
    }
    g.p = max(g.pq[0], g.pq[1]);
    g.n_vis = max(g.nq[0], g.nq[1]);
    const int64_t lo = max((int64_t)0, min(g.pq[0], g.pq[1]) - P.n_win + 1);
    g.n_main = (int)g.n_vis;
    g.n_swa = g.p >= 0 ? (int)(g.p - lo + 1) : 0;
  } else {
    query_span<PAGED>(P, q, g.b, g.p, g.n_vis);
    g.pq[0] = g.pq[1] = g.p;
    g.nq[0] = g.nq[1] = g.n_vis;
    g.n_main = P.idx ? P.n_sel : (int)g.n_vis;
    g.n_swa = (int)min((int64_t)P.n_win, g.p + 1);
  }
  if (g.n_swa < 0) g.n_swa = 0;
  g.nmp = (g.n_main + NK - 1) / NK * NK;
  g.total = g.nmp + (g.n_swa + NK - 1) / NK * NK;
  // The query's tiles, entries first then window tokens, are split by cost:
  // a window tile (rows gathered from the ring) counts kWinCost entry tiles
  // of a dense call (contiguous rows, one tile-mode copy each); in a sparse
  // call every tile is gathered and counts one.  Split `split` of C takes
  // the tiles whose cost prefix starts in [W split / C, W (split + 1) / C).
  const int mt = g.nmp / NK, wt = (g.total - g.nmp) / NK, C = P.n_split;
  const int wc = (PAGED || P.idx) ? 1 : kWinCost;   // paged entries are gathered too
  const int64_t W = mt + (int64_t)wc * wt;
  auto tile_at = [&](int64_t x) -> int {        // first tile whose cost prefix is >= x
    return (int)(x <= mt ? x : mt + (x - mt + wc - 1) / wc);
  };
  const int t0 = tile_at(W * split / C), t1 = tile_at(W * (split + 1) / C);
  g.s0 = t0 * NK;
  g.T = t1 - t0;
  return g;
}

}  // namespace

// Eight CTAs per query (16 head rows each, so that a query's 128 KB of bf16 Q
// is read by eight SMs): the query image of the main kernel.
__global__ void __launch_bounds__(64) mqa_tc_qprep_kernel(MqaParams P) {
  __shared__ float cs[32], sn[32];
  // pairs: image blockIdx.x holds query 2x in rows 0..63, 2x + 1 in rows 64..127
  const int second = (P.pair && blockIdx.y >= 4) ? 1 : 0;
  const int q = P.pair ? 2 * blockIdx.x + second : blockIdx.x;
  qimage_code_rows(reinterpret_cast<const __nv_bfloat16*>(P.Q) + (int64_t)q * P.H * 512, P.H,
                   P.q_pos[q], P.theta, P.qbuf + (int64_t)blockIdx.x * kMqaQImageStride, blockIdx.y, cs, sn,
                   P.q_rmsnorm != 0, P.eps, second ? 64 : 0);
}

// 576 threads = 18 warps: on the SM sub-partition that holds five of them at
// most 16384 / 5 registers a warp, hence 96 registers a thread
// PAIR: two consecutive queries of one sequence per CTA (see MqaParams::pair).
// PAGED: entry rows through the block table (P.pages), every main tile
// gathered; a compile-time switch, so that the per-sequence kernel carries
// none of it
template <bool PAIR, bool PAGED>
__global__ void __launch_bounds__(NTHR, 1)
    mqa_tc_kernel(MqaParams P, const __grid_constant__ Maps maps) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTAs unit * C .. unit * C + C - 1 are the key splits of one (query, half)
  const int C = P.n_split;
  const int split = (int)(blockIdx.x % (unsigned)C);
  const int unit = (int)(blockIdx.x / (unsigned)C);
  const int dh = unit & 1, q = unit >> 1;
  const Geo g = geometry<PAIR, PAGED>(P, q, split);
  // the grid barrier's generation before this CTA arrives (merging launches)
  const uint32_t bar_gen0 = (C > 1 && threadIdx.x == 0) ? ld_acquire_gpu(P.grid_bar + 1) : 0u;
  // every CTA, also one with no tiles (T = 0), takes part in the merge below

  if (threadIdx.x == 0) {
    for (int i = 0; i < KST; ++i) {
      mbar_init(&s.full[i], 32);   // the producer lanes' scale arrivals + TMA bytes
      mbar_init(&s.empty[i], NSM);   // every softmax warp, done with the stage
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.sfull[i], 1);     // QK of the buffer's tile done (one commit)
      mbar_init(&s.pfull[i], NSM);   // every softmax warp wrote its P of the tile
      mbar_init(&s.pdone[i], 1);     // PV of the buffer's tile done (one commit)
      for (int qd = 0; qd < 4; ++qd) mbar_init(&s.xbar[qd][i], KG);   // the quarter's key groups
    }
    mbar_init(&s.qready, 1);
    mbar_init(&s.ofinal, 1);
    mbar_init(&s.done, 1);
    mbar_init(&s.lbar, NSM - 4);
    fence_mbar_init();
    // the query image by four bulk copies on qready, issued before the CTA's
    // first barrier so that it overlaps the TMEM allocation and the set-up
    const uint8_t* qimg = P.qbuf + (int64_t)q * kMqaQImageStride;
    mbar_arrive_expect_tx(&s.qready, QIMG);
    for (int k = 0; k < 4; ++k) bulk_load(s.q + k * QCHUNK, qimg + k * QCHUNK, QCHUNK, &s.qready);
  }
  if (warp == 1) tmem_alloc(&s.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    // (The query image is already on its way: thread 0 issued it with the
    // barriers.)  Entry / window rows by TMA (complete_tx bytes on full[st]);
    // the 64 entry scales by cp.async,
    // zero-filled for empty slots (a stored scale is a nonzero power of two,
    // so a zero scale marks an empty slot); every lane arrives on full[st]
    // through cp.async.mbarrier.arrive.noinc once its scale copies land.
    // paged entries: rows of the pool (through the block table), else of
    // this sequence's part of the cache
    const int64_t kv_base = PAGED ? 0 : (int64_t)g.b * P.kv_rows;
    const int64_t sw_base = (int64_t)g.b * P.swa_rows;
    // global row of key r of tile vk, or -1 when the slot is empty
    auto row_of = [&](int vk, int r, bool main_tile) -> int64_t {
      if (main_tile) {
        const int jj = vk + r;
        if (jj >= g.n_main) return -1;
        const int e = P.idx ? P.idx[(int64_t)q * P.n_sel + jj] : jj;   // -1: an empty slot
        if (e < 0) return -1;
        if (e >= g.n_vis) {
          flag(P.status, ST_BAD_INDEX);
          return -1;
        }
        if constexpr (PAGED) {
          const int64_t row = page_row(P.pages, g.b, e);
          if (row < 0) flag(P.status, ST_BAD_INDEX);
          return row;
        }
        return kv_base + e;
      }
      const int w = vk - g.nmp + r;
      if (w >= g.n_swa) return -1;
      const int64_t tok = g.p - g.n_swa + 1 + w;
      return sw_base + tok % P.swa_rows;
    };
    bool issued_ok = true;
    int issued = 0;
    for (int t = 0; t < g.T; ++t) {
      const int st = t % KST, u = t / KST;
      if (u >= 1 && !mbar_wait_warp(&s.empty[st], (u - 1) & 1, P.status, 0)) {
        issued_ok = false;
        break;
      }
      issued = t + 1;
      const int vk = g.s0 + t * NK;
      const bool main_tile = vk < g.nmp;
      const bool contiguous = !PAGED && main_tile && !P.idx && vk + NK <= g.n_main;
      if (lane == 0) mbar_expect_tx(&s.full[st], TILE_BYTES);
      __syncwarp();
      if (contiguous) {
        if (lane == 0) {
          const int y = (int)(kv_base + vk);
          tma_load_2d(s.kv[st][0], &maps.kv128, &s.full[st], 0, y);
          tma_load_2d(s.kv[st][1], &maps.kv128, &s.full[st], 128, y);
          tma_load_2d(s.kv[st][2], &maps.kv128, &s.full[st], 256, y);
          tma_load_2d(s.kv3[st], &maps.kv64, &s.full[st], 384, y);
          tma_load_2d(s.kv[st][3], &maps.kv128, &s.full[st], 448, y);
        }
      } else if (lane < NK / 4) {
        // 4 rows per tile::gather4 (box one row high); an empty slot repeats
        // a valid row (its scale is zero-filled, which marks it empty)
        int rows[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int64_t row = row_of(vk, lane * 4 + k, main_tile);
          rows[k] = (int)(row >= 0 ? row : (main_tile ? kv_base : sw_base));
        }
        const CUtensorMap* m128 = main_tile ? &maps.kvg128 : &maps.swg128;
        const CUtensorMap* m64 = main_tile ? &maps.kvg64 : &maps.swg64;
        const int o128 = lane * 4 * 128, o64 = lane * 4 * 64;
        gather4(s.kv[st][0] + o128, m128, &s.full[st], 0, rows[0], rows[1], rows[2], rows[3]);
        gather4(s.kv[st][1] + o128, m128, &s.full[st], 128, rows[0], rows[1], rows[2], rows[3]);
        gather4(s.kv[st][2] + o128, m128, &s.full[st], 256, rows[0], rows[1], rows[2], rows[3]);
        gather4(s.kv3[st] + o64, m64, &s.full[st], 384, rows[0], rows[1], rows[2], rows[3]);
        gather4(s.kv[st][3] + o128, m128, &s.full[st], 448, rows[0], rows[1], rows[2], rows[3]);
      }
      // entry scales (zero for an empty slot), then this lane's arrival, which
      // fires once its scale copies have landed
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int r = lane + 32 * k;
        const int64_t row = row_of(vk, r, main_tile);
        const float* src = (main_tile ? P.kv_scale : P.swa_scale) + (row >= 0 ? row : 0);
        cp_async4(&s.kscale[st][r], src, row >= 0);
      }
      cp_async_arrive_noinc(&s.full[st]);
    }
    cp_async_wait<0>();
    if (!issued_ok) flag(P.status, ST_TIMEOUT);
    // drain: no copy may still be landing when the merge reuses the stages (or
    // the CTA exits); on a normal run these phases completed long ago
    if (lane == 0) {
      mbar_wait(&s.qready, 0);                                      // time bound only
      for (int k = 0; k < KST && k < issued; ++k) {
        const int i2 = issued - 1 - k;
        mbar_wait(&s.full[i2 % KST], (i2 / KST) & 1);
      }
    }
    __syncwarp();
    // the angles of the output's inverse RoPE (dims 448..511, one pair a
    // lane), computed here while the other warps still work through the tiles
    if (dh == 1) {
      for (int u = 0; u < (PAIR ? 2 : 1); ++u) {
        float c = 1.f, sv = 0.f;
        if (g.pq[u] >= 0) rope_cs(g.pq[u], lane, 64, P.theta, c, sv);
        s.rcs[u][lane] = c;
        s.rsn[u][lane] = sv;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    const uint64_t kq128 = smem_desc_bits(16, 1024, 2);   // K-major, 128B swizzle
    const uint64_t kq64 = smem_desc_bits(16, 512, 4);     // K-major, 64B swizzle
    const uint64_t mn128 = smem_desc_bits(NK * 128, 1024, 2);  // MN-major, 128B swizzle, 8 KB blocks
    const uint32_t id_qk8 = idesc_f(0, 0, 128, NK, false, false);
    const uint32_t id_qk16 = idesc_f(1, 1, 128, NK, false, false);
    const uint32_t id_pv = idesc_f(0, 0, 128, 256, false, true);   // f16 x f16, B MN-major
    const uint32_t O = tmem + 256;
    bool ok = mbar_wait_warp(&s.qready, 0, P.status, 1);
    // P.V of tile tt: A = P (f16) of the tile, read from its TMEM buffer
    // (tt & 1, written there by the softmax), B = the tile's V in f16
    // (s.v16, converted by the softmax warps), N = this CTA's 256 dims
    auto pv = [&](int tt) -> bool {
      const int a = tt & 1;
      if (!mbar_wait_warp(&s.pfull[a], (tt >> 1) & 1, P.status, 2)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t pb = tmem + a * 128 + PC_F16;
        const uint64_t bv = smem_desc(s.v16[0], mn128);
        for (int ks = 0; ks < 4; ++ks)                        // 16 keys (8 columns) a step
          mma_f16_ts(O, pb + 8 * ks, bv + (uint64_t)(ks * 16 * 128 >> 4), id_pv, (tt | ks) != 0);
        tc_commit(&s.pdone[a]);
      }
      __syncwarp();
      return true;
    };
    // Issue order QK(t), PV(t-1), QK(t+1), PV(t), ...: the tensor pipe runs
    // QK(t+1) while the softmax works on tile t.  QK(t) overwrites the TMEM
    // buffer of tile t-2, whose PV was issued earlier by this thread (tcgen05
    // MMAs of one thread execute in issue order).
    for (int t = 0; t < g.T && ok; ++t) {
      const int st = t % KST, a = t & 1;
      if (!mbar_wait_warp(&s.full[st], (t / KST) & 1, P.status, 3)) { ok = false; break; }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t Sn = tmem + a * 128, Sr = Sn + 64;
        for (int kb = 0; kb < 3; ++kb) {
          const uint64_t aq = smem_desc(s.q + kb * 16384, kq128), bk = smem_desc(s.kv[st][kb], kq128);
          for (int ks = 0; ks < 4; ++ks)
            mma_f8f6f4(Sn, aq + 2 * ks, bk + 2 * ks, id_qk8, (kb | ks) != 0);
        }
        {
          const uint64_t aq = smem_desc(s.q + Q_NOPE3, kq64), bk = smem_desc(s.kv3[st], kq64);
          for (int ks = 0; ks < 2; ++ks) mma_f8f6f4(Sn, aq + 2 * ks, bk + 2 * ks, id_qk8, 1);
        }
        {
          const uint64_t aq = smem_desc(s.q + Q_ROPE, kq128), bk = smem_desc(s.kv[st][3], kq128);
          for (int ks = 0; ks < 4; ++ks) mma_f16(Sr, aq + 2 * ks, bk + 2 * ks, id_qk16, ks != 0);
        }
        tc_commit(&s.sfull[a]);
      }
      __syncwarp();
      if (t >= 1 && !pv(t - 1)) { ok = false; break; }
    }
    if (ok && g.T > 0) ok = pv(g.T - 1);
    if (!ok) flag(P.status, ST_TIMEOUT);
    if (lane == 0) {
      tc_commit(&s.ofinal);
      tc_commit(&s.done);
      if (!mbar_wait(&s.done, 0)) flag(P.status, ST_TIMEOUT | (1u << (16 + 5)));   // time bound only
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;          // keys grp*KPG .. +KPG-1 of each tile
    const int h = quad * 32 + lane;           // head row == TMEM lane
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float sl2 = P.scale * 1.4426950408889634f;     // softmax scale x log2(e)
    // Ms: the row's running score maximum (log2 units), moved only when a tile
    // exceeds it by more than kTau, so P <= 2^kTau (well inside f16's range).
    float Ms = -INFINITY, l = 0.f;
    bool wrote = false;                                  // O holds a PV result
    bool live = mbar_wait_warp(&s.qready, 0, P.status, 1);
    const float qs = s.qsc[h];
    const int ctid = (warp - 2) * 32 + lane;             // 0 .. 511: share of the V conversion
    // pairs: this row's query (rows 64..127 the second): its visible entries
    // and its window [p - n_win + 1, p] among the pair's union
    const int rq = (PAIR && h >= 64) ? 1 : 0;
    const int64_t lim_e = g.nq[rq], w_lo = g.pq[rq] - P.n_win + 1, w_hi = g.pq[rq];
    const int64_t tok0 = g.p - g.n_swa + 1 - g.nmp;      // window token of key vk + g.nmp .. is tok0 + vk
    for (int t = 0; t < g.T && live; ++t) {
      const int a = t & 1, st = t % KST, xb = t & 1;
      if (!mbar_wait_warp(&s.sfull[a], (t >> 1) & 1, P.status, 6) ||
          !mbar_wait_warp(&s.full[st], (t / KST) & 1, P.status, 7)) {
        live = false;
        break;
      }
      tc_fence_after();
      uint32_t sn_[KPG], sr_[KPG];
      const uint32_t tb = tmem + lane_off + a * 128;     // this tile's TMEM buffer
      tmem_ld16_nowait(tb + grp * KPG, sn_);
      tmem_ld16_nowait(tb + 64 + grp * KPG, sr_);
      float ksc[KPG];
#pragma unroll
      for (int j = 0; j < KPG; j += 4)
        *reinterpret_cast<float4*>(&ksc[j]) =
            *reinterpret_cast<const float4*>(&s.kscale[st][grp * KPG + j]);
      tmem_ld_wait();
      float s2[KPG];
      float ms = -INFINITY;
#pragma unroll
      for (int j = 0; j < KPG; ++j) {
        const float kj = ksc[j];
        const float v = (qs * kj * __uint_as_float(sn_[j]) + __uint_as_float(sr_[j])) * sl2;
        s2[j] = (kj != 0.f) ? v : -INFINITY;             // a zero scale marks an empty slot
      }
      if (PAIR) {                                      // uniform: the row's own query only
        const int vk = g.s0 + t * NK + grp * KPG;
#pragma unroll
        for (int j = 0; j < KPG; ++j) {
          const bool ok = vk + j < g.nmp ? (vk + j < lim_e)
                                         : (tok0 + vk + j >= w_lo && tok0 + vk + j <= w_hi);
          if (!ok) s2[j] = -INFINITY;
        }
      }
#pragma unroll
      for (int j = 0; j < KPG; ++j) ms = fmaxf(ms, s2[j]);
      // the tile's row maximum: exchanged with the other key groups of the
      // same TMEM lane quarter (the same head rows); past this exchange every
      // group has read its S columns, so P may overwrite them
      s.xmax[xb][grp][h] = ms;
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.xbar[quad][xb]);
      if (!mbar_wait_warp(&s.xbar[quad][xb], (t >> 1) & 1, P.status, 10)) {
        live = false;
        break;
      }
#pragma unroll
      for (int o = 0; o < KG; ++o) ms = fmaxf(ms, s.xmax[xb][o][h]);
      const bool upd = ms > Ms + kTau;
      const float Ms_new = upd ? ms : Ms;
      const float as = (upd && Ms != -INFINITY) ? ex2f(Ms - Ms_new) : 1.f;
      const float ms_ref = (Ms_new == -INFINITY) ? 0.f : Ms_new;
      // P = exp2(s - Ms) in f16 (the A operand of P V); the row sum is taken
      // over the f16 values, i.e. the weights P V really applies
      float lsum = 0.f;
      uint32_t ph[KPG / 2];
#pragma unroll
      for (int j = 0; j < KPG; j += 2) {
        const __half2 hp = __floats2half2_rn(ex2f(s2[j] - ms_ref), ex2f(s2[j + 1] - ms_ref));
        const float2 pf = __half22float2(hp);
        lsum += pf.x + pf.y;
        ph[j >> 1] = *reinterpret_cast<const uint32_t*>(&hp);
      }
      l = l * as + lsum;
      // the previous tile's P.V has completed: O may be rescaled and the f16
      // V buffer rewritten
      if (t >= 1 && !mbar_wait_warp(&s.pdone[(t - 1) & 1], ((t - 1) >> 1) & 1, P.status, 8)) {
        live = false;
        break;
      }
      tc_fence_after();
      // Rescale this warp's share of O (columns grp*64 .. +63) when the row's
      // reference moved.  tcgen05.ld / st are warp-wide (.sync.aligned): the
      // decision is taken per warp, every lane takes part with its own factor.
      if (__any_sync(0xffffffffu, wrote && as < 1.f)) {
        const uint32_t ob = tmem + lane_off + 256;
#pragma unroll 1
        for (int cc = 0; cc < 256 / KG; cc += 32) {
          const int c = grp * (256 / KG) + cc;
          uint32_t r[32];
          tmem_ld32_nowait(ob + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * as);
          tmem_st32(ob + c, r);
        }
      }
      Ms = Ms_new;
      // this group's 16 keys of P into the tile's TMEM buffer (columns
      // PC_F16 + 8 grp ..), and this thread's share of the tile's V in f16;
      // then the stage goes back to the producer (V converted, scales read)
      tmem_st8(tb + PC_F16 + 8 * grp, ph);
      convert_v(s, st, dh, ctid);
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.empty[st]);
      fence_proxy_async_smem();                          // V16 visible to the tensor core
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.pfull[a]);
      wrote = true;
    }
    if (!live) flag(P.status, ST_TIMEOUT);
    bool fin = mbar_wait_warp(&s.ofinal, 0, P.status, 9);
    tc_fence_after();
    // row sums of all key groups
    if (grp > 0) {
      s.xl[grp - 1][h] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.lbar);
    } else {
      fin = mbar_wait_warp(&s.lbar, 0, P.status, 11) && fin;
#pragma unroll
      for (int o = 0; o < KG - 1; ++o) l += s.xl[o][h];
    }
    fin = fin && live;
    // this split's per-row results for the merge: the row maximum (log2 units;
    // -inf for no key) and the row sum, O and the sum both in units of exp2(. - Ms)
    if (grp == 0) {
      const bool any = fin && Ms != -INFINITY;
      s.mg.rms[h] = any ? Ms : -INFINITY;
      s.mg.rl[h] = any ? l : 0.f;
    }
  }

  // ------------------------------------------------------------ merge the C splits
  // C == 1: the output straight from TMEM.  C > 1 (a cooperative launch, every
  // CTA resident): each split writes its O, in units of exp2(. - its row
  // maximum), and its row maxima / sums to the workspace (L2-resident), all
  // CTAs meet at one grid barrier, then CTA `split` reduces column groups
  // [64 split / C, 64 (split + 1) / C) (four columns each) of its (query, half)
  // over the C partials and writes them.  Every thread passes the barriers
  // below exactly once (the roles above have no early exit).
  const int tid = threadIdx.x;
  tc_fence_before();
  __syncthreads();
  const float log2e = 1.4426950408889634f;
  // the output (query, head) of TMEM lane / image row hh
  auto row_q = [&](int hh) -> int64_t { return PAIR ? 2 * (int64_t)q + (hh >> 6) : q; };
  auto row_h = [&](int hh) -> int { return PAIR ? (hh & 63) : hh; };
  uint8_t* stage = &s.q[0];                             // q .. kv3: free, every MMA / copy is done
  float* fac = reinterpret_cast<float*>(stage);         // [C][128] row factors (after the copy-out)
  float* lsp = fac + C * 128;                           // [C][128] row sums
  bool merge_ok = true;
  if (C > 1) {
    // (1) this split's O / l (a weighted mean of V rows: inside f16's range)
    // as f16 rows of SSTB bytes
    if (warp >= 2) {
      const int quad = warp & 3, grp = (warp - 2) >> 2;
      const int hh = quad * 32 + lane;
      const uint32_t ob = tmem + ((uint32_t)(quad * 32) << 16) + 256;
      const float lr = s.mg.rl[hh];
      const float il = lr > 0.f ? 1.f / lr : 0.f;
#pragma unroll 1
      for (int cc = 0; cc < 256 / KG; cc += 32) {
        const int c = grp * (256 / KG) + cc;
        uint32_t r[32];
        tmem_ld32_nowait(ob + c, r);
        tmem_ld_wait();
        uint32_t hv[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const __half2 hp = __floats2half2_rn(__uint_as_float(r[2 * k]) * il,
                                               __uint_as_float(r[2 * k + 1]) * il);
          hv[k] = *reinterpret_cast<const uint32_t*>(&hp);
        }
        uint4* dst = reinterpret_cast<uint4*>(stage + hh * SSTB + c * 2);
#pragma unroll
        for (int k = 0; k < 4; ++k) dst[k] = make_uint4(hv[4 * k], hv[4 * k + 1], hv[4 * k + 2], hv[4 * k + 3]);
      }
    }
    __syncthreads();
    // (2) to this CTA's partial: [128][256] f16, then [row max | row sum][128] fp32
    uint4* po = reinterpret_cast<uint4*>(P.part_o) + (int64_t)blockIdx.x * (128 * 256 / 8);
    float* pm = P.part_ml + (int64_t)blockIdx.x * 256;
    for (int i = tid; i < 128 * 32; i += NTHR)
      __stcg(po + i, *reinterpret_cast<const uint4*>(stage + (i >> 5) * SSTB + (i & 31) * 16));
    if (tid < 128) {
      __stcg(pm + tid, s.mg.rms[tid]);
      __stcg(pm + 128 + tid, s.mg.rl[tid]);
    }
    __syncthreads();
    // (3) every split of every (query, half) written
    if (tid == 0) {
      const bool ok = grid_barrier(P.grid_bar, P.grid_bar + 1, bar_gen0, gridDim.x, P.status);
      if (!ok) flag(P.status, ST_TIMEOUT | (1u << (16 + 13)));
      s.bar_ok = ok ? 1 : 0;
    }
    __syncthreads();
    merge_ok = s.bar_ok != 0;
  }
  // this CTA's column groups [g0, g1) of every row (four columns each); with
  // few splits and at most one (row, group) item a thread, every partial the
  // thread will sum is loaded together with the row statistics, so the whole
  // merge waits for L2 once
  const int g0 = 64 * split / C, g1 = 64 * (split + 1) / C, ng = g1 - g0;
  const bool fast = C > 1 && C <= kFastSplits && 128 * ng <= NTHR;
  const uint2* po0 = reinterpret_cast<const uint2*>(P.part_o) + (int64_t)(blockIdx.x - split) * (128 * 64);
  const int f_hh = fast ? tid / max(ng, 1) : 0, f_col = fast ? 4 * (g0 + tid % max(ng, 1)) : 0;
  const bool f_item = fast && tid < 128 * ng && row_h(f_hh) < P.H;
  uint2 pre[kFastSplits];
  if (C > 1) {
    // (4) the C splits' row maxima and sums of this (query, half): every
    // thread's loads issued before its stores (C <= 64: at most 15 a thread)
    if (merge_ok && fast) {
#pragma unroll
      for (int r = 0; r < kFastSplits; ++r)
        if (r < C && f_item) pre[r] = __ldcg(po0 + (int64_t)r * (128 * 64) + f_hh * 64 + (f_col >> 2));
      const float* pm0 = P.part_ml + (int64_t)(blockIdx.x - split) * 256;
      constexpr int PERF = (kFastSplits * 128 + NTHR - 1) / NTHR;
      float mv[PERF], lv[PERF];
#pragma unroll
      for (int u = 0; u < PERF; ++u) {
        const int i = tid + u * NTHR;
        if (i < C * 128) {
          mv[u] = __ldcg(pm0 + (i >> 7) * 256 + (i & 127));
          lv[u] = __ldcg(pm0 + (i >> 7) * 256 + 128 + (i & 127));
        }
      }
#pragma unroll
      for (int u = 0; u < PERF; ++u) {
        const int i = tid + u * NTHR;
        if (i < C * 128) {
          fac[i] = mv[u];
          lsp[i] = lv[u];
        }
      }
    } else if (merge_ok) {
      const float* pm0 = P.part_ml + (int64_t)(blockIdx.x - split) * 256;
      constexpr int PER = (kMaxSplit * 128 + NTHR - 1) / NTHR;
      float mv[PER], lv[PER];
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int i = tid + u * NTHR;
        if (i < C * 128) {
          mv[u] = __ldcg(pm0 + (i >> 7) * 256 + (i & 127));
          lv[u] = __ldcg(pm0 + (i >> 7) * 256 + 128 + (i & 127));
        }
      }
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int i = tid + u * NTHR;
        if (i < C * 128) {
          fac[i] = mv[u];
          lsp[i] = lv[u];
        }
      }
    }
    __syncthreads();
  }
  if (tid < 128) {
    // the merged row maximum (with the sink, log2 units) and denominator; the
    // factor of each split: exp2(max_r - M) for O (C = 1), times l_r for the
    // normalised partials O_r / l_r (C > 1)
    const int hh = tid, head = row_h(hh);
    const float z = (P.sink && head < P.H) ? P.sink[head] * log2e : -INFINITY;
    float M = z;
    if (C == 1) {
      M = fmaxf(M, s.mg.rms[hh]);
    } else {
      for (int r = 0; r < C; ++r) M = fmaxf(M, fac[r * 128 + hh]);
    }
    float den = 0.f;
    if (C == 1) {
      const float f = (M != -INFINITY && s.mg.rms[hh] != -INFINITY) ? ex2f(s.mg.rms[hh] - M) : 0.f;
      s.mg.fself[hh] = f;
      den = f * s.mg.rl[hh];
    } else {
      for (int r = 0; r < C; ++r) {
        const float mr = fac[r * 128 + hh];
        const float f = (M != -INFINITY && mr != -INFINITY) ? ex2f(mr - M) * lsp[r * 128 + hh] : 0.f;
        fac[r * 128 + hh] = f;
        den += f;
      }
    }
    if (M != -INFINITY && z != -INFINITY) den += ex2f(z - M);
    s.mg.invl[hh] = den > 0.f ? 1.f / den : 0.f;
    if (P.lse && dh == 0 && split == 0 && head < P.H && merge_ok)
      P.lse[row_q(hh) * P.H + head] = den > 0.f ? M * 0.6931471805599453f + logf(den) : -INFINITY;
  }
  __syncthreads();
  // the final value of output column `col` (this half) of row hh from its
  // merged (summed, scaled) value: / denominator, R(-p) on RoPE pairs, stored
  auto emit4 = [&](int hh, int col, float4 a) {
    const float il = s.mg.invl[hh];
    float o[4] = {a.x * il, a.y * il, a.z * il, a.w * il};
    if (dh == 1 && col >= 192) {
      const int u = (PAIR && hh >= 64) ? 1 : 0;
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        const int k = (col + e - 192) >> 1;
        const float cs = s.rcs[u][k], sn = s.rsn[u][k];
        const float r0 = o[e] * cs + o[e + 1] * sn, r1 = -o[e] * sn + o[e + 1] * cs;
        o[e] = r0;
        o[e + 1] = r1;
      }
    }
    const int64_t off = (row_q(hh) * P.H + row_h(hh)) * 512 + dh * 256 + col;
    if (P.out_dtype == V4A_F32) {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(P.out) + off) = make_float4(o[0], o[1], o[2], o[3]);
    } else {
      const uint32_t w0 = (uint32_t)f32_to_bf16_bits(o[0]) | ((uint32_t)f32_to_bf16_bits(o[1]) << 16);
      const uint32_t w1 = (uint32_t)f32_to_bf16_bits(o[2]) | ((uint32_t)f32_to_bf16_bits(o[3]) << 16);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(P.out) + off) = make_uint2(w0, w1);
    }
  };
  if (C == 1) {
    // each epilogue thread 64 columns of its row
    if (warp >= 2) {
      const int quad = warp & 3, grp = (warp - 2) >> 2;
      const int hh = quad * 32 + lane;
      const uint32_t ob = tmem + ((uint32_t)(quad * 32) << 16) + 256;
      const float f = s.mg.fself[hh];
#pragma unroll 1
      for (int cc = 0; cc < 256 / KG; cc += 32) {
        const int c = grp * (256 / KG) + cc;
        uint32_t r[32];
        tmem_ld32_nowait(ob + c, r);
        tmem_ld_wait();
        if (row_h(hh) < P.H)
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            emit4(hh, c + k, make_float4(__uint_as_float(r[k]) * f, __uint_as_float(r[k + 1]) * f,
                                         __uint_as_float(r[k + 2]) * f, __uint_as_float(r[k + 3]) * f));
      }
    }
  } else if (merge_ok) {
    // (5) this CTA's column groups of every row, summed over the C partials
    if (fast) {
      if (f_item) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int r = 0; r < kFastSplits; ++r)
          if (r < C) {
            const float f = fac[r * 128 + f_hh];
            const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&pre[r].x));
            const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&pre[r].y));
            a.x = fmaf(f, lo.x, a.x);
            a.y = fmaf(f, lo.y, a.y);
            a.z = fmaf(f, hi.x, a.z);
            a.w = fmaf(f, hi.y, a.w);
          }
        emit4(f_hh, f_col, a);
      }
    } else
    for (int it = tid; it < 128 * ng; it += NTHR) {
      const int hh = it / ng, col = 4 * (g0 + it % ng);
      if (row_h(hh) >= P.H) continue;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int r0 = 0; r0 < C; r0 += 8) {              // eight loads in flight
        uint2 b[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (r0 + u < C) b[u] = __ldcg(po0 + (int64_t)(r0 + u) * (128 * 64) + hh * 64 + (col >> 2));
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (r0 + u < C) {
            const float f = fac[(r0 + u) * 128 + hh];
            const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&b[u].x));
            const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&b[u].y));
            a.x = fmaf(f, lo.x, a.x);
            a.y = fmaf(f, lo.y, a.y);
            a.z = fmaf(f, hi.x, a.z);
            a.w = fmaf(f, hi.y, a.w);
          }
      }
      emit4(hh, col, a);
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

bool make_rows_map_sw(CUtensorMap* map, const void* base, int64_t rows, int row_bytes,
                      int box_bytes, int box_rows, int swizzle_bytes);

int mqa_tc_check(const MqaParams& P) {
  if (P.kv_dtype != V4A_E4M3_BF16ROPE || P.d != 512 || P.d_rope != 64 || P.H > 128 ||
      P.q_dtype != V4A_BF16 || P.n_win > 1024 || P.qbuf == nullptr ||
      (P.pages.bt ? P.kv_rows : (int64_t)P.B * P.kv_rows) >= (1ll << 31) ||
      (int64_t)P.B * P.swa_rows >= (1ll << 31))
    return 2;
  if (((uintptr_t)P.qbuf & 15) || ((uintptr_t)P.kv & 15) ||
      (P.n_win > 0 && ((uintptr_t)P.swa & 15)) || ((uintptr_t)P.Q & 15))
    return 1;
  return 0;
}

cudaError_t launch_mqa_tc(const MqaParams& P, cudaStream_t st) {
  Maps m;
  const int64_t kv_rows = P.pages.bt ? P.kv_rows : (int64_t)P.B * P.kv_rows;   // rows the maps cover
  const int64_t sw_rows = (int64_t)P.B * P.swa_rows;
  const void* swa = P.swa ? (const void*)P.swa : (const void*)P.kv;
  const int64_t swr = P.swa ? sw_rows : kv_rows;
  if (!make_rows_map_sw(&m.kv128, P.kv, kv_rows, ROWB, 128, NK, 128) ||
      !make_rows_map_sw(&m.kv64, P.kv, kv_rows, ROWB, 64, NK, 64) ||
      !make_rows_map_sw(&m.kvg128, P.kv, kv_rows, ROWB, 128, 1, 128) ||
      !make_rows_map_sw(&m.kvg64, P.kv, kv_rows, ROWB, 64, 1, 64) ||
      !make_rows_map_sw(&m.swg128, swa, swr, ROWB, 128, 1, 128) ||
      !make_rows_map_sw(&m.swg64, swa, swr, ROWB, 64, 1, 64))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64) return cudaErrorInvalidDevice;
  // per device: CTAs that can be resident at once (one per SM)
  static int resident[64] = {0};
  if (resident[dev] == 0) {
    cudaError_t e = cudaSuccess;
    for (auto k : {mqa_tc_kernel<false, false>, mqa_tc_kernel<true, false>,
                   mqa_tc_kernel<false, true>, mqa_tc_kernel<true, true>})
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0, n_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, mqa_tc_kernel<false, false>, NTHR,
                                                      smem);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    resident[dev] = std::max(1, per_sm * n_sm);
  }
  // key splits per (query, half): as many as keep every CTA of the launch
  // resident (at most kMqaTcMaxCtas and kMaxSplit) while each split keeps at
  // least kMinSplitTiles key tiles in a dense call (a split's fixed cost, its
  // start and its share of the merge, is worth about that many contiguous
  // tiles; gathered tiles are bound by the copy engine of their SM, so a
  // sparse call, or a paged one, spreads them over as many SMs as it can);
  // one when fewer than two fit, which needs no partials and no grid barrier
  MqaParams Q = P;
  // Two consecutive queries per CTA (their 2 x H <= 128 head rows side by
  // side, sharing every key tile) when a dense call's queries all belong to
  // one sequence and are many: the prefill form of the HCA MQA
  Q.pair = (!P.idx && P.H <= 64 && P.B == 1 && P.n_q >= 256 && P.n_q % 2 == 0 && !P.q_ready) ? 1 : 0;
  const int64_t n_main = P.idx ? (int64_t)P.n_sel : P.max_vis;
  const int64_t tiles = (n_main + NK - 1) / NK + (P.n_win + NK - 1 + (Q.pair ? NK : 0)) / NK;
  const int64_t units = 2 * (int64_t)(Q.pair ? P.n_q / 2 : P.n_q);
  const int64_t cap = std::min<int64_t>(resident[dev], kMqaTcMaxCtas);
  int64_t C = 1;
  if (units * 2 <= cap)
    C = std::max<int64_t>(1, std::min<int64_t>({cap / units,
                                               (P.idx || P.pages.bt) ? tiles : tiles / kMinSplitTiles,
                                               (int64_t)kMaxSplit}));
  Q.n_split = (int)C;
  if (C > 1 && (Q.part_o == nullptr || Q.part_ml == nullptr || Q.grid_bar == nullptr))
    return cudaErrorInvalidValue;
  const int64_t grid = units * C;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
  if (C > 1) Q.pair = 0;                            // (never with n_q >= 256)
  if (!P.q_ready)
    mqa_tc_qprep_kernel<<<dim3((unsigned)(Q.pair ? P.n_q / 2 : P.n_q), 8), 64, 0, st>>>(Q);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(NTHR, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;        // the grid barrier needs every CTA resident
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = C > 1 ? 1 : 0;
  if (P.pages.bt)
    return Q.pair ? cudaLaunchKernelEx(&cfg, mqa_tc_kernel<true, true>, Q, m)
                  : cudaLaunchKernelEx(&cfg, mqa_tc_kernel<false, true>, Q, m);
  return Q.pair ? cudaLaunchKernelEx(&cfg, mqa_tc_kernel<true, false>, Q, m)
                : cudaLaunchKernelEx(&cfg, mqa_tc_kernel<false, false>, Q, m);
}

}  // namespace v4a
