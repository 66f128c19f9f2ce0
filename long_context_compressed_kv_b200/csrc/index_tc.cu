// Lightning-indexer scores on the 5th-generation tensor cores: block-scaled
// MXFP4 x MXFP4 MMA (tcgen05.mma kind::mxf4, E8M0 scale per 32 elements) with
// the ReLU / head-weighted reduction fused into the TMEM epilogue.
//
// Method: "DeepSeek-V4 深读" (ricardokevins.github.io), section
// "CSA：4× 压缩之后再 top-k" (64 indexer heads, ReLU scores, input-dependent
// head weights) and section "FP4 QAT、可恢复 rollout 与百万 Token RL" (MXFP4
// indexer QK path):  s_i = sum_h w_h * max(0, q_h . k_i).
//
// Shape of the contraction per query: D[128 keys][H_I heads] = K_tile . Q^T,
// K-dim = d_I = 128 (two MMAs of K = 64).  A (keys) streams from HBM through a
// multi-stage TMA ring (64-byte-swizzled K-major tiles); B (the query's H_I x
// 128 codes) stays in shared memory for the query's whole key range; the E8M0
// scales of both go to TMEM with tcgen05.cp (row m at lane m % 32 of every
// sub-partition, column m / 32, byte = 32-element block).  The key tile is
// loaded through a 3-D view of the key array (64 B x rows/4 x 4, strides 256 B
// and 64 B) so that MMA row 32c + l holds key 4l + c: in that order the key
// scales, stored row-major (4 bytes a key), are already the scale-factor
// layout, and go from the bulk-copied stage straight to TMEM with no rewrite
// through registers (which would add generic-proxy stores and a proxy fence
// per stage to the MMA warp).  The epilogue maps TMEM lane 32c + l back to key
// 4l + c.  A ring stage holds
// up to three (two CTAs per SM, N <= 64) or four (one CTA per SM, N = 128)
// consecutive 128-key tiles of one query: on this part a streaming read over
// one stage per barrier round trip reaches HBM speed only from about 32 KB per
// SM and stage on, while the work is still split between CTAs tile by tile.
// The accumulator has several TMEM stages so the epilogue of tile i overlaps
// the MMAs of the tiles after it.  The MMA warp commits once per stage
// (commits were its costliest instruction to issue); the first epilogue warp,
// once it has seen that commit, hands the ring stage (and at a query's end its
// query buffer) back to the producer.  Roles: warp 0 TMA producer, warp 1 MMA
// issuer (one lane), warps 2..5 and 6..9 two epilogue groups on alternate
// tiles (one thread per key row).  By its arithmetic intensity the indexer is
// HBM-bound (68 bytes per key against 16384 FP4 FLOP); as built, the
// streaming itself (the per-stage barrier round trips from a landed load to
// the stage's release) sets its time, the MMA issue next.
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"
#include "tc_kernels.h"

namespace v4a {

namespace {

constexpr int KT = 128;                 // keys per tile (MMA M)
constexpr int KROW = 64;                // bytes per key row (128 E2M1)
constexpr int KTILE_BYTES = KT * KROW;  // 8 KB
constexpr int SF_BYTES = 512;           // 128 rows x 4 scale bytes
constexpr int MAXQ = 1024;              // queries per launch on this path
constexpr int EPI_GROUPS = 2;           // epilogue warp groups, alternating tiles
constexpr int NTHREADS = 64 + EPI_GROUPS * 128;
constexpr int MAX_ACC = 8;              // accumulator stages in TMEM

// Per MMA width N: N <= 64 runs two CTAs per SM (each its own MMA-issuing
// thread, whose tcgen05 issue rate bounds the kernel; half of TMEM each; a
// ring of 3 stages of up to 3 tiles), N = 128 one CTA per SM (all of TMEM, 5
// stages of up to 4 tiles: 32 KB, the size from which one stage per barrier
// round trip streams at HBM speed).  Accumulators: as many as fit the CTA's
// TMEM columns next to their key scales (4 columns each) and the two
// query-scale slots (4 columns each).
template <int N>
struct Cfg {
  static constexpr int CPS = N <= 64 ? 2 : 1;
  static constexpr int STAGES = CPS == 2 ? 3 : 5;
  static constexpr int TPS = CPS == 2 ? 3 : 4;
  static constexpr uint32_t TM_COLS = CPS == 2 ? 256 : 512;
  static constexpr int NACC = ((int)TM_COLS - 8) / (N + 4) < MAX_ACC ? ((int)TM_COLS - 8) / (N + 4)
                                                                      : MAX_ACC;
};

template <int STAGES, int TPS>
struct Smem {
  alignas(1024) uint8_t keys[STAGES][TPS][KTILE_BYTES];
  alignas(1024) uint8_t q[2][128 * KROW];
  alignas(128) uint32_t sfa_raw[STAGES][TPS * KT];  // key scales as loaded (row-major)
  alignas(128) uint8_t sfb[2][SF_BYTES];
  alignas(128) uint32_t sfb_raw[2][128];
  alignas(16) float w[2][128];
  uint64_t full[STAGES], empty[STAGES], accstage[STAGES], qfull[2], qempty[2],
      accempty[MAX_ACC], done, never;
  int tile_prefix[MAXQ + 1];
  int seq[MAXQ];                                    // sequence of each query group
  uint32_t tmem_base;
  int abort;
};

struct TileIter {
  int q = -1, lt = 0, seg = -1;
  int qcur = 0;
};

}  // namespace

template <class S>
__device__ __forceinline__ void fail(S& s, uint32_t* status) {
  s.abort = 1;
  flag(status, ST_TIMEOUT);
}

// Decode tile g into (query, local tile); `it` tracks segments (query changes).
template <class S>
__device__ __forceinline__ void locate(const S& s, int n_q, int g, TileIter& t) {
  while (t.qcur + 1 <= n_q && s.tile_prefix[t.qcur + 1] <= g) ++t.qcur;
  if (t.qcur != t.q) {
    t.q = t.qcur;
    ++t.seg;
  }
  t.lt = g - s.tile_prefix[t.q];
}

// Tiles in the stage that starts at tile g: up to `tps` (at most the stage's and at
// most the accumulator count, so that the tiles of one stage never wait for
// each other's accumulator: the epilogue frees a stage's accumulators only
// after that stage's single commit), all of one query group, all inside this
// CTA's range.  Every role walks the stages with this same rule.
template <class S>
__device__ __forceinline__ int stage_tiles(const S& s, const TileIter& t, int g, int g1, int tps) {
  const int to_seg = s.tile_prefix[t.q + 1] - g, to_end = g1 - g;
  const int n = to_seg < to_end ? to_seg : to_end;
  return n < tps ? n : tps;
}

// N = MMA N: the indexer heads, or with PAIR two consecutive queries of one
// sequence side by side (2 x H_I columns), so that every key tile serves both:
// half the MMAs per score where many queries share their keys (prefill).
// PAGED: the keys are a pool of 32-key blocks (a classical block of 128 raw
// tokens holds 32 indexer keys) reached through P.pages; a 128-key tile is
// four blocks, each loaded by its own TMA box of 32 rows (tm_keys then has a
// box of {64 B, 8, 4}), so MMA row 32 kb + 8 c + l holds key 32 kb + 4 l + c
// of the tile's block kb, and the producer's lanes copy the key scales into
// the matching scale-factor order (lane 8 c + l, column kb) one 4-byte word each.
template <int N, bool PAIR, bool PAGED>
__global__ void __launch_bounds__(NTHREADS, Cfg<N>::CPS)
    index_tc_kernel(IndexParams P, const __grid_constant__ CUtensorMap tm_keys,
                    const __grid_constant__ CUtensorMap tm_q) {
  constexpr int STAGES = Cfg<N>::STAGES, TPS = Cfg<N>::TPS;
  constexpr uint32_t TM_COLS = Cfg<N>::TM_COLS;
  using Smem = v4a::Smem<STAGES, TPS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NACC = Cfg<N>::NACC;
  static_assert(NACC >= 2 && NACC * (N + 4) + 8 <= (int)TM_COLS, "TMEM budget");
  constexpr int TPS_N = NACC < TPS ? NACC : TPS;        // tiles per stage for this N
  // head weights in registers (one CTA per SM: registers to spare) or read
  // from shared memory (two CTAs per SM: at most 102 registers a thread)
  constexpr bool W_IN_REGS = N <= 64 && Cfg<N>::CPS == 1;
  constexpr int QPG = PAIR ? 2 : 1;                     // queries per MMA group
  constexpr int HG = N / QPG;                           // heads of one query
  const int n_g = P.n_q / QPG;                          // query groups (n_q even with PAIR)
  const uint32_t lim = P.wait_ns ? P.wait_ns : (uint32_t)kWaitNs;   // bound of every wait

  // keys a sequence can hold: its part of the cache, or its blocks of the pool
  const int64_t cap = PAGED ? (int64_t)P.pages.bps * P.pages.epb : P.key_rows;
  // visible keys of query q (checked); a group's tiles cover its largest
  auto visible = [&](int q) -> int64_t {
    int64_t nv = (P.q_pos[q] + 1) / P.m;
    const int b = P.q_seq ? P.q_seq[q] : P.q_base + q;
    if (b < 0 || b >= P.B) {
      flag(P.status, ST_BAD_SEQ);
      nv = 0;
    }
    if (nv > cap || nv > P.max_vis) {
      flag(P.status, ST_BAD_POSITION);
      nv = min(cap, P.max_vis);
    }
    return nv;
  };
  // set-up that needs no global memory first (barriers, TMEM), so that it
  // overlaps the position loads below
  if (threadIdx.x == 0) {
    s.abort = 0;
    for (int i = 0; i < STAGES; ++i) {
      // the producer lane's arrive + TMA / bulk bytes (paged: every producer
      // lane's arrive, once its scale copies have landed, + TMA bytes)
      mbar_init(&s.full[i], PAGED ? 32 : 1);
      mbar_init(&s.empty[i], 1);   // the epilogue's releaser, once the stage's MMAs are done
      mbar_init(&s.accstage[i], 1);   // one commit after all MMAs of a stage
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.qfull[i], 1);
      mbar_init(&s.qempty[i], 1 + 4 * EPI_GROUPS);   // releaser + every epilogue warp
    }
    for (int i = 0; i < MAX_ACC; ++i) mbar_init(&s.accempty[i], 4);
    mbar_init(&s.done, 1);
    mbar_init(&s.never, 1);   // debug stall site: nothing ever arrives on it
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&s.tmem_base, TM_COLS);
  // tiles and sequence of each query group (positions loaded in parallel,
  // one round trip), then a serial prefix over shared memory
  for (int q = threadIdx.x; q < n_g; q += NTHREADS) {
    int64_t nv = visible(q * QPG);
    if (PAIR) nv = max(nv, visible(q * QPG + 1));
    s.tile_prefix[q + 1] = (int)((nv + KT - 1) / KT);
    s.seq[q] = P.q_seq ? P.q_seq[q * QPG] : P.q_base + q * QPG;   // used only with tiles
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    s.tile_prefix[0] = 0;
    for (int q = 0; q < n_g; ++q) {
      acc += s.tile_prefix[q + 1];
      s.tile_prefix[q + 1] = acc;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int total = s.tile_prefix[n_g];
  const int g0 = (int)((int64_t)total * blockIdx.x / gridDim.x);
  const int g1 = (int)((int64_t)total * (blockIdx.x + 1) / gridDim.x);
  const uint32_t tmem = s.tmem_base;
  // TMEM columns: acc[a] at a*N; SFA[a] at NACC*N + 4a; SFB[j] after them
  const uint32_t col_sfa = NACC * N, col_sfb = NACC * N + 4 * NACC;
  auto aborted = [&]() {
    return __any_sync(0xffffffffu, *reinterpret_cast<volatile int*>(&s.abort)) != 0;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tm_keys);
      prefetch_tmap(&tm_q);
    }
    TileIter t;
    const uint32_t* ksf32 = reinterpret_cast<const uint32_t*>(P.keys_sf);
    const int64_t total_rows = (int64_t)P.B * P.key_rows;
    int stg = 0;
    int qissued = 0;                            // query-buffer loads issued
    int b = 0;                                  // sequence of the current query
    int64_t nvg = 0;                            // paged: visible keys of the current group
    for (int g = g0; g < g1 && !aborted(); ++stg) {
      const int seg_before = t.seg;
      locate(s, n_g, g, t);
      const int n = stage_tiles(s, t, g, g1, TPS_N);
      if (t.seg != seg_before) {
        b = s.seq[t.q];
        if constexpr (PAGED) {
          nvg = min((int64_t)(P.q_pos[t.q * QPG] + 1) / P.m, min(cap, P.max_vis));
          if (PAIR) nvg = max(nvg, min((int64_t)(P.q_pos[t.q * QPG + 1] + 1) / P.m, min(cap, P.max_vis)));
        }
        const int j = t.seg & 1, uq = t.seg >> 1;
        if (uq >= 1 && !mbar_wait_warp(&s.qempty[j], (uq - 1) & 1, P.status, -1, lim)) {
          fail(s, P.status);
          break;
        }
        if (lane == 0) {
          // query codes (TMA), query scales and head weights (bulk copies)
          mbar_arrive_expect_tx(&s.qfull[j], (uint32_t)(N * KROW + 2 * N * 4));
          tma_load_2d(s.q[j], &tm_q, &s.qfull[j], 0, t.q * N);
          bulk_load(s.sfb_raw[j], reinterpret_cast<const uint32_t*>(P.qI_sf) + (int64_t)t.q * N,
                    N * 4, &s.qfull[j]);
          bulk_load(s.w[j], P.w + (int64_t)t.q * N, N * 4, &s.qfull[j]);
        }
        ++qissued;
      }
      const int st = stg % STAGES, u = stg / STAGES;
      if (u >= 1 && !mbar_wait_warp(&s.empty[st], (u - 1) & 1, P.status, -1, lim)) {
        fail(s, P.status);
        break;
      }
      if constexpr (PAGED) {
        // block kb of tile k: keys (lt + k) * 128 + 32 kb .. +31 of the sequence,
        // pool rows pr .. pr + 31; blocks at or past the group's visible keys
        // are not loaded (their rows are masked in the epilogue)
        int64_t pr[TPS * 4];
        uint32_t bytes = 0;
#pragma unroll
        for (int i = 0; i < TPS * 4; ++i) {
          pr[i] = -1;
          if (i < 4 * n) {
            const int64_t e = (int64_t)(t.lt + i / 4) * KT + 32 * (i % 4);
            if (e < nvg) {
              pr[i] = page_row(P.pages, b, e);
              if (pr[i] < 0 && lane == 0) flag(P.status, ST_BAD_INDEX);
            }
            if (pr[i] >= 0) bytes += 32 * KROW;
          }
        }
        if (lane == 0) mbar_expect_tx(&s.full[st], bytes);
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int i = 0; i < TPS * 4; ++i)
            if (pr[i] >= 0)
              tma_load_3d(s.keys[st][i / 4] + (i % 4) * 32 * KROW, &tm_keys, &s.full[st], 0,
                          (int)(pr[i] >> 2), 0);
        }
        // lane 8 c + l, column kb: the scale word of key 32 kb + 4 l + c
        const int kin = 4 * (lane & 7) + (lane >> 3);
#pragma unroll
        for (int i = 0; i < TPS * 4; ++i)
          if (i < 4 * n)
            cp_async4(&s.sfa_raw[st][(i / 4) * KT + 4 * lane + (i % 4)],
                      ksf32 + (pr[i] >= 0 ? pr[i] + kin : 0), pr[i] >= 0);
        cp_async_arrive_noinc(&s.full[st]);
        g += n;
        continue;
      }
      const int64_t row0 = (int64_t)b * P.key_rows + (int64_t)t.lt * KT;
      if (lane == 0) {
        // key codes (one TMA tile per 128 keys) + their scales (bulk copy of
        // the in-range rows, 4 at a time; a ragged end of the key array goes by
        // 4-byte cp.async)
        const int64_t rows_left = total_rows - row0;
        const int nrow = (int)(rows_left < n * KT ? rows_left : n * KT);
        const int nbulk = nrow & ~3;
        mbar_expect_tx(&s.full[st], (uint32_t)(n * KTILE_BYTES + nbulk * 4));
        for (int k = 0; k < n; ++k)   // rows row0 + 4l + c land at tile row 32c + l
          tma_load_3d(s.keys[st][k], &tm_keys, &s.full[st], 0, (int)((row0 + k * KT) >> 2), 0);
        if (nbulk) bulk_load(s.sfa_raw[st], ksf32 + row0, nbulk * 4, &s.full[st]);
        for (int r = nbulk; r < nrow; ++r) cp_async4(&s.sfa_raw[st][r], ksf32 + row0 + r, true);
        cp_async_arrive_noinc(&s.full[st]);
      }
      g += n;
    }
    // drain: no load may still be landing in shared memory when the CTA exits.
    // The last use of every ring slot and query buffer is waited for (on a
    // normal run those phases completed long ago; after an abort their
    // consumers may never have waited on them)
    if (lane == 0) {
      for (int k = 0; k < STAGES && k < stg; ++k) {
        const int i2 = stg - 1 - k;
        mbar_wait(&s.full[i2 % STAGES], (i2 / STAGES) & 1);   // time bound only
      }
      for (int k = 0; k < 2 && k < qissued; ++k) {
        const int sg = qissued - 1 - k;
        mbar_wait(&s.qfull[sg & 1], (sg >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    TileIter t;
    int stg = 0;
    bool ok = true;
    if (P.stall && !mbar_wait_warp(&s.never, 0, P.status, 12, lim)) {
      // debug: a wait that nothing completes runs out here, before any MMA is
      // issued; the other roles see the status bit and return
      fail(s, P.status);
      ok = false;
    }
    const uint64_t kdesc_bits = smem_desc_bits(16, 8 * KROW, 4);    // K-major, 64B swizzle
    const uint64_t sf_bits = smem_desc_bits(16, 128, 0);            // 32 rows x 16 B
    for (int g = g0; ok && g < g1 && !aborted(); ++stg) {
      const int seg_before = t.seg;
      locate(s, n_g, g, t);
      const int n = stage_tiles(s, t, g, g1, TPS_N);
      const int j = t.seg & 1;
      if (t.seg != seg_before) {
        if (!mbar_wait_warp(&s.qfull[j], (t.seg >> 1) & 1, P.status, -1, lim)) {
          fail(s, P.status);
          break;
        }
        // query scales into the tcgen05 scale-factor order (rows >= N zero)
        for (int h = lane; h < 128; h += 32)
          *reinterpret_cast<uint32_t*>(&s.sfb[j][16 * (h & 31) + 4 * (h >> 5)]) =
              (h < N) ? s.sfb_raw[j][h] : 0u;
        fence_proxy_async_smem();
        __syncwarp();
        tc_fence_after();
        if (lane == 0) tmem_cp_32x128b_warpx4(tmem + col_sfb + 4 * j, smem_desc(s.sfb[j], sf_bits));
      }
      const int st = stg % STAGES;
      if (!mbar_wait_warp(&s.full[st], (stg / STAGES) & 1, P.status, -1, lim)) {
        fail(s, P.status);
        break;
      }
      // every accumulator of the stage free first; then all scale copies, then
      // the MMAs (a copy issued behind an MMA waits for it)
      for (int k = 0; k < n; ++k) {
        const int it = g - g0 + k, a = it % NACC, ua = it / NACC;
        if (ua >= 1 && !mbar_wait_warp(&s.accempty[a], (ua - 1) & 1, P.status, -1, lim)) {
          fail(s, P.status);
          ok = false;
          break;
        }
      }
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t sfb = tmem + col_sfb + 4 * j;
        const uint64_t db = smem_desc(s.q[j], kdesc_bits);
        for (int k = 0; k < n; ++k) {
          const int a = (g - g0 + k) % NACC;
          tmem_cp_32x128b_warpx4(tmem + col_sfa + 4 * a, smem_desc(&s.sfa_raw[st][k * KT], sf_bits));
        }
        for (int k = 0; k < n; ++k) {
          const int a = (g - g0 + k) % NACC;
          const uint32_t sfa = tmem + col_sfa + 4 * a;
          const uint64_t da = smem_desc(s.keys[st][k], kdesc_bits);
          const uint32_t d = tmem + a * N;
          // K = 0..63 (scale bytes 0,1), then K = 64..127 (scale bytes 2,3): +32 B
          mma_mxf4(d, da, db, idesc_mxf4(KT, N, 0, 0), sfa, sfb, 0);
          mma_mxf4(d, da + 2, db + 2, idesc_mxf4(KT, N, 2, 2), sfa, sfb, 1);
        }
        // one commit for the whole stage: commits are the costly tcgen05
        // instruction here; the epilogue releases the ring stage and the
        // query buffer once it has seen this one
        tc_commit(&s.accstage[st]);
      }
      __syncwarp();
      g += n;
    }
    // every MMA / copy this warp issued has completed before TMEM is released
    if (lane == 0) {
      tc_commit(&s.done);
      if (!mbar_wait(&s.done, 0)) flag(P.status, ST_TIMEOUT);   // time bound only
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // group g handles the tiles with it % 2 == g; within a group, warp w reads
    // TMEM lanes 32*(w%4) .. +31 (one key per thread)
    const int grp = (warp - 2) >> 2;
    const int quad = warp & 3;
    // key of TMEM lane 32 * quad + lane (its MMA row) within the tile
    const int r = PAGED ? 32 * quad + 4 * (lane & 7) + (lane >> 3) : 4 * lane + quad;
    {
      // keys beyond the last tile of each query (group): -inf
      const int et = threadIdx.x - 64;
      for (int q = blockIdx.x; q < n_g; q += gridDim.x) {
        const int64_t from = (int64_t)(s.tile_prefix[q + 1] - s.tile_prefix[q]) * KT;
        for (int u = 0; u < QPG; ++u)
          for (int64_t i = from + et; i < P.max_vis; i += EPI_GROUPS * 128)
            put_score(P.scores, (int64_t)(q * QPG + u) * P.scores_ld + i, -INFINITY, P.score_bf16);
      }
    }
    TileIter t;
    float wreg[W_IN_REGS ? N : 1];
    int64_t nv = 0, nv2 = 0;                    // visible keys of the group's queries
    int stg = 0;
    // warp 2 lane 0 (group 0) is the releaser: it waits for every stage's
    // commit and then frees the ring stage (and, at a query's last stage, the
    // query buffer) for the producer
    const bool releaser = warp == 2 && lane == 0;
    for (int g = g0; g < g1 && !aborted(); ++stg) {
      const int seg_before = t.seg;
      locate(s, n_g, g, t);
      const int n = stage_tiles(s, t, g, g1, TPS_N);
      const int j = t.seg & 1;
      if (t.seg != seg_before) {
        if (!mbar_wait_warp(&s.qfull[j], (t.seg >> 1) & 1, P.status, -1, lim)) {
          fail(s, P.status);
          break;
        }
        if constexpr (W_IN_REGS) {
#pragma unroll
          for (int h = 0; h < N; ++h) wreg[h] = s.w[j][h];
        }
        nv = min((int64_t)(P.q_pos[t.q * QPG] + 1) / P.m, min(P.key_rows, P.max_vis));
        if (PAIR) nv2 = min((int64_t)(P.q_pos[t.q * QPG + 1] + 1) / P.m, min(P.key_rows, P.max_vis));
      }
      const int st = stg % STAGES;
      const bool has_tile = n > 1 || ((g - g0) & 1) == grp;
      const bool seg_end = (g + n == g1) || (g + n >= s.tile_prefix[t.q + 1]);
      if (grp == 0 || has_tile) {
        if (!mbar_wait_warp(&s.accstage[st], (stg / STAGES) & 1, P.status, -1, lim)) {
          fail(s, P.status);
          break;
        }
        if (releaser) {
          mbar_arrive(&s.empty[st]);
          if (seg_end) mbar_arrive(&s.qempty[j]);
        }
      }
      tc_fence_after();
      for (int k = 0; k < n; ++k) {
        const int it = g - g0 + k;
        if ((it & 1) != grp) continue;
        const int a = it % NACC;
        const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + a * N;
        float s0 = 0.f, s1 = 0.f, u0 = 0.f, u1 = 0.f;   // even / odd heads; u: the second query
        constexpr int CH = Cfg<N>::CPS == 2 ? 32 : (N <= 64 ? N : 64);   // columns per TMEM round trip
#pragma unroll
        for (int c0 = 0; c0 < N; c0 += CH) {
          uint32_t v[CH];
#pragma unroll
          for (int c = 0; c < CH; c += 32) tmem_ld32_nowait(taddr + c0 + c, v + c);
          tmem_ld_wait();
          if (c0 + CH == N) {                     // accumulator fully read: release it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.accempty[a]);
          }
#pragma unroll
          for (int h = 0; h < CH; h += 2) {
            const float w0 = W_IN_REGS ? wreg[(c0 + h) % (W_IN_REGS ? N : 1)] : s.w[j][c0 + h];
            const float w1 = W_IN_REGS ? wreg[(c0 + h + 1) % (W_IN_REGS ? N : 1)] : s.w[j][c0 + h + 1];
            if (c0 + h < HG) {
              s0 = fmaf(w0, fmaxf(__uint_as_float(v[h]), 0.f), s0);
              s1 = fmaf(w1, fmaxf(__uint_as_float(v[h + 1]), 0.f), s1);
            } else {
              u0 = fmaf(w0, fmaxf(__uint_as_float(v[h]), 0.f), u0);
              u1 = fmaf(w1, fmaxf(__uint_as_float(v[h + 1]), 0.f), u1);
            }
          }
        }
        const int64_t i = (int64_t)(t.lt + k) * KT + r;
        if (i < P.max_vis) {
          put_score(P.scores, (int64_t)(t.q * QPG) * P.scores_ld + i, (i < nv) ? s0 + s1 : -INFINITY,
                    P.score_bf16);
          if (PAIR)
            put_score(P.scores, (int64_t)(t.q * QPG + 1) * P.scores_ld + i,
                      (i < nv2) ? u0 + u1 : -INFINITY, P.score_bf16);
        }
      }
      if (seg_end) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.qempty[j]);
      }
      g += n;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

void* tensor_map_encoder() { return reinterpret_cast<void*>(encode_fn()); }

// 2-D uint8 tensor map: rows of `row_bytes`, box of `box_rows` rows, 64B swizzle.
bool make_rows_map(CUtensorMap* map, const void* base, int64_t rows, int row_bytes, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || rows < 1 || rows > (1ll << 31)) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)row_bytes, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 2-D uint8 tensor map over rows of `row_bytes`: box of `box_bytes` x `box_rows`
// starting at any 16-byte-aligned column, with a 32/64/128-byte swizzle.
bool make_rows_map_sw(CUtensorMap* map, const void* base, int64_t rows, int row_bytes,
                      int box_bytes, int box_rows, int swizzle_bytes) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || rows < 1 || rows > (1ll << 31) || (row_bytes & 15)) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)box_bytes, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D uint8 view of the MXFP4 key codes (64-byte rows, row count divisible by
// 4): dims {64 B, rows / 4, 4} with strides {256 B, 64 B}.  A box {64, 32, 4}
// at (0, row0 / 4, 0) lands rows row0 + 4l + c at shared-memory row 32c + l,
// 64-byte swizzled; rows past the end of the array read as zero.  With
// box_l = 8 (paged keys: one 32-key block) row0 + 4l + c lands at row 8c + l.
static bool make_keys_map(CUtensorMap* map, const void* base, int64_t rows, int box_l = 32) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || rows < 4 || (rows & 3) || rows > (1ll << 31)) return false;
  cuuint64_t dims[3] = {(cuuint64_t)KROW, (cuuint64_t)(rows / 4), 4};
  cuuint64_t strides[2] = {(cuuint64_t)(4 * KROW), (cuuint64_t)KROW};
  cuuint32_t box[3] = {(cuuint32_t)KROW, (cuuint32_t)box_l, 4};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int index_tc_check(const IndexParams& P) {
  if (P.idx_dtype != V4A_MXFP4 || P.d_I != 128 || !(P.H_I == 32 || P.H_I == 64 || P.H_I == 128) ||
      P.n_q > MAXQ)
    return 2;
  // the scale and weight rows are moved by 1-D bulk copies: 16-byte aligned
  // sources, i.e. 16-byte aligned bases and a key row count divisible by 4
  // (the 3-D key view needs the latter too)
  if (P.key_rows % 4 != 0 ||
      (P.pages.bt ? P.key_rows : (int64_t)P.B * P.key_rows) > (1ll << 31))
    return 2;
  // paged keys: a pool of whole 32-key blocks (m = 4: 128 raw tokens a block)
  if (P.pages.bt && (P.pages.epb != 32 || P.key_rows % 32 != 0)) return 2;
  if (((uintptr_t)P.keys & 15) || ((uintptr_t)P.qI & 15) || ((uintptr_t)P.keys_sf & 15) ||
      ((uintptr_t)P.qI_sf & 15) || ((uintptr_t)P.w & 15))
    return 1;
  return encode_fn() != nullptr ? 0 : 2;   // the driver's tensor-map encoder
}

cudaError_t launch_index_tc(const IndexParams& P, cudaStream_t st) {
  CUtensorMap tk, tq;
  const bool paged = P.pages.bt != nullptr;
  if (!(paged ? make_keys_map(&tk, P.keys, P.key_rows, 8)
              : make_keys_map(&tk, P.keys, (int64_t)P.B * P.key_rows)))
    return cudaErrorInvalidValue;
  // two consecutive queries per MMA (N = 2 H_I) when every query belongs to
  // the one sequence of the call and they pair up evenly
  const bool pair = P.B == 1 && P.n_q >= 2 && P.n_q % 2 == 0 && P.H_I <= 64;
  const int nmma = pair ? 2 * P.H_I : P.H_I;
  if (!make_rows_map(&tq, P.qI, (int64_t)P.n_q * P.H_I, KROW, nmma)) return cudaErrorInvalidValue;
  int dev = 0;
  cudaGetDevice(&dev);
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // persistent: Cfg<N>::CPS CTAs per SM, each over a contiguous range of tiles
  auto launch = [&](auto kernel, auto cfg_tag) -> cudaError_t {
    using C = decltype(cfg_tag);
    const size_t smem = sizeof(Smem<C::STAGES, C::TPS>) + 1024;
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kernel<<<C::CPS * sms, NTHREADS, smem, st>>>(P, tk, tq);
    return cudaSuccess;
  };
  cudaError_t e = cudaSuccess;
  if (paged) {
    switch (nmma * (pair ? -1 : 1)) {
      case 32: e = launch(index_tc_kernel<32, false, true>, Cfg<32>{}); break;
      case 64: e = launch(index_tc_kernel<64, false, true>, Cfg<64>{}); break;
      case 128: e = launch(index_tc_kernel<128, false, true>, Cfg<128>{}); break;
      case -64: e = launch(index_tc_kernel<64, true, true>, Cfg<64>{}); break;
      case -128: e = launch(index_tc_kernel<128, true, true>, Cfg<128>{}); break;
      default: return cudaErrorInvalidValue;
    }
  } else {
    switch (nmma * (pair ? -1 : 1)) {
      case 32: e = launch(index_tc_kernel<32, false, false>, Cfg<32>{}); break;
      case 64: e = launch(index_tc_kernel<64, false, false>, Cfg<64>{}); break;
      case 128: e = launch(index_tc_kernel<128, false, false>, Cfg<128>{}); break;
      case -64: e = launch(index_tc_kernel<64, true, false>, Cfg<64>{}); break;
      case -128: e = launch(index_tc_kernel<128, true, false>, Cfg<128>{}); break;
      default: return cudaErrorInvalidValue;
    }
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace v4a
