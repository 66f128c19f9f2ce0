// sm_100a building blocks: mbarriers with bounded waits, TMA tensor loads,
// and the tcgen05 (5th-generation tensor core / TMEM) instructions.
//
// Descriptor formats (PTX ISA, tcgen05 "shared memory descriptor" and
// "instruction descriptor"; the same bit layout CUTLASS's UMMA::SmemDescriptor
// and UMMA::InstrDescriptor[BlockScaled] spell out):
//   smem descriptor: [0,14) start>>4, [16,30) LBO>>4, [32,46) SBO>>4,
//                    [46,48) version = 1, [49,52) base offset, [61,64) layout
//                    (0 none, 2 128B, 4 64B, 6 32B swizzle);
//   instr descriptor: [4,6) D format (1 = f32), [7,10) A format, [10,13) B
//                    format, bit 15/16 A/B MN-major, [17,23) N>>3, [24,29) M>>4;
//                    block-scaled: [4,6) B scale id, bit 23 scale type (1 =
//                    E8M0), [29,31) A scale id, bit 31 K size.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace v4a {

// Wall-clock limit of every mbarrier wait.  A failed try_wait may suspend the
// thread for a while, so the bound is in time (%globaltimer), not iterations.
// On expiry the wait reports failure; the kernel records ST_TIMEOUT in the
// status word, and every other wait of the grid that has lasted kStatusPollNs
// gives up as soon as it sees that bit, so a stuck kernel ends within about
// one limit.
constexpr unsigned long long kWaitNs = 1000000000ull;   // 1 s (< 2^32 ns)
constexpr unsigned long long kStatusPollNs = 20000ull;  // 20 us
constexpr uint32_t kStatusTimeout = 1u << 8;            // == ST_TIMEOUT

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// The same test, letting the hardware suspend the thread until the phase
// completes (or the hint runs out) instead of returning at once: waiting
// warps then take no issue slots from the warps they wait for (an MMA-issuing
// warp shares its scheduler with epilogue warps).
constexpr uint32_t kSuspendHintNs = 1000000;   // 1 ms; completion wakes the thread first
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait that, on expiry, also records its call site (bit 16 + site of
// the status word) so a report says which wait gave up.
__device__ __forceinline__ bool mbar_wait_at(uint64_t* bar, uint32_t parity, uint32_t* status,
                                             int site, uint32_t limit_ns = (uint32_t)kWaitNs);

// Bounded wait for the phase with the given parity; false on expiry or when
// `status` (the grid's status word, may be null) already records a timeout.
// The status word is read only once the wait has lasted kStatusPollNs: a
// global load on the polling path of every healthy wait would delay noticing
// the phase by a memory round trip, which under a full HBM stream is several
// hundred nanoseconds.
// `limit_ns` (default kWaitNs) is the wall-clock bound of this wait.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          const uint32_t* status = nullptr,
                                          uint32_t limit_ns = (uint32_t)kWaitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  // elapsed time in 32 bits: it wraps after 4.29 s, well above the limit
  const uint32_t t0 = (uint32_t)global_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    const uint32_t dt = (uint32_t)global_ns() - t0;
    if (dt > limit_ns) return false;
    if (status && dt > (uint32_t)kStatusPollNs &&
        (*reinterpret_cast<const volatile uint32_t*>(status) & kStatusTimeout))
      return false;
  }
}
__device__ __forceinline__ bool mbar_wait_at(uint64_t* bar, uint32_t parity, uint32_t* status,
                                             int site, uint32_t limit_ns) {
  if (mbar_wait(bar, parity, status, limit_ns)) return true;
  if (status) atomicOr(status, kStatusTimeout | (1u << (16 + (site & 15))));
  return false;
}

// Barrier of all n CTAs of a cooperative launch (co-resident by construction),
// taken by one thread of each CTA after a __syncthreads that follows the CTA's
// writes; the CTA's other threads wait at a __syncthreads after it.  `count`
// and `gen` are words of the workspace header; gen0 is `gen` as the CTA read it
// when it started (a barrier completes only after every CTA has arrived, so
// no CTA can read the new generation there).  The last CTA to arrive returns
// the count to zero and publishes the next generation; the others poll it.
// Bounded like mbar_wait: false on expiry or when `status` records a timeout.
__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ bool grid_barrier(uint32_t* count, uint32_t* gen, uint32_t gen0,
                                             uint32_t n, const uint32_t* status,
                                             uint32_t limit_ns = (uint32_t)kWaitNs) {
  __threadfence();
  uint32_t old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(old) : "l"(count) : "memory");
  if (old == n - 1) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], 0;" ::"l"(count) : "memory");
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(gen), "r"(gen0 + 1u) : "memory");
    return true;
  }
  const uint32_t t0 = (uint32_t)global_ns();
  for (;;) {
    if (ld_acquire_gpu(gen) != gen0) return true;
    const uint32_t dt = (uint32_t)global_ns() - t0;
    if (dt > limit_ns) return false;
    if (status && dt > (uint32_t)kStatusPollNs &&
        (*reinterpret_cast<const volatile uint32_t*>(status) & kStatusTimeout))
      return false;
    __nanosleep(32);
  }
}

// The same wait taken by all 32 lanes of a warp, with one answer for all of
// them: a warp never splits at a timeout, so the warp-wide (.sync.aligned)
// tcgen05 loads and stores that follow always see every lane.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, uint32_t* status,
                                               int site = -1,
                                               uint32_t limit_ns = (uint32_t)kWaitNs) {
  const bool ok = site >= 0 ? mbar_wait_at(bar, parity, status, site, limit_ns)
                            : mbar_wait(bar, parity, status, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// 4-byte asynchronous global->shared copy (zero-filled when !valid) and the
// arrive that fires on `bar` once this thread's earlier cp.async copies land.
__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}
// 16-byte copy that bypasses L1 (zero-filled when !valid); both addresses 16-byte aligned.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// Wait until at most N of this thread's committed groups are still in flight.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---------------------------------------------------------------- fences
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}
// 1-D bulk copy global -> shared through the TMA engine (16-byte aligned
// addresses, size a multiple of 16), completing as transaction bytes on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
// Allocation: one full warp executes these.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__host__ __device__ constexpr uint64_t smem_desc_bits(uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) | ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) |
         (1ull << 46) | ((uint64_t)(layout & 7) << 61);
}
__device__ __forceinline__ uint64_t smem_desc(const void* p, uint64_t bits) {
  return bits | (uint64_t)((smem_u32(p) >> 4) & 0x3FFF);
}

// kind::f16 / kind::f8f6f4 instruction descriptor, fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_f(uint32_t afmt, uint32_t bfmt, int M, int N,
                                               bool a_mn, bool b_mn) {
  return (1u << 4) | (afmt << 7) | (bfmt << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// kind::mxf4 block-scaled descriptor (E2M1 x E2M1, E8M0 scales, K = 64).
__host__ __device__ constexpr uint32_t idesc_mxf4(int M, int N, uint32_t a_sf_id,
                                                  uint32_t b_sf_id) {
  return (b_sf_id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) |
         ((uint32_t)(M >> 4) << 24) | (a_sf_id << 29);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_f8f6f4(uint32_t d_tmem, uint64_t a, uint64_t b,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;"
      "\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// Scale factors: 32 rows x 16 bytes from shared memory to TMEM columns
// [taddr, taddr+4), replicated into all four 32-lane sub-partitions.
__device__ __forceinline__ void tmem_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}
// Arrive on `bar` once every tcgen05 operation this thread issued before completes.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 bits, 32 consecutive columns -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// Issue-only variant (no wait): pair with tmem_ld_wait() after several loads.
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// Issue-only load of 16 consecutive columns (32 lanes x 32 bits).
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ bool elect_lane0() { return (threadIdx.x & 31) == 0; }

}  // namespace v4a
