// Device-side building blocks for the sm_100a kernels: mbarriers, TMA and
// bulk copies, tcgen05 (TMEM allocation, tensor-core MMA, TMEM loads/stores)
// and the bounded waits every pipeline role uses.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/qoq.h"

namespace qoq {

// ---------------------------------------------------------------- addresses

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarriers

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Upper bound on any single pipeline wait. Nothing inside one launch waits
// this long when the pipeline is healthy (waits are for on-chip hand-offs and
// HBM reads of a few KB), so running out means a lost arrival.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

// Where a bounded wait gave up (workspace word 1 after QOQ_ERR_TIMEOUT).
enum WaitSite : int {
    kSiteProducerFreed = 1,   // TMA producer waiting for a free stage
    kSiteMmaAccEmpty = 2,     // MMA warp waiting for the epilogue to drain an accumulator
    kSiteMmaOperands = 3,     // MMA warp waiting for a token tile / dequantised weights
    kSiteDequantFull = 4,     // dequant warp waiting for a stage's copies
    kSiteEpilogueAcc = 5,     // epilogue waiting for an accumulator
    kSiteOwnerFlag = 6,       // a global flag wait (the watchdog self-test)
    kSiteLastOwner = 7,       // last arriver of a split tile waiting for the owner's partial sums
    kSiteRowsDone = 8,        // fused activation quantisation: waiting for every token row
    kSiteXEmpty = 9,          // token-tile producer / dequantiser waiting for a free A/X stage
    kSiteKvTile = 10,         // KV4 attention warp waiting for its K/V code tile
};

// Shared abort flag + global status word used by the bounded waits. The CTA
// that first fails also records, after the status word, the wait site, its
// block index and a site-specific detail (unit, segment or contributor).
struct Watchdog {
    volatile int *abort_flag;  // shared memory, 0 = healthy
    int *status;               // global status word (workspace[0]); may be null
    __device__ __forceinline__ bool aborted() const { return *abort_flag != 0; }
    __device__ __forceinline__ void fail(int code, int site = 0, int detail = 0) const {
        *abort_flag = 1;
        if (status && atomicCAS(status, 0, code) == 0) {
            status[1] = site;
            status[2] = (int)blockIdx.x;
            status[3] = detail;
        }
    }
};

// Wait for the phase of `bar` with the given parity to complete. Returns
// false (after raising the CTA abort flag and the status word) when the wait
// runs past `limit_ns`, or when another role of the CTA has aborted.
__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, const Watchdog &wd, int site,
                                             int detail, uint64_t limit_ns = kWaitLimitNs) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(a, parity)) return true;
        if ((it & 31u) == 0) {
            if (wd.aborted()) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                wd.fail(QOQ_ERR_TIMEOUT, site, detail);
                return false;
            }
        }
    }
}

// Same, but ignores the abort flag: used at teardown to let copies that are
// already in flight land before the CTA exits.
__device__ __forceinline__ bool wait_drain(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(a, parity)) return true;
        if ((it & 31u) == 0 && globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// ------------------------------------------------------------ TMA and bulk

// 2-D tiled TMA load (no multicast) completing on `bar` with byte accounting.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int x,
                                            int y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

// Contiguous bulk copy global -> shared (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// 2-D tiled TMA store shared -> global, completing in this thread's current
// bulk group. Box elements outside the tensor are not written; the start
// coordinates must be non-negative and x * element size a multiple of 16 B.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *smem_src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
                 "r"(smem_u32(smem_src)), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until at most N of this thread's bulk groups are still in flight.
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) reads of them.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ------------------------------------------------------------------ tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t *smem_result, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// One 128-wide k-tile: four tcgen05.mma (K = 32 each) issued back to back,
// D[tmem] (+)= A[tmem] . B[smem]^T, kind::i8, INT32 accumulate. A columns
// a .. a+31 (8 per MMA); the B descriptor advances 32 bytes (2 units of 16 B)
// per MMA inside the 128-byte swizzle row. `accumulate` applies to the first
// MMA only; the other three always accumulate.
__device__ __forceinline__ void mma4_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%5], %6, %3, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%7], %8, %3, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%9], %10, %3, 1;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(a_tmem + 8u), "l"(b_desc + 2ull),
        "r"(a_tmem + 16u), "l"(b_desc + 4ull), "r"(a_tmem + 24u), "l"(b_desc + 6ull)
        : "memory");
}

// Instruction descriptor for kind::i8: D = S32, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_i8(int m, int n, bool a_signed, bool b_signed) {
    return (2u << 4)                                   // D format: S32
           | ((a_signed ? 1u : 0u) << 7)               // A: 1 = s8, 0 = u8
           | ((b_signed ? 1u : 0u) << 10)              // B: 1 = s8, 0 = u8
           | (static_cast<uint32_t>(n >> 3) << 17)     // N / 8
           | (static_cast<uint32_t>(m >> 4) << 24);    // M / 16
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row core groups 1024 bytes apart. Tile base 1024-aligned.
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);   // start address
    d |= static_cast<uint64_t>(1) << 16;                   // leading offset (unused here)
    d |= static_cast<uint64_t>(1024 >> 4) << 32;           // stride offset: 8 rows x 128 B
    d |= static_cast<uint64_t>(1) << 46;                   // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;                   // SWIZZLE_128B
    return d;
}

// Load + wait in one asm block so no use of the destination registers can be
// scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, uint32_t (&r)[32]) {
    __syncwarp();   // warp-collective (.sync.aligned)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld16_wait(uint32_t taddr, uint32_t (&r)[16]) {
    __syncwarp();   // warp-collective (.sync.aligned)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// 32 lanes x 32 columns store and its completion wait in one asm block, so
// the source registers are never reused early.
__device__ __forceinline__ void tmem_st32_wait(uint32_t taddr, const uint32_t (&r)[32]) {
    __syncwarp();   // warp-collective (.sync.aligned)
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// 32 lanes x 32 columns store without its completion wait. The registers are
// read when the store issues; tmem_st_wait() must still come before anything
// that publishes the stored columns (the fence and arrive that hand them to
// the MMA issuer).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    __syncwarp();   // warp-collective (.sync.aligned)
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
        "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------- CTA pairs (cta_group::2)
// A kernel uses one cta_group for all its tcgen05 instructions; the paired
// GEMM uses these forms. The pair is a cluster of two CTAs; rank 0 (the
// leader) issues the MMAs, which read A from both CTAs' tensor memory and B
// from both CTAs' shared memory (each holds half of the MMA's N), and write
// each CTA's half of the M rows into its own tensor memory.

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// All threads of both CTAs; release/acquire at cluster scope.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t *smem_result, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Arrive on this CTA's `bar` once the pair's tcgen05 operations issued so
// far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// The same, arriving on the barrier at `bar`'s offset in both CTAs of the pair.
__device__ __forceinline__ void tc_commit_pair_both(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Four paired MMAs (K = 32 each) of one 128-wide k-tile, as mma4_i8_ts.
__device__ __forceinline__ void mma4_i8_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%5], %6, %3, 1;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%7], %8, %3, 1;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%9], %10, %3, 1;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(a_tmem + 8u), "l"(b_desc + 2ull),
        "r"(a_tmem + 16u), "l"(b_desc + 4ull), "r"(a_tmem + 24u), "l"(b_desc + 6ull)
        : "memory");
}

// Arrive on the barrier at `bar`'s offset in CTA `rank` of the cluster
// (this CTA included), with the instruction's default release semantics, the
// form CUTLASS's 2-SM pipelines use for cross-CTA arrivals. (The .cluster
// scope release costs the arriving thread about a microsecond on B200: it
// waits for the SM's outstanding memory traffic.)
__device__ __forceinline__ void mbar_arrive_cluster(uint64_t *bar, uint32_t rank) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(bar)), "r"(rank));
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(ra) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// wait_bounded for barriers that CTAs of the cluster arrive on (acquire at
// cluster scope).
__device__ __forceinline__ bool wait_bounded_cluster(uint64_t *bar, uint32_t parity, const Watchdog &wd, int site,
                                                     int detail, uint64_t limit_ns = kWaitLimitNs) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait_cluster(a, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_cluster(a, parity)) return true;
        if ((it & 31u) == 0) {
            if (wd.aborted()) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                wd.fail(QOQ_ERR_TIMEOUT, site, detail);
                return false;
            }
        }
    }
}

// ------------------------------------------- programmatic dependent launch

// Block until the grids this one depends on have completed and their memory
// is visible (returns at once when launched without a programmatic edge).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Allow the next grid in the stream to start launching.
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------- cross-CTA flags (gpu scope)

__device__ __forceinline__ void st_release_gpu(int32_t *p, int32_t v) {
    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}


// Spin until *flag != 0, bounded like the pipeline waits.
__device__ __forceinline__ int32_t ld_relaxed_gpu(const int32_t *p) {
    int32_t v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Atomic add at gpu scope with acquire and release semantics; returns the old value.
__device__ __forceinline__ int32_t atom_add_acq_rel_gpu(int32_t *p, int32_t v) {
    int32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void red_add_release_gpu(int32_t *p, int32_t v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void red_or_release_gpu(int32_t *p, int32_t v) {
    asm volatile("red.release.gpu.global.or.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int32_t ld_acquire_gpu(const int32_t *p) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Orders this thread's generic-proxy accesses of global memory with its
// later async-proxy (TMA) accesses, and the other way round.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Spins until (*p & mask) == want (acquire), bounded like the pipeline waits.
__device__ __forceinline__ bool wait_word_bounded(const int32_t *p, int32_t mask, int32_t want, const Watchdog &wd,
                                                  int site, int detail, uint64_t limit_ns = kWaitLimitNs) {
    if ((ld_acquire_gpu(p) & mask) == want) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if ((ld_acquire_gpu(p) & mask) == want) return true;
        if ((it & 15u) == 0) {
            if (wd.aborted()) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                wd.fail(QOQ_ERR_TIMEOUT, site, detail);
                return false;
            }
        }
    }
}

// Spins until *flag != 0: relaxed loads back to back (a few lanes poll, so no
// sleep between them), then one acquire fence, which with the relaxed load
// that saw the releasing store orders every later access after that store.
__device__ __forceinline__ bool wait_flag_bounded(const int32_t *flag, const Watchdog &wd, int detail,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    if (ld_relaxed_gpu(flag) != 0) {
        fence_acq_rel_gpu();
        return true;
    }
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (ld_relaxed_gpu(flag) != 0) {
            fence_acq_rel_gpu();
            return true;
        }
        if ((it & 15u) == 0) {
            if (wd.aborted()) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                wd.fail(QOQ_ERR_TIMEOUT, kSiteOwnerFlag, detail);
                return false;
            }
        }
    }
}

// ------------------------------------------------------ register reallocation

// Per-warpgroup register budgets: every warp of a warpgroup executes the same
// one. The CTA's pool is what it was launched with (threads x registers per
// thread at launch); increases wait for decreases, so the budgets must add up
// to no more than that pool.
template <int N>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// -------------------------------------------------------------- misc device

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    __syncwarp();   // bar.sync is the .aligned form: the warp must arrive converged
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier over `nthreads` threads that also returns whether `pred` was
// true in any of them (every participating thread gets the same answer).
__device__ __forceinline__ bool named_bar_any(int id, int nthreads, bool pred) {
    __syncwarp();   // bar.red is the .aligned form: the warp must arrive converged
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint4 lds128(uint32_t saddr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(saddr));
    return v;
}

__device__ __forceinline__ uint32_t lds16(uint32_t saddr) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(saddr));
    return v;
}

__device__ __forceinline__ void red_add_s32(int32_t *p, int32_t v) {
    asm volatile("red.relaxed.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int32_t ld_cg_s32(const int32_t *p) {
    int32_t v;
    asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

}  // namespace qoq
