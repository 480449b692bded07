// QoQ W4A8 GEMM for sm_100a: 4-bit weights are rebuilt to INT8 inside the
// main loop and multiplied with per-token INT8 activations on the 5th-gen
// tensor cores (tcgen05.mma kind::i8, INT32 accumulators in tensor memory).
//
// QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM Serving
// (arXiv 2405.04532), paperlayer.ai summary:
//   section 3/4 -- weight-side (not partial-sum) dequantisation keeps the GEMM
//     on INT8 tensor cores; four 4-bit values are decoded per register op;
//   section 4 -- the protective range [-119, 119] guarantees q*s - z*s fits
//     INT8, so the decode needs no saturation;
//   section 5 -- subtraction after multiplication; weights pre-reordered into
//     compute order; per-channel scale (and, for the per-channel variant, the
//     zero point) applied in the epilogue; FP16 output.
//
// Design on B200 (not the pages' A100/L40S design):
//   * swap-AB: the 128 weight rows of a tile are the MMA's M dimension and
//     live in TMEM (tcgen05.mma A operand from tensor memory); tokens are the
//     MMA's N dimension (16..256), staged by TMA in shared memory with the
//     128-byte swizzle. Dequantised weights go registers -> TMEM and never
//     touch shared memory, leaving shared-memory bandwidth to the copies.
//   * one dequant thread owns one weight row of a 128-wide k-tile, which is
//     exactly one quantisation group, so the group's (s, z*s) is a per-thread
//     scalar. 8 nibbles per 32-bit word decode with and/shift, one 32-bit
//     multiply-add (q*s <= 240 and q*s + 128 - z*s in [7, 249] never carry
//     between bytes) and one xor that turns excess-128 bytes into int8.
//   * warp roles: 1 TMA producer warp, 2 MMA issuer warps (lane 0 each), and
//     either two dequant warpgroups that take alternate pipeline units and one
//     epilogue warpgroup (up to 128-token tiles), or one dequant warpgroup and
//     two epilogue warpgroups, one per accumulator half (256-token tiles).
//   * 256-token tiles run on CTA pairs where the n-tiles pair up: one
//     tcgen05.mma.cta_group::2 with M = 256 (each CTA's 128 weight rows in its
//     own tensor memory) and each CTA staging half of the token tile.
//   * a pipeline unit is up to KB consecutive k-tiles of one n-tile: one bulk
//     copy of the packed weights, one TMA per token tile, one TMEM A buffer,
//     one commit that frees both the shared-memory stage and the TMEM buffer.
//   * programmatic dependent launch: the set-up and the first weight copies
//     overlap the previous kernel in the stream; everything the previous
//     kernel may write (activations, scales, outputs, workspace) is touched
//     only after griddepcontrol.wait.
//   * persistent stream-K at k-tile granularity: the (token tile, n-tile,
//     k-tile) blocks, tiles in groups of up to 8 token tiles with the token
//     tile fastest, are split evenly over at most one CTA (pair) per SM (pair). A tile cut
//     between CTAs is finished by whichever of them arrives last on the
//     tile's counter: usually its owner (the CTA holding the tile's first
//     k-tile, which it reaches last), adding the partial sums the others
//     stored; if another CTA of the tile started late, the owner stores its
//     own partial sums instead and that CTA finishes the tile. No CTA waits
//     for one that may not have started, so no co-residency is assumed. The
//     sum is exact in any order.
#include <algorithm>
#include <cstring>

#include "gemm_common.cuh"

namespace qoq {

constexpr int kThreads = 512;            // 16 warps
constexpr int kWarpProducer = 0;
constexpr int kWarpMma = 1;             // warps 1, 2: the two MMA issuers
constexpr int kIssuers = 2;
constexpr int kWarpDequant0 = 4;         // warps 4..: the dequant warpgroups, then the epilogue warpgroups
// Register budgets of the 256-token configuration (512 threads launched with
// 128 registers each): control warpgroup 56, dequant 128, epilogue 2 x 160.
constexpr int kRegsCtlHalves = 56;
constexpr int kRegsEpiHalves = 160;
static_assert(128 * kRegsCtlHalves + 128 * 128 + 256 * kRegsEpiHalves <= kThreads * 128,
              "register split exceeds the launch pool");

template <int TOK, int MODE, bool PAIR = false>
struct GemmCfg {
    // PAIR: a cluster of two CTAs runs one 256-row MMA (tcgen05.mma.cta_group::2):
    // each CTA dequantises its own 128 weight rows into its own tensor memory
    // and stages half of the token tile (tokens rank*TOK/2 ..), so per SM the
    // token-tile bytes per MAC halve; the leader CTA issues the MMAs.
    static_assert(!PAIR || TOK == 256, "paired CTAs are built for 256-token tiles");
    static constexpr int kXRows = PAIR ? TOK / 2 : TOK;        // token rows staged by this CTA
    // KB = k-tiles per pipeline unit: two up to 128-token tiles (halves the
    // barrier and issue work per weight byte), one for 256-token tiles
    // (shared memory holds only two two-k-tile stages of those).
    static constexpr int kKB = TOK <= 128 ? 2 : 1;
    static constexpr int kXTile = kXRows * 128;                 // this CTA's token rows, 128 k
    static constexpr int kWTile = MODE == 0 ? 8448 : 8192;      // codes (+ s, z*s) per k-tile
    static constexpr int kXBytes = kKB * kXTile;
    static constexpr int kWBytes = kKB * kWTile;
    static constexpr int kStageBytes = (kXBytes + kWBytes + 1023) / 1024 * 1024;
    static constexpr int kSmemLimit = 232448;                   // 227 KB per CTA
    // After the stages: 1 KB alignment slack, the control block (3 KB) and
    // the epilogue warps' output staging (two 1 KB blocks per warp).
    static constexpr int kCtlBytes = 3072;
    static constexpr int kReserve = 1024 + kCtlBytes + (TOK == 256 ? 8 : 4) * 2048;
    // Two MMA issuers. Up to 64-token tiles (kAlt), issuer j takes the units
    // of index parity j (those its dequant warpgroup serves) into its own
    // accumulator, and the epilogue adds the two; wider tiles have no TMEM for
    // a second accumulator, and issuer j takes token columns j*TOK/2 .. of
    // every unit.
    static constexpr bool kAlt = TOK <= 64;
    static constexpr int kAccCols = kAlt ? 2 * TOK : TOK;   // TMEM columns per accumulator buffer
    static constexpr int kAccBufs = (TOK == 64 || TOK == 256) ? 1 : 2;
    static constexpr int kACol0 = kAccBufs * kAccCols;
    // 256-token tiles have no second accumulator buffer. Each issuer's half of
    // the token columns goes to the epilogue and back on its own barrier pair
    // (acc_full[k], acc_empty[k]), so issuer 0 starts the next tile as soon as
    // the epilogue has read the first half.
    static constexpr bool kHalves = TOK == 256;
    // Warpgroups after the producer/issuer warps (12 warps): two dequant and
    // one epilogue warpgroup, except for 256-token tiles, whose main loop needs
    // one k-tile decoded per 512 tensor-core cycles (one warpgroup keeps up)
    // and whose epilogue is not overlapped with the next tile's main loop:
    // there one dequant warpgroup and two epilogue warpgroups, one per half.
    static constexpr int kDqGroups = kHalves ? 1 : 2;
    static constexpr int kEpiGroups = kHalves ? 2 : 1;
    static constexpr int kWarpEpi0 = kWarpDequant0 + 4 * kDqGroups;
    static_assert(kWarpEpi0 + 4 * kEpiGroups == kThreads / 32, "warp roles must fill the CTA");
    // One CTA per SM (shared memory use guarantees it), so the CTA takes all
    // 512 TMEM columns: accumulators first, then one A buffer per stage
    // (32 columns per dequantised 128x128 k-tile).
    static constexpr int kTmemCols = 512;
    static constexpr int kStagesSmem = (kSmemLimit - kReserve) / kStageBytes;
    static constexpr int kStagesTmem = (kTmemCols - kACol0) / (kKB * 32);
    static constexpr int kStagesMin = kStagesSmem < kStagesTmem ? kStagesSmem : kStagesTmem;
    // With two dequant warpgroups even, so that stage s is always dequantised
    // by warpgroup s % 2 (they take alternate units); each warpgroup then waits
    // on every phase of the stages it reads. One warpgroup takes every stage.
    static constexpr int kStages = (kStagesMin > 16 ? 16 : kStagesMin) & (kHalves ? ~0 : ~1);
    static constexpr int kSmemBytes = kStages * kStageBytes + kReserve;
    static_assert(kStages >= 4, "pipeline too shallow");
    static_assert(kACol0 + kStages * kKB * 32 <= kTmemCols, "TMEM over-subscribed");
    static_assert(kSmemBytes > 232448 / 2, "two CTAs per SM would contend for TMEM");
    static_assert(kXTile % 1024 == 0, "token tile must keep the swizzle atom aligned");
};

struct GemmParams {
    const uint8_t *blob;
    const __half *s_x;
    const int32_t *rowsum;
    void *out;
    int32_t *status;
    int32_t *flags;         // [grid]: arrival counter of the split tile owned by schedule unit c (bit 16: owner's sums stored)
    int32_t *partials;      // [grid][2][TOK][128]: CTA c's partial sums as a contributor (0) and as an owner (1)
    long long late_arrival_ns;   // test override: contributors' arrivals delayed by this long (0)
    int M, N, K, group;
    int NT, KT, MT;
    int NTw;                // n-tiles of the schedule: NT, or NT / 2 CTA pairs' 256-row tiles
    int GM;                 // token tiles per group of the tile order
    int grid;
    uint32_t total_blocks;  // MT * NT * KT (k-tile blocks)
    uint32_t dp_tiles;      // tiles 0 .. dp_tiles-1 go whole to CTAs in data-parallel waves
    uint32_t sk_base;       // first block of the stream-K tail: dp_tiles * KT
    long long off_codes, off_scale, off_zero;
    int fp16_out;
};

struct SharedCtl {
    uint64_t full[16], freed[16], a_full[16];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t final_bar[2];
    uint32_t tmem_base;
    int abort_flag;
    int fix_old;            // the epilogue leader's arrival-counter value, broadcast
    // The owner's epilogue inputs of the current token tile, staged once per
    // tile: FP32(s_x) and (per-channel variant) the row sums.
    alignas(16) float tok_scale[256];
    int32_t tok_rowsum[256];
};
static_assert(sizeof(SharedCtl) <= GemmCfg<16, 0>::kCtlBytes, "control block outgrows its reserve");

// Four codes (bytes of b4, each 0..15) to int8 q*s - z*s, saturated to
// [-128, 127] per byte: the decode a kernel needs when dequantised weights can
// leave the INT8 range (no protective range). Each pair of codes is widened to
// 16-bit lanes, multiplied, shifted by z*s, clamped and narrowed again. With
// the protective range the clamp never acts, so the bytes equal the
// excess-128 decode's.
__device__ __forceinline__ uint32_t decode4_saturating(uint32_t b4, uint32_t s, uint32_t zs2) {
    uint32_t a = __byte_perm(b4, 0u, 0x4140) * s;   // codes 0, 1 in 16-bit lanes
    uint32_t b = __byte_perm(b4, 0u, 0x4342) * s;   // codes 2, 3
    a = __vsub2(a, zs2);
    b = __vsub2(b, zs2);
    a = __vmaxs2(__vmins2(a, 0x007F007Fu), 0xFF80FF80u);
    b = __vmaxs2(__vmins2(b, 0x007F007Fu), 0xFF80FF80u);
    return __byte_perm(a, b, 0x6420);
}

template <int TOK, int MODE, bool PAIR, bool SAT>
__global__ void __launch_bounds__(kThreads, 1)
    qoq_gemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ CUtensorMap tmap_x,
                    const __grid_constant__ CUtensorMap tmap_y) {
    using C = GemmCfg<TOK, MODE, PAIR>;
    constexpr int S = C::kStages;
    constexpr int KB = C::kKB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SharedCtl *ctl = reinterpret_cast<SharedCtl *>(smem + S * C::kStageBytes);
    // Per epilogue warp, two alternating blocks of one step's FP16 outputs
    // (16 tokens x 32 weight rows), the source of the TMA output stores.
    __half *out_stage = reinterpret_cast<__half *>(smem + S * C::kStageBytes + C::kCtlBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Watchdog wd{&ctl->abort_flag, p.status};
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;   // 0: the pair's leader (MMA issue)

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        ctl->abort_flag = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->freed[s], (C::kAlt || PAIR) ? 1 : kIssuers);
            // the four warps of one dequant warpgroup (of each CTA of a pair)
            mbar_init(&ctl->a_full[s], PAIR ? 8 : 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->acc_full[b], C::kHalves ? 1 : kIssuers);
            mbar_init(&ctl->acc_empty[b], PAIR ? 8 : 4);
        }
        mbar_init(&ctl->final_bar[0], 1);
        mbar_init(&ctl->final_bar[1], 1);
        mbar_fence_init();
        // No kernel that releases its dependents early (this GEMM, the
        // activation quantiser) writes a blob, so the blob may be read before
        // griddepcontrol.wait; read at L2, as the TMA weight copies are.
        // The five words are loaded together (one round trip), then compared.
        const int32_t *h = reinterpret_cast<const int32_t *>(p.blob);
        const int32_t h0 = ld_cg_s32(h), h1 = ld_cg_s32(h + 1), h2 = ld_cg_s32(h + 2), h3 = ld_cg_s32(h + 3),
                      h4 = ld_cg_s32(h + 4);
        if ((uint32_t)h0 != kMagic || (uint32_t)h1 != kVersion || h2 != p.N || h3 != p.K || h4 != p.group)
            ctl->abort_flag = 1;   // reported on the status word after griddepcontrol.wait
    }
    if (warp == kWarpProducer && lane == 0) prefetch_tensormap(&tmap_x);
    if (warp == C::kWarpEpi0 && lane == 0 && p.fp16_out) prefetch_tensormap(&tmap_y);
    if (warp == kWarpMma) {
        if (PAIR) {
            tmem_alloc_pair(&ctl->tmem_base, C::kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&ctl->tmem_base, C::kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    // A pair's CTAs arrive on the leader's barriers and the leader's MMAs
    // write both CTAs' tensor memory: both set-ups complete first.
    if (PAIR) cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    griddep_launch_dependents();   // the next kernel may start its own set-up
    const bool bad_blob = wd.aborted();
    if (bad_blob && threadIdx.x == 0) {
        griddep_wait();
        atomicCAS(p.status, 0, QOQ_ERR_BAD_BLOB);
    }

    // This CTA's schedule: the whole tiles blockIdx.x + w * grid below
    // p.dp_tiles (`waves` of them), then its stream-K share [b0, b1) of the
    // tail blocks [sk_base, total) in (token tile, n-tile, k-tile) order,
    // k-tile fastest.
    // With CTA pairs the schedule's unit is the pair (both CTAs walk the same
    // blocks, each for its own n-tile 2 * nt + rank).
    const uint32_t me = PAIR ? (blockIdx.x >> 1) : blockIdx.x;
    const uint32_t G = (uint32_t)p.grid;
    const int waves = p.dp_tiles > me ? (int)((p.dp_tiles - me + G - 1) / G) : 0;
    const uint32_t BS = p.total_blocks - p.sk_base;   // stream-K tail blocks
    const uint32_t b0 = p.sk_base + cta_begin(me, BS, G);
    const uint32_t b1 = p.sk_base + cta_begin(me + 1, BS, G);
    const int KT = p.KT;

    auto stage_x = [&](int s) { return smem + s * C::kStageBytes; };
    auto stage_w = [&](int s) { return smem + s * C::kStageBytes + C::kXBytes; };

    if (!bad_blob) {
        // 256-token tiles: the epilogue warpgroups hold half a tile of packed
        // FP16 results in registers (to hand the accumulator back early), so
        // the control warpgroup gives them part of its budget; each
        // warpgroup sets it at the top of its own branch.
        if (warp < kWarpDequant0) {
        if constexpr (C::kHalves) regs_dec<kRegsCtlHalves>();
        if (warp == kWarpProducer) {
            // ------------------------------------------------ TMA producer
            const uint64_t pol_w = policy_evict_first();   // weights: streamed once
            const uint64_t pol_x = policy_evict_last();    // activations: reused by every n-tile
            UnitCursor<KB> cur;
            cur.init(me, G, waves, b0, b1, KT, p.NTw, p.MT, p.GM);
            auto issue_w = [&](int s, const UnitCursor<KB> &c) {
                mbar_arrive_expect_tx(&ctl->full[s], (uint32_t)(c.nk * (C::kWTile + C::kXTile)));
                const int nt_cta = PAIR ? 2 * c.nt + (int)rank : c.nt;
                const uint8_t *wsrc = p.blob + p.off_codes + ((long long)nt_cta * KT + c.kt) * C::kWTile;
                bulk_load(stage_w(s), wsrc, (uint32_t)(c.nk * C::kWTile), &ctl->full[s], pol_w);
            };
            auto issue_x = [&](int s, const UnitCursor<KB> &c) {
                for (int j = 0; j < c.nk; ++j)
                    tma_load_2d(stage_x(s) + j * C::kXTile, &tmap_x, &ctl->full[s], (c.kt + j) * kTileK,
                                c.mt * TOK + (int)rank * C::kXRows, pol_x);
            };
            // The first S units need no free stage: start their weight copies
            // before waiting for the previous kernel, then their token tiles.
            int npre = 0;
            {
                UnitCursor<KB> c1 = cur;
                for (; npre < S && !c1.done(); ++npre) {
                    if (lane == 0) issue_w(npre, c1);
                    c1.advance();
                }
            }
            __syncwarp();
            griddep_wait();
            if (lane == 0) {
                UnitCursor<KB> c2 = cur;
                for (int i = 0; i < npre; ++i) {
                    issue_x(i, c2);
                    c2.advance();
                }
            }
            __syncwarp();
            for (int i = 0; i < npre; ++i) cur.advance();
            int issued = npre;
            int s = npre % S;
            uint32_t ph = (uint32_t)(npre / S) & 1u;
            for (int i = npre; !cur.done(); ++i) {
                const bool ok = __all_sync(0xffffffffu, wait_bounded(&ctl->freed[s], ph ^ 1u, wd, kSiteProducerFreed, i));
                if (!ok) break;
                if (lane == 0) {
                    issue_w(s, cur);
                    issue_x(s, cur);
                }
                __syncwarp();
                issued = i + 1;
                cur.advance();
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            // Let every copy that was issued land before the CTA can exit.
            if (lane == 0)
                for (int i = issued > S ? issued - S : 0; i < issued; ++i)
                    wait_drain(&ctl->full[i % S], (uint32_t)(i / S) & 1u, kDrainNs);
            __syncwarp();
        } else if (warp == kWarpMma || warp == kWarpMma + 1) {
            // ------------------------------------------------ MMA issuers
            // Lane 0 of each issuer warp runs the role. A thread's mbarrier
            // waits stall its own queued tensor-core work, so two issuers that
            // take turns keep the tensor core busy through each other's waits.
            // Up to 64-token tiles: issuer k takes the units of parity k (with
            // an even stage count always the same stages, whose every phase it
            // waits on) into its own accumulator and commits their freed[s].
            // Wider tiles: both issuers take every unit, each half of the
            // token columns, and both commit freed[s]. Both commit acc_full.
            // A pair has one issuer, lane 0 of the leader's first issuer warp:
            // one M = 256, N = TOK MMA per K = 32 step covers both CTAs.
            const int k = warp - kWarpMma;
            if (lane == 0 && (!PAIR || (rank == 0 && k == 0))) {
                constexpr bool ALT = C::kAlt;
                constexpr uint32_t idesc = idesc_i8(PAIR ? 256 : 128, (ALT || PAIR) ? TOK : TOK / 2, true, true);
                UnitCursor<KB> cur;
                cur.init(me, G, waves, b0, b1, KT, p.NTw, p.MT, p.GM);
                int s = 0, seg = 0, unit = 0;
                uint32_t ph = 0;
                bool ok = true;
                while (ok && !cur.done()) {
                    const int buf = seg % C::kAccBufs;
                    const uint32_t aph = (uint32_t)(seg / C::kAccBufs) & 1u;
                    const int bi = C::kHalves ? k : buf;   // this issuer's accumulator barrier pair
                    if (PAIR)   // both halves, released by the epilogues of both CTAs
                        ok = wait_bounded_cluster(&ctl->acc_empty[0], aph ^ 1u, wd, kSiteMmaAccEmpty, seg) &&
                             wait_bounded_cluster(&ctl->acc_empty[1], aph ^ 1u, wd, kSiteMmaAccEmpty, seg);
                    else
                        ok = wait_bounded(&ctl->acc_empty[bi], aph ^ 1u, wd, kSiteMmaAccEmpty, seg);
                    if (!ok) break;
                    const uint32_t d_tmem = tmem_base + (uint32_t)(buf * C::kAccCols + k * (ALT ? TOK : TOK / 2));
                    uint32_t acc = 0u;   // this issuer's first MMA of the segment overwrites its accumulator
                    bool seg_done = false;
                    while (!seg_done) {
                        if (!ALT || (unit & 1) == k) {
                            // The dequantised weights (TMEM) of this unit.
                            // One wait covers the token tile too: the dequant
                            // warps arrive on a_full[s] only after their own
                            // wait on full[s], which counts the token tile's
                            // bytes, and the arrivals order that completion
                            // before this thread's MMAs. Each wait of an
                            // issuing thread costs it hundreds of cycles, so
                            // the issuer waits once per unit.
                            ok = PAIR ? wait_bounded_cluster(&ctl->a_full[s], ph, wd, kSiteMmaOperands, unit)
                                      : wait_bounded(&ctl->a_full[s], ph, wd, kSiteMmaOperands, unit);
                            if (!ok) break;
                            tc_fence_after();
                            const uint32_t a_tmem = tmem_base + (uint32_t)(C::kACol0 + s * KB * 32);
                            const uint64_t bdesc = smem_desc_k_sw128(smem_u32(stage_x(s)));
                            // Per k-tile j of the unit: four MMAs; the token
                            // tile of k-tile j lies kXTile bytes further on,
                            // and (N split) issuer k's token rows k*TOK/2 ..
                            // another (TOK/2) x 128 bytes on.
                            const uint64_t bk = bdesc + (uint64_t)(ALT ? 0 : k * (TOK / 2) * 128 / 16);
                            if (PAIR) {
                                mma4_i8_ts_pair(d_tmem, a_tmem, bk, idesc, acc);
                                acc = 1u;
                                tc_commit_pair_both(&ctl->freed[s]);
                            } else {
                                mma4_i8_ts(d_tmem, a_tmem, bk, idesc, acc);
                                if (KB == 2 && cur.nk == 2)
                                    mma4_i8_ts(d_tmem, a_tmem + 32u, bk + (uint64_t)(C::kXTile >> 4), idesc, 1u);
                                acc = 1u;
                                tc_commit(&ctl->freed[s]);
                            }
                        }
                        ++unit;
                        if (++s == S) {
                            s = 0;
                            ph ^= 1u;
                        }
                        seg_done = cur.advance();
                    }
                    if (!ok) break;
                    if (PAIR) {
                        tc_commit_pair_both(&ctl->acc_full[0]);
                        tc_commit_pair_both(&ctl->acc_full[1]);
                    } else {
                        tc_commit(&ctl->acc_full[bi]);
                    }
                    ++seg;
                }
                // Every MMA must have completed before tensor memory is freed.
                if (PAIR)
                    tc_commit_pair(&ctl->final_bar[k]);
                else
                    tc_commit(&ctl->final_bar[k]);
                wait_drain(&ctl->final_bar[k], 0, kDrainNs);
            }
            __syncwarp();
        }
        } else if (warp >= kWarpDequant0 && warp < C::kWarpEpi0) {
            // ------------------------------------------------ dequant
            // With two warpgroups, warpgroup g takes the units i with
            // i % 2 == g, i.e. (the stage count being even) always the same
            // stages: it waits on every phase of those stage barriers and on no
            // others, so parity waits cannot alias. A single warpgroup takes
            // every unit. Thread (quarter, lane) decodes weight row r of each
            // k-tile.
            const int g = (warp - kWarpDequant0) >> 2;
            const int quarter = warp & 3;                    // TMEM lanes 32q .. 32q+31
            const int r = quarter * 32 + lane;               // weight row in the tile
            const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
            UnitCursor<KB> cur;
            cur.init(me, G, waves, b0, b1, KT, p.NTw, p.MT, p.GM);
            int s = 0;
            uint32_t ph = 0;
            for (int i = 0; !cur.done(); ++i, cur.advance()) {
                const int unit_s = s;
                const uint32_t unit_ph = ph;
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
                if (C::kDqGroups == 2 && (i & 1) != g) continue;
                // full[s] for this unit implies the producer saw freed[s] for
                // the unit S earlier, i.e. TMEM A buffer s is no longer read.
                const bool ok = __all_sync(0xffffffffu, wait_bounded(&ctl->full[unit_s], unit_ph, wd, kSiteDequantFull, i));
                if (!ok) break;
                tc_fence_after();   // the TMEM writes below come after the wait (and the MMA reads it implies)
                const uint32_t a_col = tmem_base + lane_addr + (uint32_t)(C::kACol0 + unit_s * KB * 32);
                const int nk = cur.nk;
                // All shared-memory loads of the unit first (four 16-byte code
                // chunks and the (s, z*s) pair per k-tile), then per k-tile the
                // decode and one 32-column TMEM store.
                uint4 v[KB][4];
                uint32_t sz[KB];
#pragma unroll
                for (int j = 0; j < KB; ++j) {
                    if (j < nk) {
                        const uint32_t wbase = smem_u32(stage_w(unit_s) + j * C::kWTile);
                        sz[j] = MODE == 0 ? lds16(wbase + 8192 + 2 * r) : 0u;
#pragma unroll
                        for (int c = 0; c < 4; ++c) v[j][c] = lds128(wbase + c * 2048 + r * 16);
                    }
                }
#pragma unroll
                for (int j = 0; j < KB; ++j) {
                    if (j < nk) {
                        const uint32_t sc = sz[j] & 0xFFu;
                        const uint32_t c4 = (uint32_t)(128 - (int)(int8_t)(sz[j] >> 8)) * 0x01010101u;
                        const uint32_t zs2 = ((uint32_t)(int32_t)(int8_t)(sz[j] >> 8) & 0xFFFFu) * 0x00010001u;
                        uint32_t o[32];
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const uint32_t w[4] = {v[j][c].x, v[j][c].y, v[j][c].z, v[j][c].w};
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const uint32_t lo = w[q] & 0x0F0F0F0Fu;
                                const uint32_t hi = (w[q] >> 4) & 0x0F0F0F0Fu;
                                if (MODE == 0 && SAT) {
                                    o[8 * c + 2 * q] = decode4_saturating(lo, sc, zs2);
                                    o[8 * c + 2 * q + 1] = decode4_saturating(hi, sc, zs2);
                                } else if (MODE == 0) {
                                    o[8 * c + 2 * q] = (lo * sc + c4) ^ 0x80808080u;
                                    o[8 * c + 2 * q + 1] = (hi * sc + c4) ^ 0x80808080u;
                                } else {
                                    o[8 * c + 2 * q] = lo;
                                    o[8 * c + 2 * q + 1] = hi;
                                }
                            }
                        }
                        tmem_st32_wait(a_col + (uint32_t)(j * 32), o);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR)
                        mbar_arrive_cluster(&ctl->a_full[unit_s], 0);   // the leader's barrier
                    else
                        mbar_arrive(&ctl->a_full[unit_s]);
                }
                __syncwarp();
            }
        } else if (warp >= C::kWarpEpi0) {
            if constexpr (C::kHalves) regs_inc<kRegsEpiHalves>();
            // ------------------------------------------------ epilogue
            // kEpiGroups warpgroups. Each reads its share of the accumulator's
            // parts: with two (256-token tiles), warpgroup e takes issuer e's
            // half of the token columns, waiting on acc_full[e] and handing it
            // back on acc_empty[e]; with one, the whole buffer. Named barrier
            // 1 + e syncs one warpgroup, barrier 3 all epilogue warps.
            constexpr int NEPI = 128 * C::kEpiGroups;
            constexpr int kBarAll = C::kEpiGroups == 2 ? 3 : 1;
            const int e = (warp - C::kWarpEpi0) >> 2;
            const int quarter = warp & 3;
            const int r = quarter * 32 + lane;
            const int te = threadIdx.x - (C::kWarpEpi0 + 4 * e) * 32;   // thread within the warpgroup
            const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
            const bool leader = (threadIdx.x == C::kWarpEpi0 * 32);
            // A part of the accumulator goes back to the issuer's CTA.
            auto acc_release = [&](uint64_t *bar) {
                if (PAIR)
                    mbar_arrive_cluster(bar, 0);
                else
                    mbar_arrive(bar);
            };
            // Flag and partial-sum slot of contributor c (a schedule unit).
            auto fidx = [&](uint32_t c) { return PAIR ? 2u * c + rank : c; };
            griddep_wait();   // outputs, scales, row sums and workspace belong to the previous kernel until now
            UnitCursor<KB> cur;
            cur.init(me, G, waves, b0, b1, KT, p.NTw, p.MT, p.GM);
            int seg = 0, ubase = 0;
            int obuf = 0;   // this warp's next output stage block
            while (!cur.done()) {
                const uint32_t seg_b = cur.b, seg_e = cur.seg_end;
                const int kt_lo = cur.kt, kt_hi = cur.kt + (int)(seg_e - seg_b);
                const int mt = cur.mt, nt = cur.nt;
                const uint32_t tile_b = seg_b - (uint32_t)kt_lo;
                int nunits = 1;
                while (!cur.advance()) ++nunits;
                // Up to 64-token tiles: the segment's first unit went to issuer
                // (ubase & 1), whose accumulator is `prim`; the other issuer's
                // (`second`) holds data only if the segment has two units or more.
                const int prim = C::kAlt ? (ubase & 1) : 0;
                ubase += nunits;
                const int buf = seg % C::kAccBufs;
                const uint32_t aph = (uint32_t)(seg / C::kAccBufs) & 1u;
                const int n = (PAIR ? 2 * nt + (int)rank : nt) * kTileN + r;
                const int64_t m0 = (int64_t)mt * TOK;
                const bool two = C::kAlt && nunits >= 2;
                // Token columns of the tile that hold tokens (>= 1): the steps
                // past them (a ragged last tile) are neither loaded nor stored.
                const int m_live = (int)(p.M - m0 < TOK ? p.M - m0 : TOK);
                // Roles in a tile: sole computer (all of its k-tiles), owner (its
                // first k-tile, not all) or contributor. The schedule units
                // sharing a split tile, t_first (the owner) .. t_last, count their
                // arrivals on the tile's counter, and whoever arrives last adds
                // the others' partial sums and writes the tile. The owner arrives
                // as it starts the tile's epilogue: with every contributor in
                // (the usual case: contributors reach their share first), it
                // finishes the tile from its accumulator; otherwise it stores its
                // partial sums in its owner slot and sets bit 16 of the counter,
                // and the last contributor, finding the owner arrived, waits only
                // for that bit. No CTA waits for one that may not have started.
                const bool owner = kt_lo == 0;
                const bool sole = owner && kt_hi == KT;
                uint32_t t_first = me, t_last = me;
                if (!sole) {
                    t_first = owner ? me : cta_of(tile_b - p.sk_base, BS, G);
                    t_last = cta_of(tile_b + (uint32_t)KT - 1 - p.sk_base, BS, G);
                }
                const int nparts = (int)(t_last - t_first + 1);
                int32_t *cnt = p.flags + fidx(t_first);
                // Contributors whose slots the finishing owner adds.
                const uint32_t c_first = t_first + 1, c_last = t_last;
                constexpr int CO = 16;   // token columns per step
                // The parts this warpgroup reads: [h_lo, h_hi) of NP, PART columns each.
                constexpr int NP = C::kHalves ? 2 : 1;
                constexpr int PART = TOK / NP;
                const int h_lo = C::kEpiGroups == 2 ? e : 0, h_hi = C::kEpiGroups == 2 ? e + 1 : NP;
                float col_scale = 0.0f;
                int col_zero = 0;
                // The tile's epilogue inputs that depend neither on the
                // accumulator nor on other CTAs: the weight row's scale (and
                // zero point), and the token scales (and row sums) of this
                // warpgroup's columns, staged in shared memory once per tile.
                // The previous segment's readers have passed its closing
                // barrier; a barrier before the first read orders these stores.
                auto stage_tile = [&]() {
                    col_scale = __half2float(reinterpret_cast<const __half *>(p.blob + p.off_scale)[n]);
                    if (MODE == 1)
                        col_zero = __half2int_rn(reinterpret_cast<const __half *>(p.blob + p.off_zero)[n]);
                    for (int j = h_lo * PART + te; j < h_hi * PART; j += 128) {
                        const int64_t m = m0 + j < p.M ? m0 + j : p.M - 1;
                        ctl->tok_scale[j] = p.fp16_out ? __half2float(p.s_x[m]) : 0.0f;
                        if (MODE == 1) ctl->tok_rowsum[j] = p.rowsum[m];
                    }
                };
                // The owner's arrival, as it starts the tile's epilogue.
                bool finish_here = sole;
                if (owner && !sole) {
                    if (leader) ctl->fix_old = atom_add_acq_rel_gpu(cnt, 1);
                    named_bar_sync(kBarAll, NEPI);
                    finish_here = (ctl->fix_old & 0xFFFF) == nparts - 1;
                }
                if (owner) stage_tile();
                // Each part is handed back to its issuer right after its last
                // TMEM load. Every lane spins on its own; the votes reconverge
                // the warps before the named barriers, and all epilogue warps
                // leave together.
                const int live_end = (m_live + CO - 1) / CO * CO;   // token columns read and stored
                const uint32_t acc_addr = tmem_base + lane_addr + (uint32_t)(buf * C::kAccCols + prim * TOK);
                const uint32_t acc2_addr = tmem_base + lane_addr + (uint32_t)(buf * C::kAccCols + (prim ^ 1) * TOK);
                // This CTA's partial-sum slot for the tile: slot 0 as a
                // contributor, slot 1 as an owner that is not the last to arrive.
                auto slot_of = [&](uint32_t c, int role) {
                    return p.partials + ((long long)fidx(c) * 2 + role) * TOK * kTileN;
                };
                int32_t *slot = slot_of(me, owner ? 1 : 0);
                bool fail = false;
                for (int h = h_lo; h < h_hi && !fail; ++h) {
                    const int bi = C::kHalves ? h : buf;
                    const uint32_t fph = C::kHalves ? (uint32_t)(seg & 1) : aph;
                    const bool ok =
                        __all_sync(0xffffffffu, wait_bounded(&ctl->acc_full[bi], fph, wd, kSiteEpilogueAcc, seg));
                    if (named_bar_any(1 + e, 128, !ok)) {
                        fail = true;
                        break;
                    }
                    tc_fence_after();
                    const int c_lo = h * PART;
                    const int c_hi = live_end < c_lo + PART ? live_end : c_lo + PART;
                    if (c_hi <= c_lo) {   // no token in this part: hand it back at once
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) acc_release(&ctl->acc_empty[bi]);
                        continue;
                    }
                    if (C::kHalves && sole && p.fp16_out) {
                        // A whole tile of this CTA (no partial sums): convert the
                        // part to FP16 in registers, hand the accumulator back,
                        // then store while the issuer runs the next tile.
                        constexpr int NS = PART / CO;
                        uint32_t pk[NS][CO / 2];
#pragma unroll
                        for (int q = 0; q < NS; ++q) {
                            const int c0 = c_lo + q * CO;
                            if (c0 < c_hi) {
                                uint32_t v[CO];
                                tmem_load<CO>(acc_addr + (uint32_t)c0, v);
                                if (c0 + CO >= c_hi) {
                                    tc_fence_before();
                                    __syncwarp();
                                    if (lane == 0) acc_release(&ctl->acc_empty[bi]);
                                }
                                convert_fp16<CO, MODE>(v, pk[q], col_scale, col_zero, ctl->tok_scale + c0,
                                                       ctl->tok_rowsum + c0);
                            }
                        }
#pragma unroll
                        for (int q = 0; q < NS; ++q) {
                            const int c0 = c_lo + q * CO;
                            if (c0 < c_hi) {
                                store_packed_fp16(&tmap_y, pk[q], m0 + c0, n - lane, lane,
                                                  out_stage + ((warp - C::kWarpEpi0) * 2 + obuf) * (16 * 32));
                                obuf ^= 1;
                            }
                        }
                        continue;
                    }
#pragma unroll 1
                    for (int c0 = c_lo; c0 < c_hi; c0 += CO) {
                        uint32_t v[CO];
                        tmem_load<CO>(acc_addr + (uint32_t)c0, v);
                        if (two) add_second<CO>(acc2_addr + (uint32_t)c0, v);
                        if (c0 + CO >= c_hi) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) acc_release(&ctl->acc_empty[bi]);
                        }
                        if (!finish_here) {
                            // Not the last to arrive: the live token columns of
                            // the partial sums go to this CTA's slot.
#pragma unroll
                            for (int j = 0; j < CO; ++j)
                                if (c0 + j < m_live) slot[(c0 + j) * kTileN + r] = (int32_t)v[j];
                            continue;
                        }
                        // Owner: add the contributors' partial sums: eight
                        // contributors per L2 round trip when at most four
                        // columns hold tokens, four otherwise. Columns past the
                        // live ones hold stale values (contributors store only
                        // the live ones); they belong to no token and are never
                        // stored.
                        if (m_live <= 4) {
#pragma unroll 1
                            for (uint32_t c = c_first; c <= c_last; c += 8) {
                                int32_t t[8][4];
#pragma unroll
                                for (int cc = 0; cc < 8; ++cc) {
                                    const int32_t *part = slot_of(c + cc, 0) + c0 * kTileN + r;
#pragma unroll
                                    for (int j = 0; j < 4; ++j)
                                        t[cc][j] = (c + cc <= c_last) ? ld_cg_s32(part + j * kTileN) : 0;
                                }
#pragma unroll
                                for (int cc = 0; cc < 8; ++cc)
#pragma unroll
                                    for (int j = 0; j < 4; ++j) v[j] += (uint32_t)t[cc][j];   // modulo 2^32: exact where the sum fits
                            }
                        } else {
#pragma unroll 1
                            for (uint32_t c = c_first; c <= c_last; c += 4) {
                                int32_t t[4][CO];
#pragma unroll
                                for (int cc = 0; cc < 4; ++cc) {
                                    const int32_t *part = slot_of(c + cc, 0) + c0 * kTileN + r;
#pragma unroll
                                    for (int j = 0; j < CO; ++j)
                                        t[cc][j] = (c + cc <= c_last) ? ld_cg_s32(part + j * kTileN) : 0;
                                }
#pragma unroll
                                for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                                    for (int j = 0; j < CO; ++j) v[j] += (uint32_t)t[cc][j];   // modulo 2^32: exact where the sum fits
                            }
                        }
                        if (p.fp16_out) {
                            store_outputs_fp16<CO, MODE>(&tmap_y, v, m0 + c0, n - lane, lane, col_scale, col_zero,
                                                         ctl->tok_scale + c0, ctl->tok_rowsum + c0,
                                                         out_stage + ((warp - C::kWarpEpi0) * 2 + obuf) * (16 * 32));
                            obuf ^= 1;
                        } else {
                            store_outputs_i32<CO, MODE>(static_cast<int32_t *>(p.out), p.M, p.N, v, m0 + c0, n, col_zero,
                                                        ctl->tok_rowsum + c0);
                        }
                    }
                }
                // Closing barrier of the segment (all epilogue warps): every
                // read of the staged scales and of other CTAs' partial sums is
                // done, and every partial-sum store of this CTA comes before the
                // leader's release (release is cumulative, so the finisher's
                // acquire sees them all). It also carries the failure vote, so
                // that all warps leave together.
                if (named_bar_any(kBarAll, NEPI, fail)) break;
                if (!sole) {
                    if (owner) {
                        if (finish_here) {
                            if (leader) *cnt = 0;   // nobody touches the counter again in this launch
                        } else {
                            if (leader) red_or_release_gpu(cnt, 0x10000);   // the owner's sums are in
                        }
                    } else {
                        // A contributor arrives; the last one finishes the tile.
                        // (QOQ_FORCE_CONFIG=lateck=us delays the arrival, so
                        // that owners arrive first and contributors finish.)
                        if (leader && p.late_arrival_ns) {
                            const uint64_t t_end = globaltimer_ns() + (uint64_t)p.late_arrival_ns;
                            while (globaltimer_ns() < t_end) __nanosleep(1000);
                        }
                        if (leader) ctl->fix_old = atom_add_acq_rel_gpu(cnt, 1);
                        named_bar_sync(kBarAll, NEPI);
                        if ((ctl->fix_old & 0xFFFF) == nparts - 1) {
                            // The owner has arrived (it is running) but may not
                            // have stored its sums yet.
                            bool got = true;
                            if (leader) got = wait_word_bounded(cnt, 0x10000, 0x10000, wd, kSiteLastOwner, (int)t_first);
                            stage_tile();
                            if (named_bar_any(kBarAll, NEPI, !got)) break;
                            for (int h = h_lo; h < h_hi; ++h) {
                                const int c_lo = h * PART;
                                const int c_hi = live_end < c_lo + PART ? live_end : c_lo + PART;
#pragma unroll 1
                                for (int c0 = c_lo; c0 < c_hi; c0 += CO) {
                                    uint32_t v[CO];
#pragma unroll
                                    for (int j = 0; j < CO; ++j) v[j] = 0u;
                                    // The owner's slot, then every contributor's
                                    // (this CTA's included); live columns only.
#pragma unroll 1
                                    for (uint32_t c = t_first; c <= t_last; ++c) {
                                        const int32_t *part = slot_of(c, c == t_first ? 1 : 0) + c0 * kTileN + r;
                                        int32_t t[CO];
#pragma unroll
                                        for (int j = 0; j < CO; ++j) t[j] = c0 + j < m_live ? ld_cg_s32(part + j * kTileN) : 0;
#pragma unroll
                                        for (int j = 0; j < CO; ++j) v[j] += (uint32_t)t[j];   // modulo 2^32: exact where the sum fits
                                    }
                                    if (p.fp16_out) {
                                        store_outputs_fp16<CO, MODE>(&tmap_y, v, m0 + c0, n - lane, lane, col_scale, col_zero,
                                                                     ctl->tok_scale + c0, ctl->tok_rowsum + c0,
                                                                     out_stage + ((warp - C::kWarpEpi0) * 2 + obuf) * (16 * 32));
                                        obuf ^= 1;
                                    } else {
                                        store_outputs_i32<CO, MODE>(static_cast<int32_t *>(p.out), p.M, p.N, v, m0 + c0, n,
                                                                    col_zero, ctl->tok_rowsum + c0);
                                    }
                                }
                            }
                            // The staged scales are read; the counter is cleared for the next launch.
                            if (named_bar_any(kBarAll, NEPI, false)) break;
                            if (leader) *cnt = 0;
                        }
                    }
                }
                ++seg;
            }
            // The output copies must have finished reading shared memory
            // before the CTA ends (their global writes complete with the grid).
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
        }
    }

    // ------------------------------------------------------------ teardown
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    // The leader's MMAs (which write the peer's tensor memory) have completed
    // and the peer's last arrivals on the leader's barriers are done before
    // either CTA frees tensor memory or exits.
    if (PAIR) cluster_sync_all();
    if (warp == kWarpMma) {
        tc_fence_after();
        if (PAIR)
            tmem_dealloc_pair(tmem_base, C::kTmemCols);
        else
            tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- host side

// Number of two-CTA clusters of the paired kernel that can be resident at
// once (clusters live inside one GPC, so this can be below SMs / 2); the
// persistent schedule launches no more than one such wave. 0 when pairs cannot
// launch.
template <int TOK, int MODE, bool SAT>
static int pair_clusters_of(int dev) {
    using C = GemmCfg<TOK, MODE, true>;
    static std::once_flag once[64];
    static int count[64];
    std::call_once(once[dev], [&] {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = C::kSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaFuncSetAttribute(qoq_gemm_kernel<TOK, MODE, true, SAT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes) != cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, qoq_gemm_kernel<TOK, MODE, true, SAT>, &cfg) != cudaSuccess)
            n = 0;
        (void)cudaGetLastError();
        count[dev] = n;
    });
    return count[dev];
}

template <int TOK, int MODE, bool PAIR, bool SAT = false>
static qoq_status launch_gemm_t(const GemmArgs &a, cudaStream_t stream, int units_max) {
    using C = GemmCfg<TOK, MODE, PAIR>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return QOQ_ERR_CUDA;

    // Opt in to the large dynamic shared memory once per device.
    static std::once_flag attr_once[64];
    static cudaError_t attr_err[64];
    std::call_once(attr_once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(qoq_gemm_kernel<TOK, MODE, PAIR, SAT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (attr_err[dev] != cudaSuccess) return QOQ_ERR_CUDA;

    CUtensorMap tmap, tmap_y;
    if (!encode_x_map(&tmap, a.X8, a.M, a.K, C::kXRows)) return QOQ_ERR_CUDA;
    if (a.fp16_out) {
        if (!encode_y_map(&tmap_y, a.out, a.M, a.N)) return QOQ_ERR_CUDA;
    } else {
        memset(&tmap_y, 0, sizeof(tmap_y));   // INT32 outputs use plain stores
    }

    const BlobLayout L = blob_layout(a.N, a.K, a.group);
    GemmParams p;
    p.blob = static_cast<const uint8_t *>(a.blob);
    p.s_x = static_cast<const __half *>(a.s_x);
    p.rowsum = a.rowsum;
    p.out = a.out;
    uint8_t *ws = static_cast<uint8_t *>(a.ws);
    p.status = reinterpret_cast<int32_t *>(ws);
    p.flags = reinterpret_cast<int32_t *>(ws + 256);
    p.late_arrival_ns = 1000ll * forced_config().lateck;
    p.partials = reinterpret_cast<int32_t *>(ws + 256 + sizeof(int32_t) * kMaxGrid);
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.group = a.group;
    p.NT = (int)(a.N / kTileN);
    p.NTw = PAIR ? p.NT / 2 : p.NT;
    p.KT = (int)(a.K / kTileK);
    p.MT = (int)((a.M + TOK - 1) / TOK);
    p.GM = p.MT < kTileGroup ? p.MT : kTileGroup;
    const long long blocks = (long long)p.MT * p.NTw * p.KT;
    if (blocks >= (1ll << 31)) return QOQ_ERR_UNSUPPORTED;
    p.total_blocks = (uint32_t)blocks;
    // Schedule units (CTAs, or CTA pairs): at most one per SM (pair), all resident.
    p.grid = (int)std::min<long long>(units_max, blocks);
    // The partial-sum slots are indexed by CTA: the workspace must hold one
    // per CTA of this grid.
    if (scratch_bytes_for_grid(TOK, PAIR ? 2 * p.grid : p.grid, 2) > a.ws_capacity) return QOQ_ERR_WORKSPACE;
    // Whole tiles in data-parallel waves while at least one to two waves of
    // tiles remain for the stream-K tail, which evens out the last wave.
    const long long tiles = (long long)p.MT * p.NTw;
    const long long dp_tiles = tiles >= 2ll * p.grid ? (tiles / p.grid - 1) * p.grid : 0;
    p.dp_tiles = (uint32_t)dp_tiles;
    p.sk_base = (uint32_t)(dp_tiles * p.KT);
    p.off_codes = L.off_codes;
    p.off_scale = L.off_scale;
    p.off_zero = L.off_zero;
    p.fp16_out = a.fp16_out ? 1 : 0;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(PAIR ? 2 * p.grid : p.grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int na = 0;
    if (kProgrammaticLaunch) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    if (PAIR) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = 2;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, qoq_gemm_kernel<TOK, MODE, PAIR, SAT>, p, tmap, tmap_y) == cudaSuccess
               ? QOQ_OK
               : QOQ_ERR_CUDA;
}

// Launch plan of a problem: token tile, CTA pairs or not, and the number of
// schedule units (CTAs, or CTA pairs) the persistent grid may use.
struct GemmPlan {
    int tok;
    bool pair;
    bool decode;    // runs on the decode kernel (token tiles up to 64, not saturating)
    int units_max;
};

static bool plan_gemm(int64_t M, int64_t N, int64_t K, int mode, bool saturating, GemmPlan *pl) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return false;
    const int sms = sm_count_of(dev);
    if (sms <= 0) return false;
    pl->tok = token_tile_for(M, N, K);
    pl->pair = false;
    pl->decode = pl->tok <= kDecodeMaxTok && !saturating;
    pl->units_max = std::min(sms, kMaxGrid);
    if (pl->tok == 256 && (N / kTileN) % 2 == 0) {
        // 256-token tiles run on CTA pairs when the n-tiles pair up.
        int clusters = 0;
        if (saturating)
            clusters = pair_clusters_of<256, 0, true>(dev);
        else
            clusters = mode == 0 ? pair_clusters_of<256, 0, false>(dev) : pair_clusters_of<256, 1, false>(dev);
        const int pairs = std::min(clusters, kMaxGrid / 2);
        if (pairs > 0) {
            pl->pair = true;
            pl->units_max = pairs;
        }
    }
    return true;
}

size_t gemm_scratch_bytes(int64_t M, int64_t N, int64_t K, int group, bool saturating) {
    GemmPlan pl;
    if (!plan_gemm(M, N, K, group ? 0 : 1, saturating, &pl)) return 0;
    const int64_t NTw = pl.pair ? N / kTileN / 2 : N / kTileN;
    const int64_t blocks = ((M + pl.tok - 1) / pl.tok) * NTw * (K / kTileK);
    const int64_t units = std::min<int64_t>(pl.units_max, blocks);
    return scratch_bytes_for_grid(pl.tok, pl.pair ? 2 * units : units, pl.decode ? 1 : 2);
}

template <int MODE>
static qoq_status launch_gemm_mode(const GemmArgs &a, cudaStream_t stream) {
    GemmPlan pl;
    if (!plan_gemm(a.M, a.N, a.K, MODE, false, &pl)) return QOQ_ERR_CUDA;
    if (pl.decode) return launch_decode_gemm(a, stream, pl.tok, pl.units_max);
    if (pl.tok == 128) return launch_gemm_t<128, MODE, false>(a, stream, pl.units_max);
    return pl.pair ? launch_gemm_t<256, MODE, true>(a, stream, pl.units_max)
                   : launch_gemm_t<256, MODE, false>(a, stream, pl.units_max);
}

// The saturating-decode ablation is built for two token tiles: 16 (decode)
// and 256 on CTA pairs (prefill).
static qoq_status launch_gemm_saturating(const GemmArgs &a, cudaStream_t stream) {
    GemmPlan pl;
    if (!plan_gemm(a.M, a.N, a.K, 0, true, &pl)) return QOQ_ERR_CUDA;
    if (pl.tok == 16) return launch_gemm_t<16, 0, false, true>(a, stream, pl.units_max);
    if (pl.tok == 256 && pl.pair) return launch_gemm_t<256, 0, true, true>(a, stream, pl.units_max);
    return QOQ_ERR_UNSUPPORTED;
}

qoq_status launch_gemm(const GemmArgs &a, cudaStream_t stream) {
    if (a.saturating) return a.group ? launch_gemm_saturating(a, stream) : QOQ_ERR_UNSUPPORTED;
    return a.group ? launch_gemm_mode<0>(a, stream) : launch_gemm_mode<1>(a, stream);
}

}  // namespace qoq
