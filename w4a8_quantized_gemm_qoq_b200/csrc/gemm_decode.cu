// QoQ W4A8 GEMM for the decode regime (token tiles of 16, 32 or 64 tokens)
// on sm_100a, optionally with the per-token activation quantisation fused in
// front of it in the same launch.
//
// QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM Serving
// (arXiv 2405.04532), paperlayer.ai summary:
//   section 3 -- at small batch the GEMM is memory-bound: the time is the
//     weight stream, so the main loop must keep HBM busy;
//   section 4 -- weights rebuilt to INT8 in the main loop from 4-bit codes
//     (q*s - z*s, no saturation thanks to the protective range);
//   section 5 -- per-token activation quantisation fused into the producer of
//     the GEMM input; per-channel scales (and the per-channel variant's zero
//     point) applied in the epilogue; FP16 output.
//
// The arithmetic is that of the general kernel (gemm.cu): swap-AB with the
// dequantised weights as the tcgen05.mma A operand in tensor memory and the
// token tile (MMA N = 16..64) staged by TMA in shared memory; exact INT32
// sums; the same FP32 epilogue. What differs is the shape of the launch,
// built for decode, where each launch streams 8-60 MB of weights in a few
// microseconds and per-launch fixed costs weigh as much as the stream:
//   * two rings: packed weights (filled by one producer warp, released by the
//     dequantisers as soon as they have read them) and A/X stages (a TMEM A
//     buffer plus the token tile, released by the MMA). Weights never depend
//     on the previous kernel, so the weight ring and the dequantisation run
//     before griddepcontrol.wait; only the token tiles (and the epilogue)
//     wait for the previous kernel. The token tile's TMA completes on the
//     same barrier the dequantisers arrive on, so the MMA issuer waits once
//     per unit;
//   * the two dequant warpgroups take alternate two-k-tile units (warpgroup g
//     the units of parity g, as do the two MMA issuers when they alternate);
//     ring sizes are even, so each waits on every phase of its own stages
//     only. A TMEM store and its completion wait cost hundreds of cycles, so
//     the first k-tile's store stays in flight while the second is decoded;
//   * one CTA per SM by default (deepest rings); a two-CTA-per-SM
//     configuration (half the shared memory, 256 TMEM columns, per-warpgroup
//     register budgets) lets consecutive launches overlap and is selectable
//     for sweeps (QOQ_FORCE_CONFIG=cps=2);
//   * stream-K fix-up by the last arriver: the CTAs sharing a tile count
//     their arrivals on a per-tile counter and add their INT32 partial sums
//     into the tile's sum buffer (red.add) before arriving; the owner (the CTA
//     with the tile's first k-tile, which reaches it last) arrives when it
//     starts the tile's epilogue, and whoever arrives last reads the buffer
//     once, writes the output and leaves buffer and counter zero for the next
//     launch. No CTA waits for one that may not have started, so the launch
//     needs no co-residency (a last contributor that finds the owner already
//     arrived waits only for that running owner's sums). A contributor reads
//     its arrival's result only at the end of its schedule;
//   * optional fused activation quantisation (qoq_w4a8_linear with
//     QOQ_FORCE_CONFIG=fuse=1): the epilogue warps, idle until the first
//     accumulator is ready, claim token rows one at a time from a grid-wide
//     counter and quantise them (the arithmetic of
//     qoq_quantize_act_per_token) into the workspace; the token tiles are
//     loaded once every row is done. Rows are claimed, not assigned, so the
//     first CTAs to start do all of them.
#include <algorithm>
#include <cstring>

#include "gemm_common.cuh"
#include "quant_math.cuh"

namespace qoq {

namespace dec {
constexpr int kThreads = 512;     // 16 warps
constexpr int kWarpProdW = 0;     // weight producer (lane 0)
constexpr int kWarpIss = 1;       // warps 1, 2: MMA issuers (lane 0)
constexpr int kWarpProdX = 3;     // token-tile producer (lane 0)
constexpr int kWarpDq = 4;        // warps 4..11: two dequant warpgroups
constexpr int kWarpEpi = 12;      // warps 12..15: epilogue warpgroup
constexpr int kBarEpi = 1;        // named barrier of the epilogue warpgroup
constexpr int kSmemPerSm = 233472;          // 228 KB of shared memory per SM
constexpr int kSmemReservedPerCta = 1024;   // the system's share of every CTA
// Two CTAs per SM: 64 registers per thread at launch (two 512-thread CTAs fill
// the SM's 65536); the control warpgroup (producers, issuers) gives 24 of its
// own so that the three compute warpgroups get 8 more each:
// 128 x 40 + 384 x 72 = 512 x 64.
constexpr int kRegsCtl = 40;
constexpr int kRegsWork = 72;
static_assert(128 * kRegsCtl + 384 * kRegsWork <= kThreads * 64, "register split exceeds the launch pool");
}  // namespace dec

constexpr int kSmemPerSmAvail = dec::kSmemPerSm;

// CPS: CTAs per SM the configuration is built for. Two: half an SM each,
// so the next launch's CTAs sit beside this one's and prefetch and
// dequantise while it runs. One: the whole SM, for the deepest weight ring
// (the main loop's HBM rate is the bytes in flight per SM over the loaded
// memory latency).
template <int TOK, int MODE, int CPS>
struct DecCfg {
    static_assert(TOK == 16 || TOK == 32 || TOK == 64, "decode token tiles");
    static_assert(CPS == 1 || CPS == 2, "one or two CTAs per SM");
    static constexpr int kKB = 2;                              // k-tiles per pipeline unit
    static constexpr int kWTile = MODE == 0 ? 8448 : 8192;     // codes (+ s, z*s) per k-tile
    static constexpr int kWStage = kKB * kWTile;
    static constexpr int kXTile = TOK * 128;                   // token tile of one k-tile
    static constexpr int kXStage = kKB * kXTile;
    // Up to 32 tokens the two issuers take alternate units, each into its own
    // accumulator; at 64 they split the token columns of every unit.
    static constexpr bool kAlt = TOK <= 32;
    static constexpr int kAccCols = kAlt ? 2 * TOK : TOK;
    static constexpr int kAccBufs = 2;
    static constexpr int kACol0 = kAccBufs * kAccCols;
    static constexpr int kTmemCols = CPS == 1 ? 512 : 256;
    // A/X stages: as many two-k-tile TMEM A buffers as fit, an even number.
    // The two dequant warpgroups take alternate units (warpgroup g the units
    // of parity g), and so do the issuers when they alternate; with an even
    // stage count unit parity fixes stage parity, so each of them waits on
    // every phase of its own stages and on no others (a parity wait cannot
    // tell a phase from the one two later).
    static constexpr int kSA = ((kTmemCols - kACol0) / (kKB * 32)) & ~1;
    static_assert(kSA >= 2, "A/X ring too shallow");
    static_assert(kACol0 + kSA * kKB * 32 <= kTmemCols, "TMEM over-subscribed");
    static constexpr int kXBytes = kSA * kXStage;              // first: 1024-aligned swizzle atoms
    static constexpr int kCtlBytes = 2048;
    static constexpr int kEpiBytes = 4 * 2 * 1024;             // per epilogue warp two 16 x 32 FP16 blocks
    static constexpr int kSmemBudget = kSmemPerSmAvail / CPS - dec::kSmemReservedPerCta;
    // Weight stages: what is left, at most 16, an even number (as above).
    static constexpr int kSWfit = (kSmemBudget - 1024 - kXBytes - kCtlBytes - kEpiBytes) / kWStage;
    static constexpr int kSW = (kSWfit > 16 ? 16 : kSWfit) & ~1;
    static_assert(kSW >= 2, "weight ring too shallow");
    static constexpr int kWBytes = kSW * kWStage;
    static constexpr int kSmemBytes = 1024 + kXBytes + kWBytes + kCtlBytes + kEpiBytes;
    static_assert(kXStage % 1024 == 0 && kXTile % 1024 == 0, "token tiles must keep the swizzle atom aligned");
    static_assert(kWStage % 16 == 0, "bulk copies move multiples of 16 bytes");
    static_assert(kSmemBytes <= 232448, "227 KB per CTA");
    static_assert(CPS * (kSmemBytes + dec::kSmemReservedPerCta) <= dec::kSmemPerSm, "CPS CTAs per SM must fit");
};

struct DecParams {
    const uint8_t *blob;
    const __half *s_x;      // token scales: the caller's, or the fused quantiser's (workspace)
    const int32_t *rowsum;  // per-token code sums (per-channel variant)
    void *out;              // int32 or fp16 [M][N]
    int32_t *status;        // workspace word 0
    int32_t *qctl;          // fused quantisation: [0] next row to claim, [1] rows done, [2] CTAs finished
    int32_t *counters;      // [kMaxGrid]: arrival counter of the split tile owned by CTA c
    int32_t *partials;      // [grid][TOK][128]: INT32 sums of the split tile owned by CTA c (zero between launches)
    const __half *X;        // fused: FP16 activations [M][K]
    int8_t *X8q;            // fused: INT8 codes [M][K] (workspace)
    __half *s_xq;           // fused: FP16 scales [M] (workspace)
    int32_t *rowsumq;       // fused: code sums [M] (workspace)
    int M, N, K, group;
    int NT, KT, MT, GM, grid;
    uint32_t total_blocks, dp_tiles, sk_base;
    long long off_codes, off_scale, off_zero;
    int fp16_out;
    long long late_arrival_ns;   // test override: contributors' arrivals delayed by this long (0)
};

struct DecCtl {
    uint64_t w_full[16], w_empty[16];
    uint64_t a_full[8], ax_empty[8];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t final_bar[2];
    uint32_t tmem_base;
    int abort_flag;
    int claim;              // fused quantisation: the row the epilogue leader claimed
    int fix_old;            // epilogue leader's arrival-counter value, broadcast
    float red_f[4];
    int red_i[4];
    alignas(16) float tok_scale[64];
    int32_t tok_rowsum[64];
};
static_assert(sizeof(DecCtl) <= 2048, "control block outgrows its reserve");

// Quantise one 16-byte chunk (eight FP16 values) of a token row: eight codes
// packed little-endian into two words; returns their sum. The arithmetic of
// qoq_quantize_act_per_token (quant_code_recip).
__device__ __forceinline__ int quant8_chunk(const uint4 &u, float s, float inv, uint2 &packed) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t p0 = 0u, p1 = 0u;
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __half2float(__ushort_as_half((unsigned short)(w[i] & 0xFFFFu)));
        const float hi = __half2float(__ushort_as_half((unsigned short)(w[i] >> 16)));
        const int q0 = quant_code_recip(lo, s, inv, 127), q1 = quant_code_recip(hi, s, inv, 127);
        sum += q0 + q1;
        const uint32_t pair = ((uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8)) << (16 * (i & 1));
        if (i < 2)
            p0 |= pair;
        else
            p1 |= pair;
    }
    packed = make_uint2(p0, p1);
    return sum;
}

__device__ __forceinline__ float absmax8(const uint4 &u, float amax) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float lo = __half2float(__ushort_as_half((unsigned short)(w[i] & 0xFFFFu)));
        const float hi = __half2float(__ushort_as_half((unsigned short)(w[i] >> 16)));
        amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
    }
    return amax;
}

// Fused per-token quantisation by the 128 epilogue threads of one CTA: claim
// rows from the grid-wide counter until none is left, quantise each, publish
// how many this CTA did, then wait until every row of the launch is done.
// Returns false if a wait ran out or the CTA aborted.
__device__ __forceinline__ bool fused_act_quant(const DecParams &p, DecCtl *ctl, int te, const Watchdog &wd) {
    const int K = p.K;
    const int lane = te & 31, w = te >> 5;
    const bool leader = te == 0;
    int mine = 0;
    for (;;) {
        if (leader) ctl->claim = atomicAdd(p.qctl, 1);
        named_bar_sync(dec::kBarEpi, 128);
        const int m = ctl->claim;
        if (m >= p.M) break;
        const __half *row = p.X + (size_t)m * K;
        float amax = 0.0f;
        for (int k = te * 8; k < K; k += 1024) amax = absmax8(*reinterpret_cast<const uint4 *>(row + k), amax);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) ctl->red_f[w] = amax;
        named_bar_sync(dec::kBarEpi, 128);
        const float a = fmaxf(fmaxf(ctl->red_f[0], ctl->red_f[1]), fmaxf(ctl->red_f[2], ctl->red_f[3]));
        const __half sh = __float2half_rn(__fdiv_rn(a, 127.0f));
        const float s = __half2float(sh), inv = __frcp_rn(s);
        int sum = 0;
        int8_t *out = p.X8q + (size_t)m * K;
        for (int k = te * 8; k < K; k += 1024) {
            uint2 pk;
            sum += quant8_chunk(*reinterpret_cast<const uint4 *>(row + k), s, inv, pk);
            *reinterpret_cast<uint2 *>(out + k) = pk;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) ctl->red_i[w] = sum;
        named_bar_sync(dec::kBarEpi, 128);
        if (leader) {
            p.s_xq[m] = sh;
            p.rowsumq[m] = ctl->red_i[0] + ctl->red_i[1] + ctl->red_i[2] + ctl->red_i[3];
        }
        ++mine;
    }
    // Every thread orders its code stores before the async-proxy (TMA) reads
    // of other CTAs; the barrier gathers them before the leader's release.
    fence_proxy_async_global();
    named_bar_sync(dec::kBarEpi, 128);
    bool ok = true;
    if (leader) {
        if (mine) red_add_release_gpu(p.qctl + 1, mine);
        ok = wait_word_bounded(p.qctl + 1, -1, p.M, wd, kSiteRowsDone, mine);
    }
    return !named_bar_any(dec::kBarEpi, 128, !ok);
}

template <int TOK, int MODE, bool FUSED, int CPS>
__global__ void __launch_bounds__(dec::kThreads, CPS)
    qoq_decode_kernel(const __grid_constant__ DecParams p, const __grid_constant__ CUtensorMap tmap_x,
                      const __grid_constant__ CUtensorMap tmap_y) {
    using C = DecCfg<TOK, MODE, CPS>;
    constexpr int SW = C::kSW, SA = C::kSA, KB = C::kKB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *xst = smem;                                   // SA token-tile stages
    uint8_t *wst = smem + C::kXBytes;                      // SW packed-weight stages
    DecCtl *ctl = reinterpret_cast<DecCtl *>(smem + C::kXBytes + C::kWBytes);
    __half *out_stage = reinterpret_cast<__half *>(smem + C::kXBytes + C::kWBytes + C::kCtlBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Watchdog wd{&ctl->abort_flag, p.status};

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        ctl->abort_flag = 0;
        for (int s = 0; s < SW; ++s) {
            mbar_init(&ctl->w_full[s], 1);
            mbar_init(&ctl->w_empty[s], 4);              // the four warps of the unit's dequant warpgroup
        }
        for (int s = 0; s < SA; ++s) {
            mbar_init(&ctl->a_full[s], 5);               // the dequant warpgroup's 4 warps + the token producer
            mbar_init(&ctl->ax_empty[s], C::kAlt ? 1 : 2);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->acc_full[b], 2);             // both issuers commit every segment
            mbar_init(&ctl->acc_empty[b], 4);            // the four epilogue warps
            mbar_init(&ctl->final_bar[b], 1);
        }
        mbar_fence_init();
        // No kernel that releases its dependents early writes a blob, so the
        // header may be read before griddepcontrol.wait (at L2, as the copies).
        const int32_t *h = reinterpret_cast<const int32_t *>(p.blob);
        const int32_t h0 = ld_cg_s32(h), h1 = ld_cg_s32(h + 1), h2 = ld_cg_s32(h + 2), h3 = ld_cg_s32(h + 3),
                      h4 = ld_cg_s32(h + 4);
        if ((uint32_t)h0 != kMagic || (uint32_t)h1 != kVersion || h2 != p.N || h3 != p.K || h4 != p.group)
            ctl->abort_flag = 1;   // reported on the status word after griddepcontrol.wait
    }
    if (warp == dec::kWarpProdX && lane == 0) prefetch_tensormap(&tmap_x);
    if (warp == dec::kWarpEpi && lane == 0 && p.fp16_out) prefetch_tensormap(&tmap_y);
    if (warp == dec::kWarpIss) {
        tmem_alloc(&ctl->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    griddep_launch_dependents();   // the next kernel may start its own set-up and weight copies
    const bool bad_blob = wd.aborted();
    if (bad_blob && threadIdx.x == 0) {
        griddep_wait();
        atomicCAS(p.status, 0, QOQ_ERR_BAD_BLOB);
    }

    // This CTA's schedule (the same as the general kernel's): whole tiles
    // me + w * grid below p.dp_tiles, then its stream-K share [b0, b1) of the
    // tail blocks.
    const uint32_t me = blockIdx.x;
    const uint32_t G = (uint32_t)p.grid;
    const int waves = p.dp_tiles > me ? (int)((p.dp_tiles - me + G - 1) / G) : 0;
    const uint32_t BS = p.total_blocks - p.sk_base;
    const uint32_t b0 = p.sk_base + cta_begin(me, BS, G);
    const uint32_t b1 = p.sk_base + cta_begin(me + 1, BS, G);
    const int KT = p.KT;

    if (!bad_blob) {
        // Each warpgroup sets its register budget at the top of its own
        // branch, so the compiler allocates each role's code with that budget.
        if (warp < 4) {
        if (CPS == 2) regs_dec<dec::kRegsCtl>();
        if (warp == dec::kWarpProdW) {
            // -------------------------------------------- weight producer
            // Runs ahead of everything else, including the previous kernel:
            // the blob is never written by a kernel that releases early.
            if (lane == 0) {
                const uint64_t pol_w = policy_evict_first();   // streamed once
                UnitCursor<KB> cur;
                cur.init(me, G, waves, b0, b1, KT, p.NT, p.MT, p.GM);
                int u = 0;
                for (; !cur.done(); ++u, cur.advance()) {
                    const int s = u % SW;
                    if (u >= SW && !wait_bounded(&ctl->w_empty[s], (uint32_t)((u / SW) - 1) & 1u, wd,
                                                 kSiteProducerFreed, u))
                        break;
                    const uint32_t bytes = (uint32_t)(cur.nk * C::kWTile);
                    mbar_arrive_expect_tx(&ctl->w_full[s], bytes);
                    const uint8_t *src = p.blob + p.off_codes + ((long long)cur.nt * KT + cur.kt) * C::kWTile;
                    bulk_load(wst + s * C::kWStage, src, bytes, &ctl->w_full[s], pol_w);
                }
                // Every issued copy lands before the CTA can exit.
                for (int i = u > SW ? u - SW : 0; i < u; ++i)
                    wait_drain(&ctl->w_full[i % SW], (uint32_t)(i / SW) & 1u, kDrainNs);
            }
            __syncwarp();
        } else if (warp == dec::kWarpProdX) {
            // ---------------------------------------- token-tile producer
            if (lane == 0) {
                griddep_wait();   // X8 (or X) belongs to the previous kernel until now
                bool ok = true;
                if (FUSED) {
                    ok = wait_word_bounded(p.qctl + 1, -1, p.M, wd, kSiteRowsDone, -1);
                    fence_proxy_async_global();   // the codes were written through the generic proxy
                }
                const uint64_t pol_x = policy_evict_last();   // reused by every n-tile
                UnitCursor<KB> cur;
                cur.init(me, G, waves, b0, b1, KT, p.NT, p.MT, p.GM);
                int u = 0;
                for (; ok && !cur.done(); ++u, cur.advance()) {
                    const int s = u % SA;
                    if (u >= SA && !wait_bounded(&ctl->ax_empty[s], (uint32_t)((u / SA) - 1) & 1u, wd, kSiteXEmpty, u))
                        break;
                    mbar_arrive_expect_tx(&ctl->a_full[s], (uint32_t)(cur.nk * C::kXTile));
                    for (int j = 0; j < cur.nk; ++j)
                        tma_load_2d(xst + s * C::kXStage + j * C::kXTile, &tmap_x, &ctl->a_full[s],
                                    (cur.kt + j) * kTileK, cur.mt * TOK, pol_x);
                }
                // The token tiles issued last land before the CTA can exit:
                // a unit's a_full phase completes only with them.
                for (int i = u > SA ? u - SA : 0; i < u; ++i)
                    wait_drain(&ctl->a_full[i % SA], (uint32_t)(i / SA) & 1u, kDrainNs);
            }
            __syncwarp();
        } else if (warp == dec::kWarpIss || warp == dec::kWarpIss + 1) {
            // ------------------------------------------------ MMA issuers
            // A thread's mbarrier waits stall its own queued tensor-core work,
            // so two issuers take turns: up to 32 tokens issuer k takes the
            // units of parity k into its own accumulator; at 64 both take
            // every unit, each half of the token columns.
            const int k = warp - dec::kWarpIss;
            if (lane == 0) {
                constexpr uint32_t idesc = idesc_i8(128, C::kAlt ? TOK : TOK / 2, true, true);
                UnitCursor<KB> cur;
                cur.init(me, G, waves, b0, b1, KT, p.NT, p.MT, p.GM);
                int seg = 0, u = 0;
                bool ok = true;
                while (ok && !cur.done()) {
                    const int buf = seg % C::kAccBufs;
                    const uint32_t aph = (uint32_t)(seg / C::kAccBufs) & 1u;
                    ok = wait_bounded(&ctl->acc_empty[buf], aph ^ 1u, wd, kSiteMmaAccEmpty, seg);
                    if (!ok) break;
                    const uint32_t d_tmem =
                        tmem_base + (uint32_t)(buf * C::kAccCols + k * (C::kAlt ? TOK : TOK / 2));
                    uint32_t acc = 0u;   // this issuer's first MMA of the segment overwrites its accumulator
                    bool seg_done = false;
                    while (!seg_done) {
                        if (!C::kAlt || (u & 1) == k) {
                            const int s = u % SA;
                            // The dequantisers' arrivals and the token tile's
                            // bytes both complete a_full[s].
                            ok = wait_bounded(&ctl->a_full[s], (uint32_t)(u / SA) & 1u, wd, kSiteMmaOperands, u);
                            if (!ok) break;
                            tc_fence_after();
                            const uint32_t a_tmem = tmem_base + (uint32_t)(C::kACol0 + s * KB * 32);
                            const uint64_t bdesc = smem_desc_k_sw128(smem_u32(xst + s * C::kXStage)) +
                                                   (uint64_t)(C::kAlt ? 0 : k * (TOK / 2) * 128 / 16);
                            mma4_i8_ts(d_tmem, a_tmem, bdesc, idesc, acc);
                            if (cur.nk == 2)
                                mma4_i8_ts(d_tmem, a_tmem + 32u, bdesc + (uint64_t)(C::kXTile >> 4), idesc, 1u);
                            acc = 1u;
                            tc_commit(&ctl->ax_empty[s]);
                        }
                        ++u;
                        seg_done = cur.advance();
                    }
                    if (!ok) break;
                    tc_commit(&ctl->acc_full[buf]);
                    ++seg;
                }
                // Every MMA completes before tensor memory is freed.
                tc_commit(&ctl->final_bar[k]);
                wait_drain(&ctl->final_bar[k], 0, kDrainNs);
            }
            __syncwarp();
        }
        } else if (warp >= dec::kWarpDq && warp < dec::kWarpEpi) {
            if (CPS == 2) regs_inc<dec::kRegsWork>();
            // ------------------------------------------------ dequant
            // Warpgroup g decodes the units of parity g, both k-tiles of each;
            // thread (quarter, lane) owns weight row r, i.e. one whole
            // quantisation group per k-tile, so (s, z*s) is a scalar. Per
            // 32-bit word of eight codes: and, shift+and, two multiply-adds
            // (q*s <= 240 and q*s + 128 - z*s in [7, 249] never carry between
            // bytes) and two xors (excess-128 to int8). A TMEM store and its
            // completion wait cost hundreds of cycles, so with registers to
            // spare (one CTA per SM) the first k-tile's store is left in
            // flight while the second is decoded. Nothing here depends on the
            // previous kernel.
            const int g = (warp - dec::kWarpDq) >> 2;
            const int quarter = warp & 3;
            const int r = quarter * 32 + lane;
            const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
            auto decode = [&](const uint4 (&v)[4], uint32_t sz, uint32_t (&o)[32]) {
                const uint32_t sc = sz & 0xFFu;
                const uint32_t c4 = (uint32_t)(128 - (int)(int8_t)(sz >> 8)) * 0x01010101u;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t wd4[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t lo = wd4[q] & 0x0F0F0F0Fu;
                        const uint32_t hi = (wd4[q] >> 4) & 0x0F0F0F0Fu;
                        if (MODE == 0) {
                            o[8 * c + 2 * q] = (lo * sc + c4) ^ 0x80808080u;
                            o[8 * c + 2 * q + 1] = (hi * sc + c4) ^ 0x80808080u;
                        } else {
                            o[8 * c + 2 * q] = lo;
                            o[8 * c + 2 * q + 1] = hi;
                        }
                    }
                }
            };
            UnitCursor<KB> cur;
            cur.init(me, G, waves, b0, b1, KT, p.NT, p.MT, p.GM);
            for (int u = 0; !cur.done(); ++u, cur.advance()) {
                if ((u & 1) != g) continue;
                const int sw = u % SW, sa = u % SA;
                bool ok = __all_sync(0xffffffffu,
                                     wait_bounded(&ctl->w_full[sw], (uint32_t)(u / SW) & 1u, wd, kSiteDequantFull, u));
                if (!ok) break;
                const int nk = cur.nk;
                uint4 v0[4], v1[4];
                uint32_t sz0 = 0u, sz1 = 0u;
                {
                    const uint32_t wbase = smem_u32(wst + sw * C::kWStage);
                    if (MODE == 0) sz0 = lds16(wbase + 8192 + 2 * r);
#pragma unroll
                    for (int c = 0; c < 4; ++c) v0[c] = lds128(wbase + c * 2048 + r * 16);
                    if (nk == 2) {
                        if (MODE == 0) sz1 = lds16(wbase + C::kWTile + 8192 + 2 * r);
#pragma unroll
                        for (int c = 0; c < 4; ++c) v1[c] = lds128(wbase + C::kWTile + c * 2048 + r * 16);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->w_empty[sw]);   // the packed weights are in registers
                // TMEM A buffer sa is free once the MMAs of unit u - SA completed.
                if (u >= SA) {
                    ok = __all_sync(0xffffffffu, wait_bounded(&ctl->ax_empty[sa], (uint32_t)((u / SA) - 1) & 1u, wd,
                                                              kSiteXEmpty, u));
                    if (!ok) break;
                }
                tc_fence_after();
                const uint32_t a_col = tmem_base + lane_addr + (uint32_t)(C::kACol0 + sa * KB * 32);
                if (CPS == 1) {
                    uint32_t o0[32], o1[32];
                    decode(v0, sz0, o0);
                    tmem_st32(a_col, o0);
                    if (nk == 2) {
                        decode(v1, sz1, o1);
                        tmem_st32(a_col + 32u, o1);
                    }
                    tmem_st_wait();
                } else {
                    uint32_t o[32];
                    decode(v0, sz0, o);
                    tmem_st32_wait(a_col, o);
                    if (nk == 2) {
                        decode(v1, sz1, o);
                        tmem_st32_wait(a_col + 32u, o);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->a_full[sa]);
                __syncwarp();
            }
        } else {
            // ------------------------------------------------ epilogue
            if (CPS == 2) regs_inc<dec::kRegsWork>();
            const int quarter = warp & 3;
            const int r = quarter * 32 + lane;
            const int te = threadIdx.x - dec::kWarpEpi * 32;
            const bool leader = te == 0;
            const bool announcer = te == 96;   // warp 15, lane 0: the owner's early arrival
            const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
            griddep_wait();   // X, scales, row sums, outputs and workspace belong to the previous kernel until now
            bool ok = true;
            if (FUSED) ok = fused_act_quant(p, ctl, te, wd);
            UnitCursor<KB> cur;
            cur.init(me, G, waves, b0, b1, KT, p.NT, p.MT, p.GM);
            int seg = 0, ubase = 0, obuf = 0;
            __half *stage_base = out_stage + (warp - dec::kWarpEpi) * 2 * (16 * 32);
            constexpr int CO = 16;   // token columns per step
            // Per-tile epilogue inputs: the weight row's scale (and zero
            // point) in registers, the tile's token scales (and row sums)
            // staged in shared memory.
            float col_scale = 0.0f;
            int col_zero = 0;
            auto stage_tile = [&](int mt, int nt) {
                const int n = nt * kTileN + r;
                col_scale = p.fp16_out ? __half2float(reinterpret_cast<const __half *>(p.blob + p.off_scale)[n]) : 0.0f;
                col_zero = MODE == 1 ? __half2int_rn(reinterpret_cast<const __half *>(p.blob + p.off_zero)[n]) : 0;
                const int64_t m0 = (int64_t)mt * TOK;
                for (int j = te; j < TOK; j += 128) {
                    const int64_t m = m0 + j < p.M ? m0 + j : p.M - 1;
                    // At L2: with the fused quantisation other CTAs wrote them in this launch.
                    ctl->tok_scale[j] = p.fp16_out ? __half2float(__ldcg(p.s_x + m)) : 0.0f;
                    if (MODE == 1) ctl->tok_rowsum[j] = __ldcg(p.rowsum + m);
                }
            };
            auto emit = [&](const uint32_t (&v)[CO], int mt, int nt, int c0) {
                const int64_t m0 = (int64_t)mt * TOK;
                const int n = nt * kTileN + r;
                if (p.fp16_out) {
                    store_outputs_fp16<CO, MODE>(&tmap_y, v, m0 + c0, n - lane, lane, col_scale, col_zero,
                                                 ctl->tok_scale + c0, ctl->tok_rowsum + c0, stage_base + obuf * 512);
                    obuf ^= 1;
                } else {
                    store_outputs_i32<CO, MODE>(static_cast<int32_t *>(p.out), p.M, p.N, v, m0 + c0, n, col_zero,
                                                ctl->tok_rowsum + c0);
                }
            };
            // The finisher's read of a split tile's sum buffer (zero at launch
            // start; every other participant added its partial sums into it
            // before arriving): live columns only, all loads in flight at
            // once; the buffer is cleared behind it for the next launch.
            auto take_sum = [&](uint32_t (&v)[CO], int32_t *tsum, int c0, int m_live) {
                int32_t t[CO];
#pragma unroll
                for (int j = 0; j < CO; ++j) t[j] = (c0 + j < m_live) ? ld_cg_s32(tsum + (c0 + j) * kTileN) : 0;
#pragma unroll
                for (int j = 0; j < CO; ++j) {
                    v[j] += (uint32_t)t[j];   // modulo 2^32: exact where the sum fits
                    if (c0 + j < m_live) tsum[(c0 + j) * kTileN] = 0;
                }
            };
            // A contributor's arrival, checked at the end: this CTA contributes
            // to at most one split tile (its first segment).
            bool pend = false;
            int pend_old = 0, pend_first = 0, pend_nparts = 0, pend_mt = 0, pend_nt = 0;
            while (ok && !cur.done()) {
                const uint32_t seg_b = cur.b, seg_e = cur.seg_end;
                const int kt_lo = cur.kt, kt_hi = cur.kt + (int)(seg_e - seg_b);
                const int mt = cur.mt, nt = cur.nt;
                const uint32_t tile_b = seg_b - (uint32_t)kt_lo;
                int nunits = 1;
                while (!cur.advance()) ++nunits;
                const int prim = C::kAlt ? (ubase & 1) : 0;   // the issuer of the segment's first unit
                const bool two = C::kAlt && nunits >= 2;
                ubase += nunits;
                const int buf = seg % C::kAccBufs;
                const uint32_t aph = (uint32_t)(seg / C::kAccBufs) & 1u;
                const int64_t m0 = (int64_t)mt * TOK;
                const int m_live = (int)(p.M - m0 < TOK ? p.M - m0 : TOK);
                const int live_end = (m_live + CO - 1) / CO * CO;
                // Roles in the tile: sole computer, owner (first k-tile, not
                // the last), or contributor.
                const bool sole = kt_lo == 0 && kt_hi == KT;
                const bool owner = kt_lo == 0 && !sole;
                uint32_t first = me, last = me;
                int32_t *cnt = nullptr;
                if (!sole) {
                    first = cta_of(tile_b - p.sk_base, BS, G);
                    last = cta_of(tile_b + (uint32_t)KT - 1 - p.sk_base, BS, G);
                    cnt = p.counters + first;
                }
                const int nparts = (int)(last - first + 1);
                int32_t *tsum = p.partials + (long long)first * TOK * kTileN + r;
                stage_tile(mt, nt);
                // The owner announces itself as soon as it starts the tile: if
                // every contributor is already in, it finishes the tile.
                if (owner && announcer) ctl->fix_old = atom_add_acq_rel_gpu(cnt, 1);
                named_bar_sync(dec::kBarEpi, 128);
                const bool finisher_owner = owner && (ctl->fix_old & 0xFFFF) == nparts - 1;
                ok = __all_sync(0xffffffffu, wait_bounded(&ctl->acc_full[buf], aph, wd, kSiteEpilogueAcc, seg));
                if (named_bar_any(dec::kBarEpi, 128, !ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t acc_addr = tmem_base + lane_addr + (uint32_t)(buf * C::kAccCols + prim * TOK);
                const uint32_t acc2_addr = tmem_base + lane_addr + (uint32_t)(buf * C::kAccCols + (prim ^ 1) * TOK);
#pragma unroll 1
                for (int c0 = 0; c0 < live_end; c0 += CO) {
                    uint32_t v[CO];
                    tmem_load<CO>(acc_addr + (uint32_t)c0, v);
                    if (two) add_second<CO>(acc2_addr + (uint32_t)c0, v);
                    if (c0 + CO >= live_end) {   // the accumulator goes back to the issuers
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&ctl->acc_empty[buf]);
                    }
                    if (sole) {
                        emit(v, mt, nt, c0);
                    } else if (finisher_owner) {
                        take_sum(v, tsum, c0, m_live);
                        emit(v, mt, nt, c0);
                    } else {
#pragma unroll
                        for (int j = 0; j < CO; ++j)
                            if (c0 + j < m_live) red_add_s32(tsum + (c0 + j) * kTileN, (int32_t)v[j]);
                    }
                }
                if (!sole) {
                    if (finisher_owner) {
                        if (leader) *cnt = 0;   // nobody touches the counter again in this launch
                    } else {
                        // Every add of this CTA precedes its arrival. The owner
                        // is not last: a contributor is still running and will
                        // finish the tile once these sums are in.
                        named_bar_sync(dec::kBarEpi, 128);
                        if (owner) {
                            if (leader) red_or_release_gpu(cnt, 0x10000);
                        } else {
                            // A contributor: arrive now, read the result later.
                            // (QOQ_FORCE_CONFIG=lateck=us delays the arrival, so
                            // that owners arrive first and contributors finish.)
                            if (leader && p.late_arrival_ns) {
                                const uint64_t t_end = globaltimer_ns() + (uint64_t)p.late_arrival_ns;
                                while (globaltimer_ns() < t_end) __nanosleep(1000);
                            }
                            if (leader) pend_old = atom_add_acq_rel_gpu(cnt, 1);
                            pend = true;
                            pend_first = (int)first;
                            pend_nparts = nparts;
                            pend_mt = mt;
                            pend_nt = nt;
                        }
                    }
                }
                // Closing barrier: the staged scales of this tile are no longer read.
                if (named_bar_any(dec::kBarEpi, 128, false)) break;
                ++seg;
            }
            if (ok && pend) {
                // Did this CTA arrive last at the tile it contributed to?
                if (leader) ctl->fix_old = pend_old;
                named_bar_sync(dec::kBarEpi, 128);
                if ((ctl->fix_old & 0xFFFF) == pend_nparts - 1) {
                    // The owner is in (it arrived), but may not have added its
                    // sums yet.
                    int32_t *cnt = p.counters + pend_first;
                    bool got = true;
                    if (leader) got = wait_word_bounded(cnt, 0x10000, 0x10000, wd, kSiteLastOwner, pend_first);
                    stage_tile(pend_mt, pend_nt);
                    if (!named_bar_any(dec::kBarEpi, 128, !got)) {
                        const int64_t m0 = (int64_t)pend_mt * TOK;
                        const int m_live = (int)(p.M - m0 < TOK ? p.M - m0 : TOK);
                        const int live_end = (m_live + CO - 1) / CO * CO;
                        int32_t *tsum = p.partials + (long long)pend_first * TOK * kTileN + r;
#pragma unroll 1
                        for (int c0 = 0; c0 < live_end; c0 += CO) {
                            uint32_t v[CO];
#pragma unroll
                            for (int j = 0; j < CO; ++j) v[j] = 0u;
                            take_sum(v, tsum, c0, m_live);
                            emit(v, pend_mt, pend_nt, c0);
                        }
                        if (leader) *cnt = 0;
                    }
                }
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
    if (FUSED && threadIdx.x == 0) {
        // The last CTA out clears the claim counters for the next launch.
        if (atom_add_acq_rel_gpu(p.qctl + 2, 1) == (int)gridDim.x - 1) {
            p.qctl[0] = 0;
            p.qctl[1] = 0;
            p.qctl[2] = 0;
        }
    }
    if (warp == dec::kWarpIss) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- host side

template <int TOK, int MODE, bool FUSED, int CPS>
static qoq_status launch_decode_t(const GemmArgs &a, cudaStream_t stream, int units_max) {
    using C = DecCfg<TOK, MODE, CPS>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64) return QOQ_ERR_CUDA;
    static std::once_flag attr_once[64];
    static cudaError_t attr_err[64];
    std::call_once(attr_once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(qoq_decode_kernel<TOK, MODE, FUSED, CPS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
        if (attr_err[dev] == cudaSuccess)
            attr_err[dev] = cudaFuncSetAttribute(qoq_decode_kernel<TOK, MODE, FUSED, CPS>,
                                                 cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    });
    if (attr_err[dev] != cudaSuccess) return QOQ_ERR_CUDA;

    const BlobLayout L = blob_layout(a.N, a.K, a.group);
    DecParams p;
    memset(&p, 0, sizeof(p));
    p.blob = static_cast<const uint8_t *>(a.blob);
    p.out = a.out;
    uint8_t *ws = static_cast<uint8_t *>(a.ws);
    p.status = reinterpret_cast<int32_t *>(ws);
    p.qctl = reinterpret_cast<int32_t *>(ws + 32);
    p.counters = reinterpret_cast<int32_t *>(ws + 256);
    p.partials = reinterpret_cast<int32_t *>(ws + QOQ_WORKSPACE_CONTROL_BYTES);
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.group = a.group;
    p.NT = (int)(a.N / kTileN);
    p.KT = (int)(a.K / kTileK);
    p.MT = (int)((a.M + TOK - 1) / TOK);
    p.GM = p.MT < kTileGroup ? p.MT : kTileGroup;
    const long long blocks = (long long)p.MT * p.NT * p.KT;
    if (blocks >= (1ll << 31)) return QOQ_ERR_UNSUPPORTED;
    p.total_blocks = (uint32_t)blocks;
    p.grid = (int)std::min<long long>(units_max, blocks);
    // The split tiles' sum buffers, one per CTA (the owner's index), must be
    // zero when the launch starts; every launch that completes leaves them so.
    if (scratch_bytes_for_grid(TOK, p.grid, 1) > a.ws_capacity) return QOQ_ERR_WORKSPACE;
    const long long tiles = (long long)p.MT * p.NT;
    const long long dp_tiles = tiles >= 2ll * p.grid ? (tiles / p.grid - 1) * p.grid : 0;
    p.dp_tiles = (uint32_t)dp_tiles;
    p.sk_base = (uint32_t)(dp_tiles * p.KT);
    p.off_codes = L.off_codes;
    p.off_scale = L.off_scale;
    p.off_zero = L.off_zero;
    p.fp16_out = a.fp16_out ? 1 : 0;
    p.late_arrival_ns = 1000ll * forced_config().lateck;
    const int8_t *x8 = a.X8;
    if (FUSED) {
        // Codes, scales and row sums of the fused quantisation live in the
        // workspace after the partial sums.
        const FusedLayout F = fused_layout(a.M, a.K, workspace_bytes_for(a.M, a.N, a.K));
        if (F.total > a.ws_capacity) return QOQ_ERR_WORKSPACE;
        p.X = static_cast<const __half *>(a.X);
        p.X8q = reinterpret_cast<int8_t *>(ws + F.off_x8);
        p.s_xq = reinterpret_cast<__half *>(ws + F.off_sx);
        p.rowsumq = reinterpret_cast<int32_t *>(ws + F.off_rowsum);
        p.s_x = p.s_xq;
        p.rowsum = p.rowsumq;
        x8 = p.X8q;
    } else {
        p.s_x = static_cast<const __half *>(a.s_x);
        p.rowsum = a.rowsum;
    }

    CUtensorMap tmap, tmap_y;
    if (!encode_x_map(&tmap, x8, a.M, a.K, TOK)) return QOQ_ERR_CUDA;
    if (a.fp16_out) {
        if (!encode_y_map(&tmap_y, a.out, a.M, a.N)) return QOQ_ERR_CUDA;
    } else {
        memset(&tmap_y, 0, sizeof(tmap_y));
    }

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.grid);
    cfg.blockDim = dim3(dec::kThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    int na = 0;
    if (kProgrammaticLaunch) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, qoq_decode_kernel<TOK, MODE, FUSED, CPS>, p, tmap, tmap_y) == cudaSuccess
               ? QOQ_OK
               : QOQ_ERR_CUDA;
}

int decode_ctas_per_sm(int64_t M, int64_t N, int64_t K) {
    if (forced_config().cps) return forced_config().cps;
    // Measured on B200 (Llama-3-8B shapes, M = 1..256): one CTA per SM is as
    // fast or faster everywhere; the deeper weight ring outweighs the overlap
    // two CTAs per SM give between consecutive launches.
    (void)M;
    (void)N;
    (void)K;
    return 1;
}

bool linear_fused(int64_t M, int64_t N, int64_t K) {
    if (forced_config().fuse) return forced_config().fuse == 2;
    // Measured on B200 (Llama-3-8B decode step, M <= 256): the fused launch's
    // grid-wide claim -> quantise -> publish -> poll chain adds about four L2
    // round trips after griddepcontrol.wait, more than the separate
    // quantiser's launch costs (0.555 vs 0.468 ms per step), so the linear
    // call uses two launches unless QOQ_FORCE_CONFIG asks for fuse=1.
    (void)M;
    (void)N;
    (void)K;
    return false;
}

template <bool FUSED, int CPS>
static qoq_status launch_decode_tok(const GemmArgs &a, cudaStream_t stream, int tok, int units_max) {
    if (a.group) {
        switch (tok) {
            case 16: return launch_decode_t<16, 0, FUSED, CPS>(a, stream, units_max);
            case 32: return launch_decode_t<32, 0, FUSED, CPS>(a, stream, units_max);
            case 64: return launch_decode_t<64, 0, FUSED, CPS>(a, stream, units_max);
        }
    } else {
        switch (tok) {
            case 16: return launch_decode_t<16, 1, FUSED, CPS>(a, stream, units_max);
            case 32: return launch_decode_t<32, 1, FUSED, CPS>(a, stream, units_max);
            case 64: return launch_decode_t<64, 1, FUSED, CPS>(a, stream, units_max);
        }
    }
    return QOQ_ERR_UNSUPPORTED;
}

qoq_status launch_decode_gemm(const GemmArgs &a, cudaStream_t stream, int tok, int units_max) {
    const int cps = decode_ctas_per_sm(a.M, a.N, a.K);
    if (a.X != nullptr)
        return cps == 1 ? launch_decode_tok<true, 1>(a, stream, tok, units_max)
                        : launch_decode_tok<true, 2>(a, stream, tok, units_max);
    return cps == 1 ? launch_decode_tok<false, 1>(a, stream, tok, units_max)
                    : launch_decode_tok<false, 2>(a, stream, tok, units_max);
}

}  // namespace qoq
