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
//   * one dequant thread owns one weight row for one 128-wide k-tile, which is
//     exactly one quantisation group, so the group's (s, z*s) is a per-thread
//     scalar. 8 nibbles per 32-bit word decode with and/shift, one 32-bit
//     multiply-add (q*s <= 240 and q*s + 128 - z*s in [7, 249] never carry
//     between bytes) and one xor that turns excess-128 bytes into int8.
//   * warp roles: 1 TMA producer, 1 MMA issuer, two dequant warpgroups that
//     alternate k-tiles, one epilogue warpgroup; mbarrier rings between them.
//   * persistent stream-K: the (token tile, n-tile, k-tile) blocks are split
//     evenly over at most one CTA per SM; a tile cut between CTAs is summed
//     exactly in INT32 in a workspace slot (integer addition is associative,
//     so the result does not depend on the order), and the last contributor
//     runs the epilogue and re-zeros the slot.
#include <algorithm>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <mutex>

#include "qoq_device.cuh"
#include "qoq_internal.h"

namespace qoq {

constexpr int kThreads = 512;            // 16 warps
constexpr int kWarpProducer = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpDequant0 = 4;         // warps 4..11: two dequant warpgroups
constexpr int kWarpEpilogue = 12;        // warps 12..15
constexpr uint64_t kDrainNs = 100ull * 1000ull * 1000ull;   // 100 ms

__device__ __forceinline__ long long lmin(long long a, long long b) { return a < b ? a : b; }

__host__ __device__ constexpr int pow2_at_least(int x) {
    int p = 32;
    while (p < x) p <<= 1;
    return p;
}

template <int TOK, int MODE>
struct GemmCfg {
    static constexpr int kXBytes = TOK * 128;                   // token tile, 128 k
    static constexpr int kWBytes = MODE == 0 ? 8448 : 8192;     // codes (+ s, z*s)
    static constexpr int kStageBytes = (kXBytes + kWBytes + 1023) / 1024 * 1024;
    static constexpr int kSmemLimit = 232448;                   // 227 KB per CTA
    static constexpr int kReserve = 2048;                       // alignment slack + barriers
    static constexpr int kStagesFit = (kSmemLimit - kReserve) / kStageBytes;
    static constexpr int kStages = kStagesFit > 16 ? 16 : kStagesFit;
    static constexpr int kAStages = 4;                          // TMEM A buffers (32 cols each)
    static constexpr int kAccBufs = TOK <= 128 ? 2 : 1;
    static constexpr int kACol0 = kAccBufs * TOK;
    static constexpr int kTmemCols = pow2_at_least(kACol0 + kAStages * 32);
    static constexpr int kSmemBytes = kStages * kStageBytes + kReserve;
    static_assert(kStages >= 3, "pipeline too shallow");
    static_assert(kTmemCols <= 512, "TMEM over-subscribed");
    static_assert(kXBytes % 1024 == 0, "token tile must keep the swizzle atom aligned");
};

struct GemmParams {
    const uint8_t *blob;
    const __half *s_x;
    const int32_t *rowsum;
    void *out;
    int32_t *status;
    int32_t *counters;
    int32_t *partials;
    int M, N, K, group;
    int NT, KT, MT;
    int grid;
    long long total_blocks;
    long long off_codes, off_scale, off_zero;
    int fp16_out;
};

struct SharedCtl {
    uint64_t full[16], empty[16];
    uint64_t a_full[4], a_empty[4];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t final_bar;
    uint32_t tmem_base;
    int abort_flag;
    int last_flag;
};

// Epilogue for CH consecutive tokens (m_first ..) of weight row n.
template <int CH, int MODE>
__device__ __forceinline__ void store_outputs(const GemmParams &p, const uint32_t (&v)[CH], int64_t m_first,
                                              int n, float col_scale, int col_zero) {
    const int64_t N = p.N;
#pragma unroll
    for (int j = 0; j < CH; ++j) {
        const int64_t m = m_first + j;
        if (m < p.M) {
            int32_t acc = (int32_t)v[j];
            if (MODE == 1) acc -= col_zero * p.rowsum[m];
            if (p.fp16_out) {
                const float sx = __half2float(p.s_x[m]);
                const float y = __fmul_rn(__int2float_rn(acc), __fmul_rn(sx, col_scale));
                static_cast<__half *>(p.out)[m * N + n] = __float2half_rn(y);
            } else {
                static_cast<int32_t *>(p.out)[m * N + n] = acc;
            }
        }
    }
}

template <int CH>
__device__ __forceinline__ void tmem_load(uint32_t taddr, uint32_t (&v)[CH]);
template <>
__device__ __forceinline__ void tmem_load<16>(uint32_t taddr, uint32_t (&v)[16]) {
    tmem_ld16_wait(taddr, v);
}
template <>
__device__ __forceinline__ void tmem_load<32>(uint32_t taddr, uint32_t (&v)[32]) {
    tmem_ld32_wait(taddr, v);
}

template <int TOK, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    qoq_gemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ CUtensorMap tmap_x) {
    using C = GemmCfg<TOK, MODE>;
    constexpr int CH = TOK < 32 ? TOK : 32;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SharedCtl *ctl = reinterpret_cast<SharedCtl *>(smem + C::kStages * C::kStageBytes);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Watchdog wd{&ctl->abort_flag, p.status};

    // ------------------------------------------------------------ set-up
    if (threadIdx.x == 0) {
        ctl->abort_flag = 0;
        ctl->last_flag = 0;
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int a = 0; a < C::kAStages; ++a) {
            mbar_init(&ctl->a_full[a], 4);
            mbar_init(&ctl->a_empty[a], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->acc_full[b], 1);
            mbar_init(&ctl->acc_empty[b], 4);
        }
        mbar_init(&ctl->final_bar, 1);
        mbar_fence_init();
        const uint32_t *h = reinterpret_cast<const uint32_t *>(p.blob);
        if (h[0] != kMagic || h[1] != kVersion || h[2] != (uint32_t)p.N || h[3] != (uint32_t)p.K ||
            h[4] != (uint32_t)p.group)
            wd.fail(QOQ_ERR_BAD_BLOB);
    }
    if (warp == kWarpProducer && lane == 0) prefetch_tensormap(&tmap_x);
    if (warp == kWarpMma) {
        tmem_alloc(&ctl->tmem_base, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;

    // Stream-K share of this CTA: blocks [b0, b1) of the (tile, k-tile) order.
    const long long B = p.total_blocks;
    const long long b0 = (long long)blockIdx.x * B / p.grid;
    const long long b1 = (long long)(blockIdx.x + 1) * B / p.grid;
    const int nblk = (int)(b1 - b0);
    const int KT = p.KT;

    auto stage_x = [&](int s) { return smem + s * C::kStageBytes; };
    auto stage_w = [&](int s) { return smem + s * C::kStageBytes + C::kXBytes; };

    if (!wd.aborted()) {
        if (warp == kWarpProducer) {
            // ------------------------------------------------ TMA producer
            if (lane == 0) {
                const uint64_t pol_w = policy_evict_first();   // weights: streamed once
                const uint64_t pol_x = policy_evict_last();    // activations: reused by every n-tile
                int issued = 0;
                for (int i = 0; i < nblk; ++i) {
                    const long long b = b0 + i;
                    const long long t = b / KT;
                    const int kt = (int)(b - t * KT);
                    const int mt = (int)(t / p.NT);
                    const int nt = (int)(t - (long long)mt * p.NT);
                    const int s = i % C::kStages;
                    const uint32_t ph = (uint32_t)(i / C::kStages) & 1u;
                    if (!wait_bounded(&ctl->empty[s], ph ^ 1u, wd)) break;
                    mbar_arrive_expect_tx(&ctl->full[s], C::kXBytes + C::kWBytes);
                    const uint8_t *wsrc = p.blob + p.off_codes + ((long long)nt * KT + kt) * C::kWBytes;
                    bulk_load(stage_w(s), wsrc, C::kWBytes, &ctl->full[s], pol_w);
                    tma_load_2d(stage_x(s), &tmap_x, &ctl->full[s], kt * kTileK, mt * TOK, pol_x);
                    issued = i + 1;
                }
                // Let every copy that was issued land before the CTA can exit.
                for (int i = issued > C::kStages ? issued - C::kStages : 0; i < issued; ++i)
                    wait_drain(&ctl->full[i % C::kStages], (uint32_t)(i / C::kStages) & 1u, kDrainNs);
            }
        } else if (warp == kWarpMma) {
            // ------------------------------------------------ MMA issuer
            if (lane == 0) {
                constexpr uint32_t idesc = idesc_i8(128, TOK, true, true);
                int i = 0, seg = 0;
                bool ok = true;
                long long b = b0;
                while (ok && b < b1) {
                    const long long t = b / KT;
                    const long long e = lmin(b1, (t + 1) * KT);
                    const int buf = seg % C::kAccBufs;
                    const uint32_t aph = (uint32_t)(seg / C::kAccBufs) & 1u;
                    if (!wait_bounded(&ctl->acc_empty[buf], aph ^ 1u, wd)) break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(buf * TOK);
                    for (long long bb = b; bb < e; ++bb, ++i) {
                        const int s = i % C::kStages;
                        const uint32_t ph = (uint32_t)(i / C::kStages) & 1u;
                        const int a = i % C::kAStages;
                        const uint32_t ap = (uint32_t)(i / C::kAStages) & 1u;
                        if (!wait_bounded(&ctl->full[s], ph, wd) || !wait_bounded(&ctl->a_full[a], ap, wd)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t bdesc = smem_desc_k_sw128(smem_u32(stage_x(s)));
                        const uint32_t a_tmem = tmem_base + (uint32_t)(C::kACol0 + a * 32);
#pragma unroll
                        for (int j = 0; j < 4; ++j)   // 4 x K=32 per 128-wide k-tile
                            mma_i8_ts(d_tmem, a_tmem + (uint32_t)(j * 8), bdesc + (uint64_t)(j * 2), idesc,
                                      (bb > b || j > 0) ? 1u : 0u);
                        tc_commit(&ctl->empty[s]);
                        tc_commit(&ctl->a_empty[a]);
                    }
                    if (!ok) break;
                    tc_commit(&ctl->acc_full[buf]);
                    ++seg;
                    b = e;
                }
                // Every MMA must have completed before tensor memory is freed.
                tc_commit(&ctl->final_bar);
                wait_drain(&ctl->final_bar, 0, kDrainNs);
            }
            __syncwarp();
        } else if (warp >= kWarpDequant0 && warp < kWarpEpilogue) {
            // ------------------------------------------------ dequant
            const int g = (warp - kWarpDequant0) >> 2;     // warpgroup 0 / 1
            const int quarter = warp & 3;                    // TMEM lanes 32q .. 32q+31
            const int r = quarter * 32 + lane;               // weight row in the tile
            const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
            for (int i = g; i < nblk; i += 2) {
                const int s = i % C::kStages;
                const uint32_t ph = (uint32_t)(i / C::kStages) & 1u;
                const int a = i % C::kAStages;
                const uint32_t ap = (uint32_t)(i / C::kAStages) & 1u;
                bool ok = wait_bounded(&ctl->full[s], ph, wd) && wait_bounded(&ctl->a_empty[a], ap ^ 1u, wd);
                if (!__all_sync(0xffffffffu, ok)) break;
                const uint32_t wbase = smem_u32(stage_w(s));
                uint32_t outw[32];
                if (MODE == 0) {
                    const uint32_t sz = lds16(wbase + 8192 + 2 * r);
                    const uint32_t sc = sz & 0xFFu;
                    const int zs = (int)(int8_t)(sz >> 8);
                    const uint32_t c4 = (uint32_t)(128 - zs) * 0x01010101u;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 v = lds128(wbase + c * 2048 + r * 16);
                        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t lo = w[j] & 0x0F0F0F0Fu;
                            const uint32_t hi = (w[j] >> 4) & 0x0F0F0F0Fu;
                            outw[8 * c + 2 * j] = (lo * sc + c4) ^ 0x80808080u;
                            outw[8 * c + 2 * j + 1] = (hi * sc + c4) ^ 0x80808080u;
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 v = lds128(wbase + c * 2048 + r * 16);
                        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            outw[8 * c + 2 * j] = w[j] & 0x0F0F0F0Fu;
                            outw[8 * c + 2 * j + 1] = (w[j] >> 4) & 0x0F0F0F0Fu;
                        }
                    }
                }
                tmem_st32_wait(tmem_base + lane_addr + (uint32_t)(C::kACol0 + a * 32), outw);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->a_full[a]);
            }
        } else if (warp >= kWarpEpilogue) {
            // ------------------------------------------------ epilogue
            const int quarter = warp & 3;
            const int r = quarter * 32 + lane;
            const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
            const bool leader = (threadIdx.x == kWarpEpilogue * 32);
            int seg = 0;
            long long b = b0;
            while (b < b1) {
                const long long t = b / KT;
                const long long e = lmin(b1, (t + 1) * KT);
                const int kt_lo = (int)(b - t * KT), kt_hi = (int)(e - t * KT);
                const int mt = (int)(t / p.NT);
                const int nt = (int)(t - (long long)mt * p.NT);
                const int buf = seg % C::kAccBufs;
                const uint32_t aph = (uint32_t)(seg / C::kAccBufs) & 1u;
                const bool ok = wait_bounded(&ctl->acc_full[buf], aph, wd);
                // All four epilogue warps leave together: the partial-tile path
                // below meets at named barriers.
                if (named_bar_any(1, 128, !ok)) break;
                tc_fence_after();
                const int n = nt * kTileN + r;
                const int64_t m0 = (int64_t)mt * TOK;
                float col_scale = 0.0f;
                int col_zero = 0;
                col_scale = __half2float(reinterpret_cast<const __half *>(p.blob + p.off_scale)[n]);
                if (MODE == 1)
                    col_zero = __half2int_rn(reinterpret_cast<const __half *>(p.blob + p.off_zero)[n]);
                const uint32_t acc_addr = tmem_base + lane_addr + (uint32_t)(buf * TOK);
                if (kt_lo == 0 && kt_hi == KT) {
                    // Whole tile computed here: straight from TMEM.
#pragma unroll 1
                    for (int c0 = 0; c0 < TOK; c0 += CH) {
                        uint32_t v[CH];
                        tmem_load<CH>(acc_addr + (uint32_t)c0, v);
                        if (c0 + CH >= TOK) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&ctl->acc_empty[buf]);
                        }
                        store_outputs<CH, MODE>(p, v, m0 + c0, n, col_scale, col_zero);
                    }
                } else {
                    // Tile shared with other CTAs: add into its slot, count the
                    // k-tiles that have arrived; the last contributor finishes.
                    const long long slot =
                        ((t * KT + 1) * (long long)p.grid + B - 1) / B - 1;   // first CTA boundary inside t
                    int32_t *part = p.partials + slot * (long long)TOK * kTileN;
#pragma unroll 1
                    for (int c0 = 0; c0 < TOK; c0 += CH) {
                        uint32_t v[CH];
                        tmem_load<CH>(acc_addr + (uint32_t)c0, v);
#pragma unroll
                        for (int j = 0; j < CH; ++j) red_add_s32(part + (c0 + j) * kTileN + r, (int32_t)v[j]);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ctl->acc_empty[buf]);
                    __threadfence();
                    named_bar_sync(1, 128);
                    if (leader) {
                        const int old = atomicAdd(p.counters + slot, kt_hi - kt_lo);
                        ctl->last_flag = (old + (kt_hi - kt_lo) == KT) ? 1 : 0;
                    }
                    named_bar_sync(1, 128);
                    if (ctl->last_flag) {
                        __threadfence();
#pragma unroll 1
                        for (int c0 = 0; c0 < TOK; c0 += CH) {
                            uint32_t v[CH];
#pragma unroll
                            for (int j = 0; j < CH; ++j) {
                                int32_t *q = part + (c0 + j) * kTileN + r;
                                v[j] = (uint32_t)ld_cg_s32(q);
                                *q = 0;
                            }
                            store_outputs<CH, MODE>(p, v, m0 + c0, n, col_scale, col_zero);
                        }
                        if (leader) p.counters[slot] = 0;
                    }
                }
                ++seg;
                b = e;
            }
        }
    }

    // ------------------------------------------------------------ teardown
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

struct DeviceInfo {
    int sm_count = 0;
};

static DeviceInfo device_info(int dev) {
    static DeviceInfo info[64];
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return DeviceInfo{};
    if (info[dev].sm_count == 0) cudaDeviceGetAttribute(&info[dev].sm_count, cudaDevAttrMultiProcessorCount, dev);
    return info[dev];
}

template <int TOK, int MODE>
static qoq_status launch_gemm_t(const GemmArgs &a, cudaStream_t stream) {
    using C = GemmCfg<TOK, MODE>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QOQ_ERR_CUDA;
    const DeviceInfo info = device_info(dev);
    if (info.sm_count <= 0) return QOQ_ERR_CUDA;

    // Opt in to the large dynamic shared memory once per device.
    static std::once_flag attr_once[64];
    static cudaError_t attr_err[64];
    if (dev >= 64) return QOQ_ERR_CUDA;
    std::call_once(attr_once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(qoq_gemm_kernel<TOK, MODE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (attr_err[dev] != cudaSuccess) return QOQ_ERR_CUDA;

    auto encode = get_encode_fn();
    if (!encode) return QOQ_ERR_CUDA;
    CUtensorMap tmap;
    const cuuint64_t gdim[2] = {(cuuint64_t)a.K, (cuuint64_t)a.M};
    const cuuint64_t gstride[1] = {(cuuint64_t)a.K};
    const cuuint32_t box[2] = {(cuuint32_t)kTileK, (cuuint32_t)TOK};
    const cuuint32_t estride[2] = {1, 1};
    CUresult cr = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(a.X8), gdim, gstride, box,
                         estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return QOQ_ERR_CUDA;

    const BlobLayout L = blob_layout(a.N, a.K, a.group);
    GemmParams p;
    p.blob = static_cast<const uint8_t *>(a.blob);
    p.s_x = static_cast<const __half *>(a.s_x);
    p.rowsum = a.rowsum;
    p.out = a.out;
    uint8_t *ws = static_cast<uint8_t *>(a.ws);
    p.status = reinterpret_cast<int32_t *>(ws);
    p.counters = reinterpret_cast<int32_t *>(ws + 256);
    p.partials = reinterpret_cast<int32_t *>(ws + 256 + sizeof(int32_t) * kMaxGrid);
    p.M = (int)a.M;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.group = a.group;
    p.NT = (int)(a.N / kTileN);
    p.KT = (int)(a.K / kTileK);
    p.MT = (int)((a.M + TOK - 1) / TOK);
    p.total_blocks = (long long)p.MT * p.NT * p.KT;
    p.grid = (int)std::min<long long>(std::min(info.sm_count, kMaxGrid), p.total_blocks);
    p.off_codes = L.off_codes;
    p.off_scale = L.off_scale;
    p.off_zero = L.off_zero;
    p.fp16_out = a.fp16_out ? 1 : 0;

    qoq_gemm_kernel<TOK, MODE><<<p.grid, kThreads, C::kSmemBytes, stream>>>(p, tmap);
    return cudaGetLastError() == cudaSuccess ? QOQ_OK : QOQ_ERR_CUDA;
}

template <int MODE>
static qoq_status launch_gemm_mode(const GemmArgs &a, cudaStream_t stream) {
    switch (token_tile_for(a.M)) {
        case 16: return launch_gemm_t<16, MODE>(a, stream);
        case 32: return launch_gemm_t<32, MODE>(a, stream);
        case 64: return launch_gemm_t<64, MODE>(a, stream);
        case 128: return launch_gemm_t<128, MODE>(a, stream);
        default: return launch_gemm_t<256, MODE>(a, stream);
    }
}

qoq_status launch_gemm(const GemmArgs &a, cudaStream_t stream) {
    return a.group ? launch_gemm_mode<0>(a, stream) : launch_gemm_mode<1>(a, stream);
}

}  // namespace qoq
