// Pieces shared by the GEMM kernels (the general kernel in gemm.cu and the
// decode-regime kernel in gemm_decode.cu): the persistent stream-K schedule,
// the fused epilogue's output stores, tensor-memory loads, and the host-side
// tensor-map encoders.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <mutex>

#include "qoq_device.cuh"
#include "qoq_internal.h"

namespace qoq {

constexpr uint64_t kDrainNs = 100ull * 1000ull * 1000ull;   // 100 ms: teardown wait for copies in flight

// First k-tile block of CTA c (the stream-K split), and the CTA holding block b.
__device__ __forceinline__ uint32_t cta_begin(uint32_t c, uint32_t B, uint32_t G) {
    return (uint32_t)(((unsigned long long)c * B) / G);
}
__device__ __forceinline__ uint32_t cta_of(uint32_t b, uint32_t B, uint32_t G) {
    return (uint32_t)((((unsigned long long)b + 1) * G + B - 1) / B) - 1;
}

// Walks this CTA's k-tile blocks as pipeline units: up to KB consecutive
// k-tiles of one tile, never crossing a tile boundary. The schedule has two
// phases. Data-parallel waves: CTA c takes whole tiles c, c + G, c + 2G, ...
// (`waves` of them), so the G tiles in flight at a time are consecutive in
// tile order and share activation and weight tiles in L2. Stream-K tail: the
// remaining tiles' k-tile blocks [sk_base, B) are split evenly over the G
// CTAs, CTA c taking blocks [sk_b0, sk_b1). Blocks are numbered
// tile * KT + k-tile in both phases. Tile order: groups of GM token tiles;
// inside a group the token tile runs fastest, then the n-tile, so that the G
// tiles in flight cover about GM token tiles x G/GM n-tiles, and each weight
// tile is read by GM CTAs at about the same time (one DRAM read, the rest L2
// hits) while the group's activations stay in L2. No division per unit.
template <int KB>
struct UnitCursor {
    uint32_t b, b1, seg_end;   // current block, end of the current range, end of the current segment
    int KT, NT, MT, GM;
    int kt, nk, nt, mt;
    uint32_t tile, G;          // data-parallel phase: current tile, tile stride
    int waves_left;            // data-parallel tiles after the current one
    bool dp;
    uint32_t sk_b0, sk_b1;
    __device__ __forceinline__ void init(uint32_t c, uint32_t G_, int waves, uint32_t sk_b0_, uint32_t sk_b1_,
                                         int KT_, int NT_, int MT_, int GM_) {
        KT = KT_;
        NT = NT_;
        MT = MT_;
        GM = GM_;
        G = G_;
        sk_b0 = sk_b0_;
        sk_b1 = sk_b1_;
        if (waves > 0) {
            dp = true;
            waves_left = waves - 1;
            tile = c;
            start_tile();
        } else {
            dp = false;
            waves_left = 0;
            start_range();
        }
    }
    // (mt, nt) of `tile` in the grouped order.
    __device__ __forceinline__ void coords() {
        const uint32_t span = (uint32_t)GM * (uint32_t)NT;
        const uint32_t grp = tile / span;
        const uint32_t idx = tile - grp * span;
        const uint32_t m_base = grp * (uint32_t)GM;
        uint32_t gm = (uint32_t)MT - m_base < (uint32_t)GM ? (uint32_t)MT - m_base : (uint32_t)GM;
        if (gm == 0) gm = 1;   // only past the last tile (an empty range), never used
        const uint32_t q = idx / gm;
        nt = (int)q;
        mt = (int)(m_base + idx - q * gm);
    }
    __device__ __forceinline__ void start_tile() {
        b = tile * (uint32_t)KT;
        b1 = b + (uint32_t)KT;
        kt = 0;
        coords();
        set_segment();
    }
    __device__ __forceinline__ void start_range() {
        b = sk_b0;
        b1 = sk_b1;
        tile = b / (uint32_t)KT;
        kt = (int)(b - tile * (uint32_t)KT);
        coords();   // unused when the range is empty
        set_segment();
    }
    __device__ __forceinline__ void set_segment() {
        const uint32_t tile_end = b - (uint32_t)kt + (uint32_t)KT;
        seg_end = tile_end < b1 ? tile_end : b1;
        set_nk();
    }
    __device__ __forceinline__ void set_nk() {
        const uint32_t left = seg_end - b;
        nk = left < (uint32_t)KB ? (int)left : KB;
    }
    __device__ __forceinline__ bool done() const { return !dp && b >= b1; }
    // Advance one unit; returns true when the current segment (tile) ends.
    __device__ __forceinline__ bool advance() {
        b += (uint32_t)nk;
        kt += nk;
        if (b < seg_end) {
            set_nk();
            return false;
        }
        if (b < b1) {   // the stream-K range goes on with the next tile
            kt = 0;
            ++tile;
            coords();
            set_segment();
            return true;
        }
        if (dp) {
            if (waves_left > 0) {
                --waves_left;
                tile += G;
                start_tile();
            } else {
                dp = false;
                start_range();   // may be empty: then done()
            }
        }
        return true;
    }
};

// Epilogue for CH consecutive tokens (m_first ..) of weight row n = n_warp +
// lane (n_warp: the warp's first of 32 rows). sx[j] is FP32(s_x[m_first + j])
// and rs[j] the row sum of that token (shared memory; values for tokens past M
// are unused).
//
// FP16: the warp writes its CH x 32 block into `stage` (token-major, 64-byte
// rows) and lane 0 stores it with one TMA copy, which leaves out the rows past
// M. The two stage blocks of a warp alternate; before one is rewritten, the
// copy issued from it two steps earlier must have finished reading it.
template <int CH, int MODE>
__device__ __forceinline__ void store_outputs_fp16(const CUtensorMap *tmap_y, const uint32_t (&v)[CH],
                                                   int64_t m_first, int n_warp, int lane, float col_scale,
                                                   int col_zero, const float *sx, const int32_t *rs,
                                                   __half *stage) {
    static_assert(CH == 16, "the output box is 16 tokens high");
    if (lane == 0) bulk_wait_group_read<1>();
    __syncwarp();
    float scale[CH];
#pragma unroll
    for (int q = 0; q < CH / 4; ++q) {
        const float4 f = reinterpret_cast<const float4 *>(sx)[q];
        scale[4 * q] = f.x;
        scale[4 * q + 1] = f.y;
        scale[4 * q + 2] = f.z;
        scale[4 * q + 3] = f.w;
    }
#pragma unroll
    for (int j = 0; j < CH; ++j) {
        int32_t acc = (int32_t)v[j];
        if (MODE == 1) acc -= col_zero * rs[j];
        const float y = __fmul_rn(__int2float_rn(acc), __fmul_rn(scale[j], col_scale));
        stage[j * 32 + lane] = __float2half_rn(y);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tmap_y, stage, n_warp, (int)m_first);
        bulk_commit_group();
    }
}

// FP16 values of CH tokens of this lane's weight row, packed in token pairs
// (pk[t]: token 2t low, 2t + 1 high); the same arithmetic as the store above.
template <int CH, int MODE>
__device__ __forceinline__ void convert_fp16(const uint32_t (&v)[CH], uint32_t *pk, float col_scale, int col_zero,
                                             const float *sx, const int32_t *rs) {
    float scale[CH];
#pragma unroll
    for (int q = 0; q < CH / 4; ++q) {
        const float4 f = reinterpret_cast<const float4 *>(sx)[q];
        scale[4 * q] = f.x;
        scale[4 * q + 1] = f.y;
        scale[4 * q + 2] = f.z;
        scale[4 * q + 3] = f.w;
    }
#pragma unroll
    for (int j = 0; j < CH; j += 2) {
        int32_t a0 = (int32_t)v[j], a1 = (int32_t)v[j + 1];
        if (MODE == 1) {
            a0 -= col_zero * rs[j];
            a1 -= col_zero * rs[j + 1];
        }
        const float y0 = __fmul_rn(__int2float_rn(a0), __fmul_rn(scale[j], col_scale));
        const float y1 = __fmul_rn(__int2float_rn(a1), __fmul_rn(scale[j + 1], col_scale));
        const __half2 h = __floats2half2_rn(y0, y1);
        pk[j / 2] = *reinterpret_cast<const uint32_t *>(&h);
    }
}

// The same store for 16 tokens already converted: pk[t] holds this lane's
// weight row at tokens 2t (low half) and 2t + 1 (high half).
__device__ __forceinline__ void store_packed_fp16(const CUtensorMap *tmap_y, const uint32_t *pk, int64_t m_first,
                                                  int n_warp, int lane, __half *stage) {
    if (lane == 0) bulk_wait_group_read<1>();
    __syncwarp();
    unsigned short *st = reinterpret_cast<unsigned short *>(stage);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        st[(2 * t) * 32 + lane] = (unsigned short)(pk[t] & 0xFFFFu);
        st[(2 * t + 1) * 32 + lane] = (unsigned short)(pk[t] >> 16);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tmap_y, stage, n_warp, (int)m_first);
        bulk_commit_group();
    }
}

// INT32 accumulators (after the per-channel zero-point term) of CH tokens.
template <int CH, int MODE>
__device__ __forceinline__ void store_outputs_i32(int32_t *out, int64_t M, int64_t N, const uint32_t (&v)[CH],
                                                  int64_t m_first, int n, int col_zero, const int32_t *rs) {
#pragma unroll
    for (int j = 0; j < CH; ++j) {
        const int64_t m = m_first + j;
        int32_t acc = (int32_t)v[j];
        if (MODE == 1) acc -= col_zero * rs[j];
        if (m < M) out[m * N + n] = acc;
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

// v += the CH columns at taddr (the second issuer's accumulator); exact INT32.
template <int CH>
__device__ __forceinline__ void add_second(uint32_t taddr, uint32_t (&v)[CH]) {
    uint32_t w[CH];
    tmem_load<CH>(taddr, w);
#pragma unroll
    for (int j = 0; j < CH; ++j) v[j] = (uint32_t)((int32_t)v[j] + (int32_t)w[j]);
}

// ---------------------------------------------------------------- host side

inline PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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

inline int sm_count_of(int dev) {
    static int count[64];
    static std::mutex mu;
    if (dev < 0 || dev >= 64) return 0;
    std::lock_guard<std::mutex> lock(mu);
    if (count[dev] == 0) cudaDeviceGetAttribute(&count[dev], cudaDevAttrMultiProcessorCount, dev);
    return count[dev];
}

// X8 [M][K] int8, boxes of 128 k x TOK tokens, 128-byte swizzle.
inline bool encode_x_map(CUtensorMap *map, const int8_t *X8, int64_t M, int64_t K, int tok) {
    auto encode = get_encode_fn();
    if (!encode) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)K};
    const cuuint32_t box[2] = {(cuuint32_t)kTileK, (cuuint32_t)tok};
    const cuuint32_t estride[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(X8), gdim, gstride, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// FP16 output Y [M][N]: boxes of 32 weight rows x 16 tokens, no swizzle (the
// epilogue's stage blocks are plain token-major 64-byte rows).
inline bool encode_y_map(CUtensorMap *map, void *Y, int64_t M, int64_t N) {
    auto encode = get_encode_fn();
    if (!encode) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)N, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)N * 2};
    const cuuint32_t box[2] = {32, 16};
    const cuuint32_t estride[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, Y, gdim, gstride, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace qoq
