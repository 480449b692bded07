// KV4 decode attention for sm_100a: per-head, dynamic, asymmetric 4-bit K/V
// caches and one-query-token-per-sequence grouped-query attention over them.
//
// QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM Serving
// (arXiv 2405.04532), paperlayer.ai summary:
//   section 3 -- at decode the attention is memory-bound, so a 4-bit cache
//     (KV4) roughly doubles its peak performance over KV8;
//   section 5 "KV4 attention" -- per-head dynamic scales and zero points,
//     attention arithmetic on CUDA cores;
//   section 6 -- per-head asymmetric INT4 KV caches; the attention kernel
//     measured at batch 64 x 1024 tokens.
//
// Cache write: one warp per vector (sequence, KV head, token): min/max by
// shuffles, FP16 scale, integer zero, codes packed two per byte; every FP32
// step one correctly rounded operation (the per-channel weight quantiser's
// arithmetic), so the codes, scales and zeros are reproducible bit for bit.
//
// Attention (B200 design): the work is HBM-bound in principle (0.53 bytes of
// cache per query-head multiply-add at D = 128, group 4), but unpacking 4-bit
// codes costs instructions, so the design is about keeping HBM busy with few
// instructions per code:
//   * a CTA takes one (sequence, KV head, span of tokens), so K and V are read
//     once for the whole query-head group; each of its 4 warps walks 64-token
//     tiles, bulk-copying (cp.async.bulk, mbarrier completion) a tile's K and
//     V codes into its own buffers and refilling each buffer as soon as it is
//     consumed, so the next tile is in flight while this one is computed;
//   * the codes become MMA operands by one AND per two codes: a nibble in
//     bits 0-3 of an FP16 half is the subnormal c * 2^-24, in bits 4-7 it is
//     c * 2^-20, both exact; the products run on tensor cores (mma.sync
//     m16n8k16, FP16 inputs, FP32 accumulation) and the zero points are
//     subtracted in FP32 afterwards (z * sum(q) per score, z * (P s) per
//     output column), so no per-code subtraction is needed;
//   * scores = K . q with the tokens as MMA rows and the group's heads as
//     columns, times the token's scale and log2(e)/sqrt(D); the online softmax
//     in FP32 once per 64-token tile; P times the value scale rounded to FP16;
//     out^T = V^T (P s)^T with the dims as rows;
//   * the warps are merged in shared memory in a fixed order, and the CTAs of
//     one (sequence, KV head) by the CTA that finishes last (a per-head
//     arrival counter; rescaling by the running maxima), which writes the
//     FP16 output; no second launch, and the counters are left zero.
// The pages put this arithmetic on CUDA cores in FP16; on B200 the legacy
// tensor-core MMA does the two contractions with FP32 accumulation for far
// fewer instructions, and the subnormal encoding removes the per-code
// dequantisation arithmetic (or with FP16 1024, subtract 1024 + z) that
// would otherwise bound the kernel's instruction issue.
#include <cuda_fp16.h>
#include <stdint.h>

#include <mutex>

#include "qoq_device.cuh"
#include "qoq_internal.h"

namespace qoq {

// ------------------------------------------------------------ cache write

template <int D>
__global__ void __launch_bounds__(256) kv4_write_kernel(const __half *__restrict__ src, int64_t nvec, int nt,
                                                         int Tmax, int t0, uint8_t *__restrict__ codes,
                                                         __half *__restrict__ scales, __half *__restrict__ zeros) {
    constexpr int VPL = D / 32;   // values per lane: 4 (D = 128) or 2 (D = 64)
    const int64_t vec = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (vec >= nvec) return;
    const int lane = threadIdx.x & 31;
    const int64_t bh = vec / nt;
    const int64_t slot = bh * Tmax + t0 + (vec - bh * nt);
    float x[VPL];
    const __half *s = src + vec * D + lane * VPL;
    if constexpr (VPL == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(s);
        x[0] = __half2float(__ushort_as_half((unsigned short)(u.x & 0xFFFFu)));
        x[1] = __half2float(__ushort_as_half((unsigned short)(u.x >> 16)));
        x[2] = __half2float(__ushort_as_half((unsigned short)(u.y & 0xFFFFu)));
        x[3] = __half2float(__ushort_as_half((unsigned short)(u.y >> 16)));
    } else {
        const uint32_t u = *reinterpret_cast<const uint32_t *>(s);
        x[0] = __half2float(__ushort_as_half((unsigned short)(u & 0xFFFFu)));
        x[1] = __half2float(__ushort_as_half((unsigned short)(u >> 16)));
    }
    // The range includes 0: lo = min(0, min x), hi = max(0, max x).
    float lo = 0.0f, hi = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        lo = fminf(lo, x[i]);
        hi = fmaxf(hi, x[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const __half sh = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f));
    const float sf = __half2float(sh);
    int z = 0;
    uint32_t q[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) q[i] = 0u;
    if (sf != 0.0f) {
        const float zf = rintf(__fdiv_rn(-lo, sf));
        z = (int)zf;
#pragma unroll
        for (int i = 0; i < VPL; ++i)
            q[i] = (uint32_t)fminf(fmaxf(rintf(__fdiv_rn(x[i], sf)) + zf, 0.0f), 15.0f);
    }
    uint8_t *dst = codes + slot * (D / 2) + lane * (VPL / 2);
    if constexpr (VPL == 4) {
        const uint32_t pk = (q[0] | (q[1] << 4)) | ((q[2] | (q[3] << 4)) << 8);
        *reinterpret_cast<uint16_t *>(dst) = (uint16_t)pk;
    } else {
        *dst = (uint8_t)(q[0] | (q[1] << 4));
    }
    if (lane == 0) {
        scales[slot] = sh;
        zeros[slot] = __int2half_rn(z);   // an integer: +0, never -0
    }
}

cudaError_t launch_kv4_cache_write(const void *src, int64_t B, int64_t Hkv, int64_t Tmax, int64_t t0, int64_t nt,
                                   int64_t D, uint8_t *codes, void *scales, void *zeros, cudaStream_t stream) {
    const int64_t nvec = B * Hkv * nt;
    const unsigned blocks = (unsigned)((nvec + 7) / 8);
    auto *s = static_cast<const __half *>(src);
    auto *sc = static_cast<__half *>(scales);
    auto *zr = static_cast<__half *>(zeros);
    if (D == 128)
        kv4_write_kernel<128><<<blocks, 256, 0, stream>>>(s, nvec, (int)nt, (int)Tmax, (int)t0, codes, sc, zr);
    else
        kv4_write_kernel<64><<<blocks, 256, 0, stream>>>(s, nvec, (int)nt, (int)Tmax, (int)t0, codes, sc, zr);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- attention

constexpr int kKvWarps = 4;                          // warps per CTA
constexpr int kKvThreads = 32 * kKvWarps;
constexpr int kKvTile = 64;                          // tokens per warp tile (one bulk copy each of K and V)
constexpr int kKvRound = kKvWarps * kKvTile;         // tokens per CTA per round of tiles
constexpr int kKvMaxGroup = 8;                       // query heads per KV head
constexpr int kKvStatusBytes = 256;                  // workspace: status words, then counters

struct Kv4Params {
    const __half *q;
    const uint8_t *kc;
    const __half *ks, *kz;
    const uint8_t *vc;
    const __half *vs, *vz;
    const int32_t *seq_lens;
    __half *out;
    int32_t *status;     // [0] code, [1] wait site, [2] block, [3] detail
    int32_t *counters;   // [B * Hkv], zero between calls
    float *part;         // [B * Hkv][splits][kKvMaxGroup * D + 2 * kKvMaxGroup]
    int B, Hq, Hkv, Tmax, G;
    int splits, tpw;     // CTAs per (sequence, KV head); tiles per warp
    float qscale;        // log2(e) / sqrt(D)
};

__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// 2^x by the PTX approximate base-2 exponential (relative error near
// 2^-22, far inside the attention's tolerance); 2^-inf = +0.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// D (16x8, FP32) += A (16x16, FP16, row-major) . B (16x8, FP16, column-major).
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t half2_bits(__half2 h) { return *reinterpret_cast<const uint32_t *>(&h); }

__device__ __forceinline__ float half_lo(uint32_t w) {
    return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu)));
}

__device__ __forceinline__ __half half_hi(uint32_t w) { return __ushort_as_half((unsigned short)(w >> 16)); }

// One CTA = one (sequence, KV head, token span of 256 * tpw); warp w takes
// the span's 64-token tiles w, w + 4, w + 8, ... Each warp owns one
// shared-memory buffer for a tile's K codes and one for its V codes, each
// filled by one bulk copy (the codes are contiguous in the cache) issued by
// the warp's lane 0 and completing on that buffer's mbarrier; the lanes fetch
// the tile's scales and zeros with plain loads, one tile ahead. The K buffer
// is refilled with the next tile's keys as soon as the scores are done, the V
// buffer as soon as the output product is done, so the next tile's codes are
// in flight while this one is computed. Each lane reads the code bytes that
// its MMA fragments need straight from the buffers; the only other
// shared-memory traffic is the 64 x 8 tile of softmax weights that changes
// fragment layout between the two products. The online softmax runs once per
// 64-token tile: the tile's score chains are independent, and there is one
// maximum, one sum and one rescale of the output per tile.
template <int D>
__global__ void __launch_bounds__(kKvThreads, 4) kv4_attn_kernel(const __grid_constant__ Kv4Params p) {
    constexpr int DB = D / 2;         // code bytes per vector
    constexpr int KW = DB / 16;       // K words a lane reads per token (bytes 4 KW tig .. 4 KW tig + 4 KW - 1)
    constexpr int VB = DB / 8;        // V bytes a lane reads per token (bytes VB gid .. VB gid + VB - 1)
    constexpr int KS = D / 16;        // k-steps of the score product
    constexpr int MT = D / 16;        // m-tiles (16 dims) of the output product
    constexpr int TB = kKvTile * DB;  // bytes of one tensor's tile
    static_assert(kKvWarps * kKvMaxGroup * D * 4 <= kKvWarps * 2 * TB, "merge buffer fits the code buffers");
    extern __shared__ __align__(128) uint8_t kv_smem[];
    __shared__ __align__(8) uint64_t bars[kKvWarps][2];   // per warp: its K buffer, its V buffer
    __shared__ float mw[kKvWarps][kKvMaxGroup], lw[kKvWarps][kKvMaxGroup];
    __shared__ float mc[kKvMaxGroup], lc[kKvMaxGroup];
    __shared__ int last_s;
    __shared__ volatile int abort_s;

    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    int T = p.Tmax;
    if (p.seq_lens) T = min(max(p.seq_lens[b], 1), p.Tmax);
    const int span = p.tpw * kKvRound;
    const int t_begin = split * span;
    if (t_begin >= T) return;   // past this sequence's tokens: no work, no arrival
    const int t_end = min(T, t_begin + span);
    const int nsplit = (T + span - 1) / span;   // CTAs of this (sequence, head) with work
    const int64_t bh = (int64_t)b * p.Hkv + h;
    const int G = p.G;
    uint8_t *kbuf = kv_smem + (size_t)warp * 2 * TB;   // this warp's K codes [64][DB], then its V codes
    uint8_t *vbuf = kbuf + TB;
    __half *pt = reinterpret_cast<__half *>(kv_smem + (size_t)kKvWarps * 2 * TB) + warp * (kKvTile * 8);
    const Watchdog wd{&abort_s, p.status};

    if (tid == 0) abort_s = 0;
    if (lane == 0) {
        mbar_init(&bars[warp][0], 1);
        mbar_init(&bars[warp][1], 1);
        mbar_fence_init();
    }
    __syncthreads();

    auto tile_t0 = [&](int k) { return t_begin + (k * kKvWarps + warp) * kKvTile; };
    const uint64_t pol = policy_evict_first();
    // Lane 0: the k-th tile's K (v = 0) or V (v = 1) codes into the warp's
    // buffer for them, completing on that buffer's barrier (phase k & 1).
    // Called only for tiles that start inside the span (1 to 64 tokens).
    auto issue = [&](int k, int v) {
        const int t0 = tile_t0(k);
        const uint32_t bytes = (uint32_t)(min(kKvTile, t_end - t0) * DB);
        uint64_t *bar = &bars[warp][v];
        mbar_arrive_expect_tx(bar, bytes);
        bulk_load(v ? vbuf : kbuf, (v ? p.vc : p.kc) + (bh * p.Tmax + t0) * DB, bytes, bar, pol);
    };
    // The k-th tile's scales and zeros: token lane + 32 r in word r, as
    // (scale | zero << 16); zero past the span, so that unwritten slots
    // contribute nothing.
    auto load_sz = [&](int k, uint32_t (&kw)[2], uint32_t (&vw)[2]) {
        const int t0 = tile_t0(k);
        const int64_t s0 = bh * p.Tmax + t0;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            kw[r] = vw[r] = 0u;
            if (t0 + lane + 32 * r < t_end) {
                const int64_t i = s0 + lane + 32 * r;
                kw[r] = (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p.ks) + i) |
                        ((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p.kz) + i) << 16);
                vw[r] = (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p.vs) + i) |
                        ((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(p.vz) + i) << 16);
            }
        }
    };
    // Tiles issued into the K and V buffers (a failed wait drains the last of
    // each before the CTA goes on). A warp whose first tile starts past the
    // span has nothing to copy.
    const bool any = tile_t0(0) < t_end;
    int nk = any ? 1 : 0, nv = any ? 1 : 0;
    if (lane == 0 && any) {
        issue(0, 0);
        issue(0, 1);
    }
    uint32_t kw[2], vw[2];
    load_sz(0, kw, vw);

    // The group's queries as the B fragments of the score product (heads
    // >= G zero). The product's k index is a permutation of the dims, fixed
    // by how a lane unpacks its code words: for the lane's word i (dims
    // d = (D/4) tig + 8 i .. d + 7; byte b holds dims d + 2b, d + 2b + 1),
    // k-step 2 i takes the low nibbles, pairing dims (d, d+4) and (d+2, d+6),
    // k-step 2 i + 1 the high nibbles, pairing (d+1, d+5) and (d+3, d+7).
    // sq: the FP32 sum of the query's dims, per head (for the zero points).
    uint32_t qf[KS][2];
    float sq2[2];
    {
        const __half *qrow = p.q + ((int64_t)b * p.Hq + (int64_t)h * G + gid) * D + tig * (D / 4);
        float sq = 0.0f;
#pragma unroll
        for (int i = 0; i < KW; ++i) {
            uint4 u = make_uint4(0u, 0u, 0u, 0u);
            if (gid < G) u = *reinterpret_cast<const uint4 *>(qrow + 8 * i);
            qf[2 * i][0] = __byte_perm(u.x, u.z, 0x5410);
            qf[2 * i][1] = __byte_perm(u.y, u.w, 0x5410);
            qf[2 * i + 1][0] = __byte_perm(u.x, u.z, 0x7632);
            qf[2 * i + 1][1] = __byte_perm(u.y, u.w, 0x7632);
            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&uw[e]));
                sq += f.x + f.y;
            }
        }
        sq += __shfl_xor_sync(0xffffffffu, sq, 1);
        sq += __shfl_xor_sync(0xffffffffu, sq, 2);   // head gid's sum in the lanes of that gid
        sq2[0] = __shfl_sync(0xffffffffu, sq, 8 * tig);       // head 2 tig
        sq2[1] = __shfl_sync(0xffffffffu, sq, 8 * tig + 4);   // head 2 tig + 1
    }

    float m2[2] = {-INFINITY, -INFINITY};   // running maximum of heads 2 tig, 2 tig + 1
    float l2[2] = {0.0f, 0.0f};             // running sum of the same heads
    float zc[2] = {0.0f, 0.0f};             // running sum over this lane's tokens of z_V * (P s), same heads
    // The output, transposed (dims x heads), in units of 2^-24 (the codes
    // enter the products as FP16 subnormals c * 2^-24). Row gid of m-tile jj
    // is dim 2 (VB gid + jj), row gid + 8 the next dim, in units of 2^-20;
    // columns are heads 2 tig, 2 tig + 1, the same heads as the lane's
    // scores, so each lane rescales with its own factors.
    float o[MT][4];
#pragma unroll
    for (int j = 0; j < MT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
    // The warp's P tile, [64 tokens][8 heads] FP16: half2 stores of a
    // lane's two heads, and transposed 8x8 loads as the B operand.
    const uint32_t pt_st = smem_u32(pt) + (uint32_t)(gid * 16 + tig * 4);
    const uint32_t pt_ld = smem_u32(pt) + (uint32_t)((lane & 15) * 16);

    bool failed = false;
    for (int k = 0; k < p.tpw; ++k) {
        const int t0 = tile_t0(k);
        if (t0 >= t_end) break;
        const int n = min(kKvTile, t_end - t0);
        const bool more = k + 1 < p.tpw && tile_t0(k + 1) < t_end;
        uint32_t kwn[2] = {0u, 0u}, vwn[2] = {0u, 0u};
        if (more) load_sz(k + 1, kwn, vwn);   // in flight while this tile is computed
        if (!wait_bounded(&bars[warp][0], (uint32_t)(k & 1), wd, kSiteKvTile, 2 * k)) {
            failed = true;
            break;
        }
        const uint8_t *kt = kbuf;
        const uint8_t *vt = vbuf;
        // 1. Scores (tokens x heads) of the tile's four 16-token steps, four
        // independent pairs of MMA chains. A lane's code words of tokens gid
        // and gid + 8 of the step become A fragments by a mask alone: low
        // nibbles are FP16 subnormals c * 2^-24, high nibbles c * 2^-20, all
        // exact, accumulated separately (acc1, acc16). The score is then
        // 2^24 acc1 + 2^20 acc16 - z * sum(q), times the token's scale.
        float sc[4][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = -INFINITY;
            if (16 * j >= n) continue;
            const uint32_t kws = kw[j >> 1];
            const int lb = (j & 1) * 16;
            const uint32_t kA = __shfl_sync(0xffffffffu, kws, lb + gid);
            const uint32_t kB = __shfl_sync(0xffffffffu, kws, lb + gid + 8);
            const uint8_t *ka = kt + (16 * j + gid) * DB + tig * (4 * KW);
            uint32_t wa[KW], wb[KW];
            if constexpr (KW == 4) {
                const uint4 x = *reinterpret_cast<const uint4 *>(ka);
                const uint4 y = *reinterpret_cast<const uint4 *>(ka + 8 * DB);
                wa[0] = x.x, wa[1] = x.y, wa[2] = x.z, wa[3] = x.w;
                wb[0] = y.x, wb[1] = y.y, wb[2] = y.z, wb[3] = y.w;
            } else {
                const uint2 x = *reinterpret_cast<const uint2 *>(ka);
                const uint2 y = *reinterpret_cast<const uint2 *>(ka + 8 * DB);
                wa[0] = x.x, wa[1] = x.y;
                wb[0] = y.x, wb[1] = y.y;
            }
            float acc1[4] = {0.0f, 0.0f, 0.0f, 0.0f}, acc16[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int i = 0; i < KW; ++i) {
                const uint32_t wa8 = wa[i] >> 8, wb8 = wb[i] >> 8;
                uint32_t a[4];
                a[0] = wa[i] & 0x000F000Fu;
                a[1] = wb[i] & 0x000F000Fu;
                a[2] = wa8 & 0x000F000Fu;
                a[3] = wb8 & 0x000F000Fu;
                mma_16816(acc1, a, qf[2 * i][0], qf[2 * i][1]);
                a[0] = wa[i] & 0x00F000F0u;
                a[1] = wb[i] & 0x00F000F0u;
                a[2] = wa8 & 0x00F000F0u;
                a[3] = wb8 & 0x00F000F0u;
                mma_16816(acc16, a, qf[2 * i + 1][0], qf[2 * i + 1][1]);
            }
            // acc[0], acc[1]: token gid, heads 2 tig, 2 tig + 1; acc[2], acc[3]: token gid + 8.
            const float zA = __half2float(half_hi(kA)), zB = __half2float(half_hi(kB));
            const float skA = half_lo(kA) * p.qscale, skB = half_lo(kB) * p.qscale;
            const bool okA = 16 * j + gid < n, okB = 16 * j + gid + 8 < n;
            const float r0 = fmaf(acc16[0], 0x1p20f, acc1[0] * 0x1p24f) - zA * sq2[0];
            const float r1 = fmaf(acc16[1], 0x1p20f, acc1[1] * 0x1p24f) - zA * sq2[1];
            const float r2 = fmaf(acc16[2], 0x1p20f, acc1[2] * 0x1p24f) - zB * sq2[0];
            const float r3 = fmaf(acc16[3], 0x1p20f, acc1[3] * 0x1p24f) - zB * sq2[1];
            sc[j][0] = okA ? r0 * skA : -INFINITY;
            sc[j][1] = okA ? r1 * skA : -INFINITY;
            sc[j][2] = okB ? r2 * skB : -INFINITY;
            sc[j][3] = okB ? r3 * skB : -INFINITY;
        }
        __syncwarp();   // every lane is done with the K buffer: refill it with the next tile's keys
        if (more) {
            if (lane == 0) issue(k + 1, 0);
            ++nk;
        }
        // 2. Online softmax over the whole tile: one maximum, one rescale. Heads
        // >= G have q = 0, so their scores are 0 (finite; their outputs are
        // never stored), and every tile holds a valid token, so the maxima are
        // finite after the first tile: no guards in the exponentials.
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            mx[0] = fmaxf(mx[0], fmaxf(sc[j][0], sc[j][2]));
            mx[1] = fmaxf(mx[1], fmaxf(sc[j][1], sc[j][3]));
        }
#pragma unroll
        for (int s = 4; s < 32; s <<= 1) {
            mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], s));
            mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], s));
        }
        float al[2], sm[2] = {0.0f, 0.0f};
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const float mn = fmaxf(m2[c], mx[c]);
            al[c] = ex2_approx(m2[c] - mn);   // 0 the first time (m2 = -inf)
            m2[c] = mn;
            zc[c] *= al[c];
        }
        // P times the value scale, FP16, into the P tile; the value zero
        // points' share, z * (P s) with the same FP16 values, summed in FP32.
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (16 * j >= n) continue;
            const uint32_t vws = vw[j >> 1];
            const int lb = (j & 1) * 16;
            const uint32_t vA = __shfl_sync(0xffffffffu, vws, lb + gid);
            const uint32_t vB = __shfl_sync(0xffffffffu, vws, lb + gid + 8);
            const float svA = half_lo(vA), svB = half_lo(vB);
            float pr[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                pr[c] = ex2_approx(sc[j][c] - m2[c & 1]);
                sm[c & 1] += pr[c];
            }
            const __half2 pA = __floats2half2_rn(pr[0] * svA, pr[1] * svA);
            const __half2 pB = __floats2half2_rn(pr[2] * svB, pr[3] * svB);
            const float2 fA = __half22float2(pA), fB = __half22float2(pB);
            const float zA = __half2float(half_hi(vA)), zB = __half2float(half_hi(vB));
            zc[0] = fmaf(zA, fA.x, fmaf(zB, fB.x, zc[0]));
            zc[1] = fmaf(zA, fA.y, fmaf(zB, fB.y, zc[1]));
            sts32(pt_st + (uint32_t)(16 * j * 16), half2_bits(pA));
            sts32(pt_st + (uint32_t)((16 * j + 8) * 16), half2_bits(pB));
        }
#pragma unroll
        for (int s = 4; s < 32; s <<= 1) {
            sm[0] += __shfl_xor_sync(0xffffffffu, sm[0], s);
            sm[1] += __shfl_xor_sync(0xffffffffu, sm[1], s);
        }
        l2[0] = l2[0] * al[0] + sm[0];
        l2[1] = l2[1] * al[1] + sm[1];
#pragma unroll
        for (int jj = 0; jj < MT; ++jj) {
            o[jj][0] *= al[0];
            o[jj][2] *= al[0];
            o[jj][1] *= al[1];
            o[jj][3] *= al[1];
        }
        __syncwarp();   // the P tile is written
        if (!wait_bounded(&bars[warp][1], (uint32_t)(k & 1), wd, kSiteKvTile, 2 * k + 1)) {
            failed = true;
            break;
        }

        // 3. out^T (dims x heads) += c_V^T (dims x tokens) . (P s)^T, 16 tokens
        // at a time. The lane's tokens 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9 of
        // the step; byte jj of each token's VB bytes gives m-tile jj: low
        // nibbles row gid (c * 2^-24), high nibbles row gid + 8 (c * 2^-20).
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (16 * j >= n) continue;
            uint32_t pb0, pb1;   // (P s)^T as the column-major B operand: tokens 2 tig.., head gid
            ldsm_x2_trans(pt_ld + (uint32_t)(16 * j * 16), pb0, pb1);
            const uint8_t *vr = vt + (16 * j + 2 * tig) * DB + gid * VB;
            constexpr int VW = VB / 4;
            uint32_t w0[VW], w1[VW], w8[VW], w9[VW];
            if constexpr (VW == 2) {
                const uint2 x0 = *reinterpret_cast<const uint2 *>(vr);
                const uint2 x1 = *reinterpret_cast<const uint2 *>(vr + DB);
                const uint2 x8 = *reinterpret_cast<const uint2 *>(vr + 8 * DB);
                const uint2 x9 = *reinterpret_cast<const uint2 *>(vr + 9 * DB);
                w0[0] = x0.x, w0[1] = x0.y, w1[0] = x1.x, w1[1] = x1.y;
                w8[0] = x8.x, w8[1] = x8.y, w9[0] = x9.x, w9[1] = x9.y;
            } else {
                w0[0] = *reinterpret_cast<const uint32_t *>(vr);
                w1[0] = *reinterpret_cast<const uint32_t *>(vr + DB);
                w8[0] = *reinterpret_cast<const uint32_t *>(vr + 8 * DB);
                w9[0] = *reinterpret_cast<const uint32_t *>(vr + 9 * DB);
            }
#pragma unroll
            for (int jj = 0; jj < MT; ++jj) {
                const uint32_t by = (uint32_t)(jj & 3);
                const uint32_t sel = by | ((4u + by) << 8);   // byte jj of the first word to byte 0, of the second to byte 2
                const uint32_t x01 = __byte_perm(w0[jj >> 2], w1[jj >> 2], sel);
                const uint32_t x89 = __byte_perm(w8[jj >> 2], w9[jj >> 2], sel);
                uint32_t a[4];
                a[0] = x01 & 0x000F000Fu;
                a[1] = x01 & 0x00F000F0u;
                a[2] = x89 & 0x000F000Fu;
                a[3] = x89 & 0x00F000F0u;
                mma_16816(o[jj], a, pb0, pb1);
            }
        }
        __syncwarp();   // every lane is done with the V buffer: refill it with the next tile's values
        if (more) {
            if (lane == 0) issue(k + 1, 1);
            ++nv;
        }
        kw[0] = kwn[0], kw[1] = kwn[1], vw[0] = vwn[0], vw[1] = vwn[1];
    }
    if (failed) {
        // Let the copies already issued land before the buffers are reused or
        // the CTA exits (each barrier has at most one phase pending); the
        // status word already holds the error.
        if (nk > 0) wait_drain(&bars[warp][0], (uint32_t)((nk - 1) & 1), kWaitLimitNs);
        if (nv > 0) wait_drain(&bars[warp][1], (uint32_t)((nv - 1) & 1), kWaitLimitNs);
    }

    // Merge the warps: maxima and sums per head, then the outputs rescaled to
    // the CTA's maxima, each warp's into its own FP32 slot over the (now
    // idle) code buffers, summed in a fixed order so that the result does not
    // depend on timing.
    if (gid == 0) {
        mw[warp][2 * tig] = m2[0];
        mw[warp][2 * tig + 1] = m2[1];
        lw[warp][2 * tig] = l2[0];
        lw[warp][2 * tig + 1] = l2[1];
    }
    __syncthreads();
    float *ow = reinterpret_cast<float *>(kv_smem);   // [kKvWarps][kKvMaxGroup][D]
    if (tid < kKvMaxGroup) {
        float M = -INFINITY;
        for (int w = 0; w < kKvWarps; ++w) M = fmaxf(M, mw[w][tid]);
        float L = 0.0f;
        for (int w = 0; w < kKvWarps; ++w) L += mw[w][tid] == -INFINITY ? 0.0f : exp2f(mw[w][tid] - M) * lw[w][tid];
        mc[tid] = M;
        lc[tid] = L;
    }
    __syncthreads();
    // The zero points' share of each head, summed over the lanes of its
    // column (xor over gid); the output in real units is 2^24 o - zc (rows
    // gid) and 2^20 o - zc (rows gid + 8).
#pragma unroll
    for (int s = 4; s < 32; s <<= 1) {
        zc[0] += __shfl_xor_sync(0xffffffffu, zc[0], s);
        zc[1] += __shfl_xor_sync(0xffffffffu, zc[1], s);
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const int g = 2 * tig + c;
        if (g < G) {
            const float f = m2[c] == -INFINITY ? 0.0f : exp2f(m2[c] - mc[g]);
            float *dst = ow + (warp * kKvMaxGroup + g) * D;
#pragma unroll
            for (int jj = 0; jj < MT; ++jj)
                *reinterpret_cast<float2 *>(dst + 2 * (VB * gid + jj)) =
                    make_float2(fmaf(o[jj][c], 0x1p24f, -zc[c]) * f, fmaf(o[jj][2 + c], 0x1p20f, -zc[c]) * f);
        }
    }
    __syncthreads();
    float *osum = ow;   // [heads][D]: warp 0's slot, summed in place over the others
    for (int i = tid; i < G * D; i += kKvThreads) {
        float sum = ow[i];
        for (int w = 1; w < kKvWarps; ++w) sum += ow[w * kKvMaxGroup * D + i];
        osum[i] = sum;   // read and written by this thread alone
    }
    __syncthreads();

    if (nsplit == 1) {
        for (int i = tid; i < G * D; i += kKvThreads)
            p.out[((int64_t)b * p.Hq + (int64_t)h * G) * D + i] = __float2half_rn(osum[i] / lc[i / D]);
        return;
    }
    // Several CTAs on this (sequence, head): store this one's unnormalised
    // sums with its maxima and weights, arrive, and let the last arriver
    // combine.
    constexpr int PSZ = kKvMaxGroup * D + 2 * kKvMaxGroup;
    float *part = p.part + (bh * p.splits + split) * PSZ;
    for (int i = tid; i < G * D; i += kKvThreads) part[i] = osum[i];
    if (tid < kKvMaxGroup) {
        part[kKvMaxGroup * D + tid] = mc[tid];
        part[kKvMaxGroup * D + kKvMaxGroup + tid] = lc[tid];
    }
    __syncthreads();   // every store of the CTA precedes the arrival (cumulative release)
    if (tid == 0) last_s = atom_add_acq_rel_gpu(p.counters + bh, 1) == nsplit - 1;
    __syncthreads();
    if (!last_s) return;
    const float *base = p.part + bh * p.splits * PSZ;
    if (tid < kKvMaxGroup) {
        float M = -INFINITY;
        for (int c = 0; c < nsplit; ++c) M = fmaxf(M, __ldcg(base + c * PSZ + kKvMaxGroup * D + tid));
        float L = 0.0f;
        for (int c = 0; c < nsplit; ++c)
            L += exp2f(__ldcg(base + c * PSZ + kKvMaxGroup * D + tid) - M) *
                 __ldcg(base + c * PSZ + kKvMaxGroup * D + kKvMaxGroup + tid);
        mc[tid] = M;
        lc[tid] = L;
    }
    __syncthreads();
    for (int i = tid; i < G * D; i += kKvThreads) {
        const int g = i / D;
        float O = 0.0f;
        for (int c = 0; c < nsplit; ++c)
            O += exp2f(__ldcg(base + c * PSZ + kKvMaxGroup * D + g) - mc[g]) * __ldcg(base + c * PSZ + i);
        p.out[((int64_t)b * p.Hq + (int64_t)h * G) * D + i] = __float2half_rn(O / lc[g]);
    }
    if (tid == 0) p.counters[bh] = 0;   // nobody arrives on it again in this call
}

// Tiles per warp: the most (up to 8) that still leave at least three CTAs
// per SM of a 148-SM GPU (four fit at once), else one; fewer, longer CTAs
// keep the next tile's copies in flight and write fewer partial results for
// the last arriver to combine.
static void kv4_split(int64_t B, int64_t Hkv, int64_t Tmax, int *splits, int *tpw) {
    const int64_t rounds = (Tmax + kKvRound - 1) / kKvRound;
    int64_t per = 1;
    const int forced = forced_config().kvt;
    if (forced > 0) {
        per = forced;
    } else {
        const int64_t want = 3 * 148;
        for (int64_t t = 2; t <= 8; ++t)
            if (B * Hkv * ((rounds + t - 1) / t) >= want) per = t;
    }
    per = per > rounds ? rounds : per;
    *tpw = (int)per;
    *splits = (int)((rounds + per - 1) / per);
}

size_t kv4_workspace_bytes(int64_t B, int64_t Hkv, int64_t Tmax, int64_t D) {
    int splits, tpw;
    kv4_split(B, Hkv, Tmax, &splits, &tpw);
    const size_t ctl = kKvStatusBytes + (size_t)align256(4 * B * Hkv);
    return ctl + sizeof(float) * (size_t)(B * Hkv * splits) * (size_t)(kKvMaxGroup * D + 2 * kKvMaxGroup);
}

template <int D>
static cudaError_t launch_attn(const Kv4Params &p, dim3 grid, cudaStream_t stream) {
    // Dynamic shared memory: per warp, one 64-token buffer of K codes and one
    // of V codes (8 KB at D = 128), then the warps' P tiles (1 KB each).
    constexpr int TB = kKvTile * D / 2;
    constexpr int smem = kKvWarps * 2 * TB + kKvWarps * kKvTile * 8 * 2;
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [] {
        attr = cudaFuncSetAttribute(kv4_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    smem);
    });
    if (attr != cudaSuccess) return attr;
    kv4_attn_kernel<D><<<grid, kKvThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_kv4_attention(const void *q, const uint8_t *kc, const void *ks, const void *kz, const uint8_t *vc,
                                 const void *vs, const void *vz, const int32_t *seq_lens, int64_t B, int64_t Hq,
                                 int64_t Hkv, int64_t Tmax, int64_t D, void *out, void *ws, cudaStream_t stream) {
    Kv4Params p;
    p.q = static_cast<const __half *>(q);
    p.kc = kc;
    p.ks = static_cast<const __half *>(ks);
    p.kz = static_cast<const __half *>(kz);
    p.vc = vc;
    p.vs = static_cast<const __half *>(vs);
    p.vz = static_cast<const __half *>(vz);
    p.seq_lens = seq_lens;
    p.out = static_cast<__half *>(out);
    p.status = static_cast<int32_t *>(ws);
    p.counters = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + kKvStatusBytes);
    p.part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kKvStatusBytes + align256(4 * B * Hkv));
    p.B = (int)B;
    p.Hq = (int)Hq;
    p.Hkv = (int)Hkv;
    p.Tmax = (int)Tmax;
    p.G = (int)(Hq / Hkv);
    kv4_split(B, Hkv, Tmax, &p.splits, &p.tpw);
    p.qscale = (float)(1.4426950408889634 / sqrt((double)D));
    const dim3 grid((unsigned)p.splits, (unsigned)Hkv, (unsigned)B);
    return D == 128 ? launch_attn<128>(p, grid, stream) : launch_attn<64>(p, grid, stream);
}

}  // namespace qoq
