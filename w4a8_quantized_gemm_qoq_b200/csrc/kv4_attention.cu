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
// Attention (B200 design): the work is HBM-bound (0.53 bytes of cache per
// query-head multiply-add at D = 128, group 4), but the contractions are
// skinny (a group of G <= 8 query heads against a chunk of tokens) and
// unpacking 4-bit codes costs CUDA-core instructions. Each CTA takes one
// (sequence, KV head, 128-token chunk), so K and V are read once for the
// whole query-head group:
//   * its 256 threads load the chunk's K and V codes (8 KB each) and
//     dequantise them to FP16 (c - z, exact integers in [-15, 15]) into
//     padded row-major tiles in shared memory, two codes per 3 instructions
//     (byte permute, and/or with the FP16 exponent of 1024, packed subtract);
//   * scores = (c - z) . q on tensor cores (mma.sync m16n8k16, FP16 inputs,
//     FP32 accumulation; tokens are the MMA rows, the group's heads its
//     columns), then times the token's scale and log2(e)/sqrt(D) in FP32;
//   * the chunk's softmax in FP32 (exp2), and P times the value scale,
//     rounded to FP16, as the A operand of the second product
//     out = (P s) (c - z) on tensor cores (heads as rows, dims as columns);
//   * the chunks of one (sequence, KV head) are combined by the CTA that
//     finishes last (a per-head arrival counter; rescaling by the running
//     maxima), which writes the FP16 output; no second launch, and the
//     counters are left zero for the next call.
// mma.sync is the right tensor-core form here: a 16-row tile covers the
// whole query-head group, and the tensor work is a few percent of the time.
#include <cuda_fp16.h>
#include <stdint.h>

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

constexpr int kKvThreads = 256;   // 8 warps
constexpr int kKvChunk = 128;     // tokens per CTA
constexpr int kKvMaxGroup = 8;    // query heads per KV head

struct Kv4Params {
    const __half *q;
    const uint8_t *kc;
    const __half *ks, *kz;
    const uint8_t *vc;
    const __half *vs, *vz;
    const int32_t *seq_lens;
    __half *out;
    int32_t *counters;   // [B * Hkv], zero between calls
    float *part;         // [B * Hkv][nchunks][kKvMaxGroup * D + 2 * kKvMaxGroup]
    int B, Hq, Hkv, Tmax, G, nchunks;
    float qscale;        // log2(e) / sqrt(D)
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

// D (16x8, FP32) += A (16x16, FP16, row-major) . B (16x8, FP16, column-major).
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16 bytes of codes (32 values of one vector, dims d0 .. d0 + 31) to FP16
// (c - z), written to a shared-memory row: per byte, a byte permute and an
// and/or put the two codes into the mantissas of 1024.0 (FP16 0x6400), and one
// packed subtract of 1024 + z leaves c - z, exact.
__device__ __forceinline__ void dequant16(const uint4 &u, __half2 zz, __half *row) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t lo4 = w[q] & 0x0F0F0F0Fu, hi4 = (w[q] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t sel = (uint32_t)k | ((uint32_t)k << 4) | ((uint32_t)(4 + k) << 8) | ((uint32_t)(4 + k) << 12);
            const uint32_t pair = (__byte_perm(lo4, hi4, sel) & 0x00FF00FFu) | 0x64006400u;
            const __half2 h = __hsub2(*reinterpret_cast<const __half2 *>(&pair), zz);
            o[4 * q + k] = *reinterpret_cast<const uint32_t *>(&h);
        }
    }
    uint4 *dst = reinterpret_cast<uint4 *>(row);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
}

template <int D>
__global__ void __launch_bounds__(kKvThreads) kv4_attn_kernel(const __grid_constant__ Kv4Params p) {
    constexpr int DB = D / 2;             // code bytes per vector
    constexpr int RS = D + 8;             // FP16 row stride of the K/V tiles (conflict-free ldmatrix)
    constexpr int PS = kKvChunk + 8;      // FP16 row stride of the P tile
    constexpr int CPT = kKvChunk * DB / 16 / kKvThreads;   // 16-byte code chunks per thread per tensor
    extern __shared__ __align__(16) uint8_t kv_smem[];
    __half *tile = reinterpret_cast<__half *>(kv_smem);                 // [kKvChunk][RS]: K, then V
    __half *qs = tile + kKvChunk * RS;                                    // [8][RS]
    __half *ps = qs + kKvMaxGroup * RS;                                   // [16][PS]
    __shared__ float sk[kKvChunk], sv[kKvChunk];
    __shared__ float red[8][kKvMaxGroup];
    __shared__ float m_s[kKvMaxGroup], l_s[kKvMaxGroup];
    __shared__ int last_s;

    const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    int T = p.Tmax;
    if (p.seq_lens) T = min(max(p.seq_lens[b], 1), p.Tmax);
    const int nch = (T + kKvChunk - 1) / kKvChunk;
    if (chunk >= nch) return;   // past this sequence's tokens: no work, no arrival
    const int t0 = chunk * kKvChunk;
    const int ntok = min(kKvChunk, T - t0);
    const int64_t bh = (int64_t)b * p.Hkv + h;
    const int64_t slot0 = bh * p.Tmax + t0;
    const int G = p.G;

    // Codes of the chunk: K and V, CPT 16-byte pieces each per thread,
    // loaded at once (V's are dequantised after the scores).
    uint4 kreg[CPT], vreg[CPT];
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int piece = tid + i * kKvThreads;
        const int t = piece / (DB / 16);
        const bool live = t < ntok;
        const uint4 *ksrc = reinterpret_cast<const uint4 *>(p.kc + (slot0 + t) * DB) + piece % (DB / 16);
        const uint4 *vsrc = reinterpret_cast<const uint4 *>(p.vc + (slot0 + t) * DB) + piece % (DB / 16);
        kreg[i] = live ? __ldcs(ksrc) : make_uint4(0u, 0u, 0u, 0u);
        vreg[i] = live ? __ldcs(vsrc) : make_uint4(0u, 0u, 0u, 0u);
    }
    // Scales and zeros of the chunk's tokens (0 past the sequence's end, so
    // that nothing read from unwritten slots reaches the sums).
    __half kz_t = __float2half(0.0f), vz_t = __float2half(0.0f);
    if (tid < kKvChunk) {
        const bool live = tid < ntok;
        sk[tid] = live ? __half2float(p.ks[slot0 + tid]) : 0.0f;
        sv[tid] = live ? __half2float(p.vs[slot0 + tid]) : 0.0f;
    }
    // The group's queries (rows >= G zero) and the P tile's padding rows.
    for (int i = tid; i < kKvMaxGroup * D / 8; i += kKvThreads) {
        const int g = i / (D / 8), c = i % (D / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (g < G) v = *reinterpret_cast<const uint4 *>(p.q + ((int64_t)b * p.Hq + (int64_t)h * G + g) * D + c * 8);
        *reinterpret_cast<uint4 *>(qs + g * RS + c * 8) = v;
    }
    for (int i = tid; i < 16 * PS / 8; i += kKvThreads) reinterpret_cast<uint4 *>(ps)[i] = make_uint4(0u, 0u, 0u, 0u);
    // K: FP16 (c - z) into the tile.
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int piece = tid + i * kKvThreads;
        const int t = piece / (DB / 16);
        if (t < ntok) kz_t = p.kz[slot0 + t];
        const __half zz = __hadd(kz_t, __float2half(1024.0f));
        dequant16(kreg[i], __halves2half2(zz, zz), tile + t * RS + (piece % (DB / 16)) * 32);
    }
    __syncthreads();

    // Scores: warp w takes tokens 16w .. 16w + 15 (the MMA rows), the group's
    // heads are the MMA columns.
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const uint32_t tile_a = smem_u32(tile);
    const uint32_t qs_a = smem_u32(qs);
    if (16 * warp < ntok) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a[4], b0, b1;
            ldsm_x4(tile_a + (uint32_t)(((16 * warp + (lane & 15)) * RS + ks * 16 + (lane >> 4) * 8) * 2), a);
            ldsm_x2(qs_a + (uint32_t)(((lane & 7) * RS + ks * 16 + ((lane >> 3) & 1) * 8) * 2), b0, b1);
            mma_16816(acc, a, b0, b1);
        }
    }
    // acc[0], acc[1]: token 16w + gid, heads 2tig, 2tig + 1; acc[2], acc[3]: token + 8.
    float sc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int t = 16 * warp + gid + (j >> 1) * 8;
        const int g = 2 * tig + (j & 1);
        sc[j] = (t < ntok && g < G) ? acc[j] * sk[t] * p.qscale : -INFINITY;
    }
    // Per-head maximum over the chunk: the two tokens of a thread, the eight
    // token rows of a warp (lanes of equal tig), then the eight warps.
    float mx[2] = {fmaxf(sc[0], sc[2]), fmaxf(sc[1], sc[3])};
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], o));
        mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], o));
    }
    if (gid == 0) {
        red[warp][2 * tig] = mx[0];
        red[warp][2 * tig + 1] = mx[1];
    }
    __syncthreads();
    if (tid < kKvMaxGroup) {
        float m = red[0][tid];
        for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w][tid]);
        m_s[tid] = m;
    }
    __syncthreads();
    float pr[4], sm[2] = {0.0f, 0.0f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int g = 2 * tig + (j & 1);
        pr[j] = sc[j] == -INFINITY ? 0.0f : exp2f(sc[j] - m_s[g]);
        sm[j & 1] += pr[j];
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        sm[0] += __shfl_xor_sync(0xffffffffu, sm[0], o);
        sm[1] += __shfl_xor_sync(0xffffffffu, sm[1], o);
    }
    // P times the value scale, FP16, as the A operand (heads x tokens) of the
    // second product.
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int t = 16 * warp + gid + (j >> 1) * 8;
        const int g = 2 * tig + (j & 1);
        ps[g * PS + t] = __float2half_rn(pr[j] * sv[t]);
    }
    __syncthreads();   // scores done with the K tile; red[] free again
    if (gid == 0) {
        red[warp][2 * tig] = sm[0];
        red[warp][2 * tig + 1] = sm[1];
    }
    // V: FP16 (c - z) into the same tile.
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
        const int piece = tid + i * kKvThreads;
        const int t = piece / (DB / 16);
        if (t < ntok) vz_t = p.vz[slot0 + t];
        const __half zz = __hadd(vz_t, __float2half(1024.0f));
        dequant16(vreg[i], __halves2half2(zz, zz), tile + t * RS + (piece % (DB / 16)) * 32);
    }
    __syncthreads();
    if (tid < kKvMaxGroup) {
        float l = 0.0f;
        for (int w = 0; w < 8; ++w) l += red[w][tid];
        l_s[tid] = l;
    }
    // out = (P s) (c - z): heads are the MMA rows (16, G used), dims the
    // columns (n-tiles of 8 split over the warps), tokens the reduction.
    constexpr int NT = D / 8;             // n-tiles
    constexpr int NTW = NT / 8;           // per warp
    const uint32_t ps_a = smem_u32(ps);
    float o[NTW][4];
#pragma unroll
    for (int j = 0; j < NTW; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
    const int kt_end = (ntok + 15) / 16;
    for (int ks = 0; ks < kt_end; ++ks) {
        uint32_t a[4];
        ldsm_x4(ps_a + (uint32_t)(((lane & 15) * PS + ks * 16 + (lane >> 4) * 8) * 2), a);
#pragma unroll
        for (int j = 0; j < NTW; ++j) {
            const int n0 = (warp * NTW + j) * 8;
            uint32_t b0, b1;
            ldsm_x2_trans(tile_a + (uint32_t)(((ks * 16 + (lane & 15)) * RS + n0) * 2), b0, b1);
            mma_16816(o[j], a, b0, b1);
        }
    }
    __syncthreads();   // l_s ready

    // o[j][0], o[j][1]: head gid, dims n0 + 2tig, + 1 (rows gid + 8 are padding).
    if (p.nchunks == 1 || nch == 1) {
        if (gid < G) {
            const float inv = 1.0f / l_s[gid];
            __half *dst = p.out + ((int64_t)b * p.Hq + (int64_t)h * G + gid) * D;
#pragma unroll
            for (int j = 0; j < NTW; ++j) {
                const int n0 = (warp * NTW + j) * 8 + 2 * tig;
                *reinterpret_cast<__half2 *>(dst + n0) = __floats2half2_rn(o[j][0] * inv, o[j][1] * inv);
            }
        }
        return;
    }
    // Several chunks: store this chunk's unnormalised sums, maxima and
    // weights, arrive, and let the last arriver combine.
    constexpr int PSZ = kKvMaxGroup * D + 2 * kKvMaxGroup;
    float *part = p.part + (bh * p.nchunks + chunk) * PSZ;
    if (gid < G) {
#pragma unroll
        for (int j = 0; j < NTW; ++j) {
            const int n0 = (warp * NTW + j) * 8 + 2 * tig;
            *reinterpret_cast<float2 *>(part + gid * D + n0) = make_float2(o[j][0], o[j][1]);
        }
    }
    if (tid < kKvMaxGroup) {
        part[kKvMaxGroup * D + tid] = m_s[tid];
        part[kKvMaxGroup * D + kKvMaxGroup + tid] = l_s[tid];
    }
    __syncthreads();   // every store of the CTA precedes the arrival (cumulative release)
    if (tid == 0) last_s = atom_add_acq_rel_gpu(p.counters + bh, 1) == nch - 1;
    __syncthreads();
    if (!last_s) return;
    const float *base = p.part + bh * p.nchunks * PSZ;
    for (int i = tid; i < G * D; i += kKvThreads) {
        const int g = i / D, d = i % D;
        float M = -INFINITY;
        for (int c = 0; c < nch; ++c) M = fmaxf(M, __ldcg(base + c * PSZ + kKvMaxGroup * D + g));
        float L = 0.0f, O = 0.0f;
        for (int c = 0; c < nch; ++c) {
            const float w = exp2f(__ldcg(base + c * PSZ + kKvMaxGroup * D + g) - M);
            L += w * __ldcg(base + c * PSZ + kKvMaxGroup * D + kKvMaxGroup + g);
            O += w * __ldcg(base + c * PSZ + g * D + d);
        }
        p.out[((int64_t)b * p.Hq + (int64_t)h * G + g) * D + d] = __float2half_rn(O / L);
    }
    if (tid == 0) p.counters[bh] = 0;   // nobody arrives on it again in this call
}

size_t kv4_workspace_bytes(int64_t B, int64_t Hkv, int64_t Tmax, int64_t D) {
    const int64_t nchunks = (Tmax + kKvChunk - 1) / kKvChunk;
    const size_t ctl = (size_t)align256(4 * B * Hkv);
    return ctl + sizeof(float) * (size_t)(B * Hkv * nchunks) * (size_t)(kKvMaxGroup * D + 2 * kKvMaxGroup);
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
    p.counters = static_cast<int32_t *>(ws);
    p.part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + align256(4 * B * Hkv));
    p.B = (int)B;
    p.Hq = (int)Hq;
    p.Hkv = (int)Hkv;
    p.Tmax = (int)Tmax;
    p.G = (int)(Hq / Hkv);
    p.nchunks = (int)((Tmax + kKvChunk - 1) / kKvChunk);
    p.qscale = (float)(1.4426950408889634 / sqrt((double)D));
    const dim3 grid((unsigned)p.nchunks, (unsigned)Hkv, (unsigned)B);
    // Dynamic shared memory: the K/V tile, the queries and the P tile (41 KB
    // at D = 128, within the default 48 KB).
    if (D == 128) {
        constexpr int smem = (kKvChunk * 136 + kKvMaxGroup * 136 + 16 * (kKvChunk + 8)) * 2;
        kv4_attn_kernel<128><<<grid, kKvThreads, smem, stream>>>(p);
    } else {
        constexpr int smem = (kKvChunk * 72 + kKvMaxGroup * 72 + 16 * (kKvChunk + 8)) * 2;
        kv4_attn_kernel<64><<<grid, kKvThreads, smem, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace qoq
