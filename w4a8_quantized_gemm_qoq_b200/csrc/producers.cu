// Fused activation producers: the layer in front of a W4A8 GEMM writes the
// GEMM's per-token INT8 activations (codes, FP16 scale, row sum) directly,
// instead of an FP16 tensor that a separate quantiser reads again.
//
// QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM Serving
// (arXiv 2405.04532), paperlayer.ai summary, section 5 "QServe Serving
// System", "Runtime and precision mapping": activation quantisation is fused
// into the preceding normalisation or activation layer. The pages give neither
// layer's arithmetic; this file computes, per token row:
//   RMSNorm:        ss = FP32(exact sum_k x^2); ms = ss / K; r = sqrt(ms + eps);
//                   h_k = (x_k / r) * gamma_k
//   SiLU-gated:     h_k = (g_k / (1 + e^-g_k)) * u_k   (gate | up halves of a row)
// then s = FP16(max_k |h| / 127), X8 = clamp(RNE(h / FP32(s)), -127, 127)
// (0 where s == 0) and rowsum = sum_k X8. Every floating-point step is one
// correctly rounded binary32 operation (no contraction), the sum of squares is
// exact (integer accumulation, then one rounding), and e^x is computed here
// from Cody and Waite's argument reduction and the degree-7 Taylor polynomial,
// so that the codes these floating-point values decide are reproducible bit
// for bit.
//
// The two divisions whose divisor is fixed for the whole row, x / r and
// h / s, are formed without a division instruction: with y = RN(1/b) (one
// correctly rounded reciprocal per row), q0 = RN(a * y), the residual
// a - b * q0 (exact in one FMA) and q = RN(q0 + residual * y) (one FMA).
// Markstein's theorem (P. Markstein, IBM J. Res. Dev. 34(1), 1990; also
// Muller et al., Handbook of Floating-Point Arithmetic, the section on
// division with an FMA) states that q is then the correctly rounded quotient
// whenever y is the correctly rounded reciprocal, q0 lies within one ulp of
// a / b and nothing overflows or underflows; both hold for every operand
// these kernels form (FP16 or bounded FP32 numerators, divisors in the normal
// range). The quotient's integer code is taken with the 1.5 * 2^23 addition,
// which rounds to nearest even exactly for |q| <= 2^22, after the clamp to
// [-127, 127]; the low byte of the sum's bit pattern is then the code.
//
// B200 layout: the row stays in registers from its load to its codes. Rows of
// up to 4096 elements (RMSNorm) or 2048 (SiLU-gated) belong to one warp each,
// four rows per CTA, and every reduction is a warp shuffle; wider rows belong
// to a CTA of 256 or 512 threads, with one shared-memory step per reduction.
// Thread t of a row owns the 8-element chunks t, t + T, t + 2T, ... (T the
// row's threads), so that every load of a chunk (16 bytes per thread) and
// every store of its codes (8 bytes) is coalesced across the warp.
#include <cuda_fp16.h>

#include "qoq_device.cuh"
#include "qoq_internal.h"

namespace qoq {

namespace {

constexpr int kWarpRows = 4;   // rows per CTA when a warp owns a row

// Threads per row (TPR), and rows and threads per CTA.
template <int TPR>
struct RowCta {
    static_assert(TPR == 32 || TPR == 256 || TPR == 512 || TPR == 1024, "row shapes");
    static constexpr int kRows = TPR == 32 ? kWarpRows : 1;
    static constexpr int kThreads = TPR * kRows;
    static constexpr int kWarps = TPR / 32;   // warps of one row
    static_assert(kWarps * 32 == TPR, "whole warps");
};

// ------------------------------------------------------------------ e^x

__device__ __forceinline__ float pow2_f32(int k) {   // 2^k, k in [-126, 127]
    return __int_as_float((k + 127) << 23);
}

// e^x in binary32: n = RNE(x * FP32(log2 e)); r = (x - n*LN2_HI) - n*LN2_LO
// (Cody-Waite: LN2_HI carries ln 2 to 16 bits so n*LN2_HI is exact); the
// Taylor polynomial sum_{k<=7} r^k / k! by Horner's rule with FP32(1/k!);
// then an exact scaling by 2^n in two factors. Outside
// [-87.33654, 88.72284] the result is 0 or +inf.
__device__ __forceinline__ float exp_cw(float x) {
    const float kOver = __int_as_float(0x42b17218);    // 88.72283935546875
    const float kUnder = __int_as_float(0xc2aeac4f);   // -87.33654022216797
    if (x > kOver) return __int_as_float(0x7f800000);
    if (x < kUnder) return 0.0f;
    const float kLog2e = __int_as_float(0x3fb8aa3b);
    const float kLn2Hi = __int_as_float(0x3f317200);
    const float kLn2Lo = __int_as_float(0x35bfbe8e);
    const float n = rintf(__fmul_rn(x, kLog2e));
    const float r = __fsub_rn(__fsub_rn(x, __fmul_rn(n, kLn2Hi)), __fmul_rn(n, kLn2Lo));
    float p = __int_as_float(0x39500d01);                    // 1/5040
    p = __fadd_rn(__fmul_rn(p, r), __int_as_float(0x3ab60b61));   // 1/720
    p = __fadd_rn(__fmul_rn(p, r), __int_as_float(0x3c088889));   // 1/120
    p = __fadd_rn(__fmul_rn(p, r), __int_as_float(0x3d2aaaab));   // 1/24
    p = __fadd_rn(__fmul_rn(p, r), __int_as_float(0x3e2aaaab));   // 1/6
    p = __fadd_rn(__fmul_rn(p, r), 0.5f);
    p = __fadd_rn(__fmul_rn(p, r), 1.0f);
    p = __fadd_rn(__fmul_rn(p, r), 1.0f);
    const int ni = (int)n;
    const int na = ni >> 1;
    return __fmul_rn(__fmul_rn(p, pow2_f32(na)), pow2_f32(ni - na));
}

// ------------------------------------------------------ exact sum of squares

struct U128 {
    unsigned long long lo, hi;
};

__device__ __forceinline__ void add128(U128 &a, const U128 &b) {
    const unsigned long long lo = a.lo + b.lo;
    a.hi += b.hi + (lo < a.lo ? 1ull : 0ull);
    a.lo = lo;
}


// S * 2^-48 rounded to binary32, ties to even. Every S formed here is 0 or at
// least 1, so the result is 0 or normal.
__device__ __forceinline__ float rn32_scaled(U128 S) {
    if (S.hi == 0 && S.lo == 0) return 0.0f;
    const int nb = S.hi ? 128 - __clzll((long long)S.hi) : 64 - __clzll((long long)S.lo);
    int drop = nb - 24;   // bits below the 24-bit significand
    unsigned long long m;
    if (drop <= 0) {
        m = S.lo;
        drop = 0;
    } else {
        // m = S >> drop (it fits 24 bits)
        m = drop >= 64 ? S.hi >> (drop - 64) : (S.lo >> drop) | (S.hi << (64 - drop));
        // the dropped bits, shifted up so that the first of them is bit 127
        const int k = 128 - drop;   // in [24, 127]
        unsigned long long dh, dl;
        if (k >= 64) {
            dh = S.lo << (k - 64);
            dl = 0ull;
        } else {
            dh = (S.hi << k) | (S.lo >> (64 - k));
            dl = S.lo << k;
        }
        const unsigned long long half = 1ull << 63;
        const bool above = dh > half || (dh == half && dl != 0ull);
        const bool tie = dh == half && dl == 0ull;
        if (above || (tie && (m & 1ull))) {
            ++m;
            if (m == (1ull << 24)) {
                m >>= 1;
                ++drop;
            }
        }
    }
    // m < 2^24 is exact in FP32; 2^(drop - 48) is an exact power of two in the
    // normal range (drop - 48 lies in [-48, 57] for S < 2^106).
    return __fmul_rn(__uint2float_rn((unsigned)m), pow2_f32(drop - 48));
}


// The exact squares of both FP16 halves of w, added to two 64-bit
// accumulators. |x| * 2^24 = m << s with m the 11-bit significand (hidden bit
// included for normal numbers) and s = max(e - 1, 0) for the exponent field e;
// a square with s < 15 is added to a0 as (m << s)^2 = x^2 * 2^48, the others to
// a1 as (m << (s - 15))^2 = x^2 * 2^48 / 2^30. Every such square is below 2^50
// (2^52 for the infinity and NaN patterns), so a thread's 128 elements at
// most, and a warp's 32 threads' sums, stay below 2^64 for finite inputs.
__device__ __forceinline__ void add_squares(uint32_t w, unsigned long long &a0, unsigned long long &a1) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const uint32_t h = k ? w >> 16 : w & 0xFFFFu;
        const uint32_t e = (h >> 10) & 31u;
        const uint32_t f = h & 0x3FFu;
        const uint32_t m = e ? (f | 0x400u) : f;
        const uint32_t s = e ? e - 1u : 0u;
        const bool up = s >= 15u;
        const uint32_t v = m << (up ? s - 15u : s);
        const unsigned long long sq = (unsigned long long)v * v;
        if (up)
            a1 += sq;
        else
            a0 += sq;
    }
}

// a / b correctly rounded, given y = RN(1/b) (Markstein's correction; the
// conditions are stated at the top of this file).
__device__ __forceinline__ float div_by_recip(float a, float b, float y) {
    const float q0 = __fmul_rn(a, y);
    const float res = __fmaf_rn(-q0, b, a);
    return __fmaf_rn(res, y, q0);
}

__device__ __forceinline__ float half_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu))); }
__device__ __forceinline__ float half_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }
__device__ __forceinline__ uint32_t word_at(const uint4 &u, int i) {   // i = 0..3
    return i < 2 ? (i == 0 ? u.x : u.y) : (i == 2 ? u.z : u.w);
}

// ------------------------------------------------------ row reductions
//
// Over the TPR threads of one row; every thread receives the result. A warp
// row reduces with shuffles alone; a CTA row adds one shared-memory exchange
// (each reduction has its own array, so no barrier guards a reuse).

struct RowRed {
    U128 sq[32];
    float mx[32];
    int sum[32];
};

template <int TPR>
__device__ __forceinline__ U128 row_sum_squares(unsigned long long a0, unsigned long long a1, RowRed &red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a0 += __shfl_xor_sync(0xffffffffu, a0, o);
        a1 += __shfl_xor_sync(0xffffffffu, a1, o);
    }
    // S = a0 + a1 * 2^30
    U128 S{a0, 0ull};
    add128(S, U128{a1 << 30, a1 >> 34});
    if constexpr (TPR > 32) {
        const int warp = threadIdx.x >> 5;
        if ((threadIdx.x & 31) == 0) red.sq[warp] = S;
        __syncthreads();
        S = red.sq[0];
#pragma unroll
        for (int w = 1; w < RowCta<TPR>::kWarps; ++w) add128(S, red.sq[w]);
    }
    return S;
}

template <int TPR>
__device__ __forceinline__ float row_max(float v, RowRed &red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if constexpr (TPR > 32) {
        const int warp = threadIdx.x >> 5;
        if ((threadIdx.x & 31) == 0) red.mx[warp] = v;
        __syncthreads();
        v = red.mx[0];
#pragma unroll
        for (int w = 1; w < RowCta<TPR>::kWarps; ++w) v = fmaxf(v, red.mx[w]);
    }
    return v;
}

template <int TPR>
__device__ __forceinline__ int row_sum(int v, RowRed &red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if constexpr (TPR > 32) {
        const int warp = threadIdx.x >> 5;
        if ((threadIdx.x & 31) == 0) red.sum[warp] = v;
        __syncthreads();
        v = 0;
#pragma unroll
        for (int w = 0; w < RowCta<TPR>::kWarps; ++w) v += red.sum[w];
    }
    return v;
}

// ------------------------------------------------------ quantisation

// Code byte of the quotient q, rounded to nearest even through the 1.5 * 2^23
// addition: the low byte of the sum's pattern is the code. kClamp first
// clamps q to [-127, 127]. Without it q must already lie below 127.5 in
// magnitude, which holds whenever the row's scale is a normal FP16 number: s is
// max|h| / 127 rounded to FP32 and then to FP16, with relative errors of at most
// 2^-24 and 2^-11, so |h / s| <= 127 / ((1 - 2^-24)(1 - 2^-11)) < 127.1.
template <bool kClamp>
__device__ __forceinline__ uint32_t code_bits(float q) {
    if constexpr (kClamp) q = fminf(fmaxf(q, -127.0f), 127.0f);
    return __float_as_uint(__fadd_rn(q, 12582912.0f));
}

// Bytes 0 of a, b, c, d as one word (a in the lowest byte).
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
}

// Codes of one chunk c (8 FP32 values h) to out[c]; returns their sum.
template <bool kClamp>
__device__ __forceinline__ int code_chunk(const float (&h)[8], float s, float y, uint2 *out, int c) {
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = code_bits<kClamp>(div_by_recip(h[i], s, y));
    const uint32_t lo = pack_low_bytes(b[0], b[1], b[2], b[3]);
    const uint32_t hi = pack_low_bytes(b[4], b[5], b[6], b[7]);
    out[c] = make_uint2(lo, hi);
    return __dp4a((int)hi, 0x01010101, __dp4a((int)lo, 0x01010101, 0));
}

// Codes of this thread's chunks: chunk j is the row's chunk c = t + TPR * j,
// valid when below nc, and row_chunk(j, c, h) yields its 8 FP32 values.
// CPT == 0: a loop over c unrolled twice, and row_chunk gets j = -1 (the
// row's values come from memory, not from per-thread arrays).
// Returns this thread's sum of the codes.
template <int TPR, int CPT, bool kClamp, typename RowChunk>
__device__ __forceinline__ int store_codes(RowChunk &row_chunk, int t, int nc, float s, float y, uint2 *out) {
    int sum = 0;
    if constexpr (CPT == 0) {
#pragma unroll 2
        for (int c = t; c < nc; c += TPR) {
            float h[8];
            row_chunk(-1, c, h);
            sum += code_chunk<kClamp>(h, s, y, out, c);
        }
    } else {
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const int c = t + TPR * j;
            if (c < nc) {
                float h[8];
                row_chunk(j, c, h);
                sum += code_chunk<kClamp>(h, s, y, out, c);
            }
        }
    }
    return sum;
}

// Quantise the FP32 row h (this thread's max |h| in amax; row_chunk as in
// store_codes) and write its codes, scale and code sum.
template <int TPR, int CPT, typename RowChunk>
__device__ __forceinline__ void quantize_row(RowChunk row_chunk, float amax, int t, int nc, int64_t m,
                                             int64_t width, int8_t *__restrict__ X8, __half *__restrict__ s_x,
                                             int32_t *__restrict__ rowsum, RowRed &red) {
    amax = row_max<TPR>(amax, red);
    const __half sh = __float2half_rn(__fdiv_rn(amax, 127.0f));
    float s = __half2float(sh);
    float y = __frcp_rn(s);
    if (!(s > 0.0f) || isinf(s)) {
        // s == 0: every code is 0 by definition; s == inf: every h / s is
        // 0. The substitute divisor 1 with reciprocal 0 gives q = 0 below.
        s = 1.0f;
        y = 0.0f;
    }
    uint2 *out = reinterpret_cast<uint2 *>(X8 + m * width);
    int sum = s >= 6.103515625e-05f   // 2^-14, the smallest normal FP16
                  ? store_codes<TPR, CPT, false>(row_chunk, t, nc, s, y, out)
                  : store_codes<TPR, CPT, true>(row_chunk, t, nc, s, y, out);
    if (rowsum != nullptr) sum = row_sum<TPR>(sum, red);
    if (t == 0) {
        s_x[m] = sh;
        if (rowsum != nullptr) rowsum[m] = sum;
    }
}

// 16-byte asynchronous copy global -> shared (both 16-byte aligned), and the
// wait for all of this thread's copies (a hardware wait, no polling).
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// h = (x / r) * gamma for the 8 elements of one chunk (yr = RN(1/r)).
__device__ __forceinline__ void rms_chunk(const uint4 &xv, const uint4 &gv, float r, float yr, float (&h)[8]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t xw = word_at(xv, i), gw = word_at(gv, i);
        h[2 * i] = __fmul_rn(div_by_recip(half_lo(xw), r, yr), half_lo(gw));
        h[2 * i + 1] = __fmul_rn(div_by_recip(half_hi(xw), r, yr), half_hi(gw));
    }
}

}  // namespace

// --------------------------------------------------------------- kernels

// Launch bounds: CTAs per SM the register budget must allow.
template <int TPR, int CPT, bool kWide>
constexpr int row_min_blocks() {
    if constexpr (TPR == 32) return kWide ? 3 : (CPT >= 16 ? 5 : 4);   // kWide: 128 FP32 values kept per thread
    return TPR == 256 ? 2 : 1;
}

// kKeepH: the normalised row stays in registers between its max and its
// codes; otherwise it is formed a second time for the codes (fewer registers,
// more CTAs per SM).
template <int TPR, int CPT, bool kKeepH>
__global__ void __launch_bounds__(RowCta<TPR>::kThreads, (row_min_blocks<TPR, CPT, kKeepH && CPT >= 16>()))
    rmsnorm_quant_kernel(const __half *__restrict__ X, const __half *__restrict__ gamma, int64_t M, int K,
                         float eps, int8_t *__restrict__ X8, __half *__restrict__ s_x,
                         int32_t *__restrict__ rowsum) {
    __shared__ RowRed red;
    griddep_wait();
    griddep_launch_dependents();
    const int t = threadIdx.x % TPR;
    const int64_t m = (int64_t)blockIdx.x * RowCta<TPR>::kRows + threadIdx.x / TPR;
    if (m >= M) return;   // warp rows only: a CTA row always exists
    const int nc = K >> 3;
    const uint4 *row = reinterpret_cast<const uint4 *>(X + m * K);
    const uint4 *g4 = reinterpret_cast<const uint4 *>(gamma);

    uint4 xv[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = t + TPR * j;
        xv[j] = c < nc ? row[c] : make_uint4(0u, 0u, 0u, 0u);
    }
    // The row's exact sum of squares (zero chunks add nothing).
    unsigned long long a0 = 0ull, a1 = 0ull;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
#pragma unroll
        for (int i = 0; i < 4; ++i) add_squares(word_at(xv[j], i), a0, a1);
    }
    const U128 S = row_sum_squares<TPR>(a0, a1, red);
    const float r = __fsqrt_rn(__fadd_rn(__fdiv_rn(rn32_scaled(S), (float)K), eps));
    const float yr = __frcp_rn(r);

    // h = (x / r) * gamma and the row's max |h|.
    float hk[kKeepH ? CPT : 1][8];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = t + TPR * j;
        if (c < nc) {
            float h[8];
            rms_chunk(xv[j], __ldg(g4 + c), r, yr, h);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                amax = fmaxf(amax, fabsf(h[i]));
                if constexpr (kKeepH) hk[j][i] = h[i];
            }
        }
    }
    auto row_chunk = [&](int j, int c, float (&h)[8]) {
        if constexpr (kKeepH) {
#pragma unroll
            for (int i = 0; i < 8; ++i) h[i] = hk[j][i];
        } else {
            rms_chunk(xv[j], __ldg(g4 + c), r, yr, h);
        }
    };
    quantize_row<TPR, CPT>(row_chunk, amax, t, nc, m, K, X8, s_x, rowsum, red);
}

// RMSNorm rows of up to 4096 elements staged in shared memory (K * 2 bytes
// per warp): one warp per row, four rows per CTA. Each lane copies its own
// chunks in and reads back only those, so no barrier is needed; the three
// passes over the row (squares, max, codes) are loops unrolled twice, which
// keeps the kernel's body small, and the normalised row is formed again for
// its codes instead of being kept.
__global__ void __launch_bounds__(kWarpRows * 32, 7)
    rmsnorm_quant_srow_kernel(const __half *__restrict__ X, const __half *__restrict__ gamma, int64_t M, int K,
                              float eps, int8_t *__restrict__ X8, __half *__restrict__ s_x,
                              int32_t *__restrict__ rowsum) {
    extern __shared__ uint4 srow[];   // [kWarpRows][K / 8]
    __shared__ RowRed red;            // unused by warp rows
    griddep_wait();
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t m = (int64_t)blockIdx.x * kWarpRows + warp;
    if (m >= M) return;
    const int nc = K >> 3;
    uint4 *xs = srow + (size_t)warp * nc;
    const uint4 *row = reinterpret_cast<const uint4 *>(X + m * K);
    const uint4 *g4 = reinterpret_cast<const uint4 *>(gamma);
    for (int c = lane; c < nc; c += 32) cp_async16(xs + c, row + c);
    cp_async_wait_all();

    unsigned long long a0 = 0ull, a1 = 0ull;
#pragma unroll 2
    for (int c = lane; c < nc; c += 32) {
        const uint4 v = xs[c];
#pragma unroll
        for (int i = 0; i < 4; ++i) add_squares(word_at(v, i), a0, a1);
    }
    const U128 S = row_sum_squares<32>(a0, a1, red);
    const float r = __fsqrt_rn(__fadd_rn(__fdiv_rn(rn32_scaled(S), (float)K), eps));
    const float yr = __frcp_rn(r);

    float amax = 0.0f;
#pragma unroll 2
    for (int c = lane; c < nc; c += 32) {
        float h[8];
        rms_chunk(xs[c], __ldg(g4 + c), r, yr, h);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(h[i]));
    }
    auto row_chunk = [&](int, int c, float (&h)[8]) { rms_chunk(xs[c], __ldg(g4 + c), r, yr, h); };
    quantize_row<32, 0>(row_chunk, amax, lane, nc, m, K, X8, s_x, rowsum, red);
}

template <int TPR, int CPT>
__global__ void __launch_bounds__(RowCta<TPR>::kThreads, (row_min_blocks<TPR, CPT, false>()))
    silu_mul_quant_kernel(const __half *__restrict__ GU, int64_t M, int I, int8_t *__restrict__ X8,
                          __half *__restrict__ s_x, int32_t *__restrict__ rowsum) {
    __shared__ RowRed red;
    griddep_wait();
    griddep_launch_dependents();
    const int t = threadIdx.x % TPR;
    const int64_t m = (int64_t)blockIdx.x * RowCta<TPR>::kRows + threadIdx.x / TPR;
    if (m >= M) return;   // warp rows only: a CTA row always exists
    const int nc = I >> 3;
    const uint4 *gate = reinterpret_cast<const uint4 *>(GU + m * 2 * (int64_t)I);
    const uint4 *up = gate + nc;

    uint4 gv[CPT], uv[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
        const int c = t + TPR * j;
        gv[j] = c < nc ? gate[c] : make_uint4(0u, 0u, 0u, 0u);
        uv[j] = c < nc ? up[c] : make_uint4(0u, 0u, 0u, 0u);
    }
    // h = (g / (1 + e^-g)) * u and the row's max |h| (zero chunks give 0).
    float hk[CPT][8];
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t gw = word_at(gv[j], i >> 1), uw = word_at(uv[j], i >> 1);
            const float gf = (i & 1) ? half_hi(gw) : half_lo(gw);
            const float uf = (i & 1) ? half_hi(uw) : half_lo(uw);
            const float sg = __fdiv_rn(gf, __fadd_rn(1.0f, exp_cw(-gf)));
            hk[j][i] = __fmul_rn(sg, uf);
            amax = fmaxf(amax, fabsf(hk[j][i]));
        }
    }
    auto row_chunk = [&](int j, int, float (&h)[8]) {
#pragma unroll
        for (int i = 0; i < 8; ++i) h[i] = hk[j][i];
    };
    quantize_row<TPR, CPT>(row_chunk, amax, t, nc, m, I, X8, s_x, rowsum, red);
}

namespace {

template <typename... KArgs, typename... Args>
cudaError_t launch_rows_smem(void (*kernel)(KArgs...), int tpr, int64_t M, size_t smem, cudaStream_t stream,
                             Args... args) {
    const int rows = tpr == 32 ? kWarpRows : 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((M + rows - 1) / rows));
    cfg.blockDim = dim3((unsigned)(tpr * rows));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = kProgrammaticLaunch ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_rows(void (*kernel)(KArgs...), int tpr, int64_t M, cudaStream_t stream, Args... args) {
    return launch_rows_smem(kernel, tpr, M, 0, stream, args...);
}

}  // namespace

// Row shapes by the number of 8-element chunks nc: a warp per row up to 512
// chunks (RMSNorm) or 256 (SiLU-gated, which holds gate and up), then CTA rows
// of 256 to 1024 threads with at most 8 chunks per thread (4096 chunks =
// kMaxProducerWidth at most).
cudaError_t launch_rmsnorm_quant(const void *X, const void *gamma, int64_t M, int64_t K, float eps, int8_t *X8,
                                 void *s_x, int32_t *rowsum, cudaStream_t stream) {
    const int nc = (int)(K / 8);
    const auto *x = static_cast<const __half *>(X);
    const auto *g = static_cast<const __half *>(gamma);
    auto *s = static_cast<__half *>(s_x);
    const int prs = forced_config().prs;
    const bool keep = prs != 2;
    if (prs == 3 && nc <= 512)   // at most 32 KB of shared memory per CTA
        return launch_rows_smem(rmsnorm_quant_srow_kernel, 32, M, (size_t)kWarpRows * K * 2, stream, x, g, M,
                                (int)K, eps, X8, s, rowsum);
#define QOQ_RMS(TPR, CPT, KEEP) \
    launch_rows(rmsnorm_quant_kernel<TPR, CPT, KEEP>, TPR, M, stream, x, g, M, (int)K, eps, X8, s, rowsum)
    if (nc <= 64) return keep ? QOQ_RMS(32, 2, true) : QOQ_RMS(32, 2, false);
    if (nc <= 128) return keep ? QOQ_RMS(32, 4, true) : QOQ_RMS(32, 4, false);
    if (nc <= 256) return keep ? QOQ_RMS(32, 8, true) : QOQ_RMS(32, 8, false);
    if (nc <= 512) return keep ? QOQ_RMS(32, 16, true) : QOQ_RMS(32, 16, false);
    if (nc <= 1024) return QOQ_RMS(256, 4, true);
    if (nc <= 2048) return QOQ_RMS(256, 8, true);
    return QOQ_RMS(512, 8, true);
#undef QOQ_RMS
}

cudaError_t launch_silu_mul_quant(const void *GU, int64_t M, int64_t I, int8_t *X8, void *s_x, int32_t *rowsum,
                                  cudaStream_t stream) {
    const int nc = (int)(I / 8);
    const auto *gu = static_cast<const __half *>(GU);
    auto *s = static_cast<__half *>(s_x);
    const bool wide = forced_config().pst == 2;
#define QOQ_SILU(TPR, CPT) launch_rows(silu_mul_quant_kernel<TPR, CPT>, TPR, M, stream, gu, M, (int)I, X8, s, rowsum)
    if (nc <= 64) return QOQ_SILU(32, 2);
    if (nc <= 128) return QOQ_SILU(32, 4);
    if (nc <= 256) return QOQ_SILU(32, 8);
    if (nc <= 512) return QOQ_SILU(256, 2);
    if (nc <= 1024) return QOQ_SILU(256, 4);
    if (nc <= 2048) return wide ? QOQ_SILU(512, 4) : QOQ_SILU(256, 8);
    return wide ? QOQ_SILU(1024, 4) : QOQ_SILU(512, 8);
#undef QOQ_SILU
}

}  // namespace qoq
