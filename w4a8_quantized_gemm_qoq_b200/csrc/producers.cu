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
// correctly rounded binary32 operation (__fdiv_rn, __fsqrt_rn, ...; the
// quantising division takes the exact reciprocal shortcut of quant_math.cuh;
// no contraction), the sum of squares is exact (128-bit integer accumulation,
// then one rounding), and e^x is computed here from Cody and Waite's argument
// reduction and the degree-7 Taylor polynomial, so that the codes these
// floating-point values decide are reproducible bit for bit.
//
// B200 layout: one 256-thread CTA per token row (memory-bound: each row is
// read once from HBM and written once as INT8). Thread t owns the 8-element
// chunks t, t+256, ...; the FP32 row h lives in shared memory between the
// passes, element i of chunk c at h[i * K/8 + c] so that a warp's accesses
// fall in distinct banks (each thread reads back only its own chunks).
#include <cuda_fp16.h>

#include "qoq_device.cuh"
#include "qoq_internal.h"
#include "quant_math.cuh"

namespace qoq {

namespace {

constexpr int kProdThreads = 256;

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

// |x| * 2^24 of an FP16 x (an integer below 2^40).
__device__ __forceinline__ unsigned long long fp16_scaled(uint32_t bits) {
    const uint32_t e = (bits >> 10) & 0x1Fu, f = bits & 0x3FFu;
    return e ? (unsigned long long)(0x400u | f) << (e - 1) : (unsigned long long)f;
}

__device__ __forceinline__ void add_square(U128 &acc, uint32_t bits16) {
    const unsigned long long v = fp16_scaled(bits16);
    add128(acc, U128{v * v, __umul64hi(v, v)});
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

// ------------------------------------------------------ block reductions

__device__ __forceinline__ U128 block_sum128(U128 v, U128 *red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        U128 w;
        w.lo = __shfl_xor_sync(0xffffffffu, v.lo, o);
        w.hi = __shfl_xor_sync(0xffffffffu, v.hi, o);
        add128(v, w);
    }
    if (lane == 0) red[warp] = v;
    __syncthreads();
    U128 t = red[0];
    for (int w = 1; w < kProdThreads / 32; ++w) add128(t, red[w]);
    return t;   // every thread gets the same exact sum
}

__device__ __forceinline__ float block_max(float v, float *red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float t = red[0];
    for (int w = 1; w < kProdThreads / 32; ++w) t = fmaxf(t, red[w]);
    return t;
}

__device__ __forceinline__ int block_sum(int v, int *red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int t = 0;
    for (int w = 0; w < kProdThreads / 32; ++w) t += red[w];
    return t;
}

__device__ __forceinline__ float half_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFFu))); }
__device__ __forceinline__ float half_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }

// Quantise the FP32 row h (shared memory, element i of chunk c at
// h[i * K/8 + c]; this thread's chunks) and write the codes, the scale and the
// row sum of token m.
__device__ __forceinline__ void quantize_row(const float *h, int K, float amax_row, int64_t m, int8_t *X8,
                                             __half *s_x, int32_t *rowsum, int *red_i) {
    __shared__ float s_shared, inv_shared;
    if (threadIdx.x == 0) {
        const __half sh = __float2half_rn(__fdiv_rn(amax_row, 127.0f));
        s_x[m] = sh;
        s_shared = __half2float(sh);
        inv_shared = __frcp_rn(__half2float(sh));
    }
    __syncthreads();
    const float s = s_shared, inv = inv_shared;
    const int nc = K / 8;
    int8_t *out = X8 + m * K;
    int sum = 0;
    for (int c = threadIdx.x; c * 8 < K; c += kProdThreads) {
        uint32_t packed[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int q = quant_code_recip(h[i * nc + c], s, inv, 127);
            sum += q;
            packed[i >> 2] |= (uint32_t)(q & 0xFF) << (8 * (i & 3));
        }
        *reinterpret_cast<uint2 *>(out + c * 8) = make_uint2(packed[0], packed[1]);
    }
    if (rowsum != nullptr) {
        const int t = block_sum(sum, red_i);
        if (threadIdx.x == 0) rowsum[m] = t;
    }
}

}  // namespace

// --------------------------------------------------------------- kernels

__global__ void __launch_bounds__(kProdThreads) rmsnorm_quant_kernel(const __half *__restrict__ X,
                                                                     const __half *__restrict__ gamma, int K,
                                                                     float eps, int8_t *__restrict__ X8,
                                                                     __half *__restrict__ s_x,
                                                                     int32_t *__restrict__ rowsum) {
    extern __shared__ float h[];   // [K]
    __shared__ U128 red128[kProdThreads / 32];
    __shared__ float red_f[kProdThreads / 32];
    __shared__ int red_i[kProdThreads / 32];
    __shared__ float r_shared;
    griddep_wait();
    griddep_launch_dependents();
    const int64_t m = blockIdx.x;
    const __half *row = X + m * K;
    const int nc = K / 8;   // chunks per row; element i of chunk c sits at h[i * nc + c] (no bank conflicts)

    // Pass 1: the row's exact sum of squares; keep x (FP32) in shared memory.
    U128 acc{0ull, 0ull};
    for (int c = threadIdx.x; c * 8 < K; c += kProdThreads) {
        const uint4 u = *reinterpret_cast<const uint4 *>(row + c * 8);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            add_square(acc, w[i] & 0xFFFFu);
            add_square(acc, w[i] >> 16);
            h[(2 * i) * nc + c] = half_lo(w[i]);
            h[(2 * i + 1) * nc + c] = half_hi(w[i]);
        }
    }
    const U128 S = block_sum128(acc, red128);
    if (threadIdx.x == 0) {
        const float ss = rn32_scaled(S);
        const float ms = __fdiv_rn(ss, (float)K);
        r_shared = __fsqrt_rn(__fadd_rn(ms, eps));
    }
    __syncthreads();
    const float r = r_shared;

    // Pass 2: h = (x / r) * gamma in place, and the row's max |h|.
    float amax = 0.0f;
    for (int c = threadIdx.x; c * 8 < K; c += kProdThreads) {
        const uint4 gu = *reinterpret_cast<const uint4 *>(gamma + c * 8);
        const uint32_t g[4] = {gu.x, gu.y, gu.z, gu.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float h0 = __fmul_rn(__fdiv_rn(h[(2 * i) * nc + c], r), half_lo(g[i]));
            const float h1 = __fmul_rn(__fdiv_rn(h[(2 * i + 1) * nc + c], r), half_hi(g[i]));
            h[(2 * i) * nc + c] = h0;
            h[(2 * i + 1) * nc + c] = h1;
            amax = fmaxf(amax, fmaxf(fabsf(h0), fabsf(h1)));
        }
    }
    amax = block_max(amax, red_f);
    quantize_row(h, K, amax, m, X8, s_x, rowsum, red_i);
}

__global__ void __launch_bounds__(kProdThreads) silu_mul_quant_kernel(const __half *__restrict__ GU, int I,
                                                                      int8_t *__restrict__ X8,
                                                                      __half *__restrict__ s_x,
                                                                      int32_t *__restrict__ rowsum) {
    extern __shared__ float h[];   // [I]
    __shared__ float red_f[kProdThreads / 32];
    __shared__ int red_i[kProdThreads / 32];
    griddep_wait();
    griddep_launch_dependents();
    const int64_t m = blockIdx.x;
    const int nc = I / 8;   // chunks per row; element i of chunk c sits at h[i * nc + c]
    const __half *gate = GU + m * 2 * (int64_t)I;
    const __half *up = gate + I;
    float amax = 0.0f;
    for (int c = threadIdx.x; c * 8 < I; c += kProdThreads) {
        const uint4 gv = *reinterpret_cast<const uint4 *>(gate + c * 8);
        const uint4 uv = *reinterpret_cast<const uint4 *>(up + c * 8);
        const uint32_t g[4] = {gv.x, gv.y, gv.z, gv.w};
        const uint32_t u[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const float gf = j ? half_hi(g[i]) : half_lo(g[i]);
                const float uf = j ? half_hi(u[i]) : half_lo(u[i]);
                const float e = exp_cw(-gf);
                const float sg = __fdiv_rn(gf, __fadd_rn(1.0f, e));
                const float hv = __fmul_rn(sg, uf);
                h[(2 * i + j) * nc + c] = hv;
                amax = fmaxf(amax, fabsf(hv));
            }
        }
    }
    amax = block_max(amax, red_f);
    quantize_row(h, I, amax, m, X8, s_x, rowsum, red_i);
}

namespace {

template <typename Kernel, typename... Args>
cudaError_t launch_row_kernel(Kernel kernel, int64_t M, int width, cudaStream_t stream, Args... args) {
    const size_t smem = (size_t)width * sizeof(float);
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (smem > 48 * 1024) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)M);
    cfg.blockDim = dim3(kProdThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = kProgrammaticLaunch ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace

cudaError_t launch_rmsnorm_quant(const void *X, const void *gamma, int64_t M, int64_t K, float eps, int8_t *X8,
                                 void *s_x, int32_t *rowsum, cudaStream_t stream) {
    return launch_row_kernel(rmsnorm_quant_kernel, M, (int)K, stream, static_cast<const __half *>(X),
                             static_cast<const __half *>(gamma), (int)K, eps, X8, static_cast<__half *>(s_x),
                             rowsum);
}

cudaError_t launch_silu_mul_quant(const void *GU, int64_t M, int64_t I, int8_t *X8, void *s_x, int32_t *rowsum,
                                  cudaStream_t stream) {
    return launch_row_kernel(silu_mul_quant_kernel, M, (int)I, stream, static_cast<const __half *>(GU), (int)I, X8,
                             static_cast<__half *>(s_x), rowsum);
}

}  // namespace qoq
