// Activation quantisation (per token) and offline weight quantisation +
// packing for the QoQ W4A8 GEMM.
//
// QServe: W4A8KV4 Quantization and System Co-design for Efficient LLM Serving
// (arXiv 2405.04532), paperlayer.ai summary:
//   section 4 "Progressive Group Quantization" -- per-channel INT8 with FP16
//     scales in the protective range [-119, 119], then per-group 4-bit codes
//     with scale and zero point;
//   section 5 -- compute-aware weight reordering (weights stored in the order
//     the GEMM consumes them);
//   section 6 -- per-token INT8 activations, g128 and per-channel variants.
// Every floating-point decision is a single correctly rounded binary32
// operation (__fdiv_rn, __float2int_rn), no contraction.
#include <cuda_fp16.h>

#include "qoq_device.cuh"
#include "qoq_internal.h"
#include "quant_math.cuh"

namespace qoq {

// ------------------------------------------------------------ activations


__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ int quant_code(float x, float s, int lim) {
    if (s == 0.0f) return 0;
    int q = __float2int_rn(__fdiv_rn(x, s));
    return max(-lim, min(lim, q));
}

// One CTA per token row: absmax (warp shuffles, then across warps), FP16
// scale, then round-half-even codes and their row sum. NCH > 0 keeps the row
// in registers (NCH 16-byte chunks per thread, one pass over HBM); NCH == 0
// reads the row twice (any K).
template <int NCH, int TH>
__global__ void __launch_bounds__(TH) act_quant_kernel(const __half *__restrict__ X, int K,
                                                                 int8_t *__restrict__ X8,
                                                                 __half *__restrict__ s_x,
                                                                 int32_t *__restrict__ rowsum) {
    __shared__ float red_f[TH / 32];
    __shared__ int red_i[TH / 32];
    __shared__ float s_shared, inv_shared;
    // X may come from the previous kernel in the stream; release the next one
    // (the GEMM) so its set-up and weight copies overlap this kernel.
    griddep_wait();
    griddep_launch_dependents();
    const int64_t m = blockIdx.x;
    const __half *row = X + m * K;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int NR = NCH > 0 ? NCH : 1;

    uint4 v[NR];
    float amax = 0.0f;
    // The eight halves of a 16-byte chunk are taken apart with shifts only:
    // no local has its address taken, so the kernel keeps no stack frame.
    auto absmax8 = [&](const uint4 &u) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float lo = __half2float(__ushort_as_half((unsigned short)(w[i] & 0xFFFFu)));
            const float hi = __half2float(__ushort_as_half((unsigned short)(w[i] >> 16)));
            amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
        }
    };
    if (NCH > 0) {
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            const int k = (i * TH + threadIdx.x) * 8;
            // The load address is clamped into the row, so no form of the
            // guard can read past the end of X; out-of-row chunks become 0.
            const uint4 u = *reinterpret_cast<const uint4 *>(row + (k < K ? k : K - 8));
            v[i] = k < K ? u : make_uint4(0u, 0u, 0u, 0u);
            absmax8(v[i]);
        }
    } else {
        for (int k = threadIdx.x * 8; k < K; k += TH * 8) absmax8(*reinterpret_cast<const uint4 *>(row + k));
    }
    amax = warp_max(amax);
    if (lane == 0) red_f[warp] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float a = red_f[0];
        for (int w = 1; w < TH / 32; ++w) a = fmaxf(a, red_f[w]);
        __half sh = __float2half_rn(__fdiv_rn(a, 127.0f));
        s_x[m] = sh;
        s_shared = __half2float(sh);
        inv_shared = __frcp_rn(__half2float(sh));
    }
    __syncthreads();
    const float s = s_shared, inv = inv_shared;

    int sum = 0;
    int8_t *out = X8 + m * K;
    auto quant8 = [&](const uint4 &u, int k) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
        uint32_t packed0 = 0u, packed1 = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float lo = __half2float(__ushort_as_half((unsigned short)(w[i] & 0xFFFFu)));
            const float hi = __half2float(__ushort_as_half((unsigned short)(w[i] >> 16)));
            const int q0 = quant_code_recip(lo, s, inv, 127), q1 = quant_code_recip(hi, s, inv, 127);
            sum += q0 + q1;
            const uint32_t pair = ((uint32_t)(q0 & 0xFF) | ((uint32_t)(q1 & 0xFF) << 8)) << (16 * (i & 1));
            if (i < 2)
                packed0 |= pair;
            else
                packed1 |= pair;
        }
        *reinterpret_cast<uint2 *>(out + k) = make_uint2(packed0, packed1);
    };
    if (NCH > 0) {
#pragma unroll
        for (int i = 0; i < NR; ++i) {
            const int k = (i * TH + threadIdx.x) * 8;
            if (k < K) quant8(v[i], k);
        }
    } else {
        for (int k = threadIdx.x * 8; k < K; k += TH * 8) quant8(*reinterpret_cast<const uint4 *>(row + k), k);
    }
    if (rowsum != nullptr) {
        sum = warp_sum(sum);
        if (lane == 0) red_i[warp] = sum;
        __syncthreads();
        if (threadIdx.x == 0) {
            int t = 0;
            for (int w = 0; w < TH / 32; ++w) t += red_i[w];
            rowsum[m] = t;
        }
    }
}

template <int NCH, int TH>
static cudaError_t launch_act_quant_t(const void *X, int64_t M, int64_t K, int8_t *X8, void *s_x,
                                      int32_t *rowsum, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)M);
    cfg.blockDim = dim3(TH);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = kProgrammaticLaunch ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, act_quant_kernel<NCH, TH>, static_cast<const __half *>(X), (int)K, X8,
                              static_cast<__half *>(s_x), rowsum);
}

template <int TH>
static cudaError_t launch_act_quant_th(const void *X, int64_t M, int64_t K, int8_t *X8, void *s_x, int32_t *rowsum,
                                       bool two_pass, cudaStream_t stream) {
    const int64_t per_pass = (int64_t)TH * 8;   // halves one pass of the CTA covers
    const int64_t nch = (K + per_pass - 1) / per_pass;
    if (two_pass) return launch_act_quant_t<0, TH>(X, M, K, X8, s_x, rowsum, stream);
    if (nch <= 1) return launch_act_quant_t<1, TH>(X, M, K, X8, s_x, rowsum, stream);
    if (nch <= 2) return launch_act_quant_t<2, TH>(X, M, K, X8, s_x, rowsum, stream);
    if (nch <= 4) return launch_act_quant_t<4, TH>(X, M, K, X8, s_x, rowsum, stream);
    if (nch <= 8) return launch_act_quant_t<8, TH>(X, M, K, X8, s_x, rowsum, stream);
    if (nch <= 12) return launch_act_quant_t<12, TH>(X, M, K, X8, s_x, rowsum, stream);
    return launch_act_quant_t<0, TH>(X, M, K, X8, s_x, rowsum, stream);
}

// CTA size and form by shape, from B200 measurements on the Llama-3-8B rows
// (K = 4096 and 14336, M = 16 .. 16384): a few rows want the most threads per
// row (the row's latency is the launch's); many rows want the most rows in
// flight per SM, i.e. few registers per thread (the two-pass form reads each
// row twice, the second time from L1/L2, and keeps nothing in registers).
// Same arithmetic in every form.
cudaError_t launch_act_quant(const void *X, int64_t M, int64_t K, int8_t *X8, void *s_x, int32_t *rowsum,
                             cudaStream_t stream) {
    int th;
    bool two_pass;
    if (M <= 256) {
        th = 512, two_pass = false;
    } else if (K > 4096) {
        th = 256, two_pass = true;
    } else if (M <= 4096) {
        th = 256, two_pass = false;
    } else {
        th = 128, two_pass = true;
    }
    if (forced_config().aqt) th = forced_config().aqt;
    if (forced_config().aq2) two_pass = forced_config().aq2 == 1;
    if (th == 128) return launch_act_quant_th<128>(X, M, K, X8, s_x, rowsum, two_pass, stream);
    if (th == 512) return launch_act_quant_th<512>(X, M, K, X8, s_x, rowsum, two_pass, stream);
    return launch_act_quant_th<256>(X, M, K, X8, s_x, rowsum, two_pass, stream);
}

// ---------------------------------------------------------------- weights

// Round half to even of a / b for integers, b > 0 (exact integer arithmetic).
__device__ __forceinline__ int div_rne(int a, int b) {
    int q = a / b, r = a % b;
    if (r < 0) {  // C truncates toward zero: move to floor division
        q -= 1;
        r += b;
    }
    if (2 * r > b || (2 * r == b && (q & 1))) q += 1;
    return q;
}

struct WeightQuantParams {
    const __half *W;
    uint8_t *blob;
    int N, K, group;
    int64_t block, off_codes, off_scale, off_zero, total;
};

// Per output channel: the level-1 FP16 scale (group mode) or the per-channel
// UINT4 scale and zero (group 0). One warp per row. CTA 0 also writes the
// header and zero-fills the alignment padding after the scale sections.
__global__ void __launch_bounds__(256) weight_rows_kernel(WeightQuantParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = blockIdx.x * 8 + warp;
    if (blockIdx.x == 0) {
        uint32_t *h32 = reinterpret_cast<uint32_t *>(p.blob);
        for (int i = threadIdx.x; i < kHeaderBytes / 4; i += blockDim.x) h32[i] = 0u;
        __syncthreads();
        if (threadIdx.x == 0) {
            h32[0] = kMagic;
            h32[1] = kVersion;
            h32[2] = (uint32_t)p.N;
            h32[3] = (uint32_t)p.K;
            h32[4] = (uint32_t)p.group;
            h32[5] = (uint32_t)p.block;
            uint64_t *h64 = reinterpret_cast<uint64_t *>(p.blob + 24);
            h64[0] = (uint64_t)p.off_codes;
            h64[1] = (uint64_t)p.off_scale;
            h64[2] = (uint64_t)p.off_zero;
            h64[3] = (uint64_t)p.total;
        }
        const int64_t pad0 = p.off_scale + 2 * (int64_t)p.N;
        const int64_t end0 = p.group ? p.total : p.off_zero;
        for (int64_t i = pad0 + threadIdx.x; i < end0; i += blockDim.x) p.blob[i] = 0;
        if (!p.group) {
            for (int64_t i = p.off_zero + 2 * (int64_t)p.N + threadIdx.x; i < p.total; i += blockDim.x)
                p.blob[i] = 0;
        }
    }
    if (n >= p.N) return;
    const __half *row = p.W + (int64_t)n * p.K;
    float amax = 0.0f, wmin = 0.0f, wmax = 0.0f;
    for (int k = lane * 8; k < p.K; k += 32 * 8) {
        uint4 v = *reinterpret_cast<const uint4 *>(row + k);
        const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __half22float2(h[i]);
            amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
            wmin = fminf(wmin, fminf(f.x, f.y));
            wmax = fmaxf(wmax, fmaxf(f.x, f.y));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        wmin = fminf(wmin, __shfl_xor_sync(0xffffffffu, wmin, o));
        wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
    }
    if (lane != 0) return;
    __half *scale = reinterpret_cast<__half *>(p.blob + p.off_scale);
    if (p.group) {
        scale[n] = __float2half_rn(__fdiv_rn(amax, 119.0f));
    } else {
        // wmin <= 0 <= wmax: the range always includes zero.
        __half sh = __float2half_rn(__fdiv_rn(__fsub_rn(wmax, wmin), 15.0f));
        float s = __half2float(sh);
        int z = (s == 0.0f) ? 0 : __float2int_rn(__fdiv_rn(-wmin, s));
        scale[n] = sh;
        reinterpret_cast<__half *>(p.blob + p.off_zero)[n] = __int2half_rn(z);
    }
}

// One CTA of 128 threads per (n-tile, k-tile) block; thread r owns row
// nt*128 + r of that block (= one quantisation group in group mode) and
// writes its four 16-byte code chunks and its (s, z*s) pair in compute order.
__global__ void __launch_bounds__(128) weight_pack_kernel(WeightQuantParams p) {
    const int r = threadIdx.x;
    const int nt = blockIdx.x, kt = blockIdx.y;
    const int KT = p.K / kTileK;
    const int n = nt * kTileN + r;
    const __half *src = p.W + (int64_t)n * p.K + (int64_t)kt * kTileK;
    uint8_t *blk = p.blob + p.off_codes + ((int64_t)nt * KT + kt) * p.block;

    const float sc = __half2float(reinterpret_cast<const __half *>(p.blob + p.off_scale)[n]);
    // Level-1 codes (group mode) or per-channel UINT4 codes, 4 per word.
    uint32_t w8[32];
    int vmin = 127, vmax = -128;
    int zpc = 0;
    if (!p.group) zpc = __half2int_rn(reinterpret_cast<const __half *>(p.blob + p.off_zero)[n]);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        uint4 v = *reinterpret_cast<const uint4 *>(src + c * 8);
        const __half2 *h = reinterpret_cast<const __half2 *>(&v);
        uint32_t lo = 0u, hi = 0u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __half22float2(h[i]);
            int a, b;
            if (p.group) {
                a = quant_code(f.x, sc, 119);
                b = quant_code(f.y, sc, 119);
                vmin = min(vmin, min(a, b));
                vmax = max(vmax, max(a, b));
            } else {
                a = (sc == 0.0f) ? 0 : max(0, min(15, __float2int_rn(__fdiv_rn(f.x, sc)) + zpc));
                b = (sc == 0.0f) ? 0 : max(0, min(15, __float2int_rn(__fdiv_rn(f.y, sc)) + zpc));
            }
            uint32_t pair = ((uint32_t)(a & 0xFF)) | ((uint32_t)(b & 0xFF) << 8);
            if (i < 2) lo |= pair << (16 * i);
            else hi |= pair << (16 * (i - 2));
        }
        w8[2 * c] = lo;
        w8[2 * c + 1] = hi;
    }

    int s = 1, zs = 0, z = 0;
    if (p.group) {
        // s = max(1, RNE((vmax - vmin) / 15)); 15 is odd so the quotient is
        // never a tie and rounding half up is round-half-even.
        s = max(1, (2 * (vmax - vmin) + 15) / 30);
        z = div_rne(-vmin, s);
        zs = z * s;
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t lo4 = w8[8 * c + 2 * j], hi4 = w8[8 * c + 2 * j + 1];
            uint32_t word = 0u;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                int vl = (int)(int8_t)((lo4 >> (8 * b)) & 0xFF);
                int vh = (int)(int8_t)((hi4 >> (8 * b)) & 0xFF);
                int ql, qh;
                if (p.group) {
                    ql = max(0, min(15, div_rne(vl, s) + z));
                    qh = max(0, min(15, div_rne(vh, s) + z));
                } else {
                    ql = vl;
                    qh = vh;
                }
                word |= (uint32_t)(ql | (qh << 4)) << (8 * b);
            }
            out[j] = word;
        }
        *reinterpret_cast<uint4 *>(blk + c * 2048 + r * 16) = make_uint4(out[0], out[1], out[2], out[3]);
    }
    if (p.group) {
        const uint16_t pair = (uint16_t)((uint32_t)s | ((uint32_t)(zs & 0xFF) << 8));
        *reinterpret_cast<uint16_t *>(blk + 8192 + 2 * r) = pair;
    }
}

cudaError_t launch_weight_quant(const void *W, int64_t N, int64_t K, int group, void *blob,
                                const BlobLayout &L, cudaStream_t stream) {
    WeightQuantParams p;
    p.W = static_cast<const __half *>(W);
    p.blob = static_cast<uint8_t *>(blob);
    p.N = (int)N;
    p.K = (int)K;
    p.group = group;
    p.block = L.block;
    p.off_codes = L.off_codes;
    p.off_scale = L.off_scale;
    p.off_zero = L.off_zero;
    p.total = L.total;
    weight_rows_kernel<<<(unsigned)((N + 7) / 8), 256, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)L.NT, (unsigned)L.KT);
    weight_pack_kernel<<<grid, 128, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace qoq
