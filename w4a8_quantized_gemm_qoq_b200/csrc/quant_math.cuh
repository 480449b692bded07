// Exact per-token quantisation arithmetic of the activation quantiser (the
// stand-alone kernel and its form inside the decode GEMM's launch).
#pragma once

#include <cuda_runtime.h>

namespace qoq {

// clamp(RNE(RN32(x / s)), -lim, lim), or 0 when s == 0, given inv = RN32(1/s)
// (0 for s = +inf), without a division in the common case: q = RN32(x * inv)
// is within |x/s| * 2^-23 (+ 2^-149) of x/s, and RN32(x/s) within half an ulp
// of it, so for |q| < 2^12 the two sit within 2^-11 of each other; unless q
// lies within 2^-10 of a half-integer both round to the same integer, and
// beyond 2^12 both clamp the same way. Near a half-integer the correctly
// rounded quotient is computed.
__device__ __forceinline__ int quant_code_recip(float x, float s, float inv, int lim) {
    if (s == 0.0f) return 0;
    const float q = __fmul_rn(x, inv);
    const float fr = __fsub_rn(q, floorf(q));
    const float qq = fabsf(__fsub_rn(fr, 0.5f)) > 0.0009765625f ? q : __fdiv_rn(x, s);
    return max(-lim, min(lim, __float2int_rn(qq)));
}

}  // namespace qoq
