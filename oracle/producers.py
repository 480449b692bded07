"""Plain CPU reference of the fused activation producers -- TEST INFRASTRUCTURE.

Only tests, the smoke check and the benchmark's CPU arms use this.

The QServe pages fuse per-token activation quantisation into the layer that
produces the GEMM's input: the preceding normalisation, or the activation
function (paperlayer.ai summary, section 5 "QServe Serving System", bullet
"Runtime and precision mapping"). They give neither layer's formula nor its
precision. The readings taken here (each named in a docstring):

  * RMSNorm (the normalisation of Llama-family models): h = (x / r) * gamma
    with r = sqrt(mean_k x^2 + eps). The sum of squares is the exact real sum
    (every x^2 of an FP16 x is exact, the sum is formed without rounding)
    rounded once to FP32; every later step is one correctly rounded FP32
    operation. The exact sum makes the result independent of summation order.
  * SiLU-gated product (the FFN activation): h = (g / (1 + e^-g)) * u for the
    gate half g and the up half u of the merged gate/up projection output.
    e^x is the function `exp_f32` below: Cody and Waite's two-constant
    argument reduction x = n ln2 + r, |r| <= ln2/2, the degree-7 Taylor
    polynomial of e^r by Horner's rule, and an exact scaling by 2^n, all in
    FP32 one operation at a time. It is within 2 ulp of e^x (checked against
    binary64 in the tests); both sides of the parity check evaluate this same
    function, so the codes it decides agree bit for bit.
  * The FP32 rows h are quantised per token exactly like the FP16 activations
    of the GEMM path: s = FP16(max_k |h| / 127), codes = clamp(RNE(h / FP32(s)),
    -127, 127), 0 where s == 0, and the int32 row sum of the codes. There is
    no FP16 rounding of h in between (the point of the fusion).
"""
from __future__ import annotations

import numpy as np

from .qoq_ref import F32, X8_RANGE, fp16

# ---------------------------------------------------------------------------
# FP32 rounding of an exact scaled integer
# ---------------------------------------------------------------------------


def rn32_from_int(S: int, shift: int) -> np.float32:
    """S * 2^-shift (S a non-negative Python integer) rounded to the nearest
    binary32, ties to even. Normal results only (callers keep the range)."""
    S = int(S)
    if S == 0:
        return F32(0.0)
    nb = S.bit_length()
    drop = nb - 24
    if drop <= 0:
        m, e = S, -shift
    else:
        m = S >> drop
        rem = S - (m << drop)
        half = 1 << (drop - 1)
        if rem > half or (rem == half and (m & 1)):
            m += 1
            if m == 1 << 24:
                m >>= 1
                drop += 1
        e = drop - shift
    return F32(np.ldexp(np.float64(m), e))


def fp16_scaled_int(x16: np.ndarray) -> np.ndarray:
    """|x| * 2^24 for FP16 x, an exact integer below 2^40 (int64)."""
    return (np.abs(np.asarray(x16, dtype=np.float16).astype(np.float64)) * float(1 << 24)).astype(np.int64)


def exact_sum_of_squares(x16: np.ndarray) -> list:
    """Per row, the exact sum of x^2 times 2^48 as a Python integer.

    Each v = |x| * 2^24 is split as v = a * 2^20 + b (a, b < 2^20) so that the
    three partial sums of a^2, a*b and b^2 stay exact in int64 for rows of up
    to 2^15 elements."""
    v = fp16_scaled_int(x16)
    a, b = v >> 20, v & ((1 << 20) - 1)
    A = (a * a).sum(axis=-1)
    B = (a * b).sum(axis=-1)
    C = (b * b).sum(axis=-1)
    return [(int(A[i]) << 40) + (int(B[i]) << 21) + int(C[i]) for i in range(v.shape[0])]


# ---------------------------------------------------------------------------
# e^x in FP32 (Cody-Waite reduction + Taylor polynomial)
# ---------------------------------------------------------------------------

EXP_LOG2E = F32(1.4426950408889634)      # FP32(log2 e)
EXP_LN2_HI = F32(0.693145751953125)      # ln 2 with its last 8 bits zero: n * LN2_HI is exact for |n| < 2^8
EXP_LN2_LO = F32(1.4286067653301870e-06)  # FP32(ln 2 - LN2_HI)
EXP_X_OVER = F32(88.72283935546875)      # above: +inf (e^x > FLT_MAX)
EXP_X_UNDER = F32(-87.33654022216797)    # below: 0 (e^x < FLT_MIN, flushed)
# 1/k! for k = 7 .. 0, rounded to FP32
EXP_TAYLOR = [F32(1.0 / 5040.0), F32(1.0 / 720.0), F32(1.0 / 120.0), F32(1.0 / 24.0), F32(1.0 / 6.0), F32(0.5),
              F32(1.0), F32(1.0)]


def _pow2_f32(k: np.ndarray) -> np.ndarray:
    """2^k as FP32 for integer k in [-126, 127] (exact)."""
    return np.ldexp(np.ones(k.shape, dtype=np.float32), k.astype(np.int32)).astype(F32)


def exp_f32(x) -> np.ndarray:
    """e^x for FP32 x, each step one correctly rounded FP32 operation:
    n = RNE(x * log2e); r = (x - n*LN2_HI) - n*LN2_LO; p = Taylor_7(r) by
    Horner; e^x = (p * 2^floor(n/2)) * 2^(n - floor(n/2)). x > EXP_X_OVER gives
    +inf, x < EXP_X_UNDER gives 0."""
    x = np.asarray(x, dtype=F32)
    xc = np.clip(x, EXP_X_UNDER, EXP_X_OVER).astype(F32)
    n = np.rint((xc * EXP_LOG2E).astype(F32)).astype(F32)
    r = ((xc - (n * EXP_LN2_HI).astype(F32)).astype(F32) - (n * EXP_LN2_LO).astype(F32)).astype(F32)
    p = np.full(x.shape, EXP_TAYLOR[0], dtype=F32)
    for c in EXP_TAYLOR[1:]:
        p = ((p * r).astype(F32) + c).astype(F32)
    ni = n.astype(np.int32)
    na = ni >> 1
    nb = ni - na
    with np.errstate(over="ignore"):
        y = ((p * _pow2_f32(na)).astype(F32) * _pow2_f32(nb)).astype(F32)
    y = np.where(x > EXP_X_OVER, F32(np.inf), y)
    y = np.where(x < EXP_X_UNDER, F32(0.0), y)
    return y.astype(F32)


# ---------------------------------------------------------------------------
# Per-token quantisation of FP32 rows (the GEMM's activation format)
# ---------------------------------------------------------------------------


def quantize_rows_f32(H: np.ndarray):
    """s[m] = FP16(max_k |H[m,k]| / 127); X8 = clamp(RNE(H / FP32(s)), -127,
    127), 0 where s == 0; rowsum = sum_k X8 (int32). Same arithmetic as the
    FP16 activation quantiser, on FP32 rows (reading: no FP16 rounding of the
    producer's output before it is quantised)."""
    H = np.asarray(H, dtype=F32)
    amax = np.abs(H).max(axis=1)
    s_x = fp16((amax / F32(X8_RANGE)).astype(F32))
    s32 = s_x.astype(F32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (H / s32).astype(F32)
    X8 = np.where(s32 == 0, F32(0), np.clip(np.rint(q), -X8_RANGE, X8_RANGE)).astype(np.int8)
    X8 = np.where(np.isnan(q), 0, X8).astype(np.int8)
    rowsum = X8.astype(np.int64).sum(axis=1).astype(np.int32)
    return X8, s_x, rowsum


# ---------------------------------------------------------------------------
# The two producers
# ---------------------------------------------------------------------------


def rmsnorm_f32(X: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm rows in FP32 (reading above):
    ss = RN32(exact sum_k x^2); ms = ss / K; r = sqrt(ms + eps);
    h = (x / r) * gamma, each an FP32 operation."""
    X16 = np.asarray(X, dtype=np.float16)
    M, K = X16.shape
    ss = np.array([rn32_from_int(S, 48) for S in exact_sum_of_squares(X16)], dtype=F32)
    ms = (ss / F32(K)).astype(F32)
    r = np.sqrt((ms + F32(eps)).astype(F32)).astype(F32)
    x32 = X16.astype(F32)
    g32 = np.asarray(gamma, dtype=np.float16).astype(F32)[None, :]
    return ((x32 / r[:, None]).astype(F32) * g32).astype(F32)


def rmsnorm_quant(X: np.ndarray, gamma: np.ndarray, eps: float):
    """Fused RMSNorm + per-token INT8 quantisation: X8 [M][K], s_x FP16 [M],
    rowsum int32 [M]."""
    return quantize_rows_f32(rmsnorm_f32(X, gamma, eps))


def silu_mul_f32(GU: np.ndarray) -> np.ndarray:
    """h = (g / (1 + exp_f32(-g))) * u per element, FP32, for GU = [gate | up]
    along the last axis (FP16 [M][2I])."""
    GU16 = np.asarray(GU, dtype=np.float16)
    I = GU16.shape[1] // 2
    g = GU16[:, :I].astype(F32)
    u = GU16[:, I:].astype(F32)
    e = exp_f32(-g)
    den = (F32(1.0) + e).astype(F32)
    with np.errstate(divide="ignore", invalid="ignore"):
        sg = (g / den).astype(F32)
    return (sg * u).astype(F32)


def silu_mul_quant(GU: np.ndarray):
    """Fused SiLU(gate) * up + per-token INT8 quantisation: X8 [M][I], s_x FP16
    [M], rowsum int32 [M]."""
    return quantize_rows_f32(silu_mul_f32(GU))
