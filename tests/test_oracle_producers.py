"""Pins for the oracle's fused activation producers (RMSNorm / SiLU-gated
product, then per-token INT8 quantisation), against things other than the
oracle itself: binary64 e^x, exact rational arithmetic (``fractions``) step by
step, and closed forms. The fusion itself is stated in the paperlayer.ai
summary of QServe, section 5, "Runtime and precision mapping"; the formulas
are the readings written in ``oracle/producers.py``.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from exact import fp16 as ex_fp16, fp32 as ex_fp32, frac, INF
from oracle import producers as P

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _ordered(a):
    b = np.asarray(a, dtype=np.float32).view(np.int32).astype(np.int64)
    return np.where(b < 0, -(b & 0x7FFFFFFF), b)


# ------------------------------------------------------------------ e^x

def test_exp_within_two_ulp_of_binary64():
    rng = np.random.default_rng(7)
    x = np.concatenate([np.linspace(-87.3, 88.7, 400_001), rng.uniform(-87.3, 88.7, 200_000),
                        rng.uniform(-1, 1, 100_000)]).astype(np.float32)
    y = P.exp_f32(x)
    ref = np.exp(x.astype(np.float64)).astype(np.float32)   # binary64 e^x rounded once to binary32
    ok = np.isfinite(ref) & (ref >= np.float32(1.1754944e-38))
    d = np.abs(_ordered(y[ok]) - _ordered(ref[ok]))
    assert d.max() <= 2, int(d.max())


def test_exp_special_values():
    assert P.exp_f32(np.float32(0.0)) == np.float32(1.0)
    assert np.isinf(P.exp_f32(np.float32(88.75))) and P.exp_f32(np.float32(88.75)) > 0
    assert P.exp_f32(np.float32(65504.0)) == np.float32(np.inf)
    assert P.exp_f32(np.float32(-88.0)) == 0.0
    assert P.exp_f32(np.float32(-65504.0)) == 0.0
    # monotone on a dense grid
    x = np.linspace(-80, 80, 200_001).astype(np.float32)
    y = P.exp_f32(x)
    assert np.all(np.diff(y.astype(np.float64)) >= 0)


def test_exp_steps_match_exact_rational_evaluation():
    """Every FP32 step of exp_f32, redone with exact rationals rounded to
    binary32 by tests/exact.py, gives the same bits."""
    rng = np.random.default_rng(3)
    xs = np.concatenate([rng.uniform(-87, 88, 300), [0.0, 1.0, -1.0, 0.5, 10.0, -10.0, 88.7, -87.3]]).astype(np.float32)
    taylor = [frac(c) for c in P.EXP_TAYLOR]
    for x in xs:
        X = frac(x)
        t = ex_fp32(X * frac(P.EXP_LOG2E))
        n = round(t)                                   # RNE of a representable value
        r = ex_fp32(ex_fp32(X - ex_fp32(n * frac(P.EXP_LN2_HI))) - ex_fp32(n * frac(P.EXP_LN2_LO)))
        p = taylor[0]
        for c in taylor[1:]:
            p = ex_fp32(ex_fp32(p * r) + c)
        na = n >> 1
        nb = n - na
        y = ex_fp32(ex_fp32(p * Fraction(2) ** na) * Fraction(2) ** nb)
        got = P.exp_f32(x)
        assert (float(y) if y not in (INF, -INF) else y) == float(got), (x, float(y), float(got))


# ------------------------------------------------------- exact sum rounding

def test_rn32_from_int_matches_exact_rounding():
    rng = np.random.default_rng(11)
    vals = [int(v) for v in rng.integers(1, 1 << 62, 2000, dtype=np.int64)]
    vals += [int(a) << int(b) for a, b in zip(rng.integers(1, 1 << 60, 500, dtype=np.int64), rng.integers(0, 35, 500))]
    # exact ties: (2^24 + odd or even mantissa) plus half a unit below it
    for m in (1 << 23, (1 << 23) + 1, (1 << 24) - 1, 12345677, 12345678):
        for k in (1, 5, 30):
            vals.append((m << k) + (1 << (k - 1)))
            vals.append((m << k) + (1 << (k - 1)) - 1)
            vals.append((m << k) + (1 << (k - 1)) + 1)
    for S in vals:
        want = ex_fp32(Fraction(S, 1 << 48))
        assert float(P.rn32_from_int(S, 48)) == float(want), S


def test_exact_sum_of_squares_is_exact():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal((3, 777)) * 30, rng.standard_normal((2, 777)) * 1e-4]).astype(np.float16)
    x[0, :5] = [65504, -65504, 6e-8, -6e-8, 0]
    got = P.exact_sum_of_squares(x)
    for i in range(x.shape[0]):
        want = sum(frac(v) ** 2 for v in x[i]) * (1 << 48)
        assert want.denominator == 1 and got[i] == want.numerator


# ------------------------------------------------------------- RMSNorm

def _sqrt32(q: Fraction) -> Fraction:
    """Correctly rounded binary32 square root of a positive rational."""
    c = np.float32(math.sqrt(float(q)))
    cands = sorted({float(c), float(np.nextafter(c, np.float32(0))), float(np.nextafter(c, np.float32(np.inf)))})
    best = None
    for v in cands:
        d = abs(Fraction(v) ** 2 - q)   # monotone in |v - sqrt(q)| near the root
        if best is None or d < best[0] or (d == best[0] and (np.float32(v).view(np.uint32) & 1) == 0):
            best = (d, v)
    # decide between the two neighbours bracketing sqrt(q) exactly via the midpoint
    v = best[1]
    lo = float(np.nextafter(np.float32(v), np.float32(0)))
    hi = float(np.nextafter(np.float32(v), np.float32(np.inf)))
    mid_lo = (Fraction(lo) + Fraction(v)) / 2
    mid_hi = (Fraction(v) + Fraction(hi)) / 2
    if q < mid_lo ** 2:
        v = lo
    elif q > mid_hi ** 2:
        v = hi
    return Fraction(v)


def _rmsnorm_exact(x16, g16, eps):
    K = x16.shape[0]
    ss = ex_fp32(sum(frac(v) ** 2 for v in x16))
    ms = ex_fp32(ss / K)
    r = _sqrt32(ex_fp32(ms + frac(np.float32(eps))))
    return [ex_fp32(ex_fp32(frac(v) / r) * frac(g)) for v, g in zip(x16, g16)]


def _quant_exact(h):
    amax = max(abs(v) for v in h)
    s = ex_fp16(ex_fp32(amax / 127))
    if s == 0:
        return [0] * len(h), s
    codes = []
    for v in h:
        q = ex_fp32(v / s)
        codes.append(int(max(-127, min(127, round(q)))))
    return codes, s


def test_rmsnorm_quant_matches_exact_rational_steps():
    rng = np.random.default_rng(21)
    for K in (8, 16, 24, 40):
        for trial in range(6):
            x = (rng.standard_normal(K) * (10.0 ** rng.uniform(-3, 2))).astype(np.float16)
            if trial == 1:
                x[rng.integers(K)] *= np.float16(20)
            g = (1 + 0.1 * rng.standard_normal(K)).astype(np.float16)
            eps = [1e-5, 1e-6, 0.5][trial % 3]
            h = P.rmsnorm_f32(x[None, :], g, eps)[0]
            want_h = _rmsnorm_exact(x, g, eps)
            assert [float(v) for v in h] == [float(v) for v in want_h], (K, trial)
            X8, s_x, rs = P.rmsnorm_quant(x[None, :], g, eps)
            codes, s = _quant_exact(want_h)
            assert float(s_x[0]) == float(s)
            assert X8[0].tolist() == codes and int(rs[0]) == sum(codes)


@pytest.mark.parametrize("c", [1.0, -3.5, 0.0078125, 300.0])
def test_rmsnorm_constant_row_closed_form(c):
    """x = c everywhere, gamma = 1: h = c / sqrt(c^2 + eps) ~ sign(c) * (1 - tiny),
    so every code is sign(c) * 127."""
    K = 4096
    x = np.full((1, K), c, dtype=np.float16)
    X8, s_x, rs = P.rmsnorm_quant(x, np.ones(K, dtype=np.float16), 1e-5)
    sgn = 1 if c > 0 else -1
    assert np.all(X8 == sgn * 127) and int(rs[0]) == sgn * 127 * K


def test_rmsnorm_one_hot_and_zero_rows():
    K = 1024
    x = np.zeros((3, K), dtype=np.float16)
    x[0, 17] = 5.0
    x[1, 1000] = -0.25
    g = np.ones(K, dtype=np.float16)
    X8, s_x, rs = P.rmsnorm_quant(x, g, 1e-6)
    assert X8[0, 17] == 127 and np.count_nonzero(X8[0]) == 1 and rs[0] == 127
    assert X8[1, 1000] == -127 and np.count_nonzero(X8[1]) == 1 and rs[1] == -127
    assert np.all(X8[2] == 0) and s_x[2] == 0 and rs[2] == 0
    # gamma = 0 gives zero rows whatever x is
    X8, s_x, rs = P.rmsnorm_quant(np.full((1, K), 2.0, dtype=np.float16), np.zeros(K, dtype=np.float16), 1e-5)
    assert np.all(X8 == 0) and s_x[0] == 0


def test_rmsnorm_close_to_binary64_definition():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((4, 4096)) * 2).astype(np.float16)
    g = (1 + 0.2 * rng.standard_normal(4096)).astype(np.float16)
    h = P.rmsnorm_f32(x, g, 1e-5)
    x64 = x.astype(np.float64)
    ref = x64 / np.sqrt((x64 ** 2).mean(axis=1, keepdims=True) + 1e-5) * g.astype(np.float64)
    rel = np.abs(h - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rel.max() < 4 * 2.0 ** -23


# ------------------------------------------------------ SiLU-gated product

def _silu_mul_exact(g16, u16):
    out = []
    for g, u in zip(g16, u16):
        e = P.exp_f32(np.float32(-np.float32(g)))       # the defined primitive
        E = INF if np.isinf(e) else frac(e)
        den = INF if E == INF else ex_fp32(1 + E)
        sg = Fraction(0) if den == INF else ex_fp32(frac(g) / den)
        out.append(ex_fp32(sg * frac(u)))
    return out


def test_silu_mul_quant_matches_exact_rational_steps():
    rng = np.random.default_rng(31)
    for I in (8, 16, 32):
        for trial in range(6):
            g = (rng.standard_normal(I) * [1, 4, 20, 0.01, 3, 90][trial]).astype(np.float16)
            u = (rng.standard_normal(I) * 2).astype(np.float16)
            gu = np.concatenate([g, u])[None, :]
            h = P.silu_mul_f32(gu)[0]
            want = _silu_mul_exact(g, u)
            assert [abs(float(a)) for a in h] == [abs(float(b)) for b in want], (I, trial)
            X8, s_x, rs = P.silu_mul_quant(gu)
            codes, s = _quant_exact(want)
            assert float(s_x[0]) == float(s) and X8[0].tolist() == codes and int(rs[0]) == sum(codes)


def test_silu_mul_closed_forms():
    I = 512
    # gate 0 or up 0: h = 0, scale 0, codes 0
    gu = np.zeros((2, 2 * I), dtype=np.float16)
    gu[1, :I] = 3.0
    X8, s_x, rs = P.silu_mul_quant(gu)
    assert np.all(X8 == 0) and np.all(s_x == 0) and np.all(rs == 0)
    # a large constant gate (e^-g below half an ulp of 1): silu(g) = g exactly, so h = g * u
    gu = np.zeros((1, 2 * I), dtype=np.float16)
    gu[0, :I] = 30.0
    gu[0, I:] = -2.0
    h = P.silu_mul_f32(gu)
    assert np.all(h == np.float32(-60.0))
    X8, s_x, rs = P.silu_mul_quant(gu)
    assert np.all(X8 == -127) and rs[0] == -127 * I
    # very negative gate: e^-g overflows, silu(g) = -0, codes 0
    gu[0, :I] = -200.0
    X8, s_x, rs = P.silu_mul_quant(gu)
    assert np.all(X8 == 0)


def test_silu_mul_close_to_binary64_definition():
    rng = np.random.default_rng(4)
    g = (rng.standard_normal((3, 2048)) * 3).astype(np.float16)
    u = rng.standard_normal((3, 2048)).astype(np.float16)
    h = P.silu_mul_f32(np.concatenate([g, u], axis=1))
    g64, u64 = g.astype(np.float64), u.astype(np.float64)
    ref = g64 / (1 + np.exp(-g64)) * u64
    ok = np.abs(ref) > 1e-30
    rel = np.abs(h[ok] - ref[ok]) / np.abs(ref[ok])
    assert rel.max() < 6 * 2.0 ** -23


def test_exact_sqrt_helper_is_correctly_rounded():
    """The rational square root used above agrees with IEEE binary32 sqrt
    (correctly rounded by the standard) on representable arguments."""
    rng = np.random.default_rng(9)
    for q in rng.uniform(1e-6, 1e6, 2000).astype(np.float32):
        assert float(_sqrt32(Fraction(float(q)))) == float(np.sqrt(q))
