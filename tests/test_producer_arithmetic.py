"""CPU checks of three arithmetic claims the fused producer kernels rest on,
each restated here in numpy from its description (no kernel code is run or
shared) and compared with the oracle or with plain definitions:

1. The exact sum of squares in two 64-bit accumulators: |x| * 2^24 = m * 2^s
   for an FP16 x (m its 11-bit significand with the hidden bit, s = max(e-1, 0)
   for the exponent field e); squares with s < 15 are summed as (m * 2^s)^2,
   the others as (m * 2^(s-15))^2, and the total is a0 + a1 * 2^30. It must
   equal the oracle's exact integer sum, and neither accumulator may wrap for
   128 elements per thread summed over a 32-lane warp.
2. The code byte: RNE(clamp(q, -127, 127)) is the low byte of the binary32 sum
   clamp(q) + 1.5 * 2^23.
3. No clamp is needed when the row's scale s = FP16(FP32(max|h| / 127)) is a
   normal FP16 number: then RN32(h / s) < 127.5 in magnitude for |h| <= max|h|.
"""
import numpy as np

from oracle import producers as P

F32 = np.float32


def _bucketed_sum_of_squares(x16: np.ndarray, split: int = 15, shift: int = 30, hidden: bool = True) -> list:
    b = np.asarray(x16, dtype=np.float16).view(np.uint16).astype(np.int64)
    e = (b >> 10) & 31
    f = b & 1023
    m = np.where(e > 0, f | 1024, f) if hidden else f
    s = np.where(e > 0, e - 1, 0)
    up = s >= split
    v = m << np.where(up, s - split, s)
    sq = v * v
    out = []
    for r in range(sq.shape[0]):
        a0 = int(sq[r][~up[r]].sum())
        a1 = int(sq[r][up[r]].sum())
        out.append(a0 + (a1 << shift))
    return out


def _test_rows() -> np.ndarray:
    rng = np.random.default_rng(7)
    every = np.arange(0, 0x7C00, dtype=np.uint16)          # every non-negative finite FP16
    every = np.concatenate([every, every | 0x8000]).view(np.float16)
    rows = [every[i:i + 4096] for i in range(0, every.size - 4096 + 1, 4096)]
    rows.append(np.full(4096, 65504, np.float16))            # the largest value everywhere
    rows.append(np.full(4096, 6e-8, np.float16))             # the smallest subnormal everywhere
    wide = rng.standard_normal(4096) * np.exp(rng.uniform(-20, 11, 4096))
    rows.append(np.clip(wide, -65504, 65504).astype(np.float16))
    return np.stack(rows)


def test_two_bucket_sum_of_squares_equals_the_exact_sum():
    X = _test_rows()
    b = np.asarray(X).view(np.uint16).astype(np.int64)
    e = (b >> 10) & 31
    v = np.where(e > 0, (b & 1023) | 1024, b & 1023) << np.where(e > 0, e - 1, 0)
    largest = int(v.max())
    # the largest square of the upper bucket, (v >> 15)^2, and of the lower, (2047 << 14)^2, are below 2^50
    assert (largest >> 15) ** 2 < 2 ** 50 and ((2 ** 11 - 1) << 14) ** 2 < 2 ** 50
    assert _bucketed_sum_of_squares(X) == [int(t) for t in P.exact_sum_of_squares(X)]


def test_planted_bucket_mistakes_are_caught():
    """Planted on the CPU: a wrong bucket boundary, a wrong scale of the
    upper bucket, or a dropped hidden bit each changes some row's sum."""
    X = _test_rows()
    want = [int(t) for t in P.exact_sum_of_squares(X)]
    assert _bucketed_sum_of_squares(X, split=14) != want
    assert _bucketed_sum_of_squares(X, shift=28) != want
    assert _bucketed_sum_of_squares(X, hidden=False) != want


def test_accumulators_cannot_wrap():
    """Worst case per accumulator: every element at its bucket's largest square
    (finite FP16), 128 elements per thread, 32 threads."""
    largest_low = ((2 ** 11 - 1) << 14) ** 2        # s = 14, m = 2047
    largest_high = ((2 ** 11 - 1) << (29 - 15)) ** 2  # s = 29 (e = 30), m = 2047
    assert 128 * largest_low < 2 ** 57 and 128 * largest_high < 2 ** 57
    assert 32 * 128 * largest_low < 2 ** 64 and 32 * 128 * largest_high < 2 ** 64
    # the 128-bit total a0 + a1 * 2^30 of a 16-warp row stays below 2^128
    assert 16 * (2 ** 64 + (2 ** 64 << 30)) < 2 ** 128


def test_code_byte_from_the_magic_sum():
    rng = np.random.default_rng(3)
    q = np.concatenate([rng.uniform(-400, 400, 200000), np.arange(-130, 131) + 0.5, np.arange(-130, 131) + 0.0,
                        [-0.0, 0.0, 127.49998, -127.49998, 127.5, -127.5]]).astype(F32)
    qc = np.clip(q, F32(-127), F32(127)).astype(F32)
    t = (qc + F32(12582912.0)).astype(F32)
    byte = (t.view(np.uint32) & 0xFF).astype(np.uint8).view(np.int8)
    assert np.array_equal(byte, np.clip(np.rint(q), -127, 127).astype(np.int8))


def test_no_clamp_needed_for_a_normal_scale():
    rng = np.random.default_rng(11)
    lo = 127.0 * 2.0 ** -14 * (1 - 2.0 ** -10)               # around the smallest normal scale
    amax = np.concatenate([np.exp(rng.uniform(np.log(lo), np.log(65504.0 * 127), 1_000_000)),
                           127.0 * np.float16(np.arange(0x0400, 0x7C00, dtype=np.uint16).view(np.float16))
                           .astype(np.float64)]).astype(F32)
    s32 = (amax / F32(127)).astype(F32)
    s = s32.astype(np.float16)
    normal = np.isfinite(s) & (s >= np.float16(2.0 ** -14))
    assert normal.sum() > 900_000
    q = (amax[normal] / s[normal].astype(F32)).astype(F32)   # |h| = max|h|, the largest quotient
    assert float(np.abs(q).max()) < 127.1
