"""Pins for the CPU reference (oracle) against things other than itself.

Each test ties one oracle function to the pages' invariants, to exact
rational arithmetic, to a closed form, to brute force with Python integers,
or to a hand-worked fixture in tests/golden/.  Section references are to the
paperlayer.ai summary of QServe (arXiv 2405.04532v3).
"""
import itertools
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from exact import fp16 as ex_fp16, fp32 as ex_fp32, frac, INF
from w4a8_quantized_gemm_qoq_b200 import inputs

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _golden(golden_dir, name):
    rows = []
    with open(os.path.join(golden_dir, name)) as f:
        for line in f:
            line = line.split("#")[0].strip() if not line.startswith("#") else ""
            if line:
                rows.append(line)
    return rows


# ---------------------------------------------------------------- FP16 rounding

def test_fp16_golden(golden_dir):
    for row in _golden(golden_dir, "fp16_rounding.txt"):
        f32_bits, f16_bits = row.split()[:2]
        x = np.array([int(f32_bits, 16)], dtype=np.uint32).view(np.float32)
        got = int(oracle.fp16(x).view(np.uint16)[0])
        assert got == int(f16_bits, 16), row


def test_fp16_against_exact_rationals():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 2 ** 32, size=4000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    # keep the interesting exponent window (subnormal .. overflow of binary16)
    x = x[(np.abs(x) < 1e6) & (np.abs(x) > 1e-9)]
    got = oracle.fp16(x)
    for xi, gi in zip(x, got):
        e = ex_fp16(frac(xi))
        if e in (INF, -INF):
            assert np.isinf(gi) and (gi > 0) == (e > 0)
        else:
            assert Fraction(float(gi)) == e, (xi, gi, e)


# ------------------------------------------------------ per-token activation quant

def _act_exact(row):
    """Per-token INT8 of one row by exact rationals (section 6: per-token INT8)."""
    vals = [frac(v) for v in row]
    amax = max(abs(v) for v in vals)
    s = ex_fp16(ex_fp32(amax / 127))
    if s == 0:
        return [0] * len(vals), s
    codes = [max(-127, min(127, round(ex_fp32(v / s)))) for v in vals]
    return codes, s


def test_act_quant_bruteforce_exact():
    X = inputs.make_activations(5, 256, seed=3)
    X[4] = (X[4].astype(np.float32) * 1e-3).astype(np.float16)   # FP16-subnormal scale
    X8, s_x, rowsum = oracle.quantize_act_per_token(X)
    for m in range(X.shape[0]):
        codes, s = _act_exact(X[m])
        assert Fraction(float(s_x[m])) == s
        assert X8[m].tolist() == codes
        assert int(rowsum[m]) == sum(codes)


def test_act_quant_golden_ties(golden_dir):
    rows = _golden(golden_dir, "act_quant_ties.txt")
    X = np.zeros((1, 128), dtype=np.float16)
    expect = np.zeros(128, dtype=np.int64)
    sx_bits = rowsum = None
    for r in rows:
        t = r.split()
        if t[0] == "s_x_bits":
            sx_bits = int(t[1], 16)
        elif t[0] == "rowsum":
            rowsum = int(t[1])
        else:
            X[0, int(t[0])] = np.float16(float(t[1]))
            expect[int(t[0])] = int(t[3])
    X8, s_x, rs = oracle.quantize_act_per_token(X)
    assert int(s_x.view(np.uint16)[0]) == sx_bits
    assert X8[0].tolist() == expect.tolist()
    assert int(rs[0]) == rowsum


def test_act_quant_closed_forms():
    K = 384
    X = np.zeros((4, K), dtype=np.float16)
    X[0, 17] = 3.5                      # one-hot: code +127 at 17, 0 elsewhere
    X[1, :] = -0.75                     # constant row: every code -127
    # row 2 stays zero: scale 0, codes 0, rowsum 0
    X[3, ::2] = 2.0; X[3, 1::2] = -2.0  # alternating: +-127, rowsum 0
    X8, s_x, rowsum = oracle.quantize_act_per_token(X)
    assert X8[0, 17] == 127 and np.count_nonzero(X8[0]) == 1
    assert np.all(X8[1] == -127) and rowsum[1] == -127 * K
    assert s_x[2] == 0 and not X8[2].any() and rowsum[2] == 0
    assert np.all(np.abs(X8[3]) == 127) and rowsum[3] == 0
    assert s_x[0] == np.float16(3.5 / 127)


def test_act_quant_invariants():
    X = inputs.make_activations(64, 1024, seed=5, token_scale_span=(-3, 1))
    X8, s_x, rowsum = oracle.quantize_act_per_token(X)
    assert np.abs(X8.astype(np.int64)).max() <= 127
    # the row absmax always maps to +-127 (scale rounding moves it by < 0.5)
    am = np.abs(X.astype(np.float32)).argmax(axis=1)
    assert np.all(np.abs(X8[np.arange(64), am]) == 127)
    assert np.array_equal(rowsum, X8.astype(np.int64).sum(axis=1))
    # scales span the requested 1e-3 .. 1e1 decade range
    assert 1e-3 * 0.9 < s_x.astype(np.float32).min() and s_x.astype(np.float32).max() < 1e1 * 1.1


# ----------------------------------------------------- level 1: per-channel INT8

def test_level1_bruteforce_exact():
    W = inputs.make_weights(6, 256, seed=7)
    W[5] = (W[5].astype(np.float32) * 1e-4).astype(np.float16)
    Q8, s_w = oracle.quantize_level1(W)
    for n in range(W.shape[0]):
        vals = [frac(v) for v in W[n]]
        s = ex_fp16(ex_fp32(max(abs(v) for v in vals) / 119))
        assert Fraction(float(s_w[n])) == s
        exp = [0 if s == 0 else max(-119, min(119, round(ex_fp32(v / s)))) for v in vals]
        assert Q8[n].tolist() == exp


def test_level1_closed_forms():
    W = np.zeros((3, 256), dtype=np.float16)
    W[0, :] = 0.02            # constant row -> all +119
    W[1, :] = -3.0            # constant negative -> all -119
    Q8, s_w = oracle.quantize_level1(W)   # row 2 zero -> scale 0, codes 0
    assert np.all(Q8[0] == 119) and np.all(Q8[1] == -119)
    assert s_w[2] == 0 and not Q8[2].any()
    Wr = inputs.make_weights(32, 512, seed=1)
    Q8, _ = oracle.quantize_level1(Wr)
    assert np.abs(Q8.astype(int)).max() == 119          # protective range reached, never passed


# --------------------------------------- level 2: exhaustive over every INT8 group

def _level2_exact(vmin, vmax, v):
    s = max(1, round(Fraction(vmax - vmin, 15)))
    z = round(Fraction(-vmin, s))
    q = min(15, max(0, round(Fraction(v, s)) + z))
    return s, z, q, (q - z) * s


def _groups_for_range(R):
    """Groups (rows of 128) covering every (vmin, v, vmax), -R <= vmin <= v <= vmax <= R."""
    rows, meta = [], []
    for vmin in range(-R, R + 1):
        for vmax in range(vmin, R + 1):
            mids = list(range(vmin, vmax + 1))
            for i in range(0, len(mids), 126):
                chunk = mids[i:i + 126]
                row = [vmin, vmax] + chunk + [vmin] * (126 - len(chunk))
                rows.append(row)
                meta.append((vmin, vmax))
    return np.asarray(rows, dtype=np.int8), meta


def test_level2_exhaustive_against_rationals():
    """Every possible group in [-119,119] (vmin and vmax fix s and z; every
    value between them is present) matches exact rational round-half-even."""
    Q8, meta = _groups_for_range(119)
    q, s, z, Wint = oracle.quantize_level2(Q8.reshape(-1, 128))
    # exact (s, z) per (vmin, vmax), checked for every group
    table = {}
    for vmin in range(-119, 120):
        for vmax in range(vmin, 120):
            table[(vmin, vmax)] = _level2_exact(vmin, vmax, vmin)[:2]
    exp_sz = np.array([table[m] for m in meta], dtype=np.int64)
    assert np.array_equal(s[:, 0].astype(np.int64), exp_sz[:, 0])
    assert np.array_equal(z[:, 0].astype(np.int64), exp_sz[:, 1])
    # exact q for every element: q depends on (v, s, z) only
    vv = Q8.astype(np.int64)
    ss = exp_sz[:, 0:1]
    zz = exp_sz[:, 1:2]
    qexp = np.empty_like(vv)
    cache = {}
    for i in range(vv.shape[0]):
        for j in range(128):
            key = (int(vv[i, j]), int(ss[i, 0]))
            r = cache.get(key)
            if r is None:
                r = cache[key] = round(Fraction(*key))
            qexp[i, j] = r
    qexp = np.clip(qexp + zz, 0, 15)
    assert np.array_equal(q.astype(np.int64), qexp)
    assert np.array_equal(Wint.astype(np.int64), (qexp - zz) * ss)


def test_level2_protective_range_is_tight():
    """The pages shrink the INT8 level to [-119, 119] so that the dequantised
    group value stays inside INT8 with no saturation (section 4).  Over every
    group: at 119 every (q - z) s and z s fit INT8 and q s stays below 256 (no
    byte carry); at 120 some group dequantises to +128."""
    Q8, _ = _groups_for_range(119)
    q, s, z, Wint = oracle.quantize_level2(Q8)
    W = (q.astype(np.int64).reshape(len(s), 128) - z.astype(np.int64)) * s.astype(np.int64)
    assert W.min() >= -128 and W.max() <= 127
    assert np.array_equal(W, Wint.astype(np.int64))
    assert W.min() == -121 and W.max() == 121
    zs = z.astype(np.int64) * s.astype(np.int64)
    assert zs.min() >= -119 and zs.max() <= 121
    assert (q.astype(np.int64) * s.astype(np.int64)[:, :1]).max() <= 240
    # one range step wider breaks the INT8 bound (exact arithmetic, no oracle)
    worst = max(abs(_level2_exact(vmin, vmax, v)[3])
                for vmin in range(-120, 121) for vmax in (120,) for v in (vmin, vmax))
    assert worst >= 128


def test_level2_golden_groups(golden_dir):
    for row in _golden(golden_dir, "level2_groups.txt"):
        head, tail = row.split("|")
        name, vmin, vmax, s_e, z_e = head.split()
        vmin, vmax, s_e, z_e = int(vmin), int(vmax), int(s_e), int(z_e)
        triples = [tuple(int(t) for t in tok.split(":")) for tok in tail.split()]
        grp = [vmin, vmax] + [t[0] for t in triples]
        grp += [vmin] * (128 - len(grp))
        q, s, z, Wint = oracle.quantize_level2(np.array([grp], dtype=np.int8))
        assert (int(s[0, 0]), int(z[0, 0])) == (s_e, z_e), name
        for i, (v, q_e, w_e) in enumerate(triples):
            assert (int(q[0, 2 + i]), int(Wint[0, 2 + i])) == (q_e, w_e), (name, v)


def test_level2_grid_groups_roundtrip():
    """Groups whose values lie on a zero-aligned grid {k s : k0 <= k <= k0+15}
    with both ends present reproduce the INT8 intermediate exactly (range
    15 s gives scale s, zero -k0 and code k - k0)."""
    rng = np.random.default_rng(11)
    rows = []
    for s in range(1, 17):
        kmax = 119 // s
        if 2 * kmax < 15:
            continue                     # no 16-point grid of step s fits in [-119, 119]
        for _ in range(20):
            k0 = int(rng.integers(-kmax, kmax - 15 + 1))
            ks = rng.integers(k0, k0 + 16, size=128)
            ks[0], ks[1] = k0, k0 + 15
            rows.append(ks * s)
    Q8 = np.asarray(rows, dtype=np.int64)
    assert np.abs(Q8).max() <= 119 and len(rows) == 20 * 14
    _, _, _, Wint = oracle.quantize_level2(Q8.astype(np.int8))
    assert np.array_equal(Wint.astype(np.int64), Q8)


# ------------------------------------------- saturating decode (no protective range)

def _saturating_golden_rows(golden_dir):
    return [tuple(int(t) for t in row.split()) for row in _golden(golden_dir, "saturating_decode.txt")]


def _check_saturating_golden(fn, rows):
    """Each hand-worked (q, s, zs) -> Wsat row sits in its own group of a
    two-group row: group 0 holds row i's code at column i, group 1 row
    (i + 1)'s code at column 128 + i; the other codes are 0."""
    n = len(rows)
    q = np.zeros((n, 256), dtype=np.uint8)
    s = np.zeros((n, 2), dtype=np.uint8)
    zs = np.zeros((n, 2), dtype=np.int8)
    want = np.zeros((n, 2), dtype=np.int64)
    for i in range(n):
        a, b = rows[i], rows[(i + 1) % n]
        q[i, i], s[i, 0], zs[i, 0], want[i, 0] = a
        q[i, 128 + i], s[i, 1], zs[i, 1], want[i, 1] = b
    got = fn(q, s, zs).astype(np.int64)
    return all(got[i, i] == want[i, 0] and got[i, 128 + i] == want[i, 1] for i in range(n))


def test_saturating_decode_golden(golden_dir):
    rows = _saturating_golden_rows(golden_dir)
    assert len(rows) >= 10
    assert _check_saturating_golden(oracle.dequantize_saturating, rows)


def test_saturating_decode_planted_mistakes_fail_the_golden(golden_dir):
    """A top bound of 128 (a 16-bit clamp), an added instead of subtracted
    zero term, and the group index taken modulo instead of divided each fail
    the hand-worked rows."""
    rows = _saturating_golden_rows(golden_dir)

    def top128(q, s, zs):
        raw = q.astype(np.int64).reshape(len(q), 2, 128) * s.astype(np.int64)[:, :, None] - \
            zs.astype(np.int64)[:, :, None]
        return np.clip(raw, -128, 128).reshape(len(q), 256)

    def plus_zero(q, s, zs):
        return oracle.dequantize_saturating(q, s, -zs.astype(np.int64).clip(-127, 127).astype(np.int8))

    def group_mod(q, s, zs):
        j = np.arange(256) % 2
        raw = q.astype(np.int64) * s.astype(np.int64)[:, j] - zs.astype(np.int64)[:, j]
        return np.clip(raw, -128, 127)

    for bad in (top128, plus_zero, group_mod):
        assert not _check_saturating_golden(bad, rows), bad.__name__


def test_saturating_decode_reduces_to_level2_on_protective_groups():
    """On groups from the protective range the clamp never acts: the
    saturating decode equals the second level's own dequantised weights."""
    rng = np.random.default_rng(21)
    Q8 = rng.integers(-119, 120, size=(64, 1024)).astype(np.int8)
    Q8[:8] = np.clip(rng.integers(-119, 120, size=(8, 1)) + rng.integers(-3, 4, size=(8, 1024)), -119, 119)
    q, s, z, Wint = oracle.quantize_level2(Q8)
    zs = (z.astype(np.int64) * s.astype(np.int64)).astype(np.int8)
    assert np.array_equal(oracle.dequantize_saturating(q, s, zs), Wint)


def test_saturating_decode_bounds_and_monotone():
    """Over random codes, scales and zero terms that leave INT8: every value
    is in [-128, 127], values are non-decreasing in the code for a fixed
    (s, zs), and the clamp acts on a good share of them."""
    rng = np.random.default_rng(22)
    N, K = 32, 2048
    s = rng.integers(0, 256, size=(N, K // 128)).astype(np.uint8)
    zs = rng.integers(-128, 128, size=(N, K // 128)).astype(np.int8)
    q = np.tile(np.arange(16, dtype=np.uint8), (N, K // 16))
    W = oracle.dequantize_saturating(q, s, zs).astype(np.int64)
    assert W.min() >= -128 and W.max() <= 127
    steps = np.diff(W.reshape(N, K // 16, 16), axis=2)
    assert steps.min() >= 0
    assert (W == 127).mean() > 0.3


# -------------------------------------------------------------- per-channel variant

def test_per_channel_bruteforce_exact():
    W = inputs.make_weights(5, 256, seed=9)
    W[3] = np.abs(W[3])                  # all-positive row
    W[4] = 0                             # zero row
    d = oracle.quantize_weights_per_channel(W)
    for n in range(W.shape[0]):
        vals = [frac(v) for v in W[n]]
        lo, hi = min(min(vals), Fraction(0)), max(max(vals), Fraction(0))
        s = ex_fp16(ex_fp32(ex_fp32(hi - lo) / 15))
        assert Fraction(float(d["s"][n])) == s
        if s == 0:
            assert d["z"][n] == 0 and not d["q"][n].any()
            continue
        z = round(ex_fp32(-lo / s))
        assert float(d["z"][n]) == z
        exp = [min(15, max(0, round(ex_fp32(v / s)) + z)) for v in vals]
        assert d["q"][n].tolist() == exp


def test_per_channel_closed_forms():
    W = np.zeros((2, 128), dtype=np.float16)
    W[0, :] = 0.5          # range [0, 0.5]: s = FP16(0.5/15), z = 0, q = 15 everywhere
    W[1, :] = -0.25        # range [-0.25, 0]: z = 15, q = 0 everywhere
    d = oracle.quantize_weights_per_channel(W)
    assert d["s"][0] == np.float16(np.float32(0.5) / np.float32(15))
    assert d["z"][0] == 0 and np.all(d["q"][0] == 15)
    assert d["z"].view(np.uint16)[0] == 0          # integer zero point: +0, never -0
    assert d["z"][1] == 15 and np.all(d["q"][1] == 0)


# ----------------------------------------------------------- packing (compute order)

def test_pack_golden_block(golden_dir):
    r = np.arange(128)[:, None]
    k = np.arange(128)[None, :]
    q = ((r + k) % 16).astype(np.uint8)
    s = (1 + np.arange(128) % 16).astype(np.uint8)[:, None]
    zs = ((np.arange(128) % 7) - 3).astype(np.int8)[:, None]
    s_w = np.ones(128, dtype=np.float16)
    blob = oracle.pack_blob_group(q, s, zs, s_w)
    assert blob.size == 8960
    for row in _golden(golden_dir, "pack_block.txt"):
        off, val = row.split()[:2]
        assert int(blob[int(off)]) == int(val, 16), row


def test_pack_roundtrip_both_modes():
    W = inputs.make_weights(384, 640, seed=2)
    blob, d = oracle.quantize_weights(W, 128)
    u = oracle.unpack_blob(blob)
    assert (u["N"], u["K"], u["group"]) == (384, 640, 128)
    assert np.array_equal(u["q"], d["q"])
    assert np.array_equal(u["s"], d["s"]) and np.array_equal(u["zs"], d["zs"])
    assert np.array_equal(u["scale"].view(np.uint16), d["s_w"].view(np.uint16))
    blob, d = oracle.quantize_weights(W, 0)
    u = oracle.unpack_blob(blob)
    assert u["group"] == 0 and np.array_equal(u["q"], d["q"])
    assert np.array_equal(u["z"].view(np.uint16), d["z"].view(np.uint16))
    assert blob.size == oracle.blob_layout(384, 640, 0)["total"]


# --------------------------------------------------------------------- integer GEMM

def test_gemm_bruteforce_python_ints():
    rng = np.random.default_rng(4)
    for M, N, K in [(1, 1, 128), (3, 5, 128), (8, 8, 256), (7, 2, 384)]:
        X8 = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
        W = rng.integers(-121, 122, size=(N, K)).astype(np.int8)
        acc = oracle.gemm_int(X8, W)
        for m, n in itertools.product(range(M), range(N)):
            assert int(acc[m, n]) == sum(int(a) * int(b) for a, b in zip(X8[m], W[n]))


def test_gemm_matches_numpy_int64_matmul():
    rng = np.random.default_rng(5)
    X8 = rng.integers(-127, 128, size=(33, 640)).astype(np.int8)
    W = rng.integers(-121, 122, size=(70, 640)).astype(np.int8)
    ref = X8.astype(np.int64) @ W.astype(np.int64).T
    assert np.array_equal(oracle.gemm_int(X8, W).astype(np.int64), ref)


def test_gemm_closed_forms():
    W = inputs.make_weights(256, 512, seed=6)
    W[5, :] = 0.01
    W[6, :] = -1.0
    d = oracle.quantize_weights_group(W)
    K = 512
    # constant W rows dequantise to +-119 exactly: acc = +-119 * rowsum
    X = inputs.make_activations(16, K, seed=6)
    X8, s_x, rowsum = oracle.quantize_act_per_token(X)
    acc = oracle.gemm_int(X8, d["Wint"])
    assert np.array_equal(acc[:, 5], 119 * rowsum) and np.array_equal(acc[:, 6], -119 * rowsum)
    # one-hot activations (a scaled identity) read back the dequantised weights
    Xi = np.zeros((K, K), dtype=np.float16)
    Xi[np.arange(K), np.arange(K)] = 1.0
    X8, _, _ = oracle.quantize_act_per_token(Xi)
    acc = oracle.gemm_int(X8, d["Wint"])
    assert np.array_equal(acc, 127 * d["Wint"].astype(np.int32).T)
    # constant activation rows: acc = 127 * sum_k Wint
    Xc = np.full((2, K), 0.3, dtype=np.float16)
    Xc[1] = -0.3
    X8, _, _ = oracle.quantize_act_per_token(Xc)
    acc = oracle.gemm_int(X8, d["Wint"])
    tot = d["Wint"].astype(np.int64).sum(axis=1)
    assert np.array_equal(acc[0], 127 * tot) and np.array_equal(acc[1], -127 * tot)


def test_gemm_int32_headroom():
    """|acc| <= K * 127 * 121 stays below 2^31 up to the largest K (24576)."""
    assert 24576 * 127 * 121 < 2 ** 31
    X8 = np.full((1, 24576), 127, dtype=np.int8)
    W = np.full((1, 24576), 121, dtype=np.int8)
    assert int(oracle.gemm_int(X8, W)[0, 0]) == 24576 * 127 * 121


def test_per_channel_correction_is_exact():
    rng = np.random.default_rng(8)
    X8 = rng.integers(-127, 128, size=(6, 256)).astype(np.int8)
    rowsum = X8.astype(np.int64).sum(axis=1).astype(np.int32)
    q = rng.integers(0, 16, size=(4, 256)).astype(np.uint8)
    z = np.array([0, 3, 15, 7], dtype=np.float16)
    t = oracle.w4a8_gemm_per_channel(X8, rowsum, q, z)
    for m in range(6):
        for n in range(4):
            assert int(t[m, n]) == sum(int(x) * (int(qq) - int(z[n])) for x, qq in zip(X8[m], q[n]))


# ------------------------------------------------------------------------ epilogue

def test_epilogue_exact_fp32_steps():
    rng = np.random.default_rng(10)
    acc = rng.integers(-2 ** 31 + 1, 2 ** 31 - 1, size=(4, 6)).astype(np.int32)
    acc[0, 0] = 16777217          # not representable in binary32: rounds to even
    s_x = oracle.fp16(rng.uniform(1e-4, 1e1, size=4))
    s_w = oracle.fp16(rng.uniform(1e-5, 1e-2, size=6))
    Y = oracle.epilogue_fp16(acc, s_x, s_w)
    for m in range(4):
        for n in range(6):
            e = ex_fp16(ex_fp32(ex_fp32(Fraction(int(acc[m, n]))) *
                                ex_fp32(frac(s_x[m]) * frac(s_w[n]))))
            y = Y[m, n]
            if e in (INF, -INF):
                assert np.isinf(y)
            else:
                assert Fraction(float(y)) == e


def test_epilogue_within_one_ulp_of_fp64():
    W = inputs.make_weights(256, 1024, seed=12)
    X = inputs.make_activations(32, 1024, seed=12, token_scale_span=(-3, 1))
    r = oracle.reference_forward(X, W, 128)
    y64 = (r["acc"].astype(np.float64) * r["s_x"].astype(np.float64)[:, None]
           * r["w"]["s_w"].astype(np.float64)[None, :]).astype(np.float16)
    assert oracle.fp16_ulp_distance(r["Y"], y64).max() <= 1


def test_ulp_distance_definition():
    a = np.array([0.0, -0.0, 1.0, 1.0, np.inf, 65504.0], dtype=np.float16)
    b = np.array([-0.0, 0.0, np.float16(1.0009766), 1.0, np.inf, np.inf], dtype=np.float16)
    assert oracle.fp16_ulp_distance(a, b).tolist() == [0, 0, 1, 0, 0, 1]


def test_whole_path_dequant_error_bound():
    """End to end, the dequantised weight (Wint * s_w) tracks W within the two
    quantisation steps: |W - Wint s_w| <= (0.5 + 14) s_w (level 1 rounds to
    half a step, level 2 moves a value by at most 14 steps, proven by the
    exhaustive enumeration)."""
    W = inputs.make_weights(128, 1024, seed=13)
    d = oracle.quantize_weights_group(W)
    err = np.abs(W.astype(np.float64) - d["Wint"].astype(np.float64) * d["s_w"].astype(np.float64)[:, None])
    assert np.all(err <= 14.5 * d["s_w"].astype(np.float64)[:, None] * (1 + 1e-3))
    assert np.abs(d["Q8"].astype(int) - d["Wint"].astype(int)).max() <= 14
