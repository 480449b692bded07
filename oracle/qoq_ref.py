"""Plain CPU reference of the QoQ W4A8 GEMM path -- TEST INFRASTRUCTURE.

Only tests, the smoke check and the benchmark's CPU-baseline arm use this.

Sources (web summaries of QServe: W4A8KV4 Quantization and System Co-design
for Efficient LLM Serving, arXiv 2405.04532):
  [P3-4]  paperlayer.ai summary, section 4 "QoQ Quantization" -- progressive
          group quantization: per-channel INT8 with FP16 scales, then per-group
          4-bit codes with scales and zero points; protective INT8 range
          [-119, 119] so the dequantised weight never leaves INT8.
  [P3-5]  same page, section 5 "QServe Serving System" -- GEMMs on INT8 tensor
          cores with FP16 outputs; subtraction after multiplication; per-channel
          scale and zero-point correction fused into the epilogue; weights
          stored in compute order.
  [P3-6]  same page, section 6 "Evaluation" -- per-token INT8 activations;
          "g128" = group size 128; the per-channel variant has no group level.
  [P5]    study.space summary -- first level 8 bits with per-channel FP16
          scales, then 4 bits; all GEMMs on INT8 tensor cores.

The pages give no formulas. Where they are silent the plainest reading is
taken and named in the docstring ("reading:"). Floating point follows the
precision the CUDA kernels use for the same decision (IEEE binary32, one
correctly rounded operation at a time, no fused multiply-add), because the
pages fix only the storage types (FP16 scales, INT8/UINT4 codes).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

GROUP = 128          # g128 [P3-6]
Q8_RANGE = 119       # protective range [-119, 119] [P3-4]
X8_RANGE = 127       # symmetric per-token INT8
U4_MAX = 15

F32 = np.float32

# ---------------------------------------------------------------------------
# Rounding helpers
# ---------------------------------------------------------------------------


def fp16(x) -> np.ndarray:
    """binary32 -> binary16, round to nearest even, overflow to +-inf."""
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float32).astype(np.float16)


def rne(x) -> np.ndarray:
    """Round half to even to an integer value (same floating type)."""
    return np.rint(x)


# ---------------------------------------------------------------------------
# Activations: per-token INT8 [P3-6]
# ---------------------------------------------------------------------------


def quantize_act_per_token(X: np.ndarray):
    """Per-token symmetric INT8 quantisation of FP16 activations [M][K].

    amax_m = max_k |X[m,k]|                 (exact)
    s_x[m] = FP16(amax_m / 127)             (FP32 divide, rounded once to FP16)
    X8     = clamp(RNE(X / FP32(s_x)), -127, 127), and 0 where s_x == 0
    rowsum = sum_k X8[m,k]                  (int32; used by the per-channel
                                             variant's zero correction)
    reading: the scale is FP16 like the other scales of the method, and the
    stored FP16 value is what the codes are divided by.
    """
    X32 = np.asarray(X, dtype=np.float16).astype(F32)
    amax = np.abs(X32).max(axis=1)
    s_x = fp16(amax / F32(X8_RANGE))
    s32 = s_x.astype(F32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        r = X32 / s32
    X8 = np.where(s32 == 0, F32(0), np.clip(rne(r), -X8_RANGE, X8_RANGE)).astype(np.int8)
    rowsum = X8.astype(np.int64).sum(axis=1).astype(np.int32)
    return X8, s_x, rowsum


# ---------------------------------------------------------------------------
# Weights, level 1: per-output-channel INT8 in the protective range [P3-4][P5]
# ---------------------------------------------------------------------------


def quantize_level1(W: np.ndarray):
    """Per-channel symmetric INT8 with FP16 scale, range [-119, 119].

    s_w[n] = FP16(max_k |W[n,k]| / 119)
    Q8     = clamp(RNE(W / FP32(s_w)), -119, 119), and 0 where s_w == 0
    """
    W32 = np.asarray(W, dtype=np.float16).astype(F32)
    amax = np.abs(W32).max(axis=1)
    s_w = fp16(amax / F32(Q8_RANGE))
    s32 = s_w.astype(F32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        r = W32 / s32
    Q8 = np.where(s32 == 0, F32(0), np.clip(rne(r), -Q8_RANGE, Q8_RANGE)).astype(np.int8)
    return Q8, s_w


# ---------------------------------------------------------------------------
# Weights, level 2: per-group (g = 128 along K) UINT4 with integer scale/zero
# ---------------------------------------------------------------------------


def quantize_level2(Q8: np.ndarray, g: int = GROUP):
    """Asymmetric min-max UINT4 quantisation of each group of g INT8 values.

    For row n and group j (columns jg .. jg+g-1), with vmin/vmax the group's
    smallest/largest Q8 value:
      s = max(1, RNE((vmax - vmin) / 15))   integer scale in [1, 16]
      z = RNE(-vmin / s)                    integer zero in [-119, 119]
      q = clamp(RNE(v / s) + z, 0, 15)      UINT4 code
      Wint = (q - z) * s                    dequantised INT8 weight
    Returns q (uint8 [N][K]), s (uint8 [N][K/g]), z (int8 [N][K/g]) and
    Wint (int8 [N][K]).

    readings: the pages call the group scale "INT4 scales" in one summary; the
    scale here is an integer (it must be, for the dequantised value to be an
    integer that the INT8 tensor core can consume) stored in 8 bits. RNE is
    used for every rounding; z is not clamped to the code range.

    The quotients are formed in float64: numerator and denominator are small
    integers, a tie (exact half) is exactly representable and any non-tie sits
    at least 1/32 away from a tie, so ``rint`` of the float64 quotient is the
    round-half-even of the exact rational.
    """
    Q8 = np.asarray(Q8, dtype=np.int8)
    N, K = Q8.shape
    assert K % g == 0
    v = Q8.reshape(N, K // g, g).astype(np.int64)
    vmin = v.min(axis=2)
    vmax = v.max(axis=2)
    s = np.maximum(1, rne((vmax - vmin) / 15.0)).astype(np.int64)
    z = rne(-vmin / s).astype(np.int64)
    q = np.clip(rne(v / s[:, :, None]).astype(np.int64) + z[:, :, None], 0, U4_MAX)
    Wint = (q - z[:, :, None]) * s[:, :, None]
    assert Wint.min() >= -128 and Wint.max() <= 127, "dequantised weight left INT8"
    return (q.reshape(N, K).astype(np.uint8), s.astype(np.uint8), z.astype(np.int8),
            Wint.reshape(N, K).astype(np.int8))


def quantize_weights_group(W: np.ndarray, g: int = GROUP):
    """Progressive group quantisation (level 1 then level 2) [P3-4][P5].

    Returns dict with Q8, s_w, q, s, z, zs (= z*s) and Wint."""
    Q8, s_w = quantize_level1(W)
    q, s, z, Wint = quantize_level2(Q8, g)
    zs = (z.astype(np.int64) * s.astype(np.int64))
    assert zs.min() >= -128 and zs.max() <= 127
    return dict(Q8=Q8, s_w=s_w, q=q, s=s, z=z, zs=zs.astype(np.int8), Wint=Wint)


# ---------------------------------------------------------------------------
# Per-channel variant: UINT4 per output channel, FP16 scale and zero [P3-6][P3-5]
# ---------------------------------------------------------------------------


def quantize_weights_per_channel(W: np.ndarray):
    """Asymmetric UINT4 per output channel straight from FP16 (no INT8 level).

    wlo = min(0, min_k W), whi = max(0, max_k W)   (range includes zero)
    s   = FP16((whi - wlo) / 15)                   (FP32 ops)
    z   = RNE(-wlo / FP32(s))                      (integer, stored as FP16)
    q   = clamp(RNE(W / FP32(s)) + z, 0, 15)
    and s == 0 gives z = 0, q = 0.  The dequantised weight is (q - z) * s.

    reading: the pages only name a "per-channel counterpart" of the g128
    scheme with the zero-point correction moved into the epilogue; the range
    is extended to include 0 so that z is a small integer (0..15 for normal
    scales) that FP16 stores exactly.
    """
    W32 = np.asarray(W, dtype=np.float16).astype(F32)
    wlo = np.minimum(W32.min(axis=1), F32(0))
    whi = np.maximum(W32.max(axis=1), F32(0))
    s = fp16((whi - wlo) / F32(U4_MAX))
    s32 = s.astype(F32)
    with np.errstate(divide="ignore", invalid="ignore"):
        z32 = np.where(s32 == 0, F32(0), rne(-wlo / s32))
        r = W32 / s32[:, None]
    q = np.where(s32[:, None] == 0, F32(0), np.clip(rne(r) + z32[:, None], 0, U4_MAX))
    zi = z32.astype(np.int64)                 # the zero point is an integer (no signed zero)
    z = zi.astype(np.float16)
    assert np.all(z.astype(np.int64) == zi), "zero point not exact in FP16"
    return dict(q=q.astype(np.uint8), s=s, z=z)


# ---------------------------------------------------------------------------
# Packed weight blob: compute-order layout [P3-5]
# ---------------------------------------------------------------------------
#
# Our own layout, not the pages' (theirs targets 32x32 tiles of mma.sync).
#   header   256 bytes, little-endian:
#              u32 magic 'QOQW', u32 version 1, u32 N, u32 K,
#              u32 group (128, or 0 = per-channel), u32 block_bytes,
#              u64 off_codes, u64 off_scale, u64 off_zero, u64 total_bytes
#   codes    for n-tile nt (128 rows) major, k-tile kt (128 columns) minor,
#            one block of block_bytes:
#              [chunk c = 0..3][row r = 0..127][16 bytes]
#            chunk c of row r holds columns 32c .. 32c+31 of that k-tile as 4
#            little-endian 32-bit words; word j covers k0 = 32c + 8j and its
#            byte b (0..3) is  q[k0 + b] | q[k0 + b + 4] << 4.
#            group mode appends [row r][u8 s, s8 z*s] for the block's group.
#   scale    FP16 [N]: s_w (group mode) or s (per-channel mode), 256-aligned
#   zero     FP16 [N]: z (per-channel mode only), 256-aligned
# ---------------------------------------------------------------------------

MAGIC = 0x57514F51   # bytes 'Q','O','Q','W'
VERSION = 1
HEADER_BYTES = 256
TILE_N = 128
TILE_K = 128


def _align256(x: int) -> int:
    return (x + 255) // 256 * 256


def blob_layout(N: int, K: int, group: int) -> dict:
    nt, kt = N // TILE_N, K // TILE_K
    block = 8192 + (256 if group else 0)
    off_codes = HEADER_BYTES
    off_scale = off_codes + nt * kt * block
    if group:
        off_zero = 0
        total = off_scale + _align256(2 * N)
    else:
        off_zero = off_scale + _align256(2 * N)
        total = off_zero + _align256(2 * N)
    return dict(NT=nt, KT=kt, block=block, off_codes=off_codes, off_scale=off_scale,
                off_zero=off_zero, total=total)


def _header(N: int, K: int, group: int, L: dict) -> np.ndarray:
    h = np.zeros(HEADER_BYTES, dtype=np.uint8)
    words = np.array([MAGIC, VERSION, N, K, group, L["block"]], dtype="<u4")
    h[0:24] = words.view(np.uint8)
    h[24:56] = np.array([L["off_codes"], L["off_scale"], L["off_zero"], L["total"]],
                        dtype="<u8").view(np.uint8)
    return h


def _pack_codes(q: np.ndarray) -> np.ndarray:
    """q uint8 [N][K] (0..15) -> code bytes [NT][KT][8192] in the layout above."""
    N, K = q.shape
    NT, KT = N // TILE_N, K // TILE_K
    # axes: nt, r, kt, c, j, half, b   (column = 32c + 8j + 4*half + b)
    t = q.reshape(NT, TILE_N, KT, 4, 4, 2, 4).astype(np.uint8)
    byte = t[:, :, :, :, :, 0, :] | (t[:, :, :, :, :, 1, :] << 4)   # nt, r, kt, c, j, b
    byte = byte.transpose(0, 2, 3, 1, 4, 5)                          # nt, kt, c, r, j, b
    return np.ascontiguousarray(byte).reshape(NT, KT, 8192)


def pack_blob_group(q, s, zs, s_w) -> np.ndarray:
    """Blob for the g128 scheme from codes q [N][K], s/zs [N][K/128], s_w [N]."""
    q = np.asarray(q, dtype=np.uint8)
    N, K = q.shape
    L = blob_layout(N, K, GROUP)
    out = np.zeros(L["total"], dtype=np.uint8)
    out[:HEADER_BYTES] = _header(N, K, GROUP, L)
    codes = _pack_codes(q)
    NT, KT = L["NT"], L["KT"]
    sz = np.empty((N, KT, 2), dtype=np.uint8)
    sz[:, :, 0] = np.asarray(s, dtype=np.uint8)
    sz[:, :, 1] = np.asarray(zs, dtype=np.int8).view(np.uint8)
    sz = sz.reshape(NT, TILE_N, KT, 2).transpose(0, 2, 1, 3).reshape(NT, KT, 256)
    blocks = np.concatenate([codes, sz], axis=2)
    out[L["off_codes"]:L["off_scale"]] = blocks.reshape(-1)
    out[L["off_scale"]:L["off_scale"] + 2 * N] = np.asarray(s_w, dtype=np.float16).view(np.uint8)
    return out


def pack_blob_per_channel(q, s, z) -> np.ndarray:
    """Blob for the per-channel scheme from codes q [N][K], s [N], z [N] (FP16)."""
    q = np.asarray(q, dtype=np.uint8)
    N, K = q.shape
    L = blob_layout(N, K, 0)
    out = np.zeros(L["total"], dtype=np.uint8)
    out[:HEADER_BYTES] = _header(N, K, 0, L)
    out[L["off_codes"]:L["off_scale"]] = _pack_codes(q).reshape(-1)
    out[L["off_scale"]:L["off_scale"] + 2 * N] = np.asarray(s, dtype=np.float16).view(np.uint8)
    out[L["off_zero"]:L["off_zero"] + 2 * N] = np.asarray(z, dtype=np.float16).view(np.uint8)
    return out


def unpack_blob(blob: np.ndarray) -> dict:
    """Inverse of the packers: header fields, q, and the per-row/group scales."""
    blob = np.asarray(blob, dtype=np.uint8)
    w = blob[:24].view("<u4")
    o = blob[24:56].view("<u8")
    magic, version, N, K, group, block = (int(x) for x in w)
    if magic != MAGIC or version != VERSION:
        raise ValueError("not a QoQ weight blob")
    NT, KT = N // TILE_N, K // TILE_K
    off_codes, off_scale, off_zero, total = (int(x) for x in o)
    blocks = blob[off_codes:off_scale].reshape(NT, KT, block)
    byte = blocks[:, :, :8192].reshape(NT, KT, 4, TILE_N, 4, 4).transpose(0, 3, 1, 2, 4, 5)
    q = np.empty((NT, TILE_N, KT, 4, 4, 2, 4), dtype=np.uint8)
    q[..., 0, :] = byte & 0x0F
    q[..., 1, :] = byte >> 4
    res = dict(N=N, K=K, group=group, block=block, q=q.reshape(N, K),
               scale=blob[off_scale:off_scale + 2 * N].view(np.float16).copy())
    if group:
        sz = blocks[:, :, 8192:].reshape(NT, KT, TILE_N, 2).transpose(0, 2, 1, 3).reshape(N, KT, 2)
        res["s"] = sz[:, :, 0].copy()
        res["zs"] = sz[:, :, 1].view(np.int8).copy()
    else:
        res["z"] = blob[off_zero:off_zero + 2 * N].view(np.float16).copy()
    return res


def quantize_weights(W: np.ndarray, group: int = GROUP):
    """Full offline weight preparation: (blob bytes, canonical dict)."""
    if group:
        d = quantize_weights_group(W, group)
        return pack_blob_group(d["q"], d["s"], d["zs"], d["s_w"]), d
    d = quantize_weights_per_channel(W)
    return pack_blob_per_channel(d["q"], d["s"], d["z"]), d


# ---------------------------------------------------------------------------
# Integer GEMM: plain int64 triple loop in C (qoq_gemm.c)
# ---------------------------------------------------------------------------

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_build", "libqoq_oracle.so")
_lib = None
_lock = threading.Lock()


def build_c_oracle(force: bool = False) -> str:
    """Compile qoq_gemm.c with gcc (plain -O2, no fast-math, OpenMP over output
    elements) into oracle/_build/."""
    src = os.path.join(_HERE, "qoq_gemm.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        os.makedirs(os.path.dirname(_SO), exist_ok=True)
        tmp = _SO + ".%d.tmp" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fopenmp",
                               "-o", tmp, src])
        os.replace(tmp, _SO)
    return _SO


def _c():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build_c_oracle())
            lib.oracle_gemm_s8s8_i64.restype = ctypes.c_int64
            lib.oracle_gemm_s8s8_i64.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3
            lib.oracle_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def gemm_threads() -> int:
    """Host threads the integer GEMM runs on."""
    return int(_c().oracle_threads())


def gemm_int(X8: np.ndarray, Wint: np.ndarray) -> np.ndarray:
    """acc[m,n] = sum_k X8[m,k] * Wint[n,k], exact, returned as int32.

    Asserts the exact sum fits int32 (the INT32 tensor-core accumulator)."""
    X8 = np.ascontiguousarray(X8, dtype=np.int8)
    Wint = np.ascontiguousarray(Wint, dtype=np.int8)
    M, K = X8.shape
    N, K2 = Wint.shape
    assert K == K2
    acc = np.empty((M, N), dtype=np.int64)
    amax = _c().oracle_gemm_s8s8_i64(X8.ctypes.data, Wint.ctypes.data, acc.ctypes.data, M, N, K)
    assert amax < 2 ** 31, "accumulator overflows int32"
    return acc.astype(np.int32)


# ---------------------------------------------------------------------------
# Epilogue: per-token and per-channel scales fused after the integer GEMM [P3-5]
# ---------------------------------------------------------------------------


def epilogue_fp16(acc: np.ndarray, s_x: np.ndarray, s_w: np.ndarray) -> np.ndarray:
    """Y[m,n] = FP16( FP32(acc[m,n]) * (FP32(s_x[m]) * FP32(s_w[n])) ).

    FP32 products, each rounded once; one final rounding to FP16.
    reading: the pages fuse the per-channel scale into the epilogue and output
    FP16; the order (token scale times channel scale first) is ours."""
    a = np.asarray(acc).astype(F32)
    scale = np.asarray(s_x, dtype=np.float16).astype(F32)[:, None] * \
        np.asarray(s_w, dtype=np.float16).astype(F32)[None, :]
    return fp16(a * scale)


def w4a8_gemm_group(X8, Wint) -> np.ndarray:
    """INT32 result of the g128 scheme: exact X8 . Wint^T."""
    return gemm_int(X8, Wint)


def per_channel_correct(accq: np.ndarray, rowsum: np.ndarray, z: np.ndarray) -> np.ndarray:
    """t[m,n] = accq[m,n] - z[n] * rowsum[m]  (exact int32): the zero-point
    correction moved out of the main loop into the epilogue [P3-5]."""
    zi = np.asarray(z, dtype=np.float16).astype(np.int64)
    t = np.asarray(accq, dtype=np.int64) - zi[None, :] * np.asarray(rowsum, dtype=np.int64)[:, None]
    assert np.abs(t).max(initial=0) < 2 ** 31
    return t.astype(np.int32)


def w4a8_gemm_per_channel(X8, rowsum, q, z) -> np.ndarray:
    """INT32 result of the per-channel scheme: sum_k X8*(q - z) via the
    epilogue correction."""
    accq = gemm_int(X8, np.asarray(q, dtype=np.uint8).astype(np.int8))
    return per_channel_correct(accq, rowsum, z)


# ---------------------------------------------------------------------------
# Saturating weight decode: what a kernel without the protective range does
# [P3-4]
# ---------------------------------------------------------------------------


def dequantize_saturating(q: np.ndarray, s: np.ndarray, zs: np.ndarray, g: int = GROUP) -> np.ndarray:
    """Second-level decode clamped to INT8, for codes that may leave it.

    Wsat[n,k] = clamp(q[n,k] * s[n,j] - zs[n,j], -128, 127),  j = k // g

    with q the UINT4 codes [N][K], s the integer group scales (uint8)
    [N][K/g] and zs = z*s (int8) [N][K/g]. The products are exact integers.

    reading: [P3-4] shrinks the first level to [-119, 119] so that the
    dequantised value q*s - z*s never leaves INT8; without that range the
    main loop must saturate, which the pages say costs up to 67% of the
    GEMM's throughput. Saturation is read as the usual clamp of the exact
    integer to the INT8 range. On protective-range groups the clamp never
    acts and Wsat equals the level-2 Wint.
    """
    q = np.asarray(q, dtype=np.uint8).astype(np.int64)
    N, K = q.shape
    s = np.asarray(s, dtype=np.uint8).astype(np.int64)
    zs = np.asarray(zs, dtype=np.int8).astype(np.int64)
    assert s.shape == (N, K // g) and zs.shape == (N, K // g)
    raw = q.reshape(N, K // g, g) * s[:, :, None] - zs[:, :, None]
    return np.clip(raw, -128, 127).reshape(N, K).astype(np.int8)


def gemm_fp16_saturating(X8: np.ndarray, s_x: np.ndarray, q, s, zs, s_w) -> np.ndarray:
    """FP16 output of the GEMM whose weights are decoded with saturation:
    the exact INT32 product with Wsat, then the epilogue."""
    return epilogue_fp16(gemm_int(X8, dequantize_saturating(q, s, zs)), s_x, s_w)


def reference_forward(X: np.ndarray, W: np.ndarray, group: int = GROUP) -> dict:
    """Whole path on FP16 inputs: act quant, weight quant + pack, GEMM, epilogue."""
    X8, s_x, rowsum = quantize_act_per_token(X)
    blob, d = quantize_weights(W, group)
    if group:
        acc = w4a8_gemm_group(X8, d["Wint"])
        Y = epilogue_fp16(acc, s_x, d["s_w"])
    else:
        acc = w4a8_gemm_per_channel(X8, rowsum, d["q"], d["z"])
        Y = epilogue_fp16(acc, s_x, d["s"])
    return dict(X8=X8, s_x=s_x, rowsum=rowsum, blob=blob, acc=acc, Y=Y, **{"w": d})


# ---------------------------------------------------------------------------
# Output comparison used by the parity tests
# ---------------------------------------------------------------------------


def fp16_ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in units in the last place between FP16 arrays, counted on the
    ordered bit patterns (so +0 and -0 are equal; inf only matches inf)."""
    def ordered(x):
        u = np.asarray(x, dtype=np.float16).view(np.uint16).astype(np.int64)
        mag = u & 0x7FFF
        return np.where(u & 0x8000, -mag, mag)
    return np.abs(ordered(a) - ordered(b))
