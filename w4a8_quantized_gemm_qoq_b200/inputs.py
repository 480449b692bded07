"""Seeded synthetic inputs for the QoQ W4A8 GEMM workloads.

This module only draws random numbers and shapes them; it holds none of the
quantisation or GEMM arithmetic. Both the CUDA path's tests/benchmark and the
CPU reference ("oracle") are fed from here, and it imports neither of them.

Value recipe (the pages evaluate on LLM linear layers whose weights and
activations are not available here, so these stand in for them):
  * X (activations, FP16, [M][K]): i.i.d. N(0, 1); then 4 distinct random
    K-columns (drawn first) are multiplied by 20 to mimic activation outlier
    channels.  With ``token_scale_span`` set, row m is then rescaled so that
    its absmax becomes 127 * 10**u_m, u_m ~ U(lo, hi); its per-token INT8
    scale then lands near 10**u_m (the prefill workload uses 1e-3 .. 1e1).
  * W (weights, FP16, [N][K]): i.i.d. N(0, std), std = 0.02 (Llama shapes) or
    0.01 (Qwen shapes).
  * gamma (RMSNorm weight, FP16, [K]): 1 + 0.1 * N(0, 1), the spread of a
    trained normalisation weight around 1.
  * GU (merged gate/up projection output, FP16, [M][2I]): gate half
    N(0, 2^2) so that SiLU sees both its negative tail and its linear part,
    up half N(0, 1); 4 outlier columns x20 in each half.
  * decode attention (GQA, one query token per sequence): q [B][Hq][D],
    K and V [B][Hkv][T][D], FP16, i.i.d. N(0, 1); in K, 2 channels per KV
    head (drawn first) are multiplied by 8, the outlier Key channels the
    pages describe.
Streams: numpy ``Generator(PCG64([seed, 1]))`` for W,
``Generator(PCG64([seed, 2]))`` for X, ``[seed, 4]`` for gamma,
``[seed, 5]`` for GU and ``[seed, 6]`` for the attention inputs, so each can
be drawn independently.
"""
from __future__ import annotations

import numpy as np

# Linear-layer (K -> N) shapes named by the model whose layer they mimic.
LLAMA3_8B = [(4096, 6144, "qkv"), (4096, 4096, "o"), (4096, 28672, "gate_up"), (14336, 4096, "down")]
QWEN15_72B = [(8192, 24576, "qkv"), (8192, 8192, "o"), (8192, 49152, "gate_up"), (24576, 8192, "down")]
LLAMA2_7B = [(4096, 12288, "qkv"), (4096, 4096, "o"), (4096, 22016, "gate_up"), (11008, 4096, "down")]

DECODE_M = [1, 4, 16, 64, 256]
PREFILL_M = [2048, 8192, 16384]
QWEN_M = [1, 16, 128, 512, 4096]
PER_CHANNEL_M = [1 << i for i in range(11)]

N_OUTLIERS = 4
OUTLIER_GAIN = 20.0


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([int(seed), int(stream)]))


def make_weights(N: int, K: int, seed: int = 0, std: float = 0.02) -> np.ndarray:
    """FP16 weights [N][K] ~ N(0, std)."""
    rng = _rng(seed, 1)
    w = rng.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(std)
    return w.astype(np.float16)


def make_activations(M: int, K: int, seed: int = 0, token_scale_span=None) -> np.ndarray:
    """FP16 activations [M][K]: N(0,1) with 4 outlier columns x20.

    ``token_scale_span=(lo, hi)`` rescales each row so its absmax is
    127 * 10**u, u ~ U(lo, hi)."""
    rng = _rng(seed, 2)
    cols = rng.choice(K, size=min(N_OUTLIERS, K), replace=False)
    x = rng.standard_normal((M, K), dtype=np.float32)
    x[:, cols] *= np.float32(OUTLIER_GAIN)
    if token_scale_span is not None:
        lo, hi = token_scale_span
        u = rng.uniform(lo, hi, size=M).astype(np.float64)
        amax = np.abs(x).max(axis=1).astype(np.float64)
        amax[amax == 0] = 1.0
        c = (127.0 * np.power(10.0, u) / amax).astype(np.float32)
        x *= c[:, None]
    return x.astype(np.float16)


def outlier_columns(K: int, seed: int = 0) -> np.ndarray:
    """The outlier columns ``make_activations`` picks for this (K, seed)."""
    rng = _rng(seed, 2)
    return rng.choice(K, size=min(N_OUTLIERS, K), replace=False)


def sample_rows(M: int, count: int = 64, seed: int = 0) -> np.ndarray:
    """Deterministic sorted row sample: first, last, tile-boundary rows and random rows."""
    picks = {0, M - 1}
    for t in (16, 32, 64, 128, 256):
        for b in range(t, M, t * max(1, M // (t * 8))):
            picks.update({b - 1, b})
    rng = _rng(seed, 3)
    extra = rng.choice(M, size=min(M, count), replace=False)
    picks.update(int(e) for e in extra)
    out = sorted(p for p in picks if 0 <= p < M)
    if len(out) > count:
        keep = [0, M - 1] + [p for p in out if p not in (0, M - 1)]
        out = sorted(set(keep[:count]))
    return np.asarray(out, dtype=np.int64)


def make_norm_weight(K: int, seed: int = 0) -> np.ndarray:
    """FP16 RMSNorm weight [K] ~ 1 + 0.1 * N(0, 1)."""
    rng = _rng(seed, 4)
    return (1.0 + 0.1 * rng.standard_normal(K, dtype=np.float32)).astype(np.float16)


def make_gate_up(M: int, I: int, seed: int = 0) -> np.ndarray:
    """FP16 merged gate/up output [M][2I]: gate ~ N(0, 4), up ~ N(0, 1), each
    half with 4 outlier columns x20."""
    rng = _rng(seed, 5)
    gu = rng.standard_normal((M, 2 * I), dtype=np.float32)
    gu[:, :I] *= np.float32(2.0)
    for half in (0, 1):
        cols = half * I + rng.choice(I, size=min(N_OUTLIERS, I), replace=False)
        gu[:, cols] *= np.float32(OUTLIER_GAIN)
    return gu.astype(np.float16)


LLAMA3_8B_ATTN = dict(Hq=32, Hkv=8, D=128)   # Llama-3-8B attention heads (GQA 4:1)
N_KEY_OUTLIERS = 2
KEY_OUTLIER_GAIN = 8.0


def make_decode_attention(B: int, T: int, Hq: int, Hkv: int, D: int, seed: int = 0):
    """FP16 (q [B][Hq][D], K [B][Hkv][T][D], V [B][Hkv][T][D]) ~ N(0, 1), with
    2 outlier channels x8 per KV head in K."""
    rng = _rng(seed, 6)
    cols = np.stack([rng.choice(D, size=min(N_KEY_OUTLIERS, D), replace=False) for _ in range(Hkv)])
    q = rng.standard_normal((B, Hq, D), dtype=np.float32)
    K = rng.standard_normal((B, Hkv, T, D), dtype=np.float32)
    V = rng.standard_normal((B, Hkv, T, D), dtype=np.float32)
    for h in range(Hkv):
        K[:, h, :, cols[h]] *= np.float32(KEY_OUTLIER_GAIN)
    return q.astype(np.float16), K.astype(np.float16), V.astype(np.float16)
