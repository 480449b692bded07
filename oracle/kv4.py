"""Plain CPU reference of KV4 decode attention -- TEST INFRASTRUCTURE.

Only tests, the smoke check and the benchmark's CPU-baseline arm may use this
module. Like the rest of ``oracle/``, it shares no code with the CUDA library
(whose kernels implement the same definitions in kv4_attention.cu).

Sources (web summaries of QServe: W4A8KV4 Quantization and System Co-design
for Efficient LLM Serving, arXiv 2405.04532):
  [P3-5]  paperlayer.ai summary, section 5 "QServe Serving System" -- KV4
          attention needs per-head dynamic KV4 scaling factors and zero
          points; attention computes in FP16 on CUDA cores.
  [P3-6]  same page, section 6 "Evaluation" -- per-head asymmetric INT4 KV
          caches.
  [P3-3]  same page, section 3 -- KV4 doubles the peak attention performance
          over KV8 (attention is memory-bound at decode).

The pages fix the granularity (per head, dynamic, asymmetric, 4-bit) and not
the formulas. Readings ("reading:" in the docstrings):
  * One (scale, zero) pair per (sequence, KV head, token): the head_dim values
    of that token's key (or value) vector for that head, computed when the
    token is written ("dynamic"), nothing calibrated.
  * The quantiser is this repository's per-channel UINT4 reading (range
    extended to include 0, FP16 scale, integer zero stored exactly in FP16),
    applied to each such vector.
  * Decode attention (one query token per sequence), grouped-query: query head
    hq reads KV head hq // (Hq / Hkv). Scores q . k_hat / sqrt(D), softmax over
    the T cached tokens, output sum_t p_t v_hat_t, with k_hat and v_hat the
    dequantised vectors (q - z) * s. The pages put the arithmetic in FP16 on
    CUDA cores but fix no order of operations; the reference is the exact
    mathematics, evaluated in binary64 from the dequantised values (which are
    exact in binary32), and a kernel is compared against it with a tolerance.
"""
from __future__ import annotations

import numpy as np

from .qoq_ref import quantize_weights_per_channel


def quantize_kv4(X: np.ndarray):
    """FP16 [..., D] -> dict(q uint8 [..., D], s FP16 [...], z FP16 [...]).

    Each length-D vector along the last axis gets its own asymmetric UINT4
    scale and zero (per head, per token) [P3-5], [P3-6].
    reading: the per-channel quantiser of the W4A8 path, applied per vector:
    lo = min(0, min x), hi = max(0, max x), s = FP16((hi - lo) / 15),
    z = RNE(-lo / s), q = clamp(RNE(x / s) + z, 0, 15); s == 0 gives q = z = 0.
    """
    X = np.asarray(X, dtype=np.float16)
    lead, D = X.shape[:-1], X.shape[-1]
    d = quantize_weights_per_channel(X.reshape(-1, D))
    return dict(q=d["q"].reshape(*lead, D), s=d["s"].reshape(lead), z=d["z"].reshape(lead))


def pack_kv4(q: np.ndarray) -> np.ndarray:
    """Codes [..., D] (0..15) -> the cache's bytes [..., D/2]: byte j holds
    q[2j] in its low nibble and q[2j+1] in its high nibble (this repository's
    layout; the pages fix only the 4-bit width)."""
    q = np.asarray(q, dtype=np.uint8)
    return (q[..., 0::2] | (q[..., 1::2] << 4)).astype(np.uint8)


def dequantize_kv4(q: np.ndarray, s: np.ndarray, z: np.ndarray) -> np.ndarray:
    """(q - z) * s in binary32. (q - z) is an integer in [-15, 15] and s an FP16
    value, so every product is exact in binary32 (at most 15 significant bits)."""
    qi = q.astype(np.int32) - z.astype(np.float32).astype(np.int32)[..., None]
    return qi.astype(np.float32) * s.astype(np.float32)[..., None]


def decode_attention(q: np.ndarray, Kq: dict, Vq: dict) -> np.ndarray:
    """One query token per sequence against a KV4 cache, grouped-query.

    q [B][Hq][D] FP16; Kq, Vq from quantize_kv4 on [B][Hkv][T][D]. Returns the
    binary64 output [B][Hq][D]:
        k_hat, v_hat = dequantised K, V;  h = hq // (Hq / Hkv)
        score_t = (q . k_hat_t) / sqrt(D);  p = softmax(score);  o = sum_t p_t v_hat_t
    reading: exact mathematics in binary64 (see the module docstring).
    """
    q64 = np.asarray(q, dtype=np.float16).astype(np.float64)
    B, Hq, D = q64.shape
    k = dequantize_kv4(Kq["q"], Kq["s"], Kq["z"]).astype(np.float64)
    v = dequantize_kv4(Vq["q"], Vq["s"], Vq["z"]).astype(np.float64)
    Hkv = k.shape[1]
    if Hq % Hkv:
        raise ValueError("query heads must be a multiple of KV heads")
    group = Hq // Hkv
    out = np.empty((B, Hq, D), dtype=np.float64)
    for b in range(B):
        for hq in range(Hq):
            h = hq // group
            score = (k[b, h] @ q64[b, hq]) / np.sqrt(D)
            e = np.exp(score - score.max())
            p = e / e.sum()
            out[b, hq] = p @ v[b, h]
    return out


def decode_attention_fp16(q, K, V) -> np.ndarray:
    """The whole path from FP16 q, K, V: KV4 quantisation, then attention,
    output rounded once to FP16."""
    return decode_attention(q, quantize_kv4(K), quantize_kv4(V)).astype(np.float16)
