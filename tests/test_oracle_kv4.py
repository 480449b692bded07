"""Pins of the KV4 decode-attention reference (oracle/kv4.py) against closed
forms, bounds and invariants, so that a plausible mistake (wrong quantisation
granularity, a flipped zero point, a dropped 1/sqrt(D), the softmax over the
wrong axis, the wrong query-head to KV-head map, K and V swapped) fails."""
import math

import numpy as np
import pytest

from oracle import kv4
from w4a8_quantized_gemm_qoq_b200 import inputs


def test_quantisation_is_per_token_per_head():
    """Each length-D vector has its own scale and zero: quantising the whole
    cache equals quantising every vector on its own."""
    _, K, _ = inputs.make_decode_attention(2, 5, 8, 4, 32, seed=1)
    d = kv4.quantize_kv4(K)
    assert d["q"].shape == K.shape and d["s"].shape == K.shape[:-1] and d["z"].shape == K.shape[:-1]
    for b in range(2):
        for h in range(4):
            for t in range(5):
                one = kv4.quantize_kv4(K[b, h, t][None])
                assert np.array_equal(one["q"][0], d["q"][b, h, t])
                assert one["s"][0] == d["s"][b, h, t] and one["z"][0] == d["z"][b, h, t]


def test_quantisation_closed_forms():
    """Vectors that the 16-level grid holds exactly come back exactly: a
    positive constant 15/8 (s = 1/8, z = 0, codes 15), its negation (z = 15,
    codes 0), zeros (s = 0), and points of the grid {(j - z) s}."""
    X = np.zeros((4, 8), dtype=np.float16)
    X[0] = 1.875
    X[1] = -1.875
    X[3] = (np.array([0, 3, 7, 15, 1, 2, 9, 12]) - 4) * 0.25   # lo = -1, hi = 2.75 -> s = 0.25, z = 4
    d = kv4.quantize_kv4(X)
    assert d["s"][0] == np.float16(0.125) and d["z"][0] == 0 and np.all(d["q"][0] == 15)
    assert d["s"][1] == np.float16(0.125) and d["z"][1] == 15 and np.all(d["q"][1] == 0)
    assert d["s"][2] == 0 and d["z"][2] == 0 and np.all(d["q"][2] == 0)
    assert d["s"][3] == np.float16(0.25) and d["z"][3] == 4
    back = kv4.dequantize_kv4(d["q"], d["s"], d["z"])
    assert np.array_equal(back, X.astype(np.float32))


def test_dequantisation_error_bound():
    """|x_hat - x| <= s/2, up to the FP16 rounding of the scale at the range's
    ends (where a code can round one step past the range and be clamped)."""
    _, K, V = inputs.make_decode_attention(3, 17, 8, 2, 128, seed=2)
    for X in (K, V):
        d = kv4.quantize_kv4(X)
        err = np.abs(kv4.dequantize_kv4(d["q"], d["s"], d["z"]) - X.astype(np.float32))
        s = d["s"].astype(np.float32)[..., None]
        span = (np.maximum(X.max(-1), 0) - np.minimum(X.min(-1), 0)).astype(np.float32)[..., None]
        assert np.all(err <= 0.5 * s + span * 2.0 ** -10 + 1e-7)
        assert np.mean(err <= 0.5 * s + 1e-7) > 0.999


def _cache(K, V):
    return kv4.quantize_kv4(K), kv4.quantize_kv4(V)


def test_single_token_returns_its_value():
    """T = 1: the softmax of one score is 1, so every query head reads back the
    dequantised value vector of its KV head."""
    q, K, V = inputs.make_decode_attention(2, 1, 8, 2, 64, seed=3)
    Kq, Vq = _cache(K, V)
    o = kv4.decode_attention(q, Kq, Vq)
    v = kv4.dequantize_kv4(Vq["q"], Vq["s"], Vq["z"]).astype(np.float64)
    for hq in range(8):
        assert np.array_equal(o[:, hq], v[:, hq // 4, 0])


def test_zero_query_averages_the_values():
    """q = 0: all scores are equal, so the output is the mean of the values."""
    _, K, V = inputs.make_decode_attention(1, 9, 4, 4, 16, seed=4)
    q = np.zeros((1, 4, 16), dtype=np.float16)
    Kq, Vq = _cache(K, V)
    o = kv4.decode_attention(q, Kq, Vq)
    v = kv4.dequantize_kv4(Vq["q"], Vq["s"], Vq["z"]).astype(np.float64)
    assert np.allclose(o[0], v[0].mean(axis=1), rtol=0, atol=1e-12)


def test_two_tokens_follow_the_logistic():
    """Keys 0 and (15/8, 0, 0, 0) with query (1, 0, 0, 0), D = 4: scores 0 and
    15/8 / sqrt(4), so the second token's weight is 1 / (1 + e^(-15/16))."""
    K = np.zeros((1, 1, 2, 4), dtype=np.float16)
    K[0, 0, 1, 0] = 1.875
    V = np.array([[[[1.0, -2.0, 0.5, 0.0], [3.0, 1.0, -1.0, 2.0]]]], dtype=np.float16)
    q = np.array([[[1.0, 0.0, 0.0, 0.0]]], dtype=np.float16)
    Kq, Vq = _cache(K, V)
    assert np.array_equal(kv4.dequantize_kv4(Kq["q"], Kq["s"], Kq["z"]), K.astype(np.float32))
    v = kv4.dequantize_kv4(Vq["q"], Vq["s"], Vq["z"]).astype(np.float64)[0, 0]
    p1 = 1.0 / (1.0 + math.exp(-1.875 / 2.0))
    want = (1.0 - p1) * v[0] + p1 * v[1]
    assert np.allclose(kv4.decode_attention(q, Kq, Vq)[0, 0], want, rtol=0, atol=1e-14)


def test_grouped_query_heads_map_to_their_kv_head():
    """Hq = 4, Hkv = 2: query heads 0, 1 read KV head 0 and 2, 3 read head 1.
    Equal queries in one group give equal outputs; swapping the two KV heads
    swaps the two groups' outputs."""
    q, K, V = inputs.make_decode_attention(1, 6, 4, 2, 32, seed=5)
    q[0, 1] = q[0, 0]
    q[0, 3] = q[0, 2]
    Kq, Vq = _cache(K, V)
    o = kv4.decode_attention(q, Kq, Vq)
    assert np.array_equal(o[0, 0], o[0, 1]) and np.array_equal(o[0, 2], o[0, 3])
    qs = q[:, [2, 3, 0, 1]]
    Ks, Vs = _cache(K[:, ::-1].copy(), V[:, ::-1].copy())
    os_ = kv4.decode_attention(qs, Ks, Vs)
    assert np.allclose(os_[0], o[0, [2, 3, 0, 1]], rtol=0, atol=1e-12)


def test_token_order_does_not_matter():
    q, K, V = inputs.make_decode_attention(2, 11, 8, 2, 32, seed=6)
    perm = np.random.default_rng(0).permutation(11)
    a = kv4.decode_attention(q, *_cache(K, V))
    b = kv4.decode_attention(q, *_cache(K[:, :, perm].copy(), V[:, :, perm].copy()))
    assert np.allclose(a, b, rtol=0, atol=1e-12)


def test_dominant_score_selects_its_value():
    """One key aligned with the query far above the others: the output is that
    token's value to within e^(-gap)."""
    D = 8
    K = np.zeros((1, 1, 4, D), dtype=np.float16)
    K[0, 0, 2, :] = 7.5                      # score 8 * 7.5 * 2 / sqrt(8), others 0
    V = inputs.make_decode_attention(1, 4, 1, 1, D, seed=7)[2]
    q = np.full((1, 1, D), 2.0, dtype=np.float16)
    Kq, Vq = _cache(K, V)
    v = kv4.dequantize_kv4(Vq["q"], Vq["s"], Vq["z"]).astype(np.float64)[0, 0]
    gap = 8 * 7.5 * 2.0 / math.sqrt(D)
    o = kv4.decode_attention(q, Kq, Vq)[0, 0]
    assert np.allclose(o, v[2], rtol=0, atol=4 * math.exp(-gap) * np.abs(v).max() + 1e-12)


def test_fp16_output_is_the_rounded_reference():
    q, K, V = inputs.make_decode_attention(1, 16, 8, 2, 128, seed=8)
    o = kv4.decode_attention_fp16(q, K, V)
    assert o.dtype == np.float16
    assert np.array_equal(o, kv4.decode_attention(q, *_cache(K, V)).astype(np.float16))


@pytest.mark.parametrize("D", [64, 128])
def test_llama3_8b_heads_shape(D):
    q, K, V = inputs.make_decode_attention(2, 8, inputs.LLAMA3_8B_ATTN["Hq"], inputs.LLAMA3_8B_ATTN["Hkv"], D,
                                           seed=9)
    o = kv4.decode_attention(q, *_cache(K, V))
    assert o.shape == (2, 32, D) and np.all(np.isfinite(o))


def test_pack_kv4_hand_worked():
    """Codes 1, 2, 3, ..., 8 pack to bytes 0x21, 0x43, 0x65, 0x87 (low nibble
    the even dimension); 15, 0 -> 0x0F; 0, 15 -> 0xF0."""
    q = np.array([[1, 2, 3, 4, 5, 6, 7, 8], [15, 0, 0, 15, 9, 9, 0, 0]], dtype=np.uint8)
    assert kv4.pack_kv4(q).tolist() == [[0x21, 0x43, 0x65, 0x87], [0x0F, 0xF0, 0x99, 0x00]]
