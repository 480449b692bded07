"""KV4 cache and decode attention on the GPU against the CPU oracle
(oracle/kv4.py), through the C ABI.

Bar: the cache write (codes, FP16 scales, FP16 zeros) bit-exact; the
attention output within the tolerance stated in tests/kv4_check.py, which
holds the shared attention checks and is also run in processes of its own
with longer warp walks forced.
"""
import numpy as np
import pytest

from oracle import kv4
from w4a8_quantized_gemm_qoq_b200 import inputs, qoq
from gpu_helpers import dev, host, torch
from kv4_check import check_attention, run_attention

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch().cuda.is_available(), "GPU tests need a CUDA device"
    from w4a8_quantized_gemm_qoq_b200 import build
    build.build()
    yield


def _check_cache(cache, X, t0=0):
    """The cache's slots t0 .. t0 + n against the oracle's quantiser of X."""
    d = kv4.quantize_kv4(X)
    n = X.shape[2]
    codes = host(cache.codes)[:, :, t0:t0 + n]
    s = host(cache.scales)[:, :, t0:t0 + n]
    z = host(cache.zeros)[:, :, t0:t0 + n]
    assert np.array_equal(codes, kv4.pack_kv4(d["q"])), "codes"
    assert np.array_equal(s.view(np.uint16), d["s"].view(np.uint16)), "scales"
    assert np.array_equal(z.view(np.uint16), d["z"].view(np.uint16)), "zeros"


@pytest.mark.parametrize("D", [64, 128])
def test_cache_write_bit_exact(D):
    """Random heads plus degenerate vectors: zeros, positive and negative
    constants, one-hot, FP16 extremes and subnormals."""
    _, K, V = inputs.make_decode_attention(3, 37, 8, 4, D, seed=D)
    K[0, 0, 0] = 0
    K[0, 0, 1] = 1.875
    K[0, 0, 2] = -1.875
    K[0, 0, 3] = 0
    K[0, 0, 3, 5] = -3.0
    K[0, 1, 0] = 65504.0
    K[0, 1, 1, ::2] = -65504.0
    K[0, 1, 2] = np.float16(6e-8)
    K[0, 1, 3] = np.linspace(-1e-5, 3e-6, D).astype(np.float16)
    for X in (K, V):
        c = qoq.KV4Cache(3, 4, 40, D).write(dev(X))
        torch().cuda.synchronize()
        _check_cache(c, X)


def test_cache_append_one_token():
    """A full write of T - 1 tokens, then the decode step's new token into
    slot T - 1 of a larger cache: every slot equals the oracle's."""
    _, K, _ = inputs.make_decode_attention(4, 25, 32, 8, 128, seed=3)
    c = qoq.KV4Cache(4, 8, 64, 128)
    c.write(dev(np.ascontiguousarray(K[:, :, :24])))
    c.write(dev(np.ascontiguousarray(K[:, :, 24:25])), t0=24)
    torch().cuda.synchronize()
    _check_cache(c, K)


_attention = run_attention
_check_attention = check_attention


@pytest.mark.parametrize("B,T,Hq,Hkv,D", [(2, 1, 8, 8, 128), (3, 7, 8, 2, 64), (2, 128, 32, 8, 128),
                                          (2, 129, 32, 8, 128), (4, 300, 4, 1, 128), (2, 1000, 16, 2, 64),
                                          (3, 517, 24, 3, 128)])
def test_decode_attention_matches_oracle(B, T, Hq, Hkv, D):
    """One chunk (direct output), several chunks (combined by the last
    arriving CTA), ragged last chunks, group sizes 1 to 8, D = 64 and 128."""
    q, K, V = inputs.make_decode_attention(B, T, Hq, Hkv, D, seed=T + D)
    out, _ = _attention(q, K, V)
    _check_attention(out, q, K, V)


def test_decode_attention_ragged_sequence_lengths():
    """Per-sequence lengths inside a 600-slot cache: sequences of 1, 128, 129,
    450 and 600 tokens; slots past a sequence's length hold other data and
    must not count."""
    lens = [1, 128, 129, 450, 600]
    q, K, V = inputs.make_decode_attention(5, 600, 32, 8, 128, seed=11)
    out, _ = _attention(q, K, V, seq_lens=lens)
    _check_attention(out, q, K, V, seq_lens=lens)


def test_decode_attention_llama3_8b_batch64_1k():
    """The pages' attention measurement shape: batch 64, 1024 cached tokens,
    Llama-3-8B heads (32 query heads over 8 KV heads, D = 128)."""
    a = inputs.LLAMA3_8B_ATTN
    q, K, V = inputs.make_decode_attention(64, 1024, a["Hq"], a["Hkv"], a["D"], seed=12)
    out, _ = _attention(q, K, V)
    _check_attention(out, q, K, V)


def test_decode_attention_graph_replays():
    """Back-to-back calls in a CUDA graph, 20 replays: outputs identical to
    the eager call's, counters left zero every time."""
    t = torch()
    q, K, V = inputs.make_decode_attention(8, 700, 32, 8, 128, seed=13)
    out0, (kc, vc, ws, _) = _attention(q, K, V)
    qd = dev(q)
    out = t.empty((8, 32, 128), dtype=t.float16, device="cuda")
    stream = t.cuda.Stream()
    stream.wait_stream(t.cuda.current_stream())
    with t.cuda.stream(stream):
        qoq.kv4_decode_attention(qd, kc, vc, ws=ws, out=out)
    stream.synchronize()
    g = t.cuda.CUDAGraph()
    with t.cuda.graph(g, stream=stream):
        for _ in range(3):
            qoq.kv4_decode_attention(qd, kc, vc, ws=ws, out=out)
    for _ in range(20):
        with t.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        assert np.array_equal(host(out).view(np.uint16), out0.view(np.uint16))
        assert not bool(ws.buf[:256 + 4 * 8 * 8].any().item())


@pytest.mark.parametrize("kvt", [2, 3, 8])
def test_decode_attention_longer_warp_walks(kvt):
    """Every warp walks up to kvt 64-token tiles (QOQ_FORCE_CONFIG=kvt=N, in a
    process of its own), refilling its K and V buffers while it computes:
    ragged last tiles, warps with fewer tiles than others, spans longer than
    the sequence."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, QOQ_FORCE_CONFIG="kvt=%d" % kvt)
    r = subprocess.run([sys.executable, os.path.join(here, "kv4_check.py")], env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0 and "kv4_check ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
