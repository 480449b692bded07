"""KV4 decode attention against the CPU oracle (oracle/kv4.py), shared by
tests/test_gpu_kv4.py and run as a script in a process of its own, so that
the launch configuration (QOQ_FORCE_CONFIG, read once per process) can be
set: with kvt=N every warp walks up to N 64-token tiles, refilling its K and
V buffers while it computes.

    QOQ_FORCE_CONFIG=kvt=3 python tests/kv4_check.py

Bar: |o - o*| <= 2^-10 * max_t |v_hat_t| + 2^-24 per (sequence, query head),
with o* the exact mathematics (binary64) and max_t |v_hat_t| the largest
dequantised value of that sequence's V. The bound: the kernel rounds the
softmax weights times the value scale to FP16 for the tensor-core product
(relative error <= 2^-11 per weight, so at most 2^-11 max|v_hat| on the
weighted mean), rounds the output once to FP16 (at most 2^-11 |o*| <=
2^-11 max|v_hat|), and sums in FP32 (errors near 2^-20 relative, inside the
slack of the first two terms' worst cases).
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

from oracle import kv4  # noqa: E402
from gpu_helpers import dev, host, torch  # noqa: E402
from w4a8_quantized_gemm_qoq_b200 import build, inputs, qoq  # noqa: E402


def run_attention(q, K, V, Tmax=None, seq_lens=None):
    """Caches written from K and V, one attention call; checks that the
    workspace's status words and arrival counters are left zero."""
    B, Hkv, T, D = K.shape
    Hq = q.shape[1]
    Tmax = Tmax or T
    kc = qoq.KV4Cache(B, Hkv, Tmax, D).write(dev(K))
    vc = qoq.KV4Cache(B, Hkv, Tmax, D).write(dev(V))
    ws = qoq.Workspace(qoq.kv4_workspace_bytes(B, Hq, Hkv, Tmax, D))
    sl = dev(np.asarray(seq_lens, dtype=np.int32)) if seq_lens is not None else None
    out = qoq.kv4_decode_attention(dev(q), kc, vc, seq_lens=sl, ws=ws)
    torch().cuda.synchronize()
    assert not bool(ws.buf[:256 + 4 * B * Hkv].any().item()), "status word set or counters not left zero"
    return host(out), (kc, vc, ws, sl)


def check_attention(out, q, K, V, seq_lens=None):
    """The bar above for every (sequence, query head); returns the worst
    error as a fraction of its bound."""
    B, Hkv, T, D = K.shape
    Hq = q.shape[1]
    G = Hq // Hkv
    worst = 0.0
    for b in range(B):
        Tb = T if seq_lens is None else int(seq_lens[b])
        Kb = kv4.quantize_kv4(K[b:b + 1, :, :Tb])
        Vb = kv4.quantize_kv4(V[b:b + 1, :, :Tb])
        want = kv4.decode_attention(q[b:b + 1], Kb, Vb)[0]
        vh = np.abs(kv4.dequantize_kv4(Vb["q"], Vb["s"], Vb["z"]).astype(np.float64))[0]
        for hq in range(Hq):
            vmax = vh[hq // G].max()
            err = np.abs(out[b, hq].astype(np.float64) - want[hq]).max()
            tol = 2.0 ** -10 * vmax + 2.0 ** -24
            assert err <= tol, "b=%d hq=%d: error %.3g above %.3g" % (b, hq, err, tol)
            worst = max(worst, err / tol)
    return worst


CASES = [(2, 1000, 16, 2, 64), (3, 517, 24, 3, 128), (4, 300, 4, 1, 128), (2, 129, 32, 8, 128),
         (8, 1024, 32, 8, 128), (1, 2000, 8, 1, 64)]


def main():
    build.build()
    worst = 0.0
    for B, T, Hq, Hkv, D in CASES:
        q, K, V = inputs.make_decode_attention(B, T, Hq, Hkv, D, seed=T + D + 1)
        out, _ = run_attention(q, K, V)
        worst = max(worst, check_attention(out, q, K, V))
    lens = [1, 128, 129, 450, 600]
    q, K, V = inputs.make_decode_attention(5, 600, 32, 8, 128, seed=21)
    out, _ = run_attention(q, K, V, seq_lens=lens)
    worst = max(worst, check_attention(out, q, K, V, seq_lens=lens))
    print("kv4_check ok (worst error %.3f of its bound)" % worst)


if __name__ == "__main__":
    main()
