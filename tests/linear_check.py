"""Checks of qoq_w4a8_linear run in a process of their own, so that the
launch configuration (QOQ_FORCE_CONFIG, read once per process) can be set
for it: the one-call output against the two-call path (bit for bit) and the
CPU oracle (within 1 ulp), and graph replays of back-to-back calls.

    QOQ_FORCE_CONFIG=fuse=1 python tests/linear_check.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle  # noqa: E402
from gpu_helpers import assert_fp16_close, dev, host, sample_tiles, torch  # noqa: E402
from w4a8_quantized_gemm_qoq_b200 import build, inputs, qoq  # noqa: E402


def oracle_tile(X, W, nt, group):
    X8, s_x, rs = oracle.quantize_act_per_token(X)
    _, d = oracle.quantize_weights(W[nt * 128:(nt + 1) * 128], group)
    if group:
        return oracle.epilogue_fp16(oracle.gemm_int(X8, d["Wint"]), s_x, d["s_w"])
    return oracle.epilogue_fp16(oracle.w4a8_gemm_per_channel(X8, rs, d["q"], d["z"]), s_x, d["s"])


def main():
    t = torch()
    build.build()
    expect = int(sys.argv[1]) if len(sys.argv) > 1 else None   # launches per decode call expected
    cases = [(1, 4096, 4096), (7, 384, 640), (16, 6144, 4096), (33, 28672, 4096), (64, 4096, 14336),
             (100, 512, 640), (256, 4096, 4096)]
    for group in (128, 0):
        for M, N, K in cases:
            tok, nl = qoq.plan(M, N, K)
            if expect is not None and tok <= 64:
                assert nl == expect, "M=%d N=%d K=%d: %d launches, expected %d" % (M, N, K, nl, expect)
            X = inputs.make_activations(M, K, seed=900 + M)
            W = inputs.make_weights(N, K, seed=900 + N)
            Xd = dev(X)
            blob = qoq.quantize_weights(dev(W), group)
            ws = qoq.Workspace.for_linear(M, N, K, group)
            Y = qoq.linear(Xd, blob, N, K, group, ws=ws)
            X8, s_x, rs = qoq.quantize_act_per_token(Xd)
            Y2 = qoq.gemm_fp16_out(X8, s_x, blob, N, K, group, rowsum=rs)
            t.cuda.synchronize()
            assert ws.status() == 0, "status %d %s" % (ws.status(), ws.timeout_site())
            assert ws.control_clear()
            assert t.equal(Y.view(t.int16), Y2.view(t.int16)), "M=%d N=%d K=%d g=%d: paths differ" % (M, N, K, group)
            Yh = host(Y)
            for nt in sample_tiles(N // 128, count=2, seed=M):
                assert_fp16_close(Yh[:, nt * 128:(nt + 1) * 128], oracle_tile(X, W, nt, group), "linear tile")
    # back-to-back calls in a graph, 20 replays
    probs = []
    for i, (K, N, _) in enumerate(inputs.LLAMA3_8B):
        M = (1, 16, 33, 64)[i]
        X = inputs.make_activations(M, K, seed=950 + i)
        W = inputs.make_weights(N, K, seed=950 + i)
        probs.append(dict(N=N, K=K, Xd=dev(X), blob=qoq.quantize_weights(dev(W), 128),
                          Y=t.empty((M, N), dtype=t.float16, device="cuda"), ws=qoq.Workspace.for_linear(M, N, K)))
    stream = t.cuda.Stream()
    stream.wait_stream(t.cuda.current_stream())

    def step():
        for p in probs:
            qoq.linear(p["Xd"], p["blob"], p["N"], p["K"], 128, ws=p["ws"], Y=p["Y"])
    with t.cuda.stream(stream):
        step()
    stream.synchronize()
    ref = [p["Y"].clone() for p in probs]
    g = t.cuda.CUDAGraph()
    with t.cuda.graph(g, stream=stream):
        step()
    for r in range(20):
        with t.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        for i, p in enumerate(probs):
            assert p["ws"].status() == 0 and p["ws"].control_clear(), "replay %d case %d" % (r, i)
            assert t.equal(p["Y"], ref[i]), "replay %d case %d differs" % (r, i)
    print("linear_check ok")


if __name__ == "__main__":
    main()
