"""The allocation-free GEMM entry point (qoq_gemm_fp16_out_static_ws).

Some callers cannot allocate device memory: code that runs inside a memory
arena planned at start-up, a host thread that must stay out of the device
allocator while other work owns it, or an embedding runtime that forbids
cudaMalloc after initialisation. This entry point keeps its stream-K scratch
in a fixed device array inside the library instead of a caller workspace.
It runs the same kernel as qoq_gemm_fp16_out, so its output must equal that
call's bit for bit, call after call, and match the CPU oracle. Collected
last, and self-contained so it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

QOQ_ERR_WORKSPACE = 4
QOQ_ERR_BAD_BLOB = 5


def _fn():
    from w4a8_quantized_gemm_qoq_b200 import build, qoq
    build.build()
    f = qoq.lib().qoq_gemm_fp16_out_static_ws
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [vp, vp, vp, vp, i64, i64, i64, ctypes.c_int, vp, vp, vp]
    f.restype = ctypes.c_int
    return f


def _call(f, X8, s_x, rowsum, blob, M, N, K, Y, status, group=128):
    import torch
    p = lambda t: ctypes.c_void_p(t.data_ptr())   # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return f(p(X8), p(s_x), p(rowsum), p(blob), M, N, K, group, p(Y), p(status), stream)


def _oracle_tiles(X, W, Y, tiles):
    """Oracle FP16 output on the given 128-row n-tiles, compared with Y."""
    import oracle
    X8, s_x, _ = oracle.quantize_act_per_token(X)
    for nt in tiles:
        _, d = oracle.quantize_weights(W[nt * 128:(nt + 1) * 128], 128)
        want = oracle.epilogue_fp16(oracle.gemm_int(X8, d["Wint"]), s_x, d["s_w"])
        got = Y[:, nt * 128:(nt + 1) * 128]
        dist = oracle.fp16_ulp_distance(got, want)
        assert dist.max() <= 1, "tile %d: %d ulp from the oracle" % (nt, dist.max())


@pytest.mark.parametrize("N,K,Ms", [(4096, 4096, (16, 64)), (28672, 4096, (64, 33))])
def test_static_scratch_matches_workspace_gemm_twice(N, K, Ms):
    """Two calls in a row on one weight matrix: each output equals the
    workspace call's bit for bit and the oracle on sampled n-tiles. The second
    shape makes the library pick 64-token tiles at M = 64, the largest scratch
    it accepts (148 CTAs x 64 x 128 INT32 partial sums)."""
    import torch
    from w4a8_quantized_gemm_qoq_b200 import inputs, qoq
    assert torch.cuda.is_available()
    f = _fn()
    W = inputs.make_weights(N, K, seed=21)
    blob = qoq.quantize_weights(torch.from_numpy(W).cuda(), 128)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call, M in enumerate(Ms):
        X = inputs.make_activations(M, K, seed=22 + call)
        X8, s_x, rowsum = qoq.quantize_act_per_token(torch.from_numpy(X).cuda())
        ref = qoq.gemm_fp16_out(X8, s_x, blob, N, K, 128, rowsum=rowsum)
        Y = torch.full((M, N), 7.0, dtype=torch.float16, device="cuda")
        rc = _call(f, X8, s_x, rowsum, blob, M, N, K, Y, status)
        assert rc == 0, "call %d returned %d" % (call, rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(Y.view(torch.int16), ref.view(torch.int16)), "call %d differs from the workspace GEMM" % call
        _oracle_tiles(X, W, Y.cpu().numpy(), [0, N // 256, N // 128 - 1])


def test_static_scratch_bad_blob_then_good_call():
    """A call whose blob header does not match its arguments reports
    QOQ_ERR_BAD_BLOB in its status without touching the output; the next
    good call on the same shared array starts from cleared control words and
    reports 0 with the right result."""
    import torch
    from w4a8_quantized_gemm_qoq_b200 import inputs, qoq
    f = _fn()
    N, K, M = 4096, 4096, 16
    W = inputs.make_weights(N, K, seed=24)
    blob = qoq.quantize_weights(torch.from_numpy(W).cuda(), 128)
    X = inputs.make_activations(M, K, seed=25)
    X8, s_x, rowsum = qoq.quantize_act_per_token(torch.from_numpy(X).cuda())
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    Yb = torch.full((M, N // 2), 7.0, dtype=torch.float16, device="cuda")
    assert _call(f, X8, s_x, rowsum, blob, M, N // 2, K, Yb, status) == 0   # claims N/2 for an N-row blob
    torch.cuda.synchronize()
    assert int(status.item()) == QOQ_ERR_BAD_BLOB
    assert bool((Yb == 7.0).all().item())
    ref = qoq.gemm_fp16_out(X8, s_x, blob, N, K, 128, rowsum=rowsum)
    Y = torch.full((M, N), 7.0, dtype=torch.float16, device="cuda")
    assert _call(f, X8, s_x, rowsum, blob, M, N, K, Y, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(Y.view(torch.int16), ref.view(torch.int16))


def test_static_scratch_rejects_too_large():
    f = _fn()
    p = ctypes.c_void_p(1 << 20)   # never dereferenced: the size check fails first
    rc = f(p, p, None, p, 4096, 4096, 4096, 128, p, None, None)
    assert rc == QOQ_ERR_WORKSPACE
