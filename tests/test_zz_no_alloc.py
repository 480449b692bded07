"""The allocation-free GEMM entry point (qoq_gemm_fp16_out_static_ws).

Some callers cannot allocate device memory (pre-planned arenas, threads that
must stay out of the device allocator, runtimes that forbid cudaMalloc after
start-up); this entry point keeps its stream-K scratch in a fixed device
array inside the library. Its output must match qoq_gemm_fp16_out with a
caller workspace, call after call. Collected last, and self-contained so it
also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _fn():
    from w4a8_quantized_gemm_qoq_b200 import build, qoq
    build.build()
    f = qoq.lib().qoq_gemm_fp16_out_static_ws
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [vp, vp, vp, vp, i64, i64, i64, ctypes.c_int, vp, vp, vp]
    f.restype = ctypes.c_int
    return f


def test_static_scratch_matches_workspace_gemm_twice():
    import torch
    import oracle
    from w4a8_quantized_gemm_qoq_b200 import inputs, qoq
    assert torch.cuda.is_available()
    f = _fn()
    N, K = 4096, 4096   # decode shape: every tile is shared between CTAs
    W = torch.from_numpy(inputs.make_weights(N, K, seed=21)).cuda()
    blob = qoq.quantize_weights(W, 128)
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call, (M, seed) in enumerate([(16, 22), (64, 23)]):
        X = torch.from_numpy(inputs.make_activations(M, K, seed=seed)).cuda()
        X8, s_x, rowsum = qoq.quantize_act_per_token(X)
        ref = qoq.gemm_fp16_out(X8, s_x, blob, N, K, 128, rowsum=rowsum)
        Y = torch.full((M, N), 7.0, dtype=torch.float16, device="cuda")
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        rc = f(ctypes.c_void_p(X8.data_ptr()), ctypes.c_void_p(s_x.data_ptr()), ctypes.c_void_p(rowsum.data_ptr()),
               ctypes.c_void_p(blob.data_ptr()), M, N, K, 128, ctypes.c_void_p(Y.data_ptr()),
               ctypes.c_void_p(status.data_ptr()), stream)
        assert rc == 0, "call %d returned %d" % (call, rc)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        d = oracle.fp16_ulp_distance(Y.cpu().numpy(), ref.cpu().numpy())
        assert d.max() <= 1, "call %d: %d ulp" % (call, d.max())


def test_static_scratch_rejects_too_large():
    import torch
    from w4a8_quantized_gemm_qoq_b200 import qoq
    f = _fn()
    p = ctypes.c_void_p(1 << 20)   # never dereferenced: the size check fails first
    rc = f(p, p, None, p, 4096, 4096, 4096, 128, p, None, None)
    assert rc == 4   # QOQ_ERR_WORKSPACE
