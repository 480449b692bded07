"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/qoq.h declares, answers size queries, and rejects bad
arguments before launching anything."""
import ctypes
import os
import re

import pytest

from w4a8_quantized_gemm_qoq_b200 import qoq
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names.update(re.findall(r"\b(qoq_[a-z0-9_]+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def L():
    from w4a8_quantized_gemm_qoq_b200 import build
    build.build()
    return qoq.lib()


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert {"qoq_quantize_weights", "qoq_quantize_act_per_token", "qoq_w4a8_gemm",
            "qoq_gemm_fp16_out"} <= names
    for n in sorted(names):
        assert hasattr(L, n), n
    assert L.qoq_status_string(4) == b"QOQ_ERR_WORKSPACE"


def test_blob_size_query_matches_layout(L):
    for N, K, g in [(128, 128, 128), (256, 512, 128), (4096, 14336, 128), (12288, 4096, 0), (384, 640, 0)]:
        assert qoq.blob_bytes(N, K, g) == oracle.blob_layout(N, K, g)["total"]


def test_linear_workspace_size_query(L):
    """qoq_w4a8_linear's workspace holds the GEMM's scratch and, after it, the
    quantised activations: codes [M][K], FP16 scales and int32 row sums."""
    for M, N, K in [(1, 4096, 4096), (64, 28672, 4096), (300, 512, 640), (2048, 4096, 14336)]:
        gemm = qoq.workspace_bytes(M, N, K)
        lin = qoq.linear_workspace_bytes(M, N, K)
        assert lin >= gemm + M * K + 2 * M + 4 * M
        assert lin <= gemm + M * K + 6 * M + 3 * 256


def test_plan_query(L):
    """Token tiles and launch counts of the one-call linear path: two launches
    (quantiser, then GEMM) unless the token tile is at most 64 and the fused
    launch is selected, and always two for prefill batches."""
    tok, nl = qoq.plan(1, 4096, 4096)
    assert tok == 16 and nl in (1, 2)
    assert qoq.plan(64, 28672, 4096)[0] == 64
    assert qoq.plan(2048, 28672, 4096) == (256, 2)
    assert L.qoq_plan(4, 100, 128, None, None) == 2


def test_kv4_argument_validation_without_launch(L):
    dummy = ctypes.c_void_p(16 * 1024)   # never dereferenced: every call below fails validation first
    w = L.qoq_kv4_cache_write
    assert w(dummy, 2, 8, 64, 0, 64, 96, dummy, dummy, dummy, None) == 2      # D not 64 or 128
    assert w(dummy, 2, 8, 64, 10, 60, 128, dummy, dummy, dummy, None) == 1    # past max_tokens
    assert w(None, 2, 8, 64, 0, 4, 128, dummy, dummy, dummy, None) == 1       # no source
    assert w(ctypes.c_void_p(16 * 1024 + 8), 2, 8, 64, 0, 4, 128, dummy, dummy, dummy, None) == 3
    assert w(None, 0, 8, 64, 0, 4, 128, None, None, None, None) == 0          # B = 0: no-op
    a = L.qoq_kv4_decode_attention
    n = ctypes.c_size_t(0)
    assert a(*([None] * 8), 64, 32, 8, 1024, 128, None, None, ctypes.byref(n), None) == 0
    assert n.value == qoq.kv4_workspace_bytes(64, 32, 8, 1024, 128) > 4 * 64 * 8
    assert a(*([dummy] * 8), 2, 30, 8, 64, 128, dummy, dummy, _sz(1 << 30), None) == 2   # Hq % Hkv
    assert a(*([dummy] * 8), 2, 72, 8, 64, 128, dummy, dummy, _sz(1 << 30), None) == 2   # group of 9
    assert a(*([dummy] * 8), 2, 32, 8, 64, 128, dummy, dummy, _sz(8), None) == 4         # workspace too small
    assert a(*([dummy] * 8), 2, 32, 8, 64, 128, dummy, ctypes.c_void_p(16 * 1024 + 16), _sz(1 << 30),
             None) == 3                                                                    # workspace alignment


def test_workspace_size_query(L):
    small = qoq.workspace_bytes(1, 4096, 4096)
    big = qoq.workspace_bytes(4096, 4096, 4096)
    assert 0 < small < big
    assert qoq.workspace_bytes(0, 128, 128) > 0


def _sz(v=0):
    return ctypes.byref(ctypes.c_size_t(v))


def test_argument_validation_without_launch(L):
    dummy = ctypes.c_void_p(16 * 1024)   # never dereferenced: every call below fails validation first
    # N / K not multiples of 128, or K too large
    assert L.qoq_quantize_weights(dummy, 100, 128, 128, dummy, _sz(1 << 30), None) == 2
    assert L.qoq_quantize_weights(dummy, 128, 130, 128, dummy, _sz(1 << 30), None) == 2
    assert L.qoq_quantize_weights(dummy, 128, 131072, 128, dummy, _sz(1 << 30), None) == 2
    # bad group size, negative sizes, null size pointer
    assert L.qoq_quantize_weights(dummy, 128, 128, 64, dummy, _sz(1 << 30), None) == 1
    assert L.qoq_quantize_weights(dummy, -128, 128, 128, dummy, _sz(1 << 30), None) == 1
    assert L.qoq_quantize_weights(dummy, 128, 128, 128, dummy, None, None) == 1
    # capacity too small
    assert L.qoq_quantize_weights(dummy, 128, 128, 128, dummy, _sz(100), None) == 4
    # misaligned weights
    assert L.qoq_quantize_weights(ctypes.c_void_p(16 * 1024 + 2), 128, 128, 128, dummy, _sz(1 << 30), None) == 3
    # activation quant
    assert L.qoq_quantize_act_per_token(dummy, -1, 128, dummy, dummy, None, None) == 1
    assert L.qoq_quantize_act_per_token(dummy, 4, 100, dummy, dummy, None, None) == 2
    assert L.qoq_quantize_act_per_token(ctypes.c_void_p(8), 4, 128, dummy, dummy, None, None) == 3
    assert L.qoq_quantize_act_per_token(None, 4, 128, dummy, dummy, None, None) == 1
    assert L.qoq_quantize_act_per_token(None, 0, 128, None, None, None, None) == 0   # empty: no-op
    # GEMM
    ws = _sz(1 << 30)
    assert L.qoq_gemm_fp16_out(dummy, dummy, None, dummy, 4, 128, 128, 128, dummy, dummy, None, None) == 1
    assert L.qoq_gemm_fp16_out(dummy, dummy, None, dummy, 4, 127, 128, 128, dummy, dummy, ws, None) == 2
    assert L.qoq_gemm_fp16_out(dummy, dummy, None, dummy, 4, 128, 128, 128, dummy, dummy, _sz(8), None) == 4
    assert L.qoq_gemm_fp16_out(dummy, None, None, dummy, 4, 128, 128, 128, dummy, dummy, ws, None) == 1
    assert L.qoq_w4a8_gemm(dummy, None, dummy, 4, 128, 128, 0, dummy, dummy, ws, None) == 1   # rowsum needed
    assert L.qoq_w4a8_gemm(ctypes.c_void_p(16 * 1024 + 8), None, dummy, 4, 128, 128, 128, dummy, dummy, ws,
                           None) == 3
    assert L.qoq_w4a8_gemm(dummy, None, dummy, 0, 128, 128, 128, dummy, dummy, ws, None) == 0   # M = 0
    # the whole linear layer (act quant + GEMM)
    assert L.qoq_w4a8_linear(dummy, dummy, 4, 128, 128, 128, dummy, dummy, None, None) == 1     # no size pointer
    assert L.qoq_w4a8_linear(dummy, dummy, 4, 128, 100, 128, dummy, dummy, ws, None) == 2      # K % 128
    assert L.qoq_w4a8_linear(dummy, dummy, 4, 128, 128, 64, dummy, dummy, ws, None) == 1       # group size
    assert L.qoq_w4a8_linear(dummy, dummy, 4, 128, 128, 128, dummy, dummy, _sz(8), None) == 4  # too small
    assert L.qoq_w4a8_linear(None, dummy, 4, 128, 128, 128, dummy, dummy, ws, None) == 1       # no X
    assert L.qoq_w4a8_linear(ctypes.c_void_p(16 * 1024 + 8), dummy, 4, 128, 128, 128, dummy, dummy, ws,
                             None) == 3                                                        # X misaligned
    assert L.qoq_w4a8_linear(dummy, dummy, 4, 128, 128, 128, dummy, ctypes.c_void_p(16 * 1024 + 16), ws,
                             None) == 3                                                        # workspace 256-aligned
    assert L.qoq_w4a8_linear(None, None, 0, 128, 128, 128, None, dummy, ws, None) == 0         # M = 0
    # fused producers
    f = ctypes.c_float
    assert L.qoq_rmsnorm_quant(dummy, dummy, -1, 4096, f(1e-5), dummy, dummy, None, None) == 1
    assert L.qoq_rmsnorm_quant(dummy, dummy, 4, 4096, f(0.0), dummy, dummy, None, None) == 1      # eps > 0
    assert L.qoq_rmsnorm_quant(dummy, dummy, 4, 4096, f(float("inf")), dummy, dummy, None, None) == 1
    assert L.qoq_rmsnorm_quant(dummy, dummy, 4, 4100, f(1e-5), dummy, dummy, None, None) == 2     # K % 8
    assert L.qoq_rmsnorm_quant(dummy, dummy, 4, 65536, f(1e-5), dummy, dummy, None, None) == 2    # too wide
    assert L.qoq_rmsnorm_quant(dummy, None, 4, 4096, f(1e-5), dummy, dummy, None, None) == 1
    assert L.qoq_rmsnorm_quant(dummy, ctypes.c_void_p(16 * 1024 + 2), 4, 4096, f(1e-5), dummy, dummy, None,
                               None) == 3
    assert L.qoq_rmsnorm_quant(None, None, 0, 4096, f(1e-5), None, None, None, None) == 0        # M = 0
    assert L.qoq_silu_mul_quant(dummy, 4, 0, dummy, dummy, None, None) == 1
    assert L.qoq_silu_mul_quant(dummy, 4, 14340, dummy, dummy, None, None) == 2                  # I % 8
    assert L.qoq_silu_mul_quant(dummy, 4, 14336, ctypes.c_void_p(16 * 1024 + 4), dummy, None, None) == 3
    assert L.qoq_silu_mul_quant(dummy, 4, 14336, dummy, ctypes.c_void_p(16 * 1024 + 1), None, None) == 3
    assert L.qoq_silu_mul_quant(None, 0, 14336, None, None, None, None) == 0
    # saturating-decode ablation: group 128 only; M <= 16, or M > 512 on paired n-tiles
    S = L.qoq_gemm_fp16_out_saturating
    assert S(dummy, dummy, dummy, 4, 256, 512, 0, dummy, dummy, ws, None) == 2      # per-channel
    assert S(dummy, dummy, dummy, 64, 256, 512, 128, dummy, dummy, ws, None) == 2   # 16 < M <= 512
    assert S(dummy, dummy, dummy, 600, 384, 512, 128, dummy, dummy, ws, None) == 2  # N / 128 odd
    assert S(dummy, dummy, dummy, 4, 256, 512, 128, dummy, dummy, _sz(8), None) == 4
    assert S(dummy, None, dummy, 4, 256, 512, 128, dummy, dummy, ws, None) == 1     # s_x needed
    assert S(None, None, None, 0, 256, 512, 128, None, dummy, ws, None) == 0        # M = 0


def test_watchdog_selftest_validation_without_launch(L):
    """Argument errors return before any CUDA call (so they work with no GPU)."""
    assert L.qoq_watchdog_selftest(None, 1000, None) == 1            # QOQ_ERR_INVALID_ARG
    assert L.qoq_watchdog_selftest(ctypes.c_void_p(16), 0, None) == 1
    assert L.qoq_watchdog_selftest(ctypes.c_void_p(16), 3_000_000_000, None) == 1
    assert L.qoq_watchdog_selftest(ctypes.c_void_p(18), 1000, None) == 3   # QOQ_ERR_ALIGNMENT
