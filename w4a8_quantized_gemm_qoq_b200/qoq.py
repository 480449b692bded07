"""ctypes binding of libqoq.so (the C ABI in include/qoq.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. PyTorch supplies device memory and the current stream. There is no
CPU fallback: if the library is missing or no CUDA device is present the calls
raise.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqoq.so")

QOQ_OK = 0
QOQ_ERR_TIMEOUT = 7
STATUS = {0: "QOQ_OK", 1: "QOQ_ERR_INVALID_ARG", 2: "QOQ_ERR_UNSUPPORTED", 3: "QOQ_ERR_ALIGNMENT",
          4: "QOQ_ERR_WORKSPACE", 5: "QOQ_ERR_BAD_BLOB", 6: "QOQ_ERR_CUDA", 7: "QOQ_ERR_TIMEOUT"}
TILE = 128
GROUP = 128
WORKSPACE_CONTROL_BYTES = 1280   # status word + per-tile arrival counters (include/qoq.h)

_lib = None


class QoQError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__("%s failed: %s (%d)" % (fn, STATUS.get(code, "?"), code))
        self.code = code


def lib() -> ctypes.CDLL:
    """Open libqoq.so (built in-tree by w4a8_quantized_gemm_qoq_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libqoq.so is not built (%s); run python -m w4a8_quantized_gemm_qoq_b200.build"
                              % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)
        L.qoq_quantize_act_per_token.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        L.qoq_quantize_weights.argtypes = [vp, i64, i64, i32, vp, sz, vp]
        L.qoq_rmsnorm_quant.argtypes = [vp, vp, i64, i64, ctypes.c_float, vp, vp, vp, vp]
        L.qoq_silu_mul_quant.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        L.qoq_w4a8_gemm.argtypes = [vp, vp, vp, i64, i64, i64, i32, vp, vp, sz, vp]
        L.qoq_gemm_fp16_out.argtypes = [vp, vp, vp, vp, i64, i64, i64, i32, vp, vp, sz, vp]
        L.qoq_gemm_fp16_out_saturating.argtypes = [vp, vp, vp, i64, i64, i64, i32, vp, vp, sz, vp]
        L.qoq_gemm_fp16_out_saturating.restype = ctypes.c_int
        L.qoq_w4a8_linear.argtypes = [vp, vp, i64, i64, i64, i32, vp, vp, sz, vp]
        L.qoq_w4a8_linear.restype = ctypes.c_int
        L.qoq_kv4_cache_write.argtypes = [vp, i64, i64, i64, i64, i64, i64, vp, vp, vp, vp]
        L.qoq_kv4_cache_write.restype = ctypes.c_int
        L.qoq_kv4_decode_attention.argtypes = [vp] * 8 + [i64] * 5 + [vp, vp, sz, vp]
        L.qoq_kv4_decode_attention.restype = ctypes.c_int
        L.qoq_plan.argtypes = [i64, i64, i64, vp, vp]
        L.qoq_plan.restype = ctypes.c_int
        L.qoq_watchdog_selftest.argtypes = [vp, i64, vp]
        L.qoq_watchdog_selftest.restype = ctypes.c_int
        L.qoq_status_string.argtypes = [ctypes.c_int]
        L.qoq_status_string.restype = ctypes.c_char_p
        for f in (L.qoq_quantize_act_per_token, L.qoq_quantize_weights, L.qoq_w4a8_gemm, L.qoq_gemm_fp16_out):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def _check(fn, code):
    if code != QOQ_OK:
        raise QoQError(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _cuda_tensor(t, dtype, name):
    import torch
    if not (isinstance(t, torch.Tensor) and t.is_cuda):
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


# ------------------------------------------------------------------ sizes

def blob_bytes(N: int, K: int, group_size: int = GROUP) -> int:
    n = ctypes.c_size_t(0)
    _check("qoq_quantize_weights", lib().qoq_quantize_weights(None, N, K, group_size, None, ctypes.byref(n), None))
    return n.value


def workspace_bytes(M: int, N: int, K: int, group_size: int = GROUP) -> int:
    n = ctypes.c_size_t(0)
    _check("qoq_gemm_fp16_out", lib().qoq_gemm_fp16_out(None, None, None, None, M, N, K, group_size, None, None,
                                                        ctypes.byref(n), None))
    return n.value


def linear_workspace_bytes(M: int, N: int, K: int, group_size: int = GROUP) -> int:
    n = ctypes.c_size_t(0)
    _check("qoq_w4a8_linear", lib().qoq_w4a8_linear(None, None, M, N, K, group_size, None, None, ctypes.byref(n),
                                                    None))
    return n.value


def plan(M: int, N: int, K: int):
    """(token tile, kernels qoq_w4a8_linear launches) for an M x N x K problem."""
    tok, nl = ctypes.c_int32(0), ctypes.c_int32(0)
    _check("qoq_plan", lib().qoq_plan(M, N, K, ctypes.byref(tok), ctypes.byref(nl)))
    return tok.value, nl.value


# ------------------------------------------------------------------ calls

def quantize_act_per_token(X, X8=None, s_x=None, rowsum=None, stream=None):
    """X [M][K] fp16 -> (X8 int8 [M][K], s_x fp16 [M], rowsum int32 [M])."""
    import torch
    X = _cuda_tensor(X, torch.float16, "X")
    M, K = X.shape
    X8 = torch.empty((M, K), dtype=torch.int8, device=X.device) if X8 is None else X8
    s_x = torch.empty((M,), dtype=torch.float16, device=X.device) if s_x is None else s_x
    rowsum = torch.empty((M,), dtype=torch.int32, device=X.device) if rowsum is None else rowsum
    _check("qoq_quantize_act_per_token",
           lib().qoq_quantize_act_per_token(_ptr(X), M, K, _ptr(X8), _ptr(s_x), _ptr(rowsum), _stream(stream)))
    return X8, s_x, rowsum


def rmsnorm_quant(X, gamma, eps: float, X8=None, s_x=None, rowsum=None, stream=None):
    """Fused RMSNorm + per-token INT8 quantisation: X [M][K] fp16, gamma [K]
    fp16 -> (X8 int8 [M][K], s_x fp16 [M], rowsum int32 [M])."""
    import torch
    X = _cuda_tensor(X, torch.float16, "X")
    gamma = _cuda_tensor(gamma, torch.float16, "gamma")
    M, K = X.shape
    if tuple(gamma.shape) != (K,):
        raise ValueError("gamma must have shape (%d,)" % K)
    X8 = torch.empty((M, K), dtype=torch.int8, device=X.device) if X8 is None else X8
    s_x = torch.empty((M,), dtype=torch.float16, device=X.device) if s_x is None else s_x
    rowsum = torch.empty((M,), dtype=torch.int32, device=X.device) if rowsum is None else rowsum
    _check("qoq_rmsnorm_quant", lib().qoq_rmsnorm_quant(_ptr(X), _ptr(gamma), M, K, float(eps), _ptr(X8),
                                                        _ptr(s_x), _ptr(rowsum), _stream(stream)))
    return X8, s_x, rowsum


def silu_mul_quant(GU, X8=None, s_x=None, rowsum=None, stream=None):
    """Fused SiLU(gate) * up + per-token INT8 quantisation: GU [M][2I] fp16
    (gate | up) -> (X8 int8 [M][I], s_x fp16 [M], rowsum int32 [M])."""
    import torch
    GU = _cuda_tensor(GU, torch.float16, "GU")
    M, I2 = GU.shape
    if I2 % 2:
        raise ValueError("GU must have an even number of columns (gate | up)")
    I = I2 // 2
    X8 = torch.empty((M, I), dtype=torch.int8, device=GU.device) if X8 is None else X8
    s_x = torch.empty((M,), dtype=torch.float16, device=GU.device) if s_x is None else s_x
    rowsum = torch.empty((M,), dtype=torch.int32, device=GU.device) if rowsum is None else rowsum
    _check("qoq_silu_mul_quant", lib().qoq_silu_mul_quant(_ptr(GU), M, I, _ptr(X8), _ptr(s_x), _ptr(rowsum),
                                                          _stream(stream)))
    return X8, s_x, rowsum


def quantize_weights(W, group_size: int = GROUP, blob=None, stream=None):
    """W [N][K] fp16 -> packed blob (uint8 tensor) in compute order."""
    import torch
    W = _cuda_tensor(W, torch.float16, "W")
    N, K = W.shape
    need = blob_bytes(N, K, group_size)
    blob = torch.empty((need,), dtype=torch.uint8, device=W.device) if blob is None else blob
    n = ctypes.c_size_t(blob.numel())
    _check("qoq_quantize_weights",
           lib().qoq_quantize_weights(_ptr(W), N, K, group_size, _ptr(blob), ctypes.byref(n), _stream(stream)))
    return blob


class Workspace:
    """Zero-filled device workspace for the GEMM calls. Its leading control
    bytes (the device status word, then per-tile arrival counters) are left zero by
    every call that completes; the rest is scratch."""

    def __init__(self, nbytes: int, device="cuda"):
        import torch
        self.buf = torch.zeros((nbytes + 15) // 16 * 16, dtype=torch.uint8, device=device)

    @classmethod
    def for_shape(cls, M, N, K, group_size=GROUP, device="cuda"):
        return cls(workspace_bytes(M, N, K, group_size), device)

    @classmethod
    def for_linear(cls, M, N, K, group_size=GROUP, device="cuda"):
        """Workspace of qoq_w4a8_linear (GEMM scratch plus the quantised activations)."""
        return cls(linear_workspace_bytes(M, N, K, group_size), device)

    def status(self) -> int:
        return int(self.buf[:4].view(dtype=__import__("torch").int32).item())

    def timeout_site(self):
        """(wait site, block index, detail) recorded with QOQ_ERR_TIMEOUT."""
        import torch
        w = self.buf[:16].view(dtype=torch.int32).tolist()
        return tuple(w[1:4])

    def control_clear(self) -> bool:
        return not bool(self.buf[:WORKSPACE_CONTROL_BYTES].any().item())

    def reset(self):
        self.buf.zero_()


def watchdog_selftest(limit_ns=50_000_000, stream=None):
    """Run the device bounded-wait self-test; returns the 32 status words
    (the mbarrier wait's record at [0:4], the flag wait's at [8:12])."""
    import torch
    status = torch.zeros(32, dtype=torch.int32, device="cuda")
    _check("qoq_watchdog_selftest", lib().qoq_watchdog_selftest(_ptr(status), int(limit_ns), _stream(stream)))
    torch.cuda.synchronize()
    return status.cpu().tolist()


def w4a8_gemm(X8, blob, N, K, group_size=GROUP, rowsum=None, ws=None, acc=None, stream=None):
    """Exact INT32 GEMM: acc [M][N]."""
    import torch
    X8 = _cuda_tensor(X8, torch.int8, "X8")
    M = X8.shape[0]
    ws = ws or Workspace.for_shape(M, N, K, group_size, X8.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=X8.device) if acc is None else acc
    n = ctypes.c_size_t(ws.buf.numel())
    _check("qoq_w4a8_gemm", lib().qoq_w4a8_gemm(_ptr(X8), _ptr(rowsum), _ptr(blob), M, N, K, group_size, _ptr(acc),
                                                _ptr(ws.buf), ctypes.byref(n), _stream(stream)))
    return acc


def gemm_fp16_out(X8, s_x, blob, N, K, group_size=GROUP, rowsum=None, ws=None, Y=None, stream=None):
    """W4A8 GEMM with fused FP16 epilogue: Y [M][N] fp16."""
    import torch
    X8 = _cuda_tensor(X8, torch.int8, "X8")
    M = X8.shape[0]
    ws = ws or Workspace.for_shape(M, N, K, group_size, X8.device)
    Y = torch.empty((M, N), dtype=torch.float16, device=X8.device) if Y is None else Y
    n = ctypes.c_size_t(ws.buf.numel())
    _check("qoq_gemm_fp16_out", lib().qoq_gemm_fp16_out(_ptr(X8), _ptr(s_x), _ptr(rowsum), _ptr(blob), M, N, K,
                                                        group_size, _ptr(Y), _ptr(ws.buf), ctypes.byref(n),
                                                        _stream(stream)))
    return Y


def gemm_fp16_out_saturating(X8, s_x, blob, N, K, ws=None, Y=None, stream=None):
    """The same GEMM with a saturating weight decode (the protective-range
    ablation; group_size 128; M <= 16, or M > 512 with N / 128 even)."""
    import torch
    X8 = _cuda_tensor(X8, torch.int8, "X8")
    M = X8.shape[0]
    ws = ws or Workspace.for_shape(M, N, K, GROUP, X8.device)
    Y = torch.empty((M, N), dtype=torch.float16, device=X8.device) if Y is None else Y
    n = ctypes.c_size_t(ws.buf.numel())
    _check("qoq_gemm_fp16_out_saturating",
           lib().qoq_gemm_fp16_out_saturating(_ptr(X8), _ptr(s_x), _ptr(blob), M, N, K, GROUP, _ptr(Y),
                                              _ptr(ws.buf), ctypes.byref(n), _stream(stream)))
    return Y


def linear(X, blob, N, K, group_size=GROUP, ws=None, Y=None, stream=None):
    """The whole hot path in one call (qoq_w4a8_linear): per-token
    quantisation of X [M][K] fp16, then the W4A8 GEMM with the FP16 epilogue;
    two launches, or one for token tiles of at most 64 tokens when
    QOQ_FORCE_CONFIG holds fuse=1 (plan() reports which). Y [M][N] fp16."""
    import torch
    X = _cuda_tensor(X, torch.float16, "X")
    M = X.shape[0]
    if X.shape[1] != K:
        raise ValueError("X must have K = %d columns" % K)
    ws = ws or Workspace.for_linear(M, N, K, group_size, X.device)
    Y = torch.empty((M, N), dtype=torch.float16, device=X.device) if Y is None else Y
    n = ctypes.c_size_t(ws.buf.numel())
    _check("qoq_w4a8_linear", lib().qoq_w4a8_linear(_ptr(X), _ptr(blob), M, N, K, group_size, _ptr(Y), _ptr(ws.buf),
                                                    ctypes.byref(n), _stream(stream)))
    return Y


# ------------------------------------------------------------------ KV4

class KV4Cache:
    """A per-head, dynamic, asymmetric 4-bit cache of one tensor (K or V):
    codes uint8 [B][Hkv][max_tokens][D/2], scales and zeros FP16
    [B][Hkv][max_tokens] (include/qoq.h, qoq_kv4_cache_write)."""

    def __init__(self, B, Hkv, max_tokens, D, device="cuda"):
        import torch
        self.B, self.Hkv, self.T, self.D = B, Hkv, max_tokens, D
        self.codes = torch.zeros((B, Hkv, max_tokens, D // 2), dtype=torch.uint8, device=device)
        self.scales = torch.zeros((B, Hkv, max_tokens), dtype=torch.float16, device=device)
        self.zeros = torch.zeros((B, Hkv, max_tokens), dtype=torch.float16, device=device)

    def write(self, src, t0=0, stream=None):
        """Quantise src [B][Hkv][n][D] FP16 into slots t0 .. t0 + n - 1."""
        import torch
        src = _cuda_tensor(src, torch.float16, "src")
        B, H, n, D = src.shape
        if (B, H, D) != (self.B, self.Hkv, self.D):
            raise ValueError("src shape %s does not match the cache" % (tuple(src.shape),))
        _check("qoq_kv4_cache_write", lib().qoq_kv4_cache_write(_ptr(src), B, H, self.T, t0, n, D, _ptr(self.codes),
                                                                _ptr(self.scales), _ptr(self.zeros),
                                                                _stream(stream)))
        return self


def kv4_workspace_bytes(B, Hq, Hkv, max_tokens, D) -> int:
    n = ctypes.c_size_t(0)
    _check("qoq_kv4_decode_attention", lib().qoq_kv4_decode_attention(*([None] * 8), B, Hq, Hkv, max_tokens, D, None,
                                                                      None, ctypes.byref(n), None))
    return n.value


def kv4_decode_attention(q, kcache, vcache, seq_lens=None, ws=None, out=None, stream=None):
    """q [B][Hq][D] FP16 against the KV4 caches -> out [B][Hq][D] FP16."""
    import torch
    q = _cuda_tensor(q, torch.float16, "q")
    B, Hq, D = q.shape
    if seq_lens is not None:
        seq_lens = _cuda_tensor(seq_lens, torch.int32, "seq_lens")
    ws = ws or Workspace(kv4_workspace_bytes(B, Hq, kcache.Hkv, kcache.T, D), q.device)
    out = torch.empty((B, Hq, D), dtype=torch.float16, device=q.device) if out is None else out
    n = ctypes.c_size_t(ws.buf.numel())
    _check("qoq_kv4_decode_attention", lib().qoq_kv4_decode_attention(
        _ptr(q), _ptr(kcache.codes), _ptr(kcache.scales), _ptr(kcache.zeros), _ptr(vcache.codes),
        _ptr(vcache.scales), _ptr(vcache.zeros), _ptr(seq_lens), B, Hq, kcache.Hkv, kcache.T, D, _ptr(out),
        _ptr(ws.buf), ctypes.byref(n), _stream(stream)))
    return out
