"""GPU parity of the fused activation producers (qoq_rmsnorm_quant,
qoq_silu_mul_quant) against the CPU oracle: bit-exact INT8 codes, FP16 scales
and row sums, through the C ABI. The fusion is the one the paperlayer.ai
summary of QServe describes in section 5 ("Runtime and precision mapping");
the arithmetic is the reading written in oracle/producers.py."""
import numpy as np
import pytest

from oracle import producers as P
from w4a8_quantized_gemm_qoq_b200 import inputs, qoq
from gpu_helpers import dev, host

pytestmark = pytest.mark.gpu


def _same(got, want, what):
    X8, s_x, rs = (host(t) for t in got)
    wX8, ws_x, wrs = want
    assert np.array_equal(s_x.view(np.uint16), ws_x.view(np.uint16)), what + " s_x"
    assert np.array_equal(X8, wX8), what + " X8 (%d codes differ)" % int((X8 != wX8).sum())
    assert np.array_equal(rs, wrs), what + " rowsum"


@pytest.mark.parametrize("M,K,eps", [(1, 4096, 1e-5), (7, 4096, 1e-6), (33, 14336, 1e-5), (130, 8192, 1e-5),
                                     (3, 32768, 1e-6), (5, 8, 1e-5), (260, 1024, 0.25), (17, 11008, 1e-5),
                                     (5, 2048, 1e-5), (9, 512, 1e-5), (6, 6144, 1e-5)])
def test_rmsnorm_quant_parity(M, K, eps):
    X = inputs.make_activations(M, K, seed=M + K, token_scale_span=(-3, 1))
    g = inputs.make_norm_weight(K, seed=K)
    _same(qoq.rmsnorm_quant(dev(X), dev(g), eps), P.rmsnorm_quant(X, g, eps), "rmsnorm %dx%d" % (M, K))


def test_rmsnorm_quant_degenerate_rows():
    K = 4096
    X = inputs.make_activations(12, K, seed=5)
    X[0] = 0                       # zero row: scale 0, codes 0
    X[1] = 2.5                     # constant row
    X[2] = 0
    X[2, 77] = -3.0                # one-hot
    X[3] = np.float16(65504)       # largest FP16
    X[4] = np.float16(6e-8)        # subnormal FP16 everywhere
    X[5, ::2] = np.float16(-65504)
    X[6] = X[6] * np.float16(1e-4)
    g = inputs.make_norm_weight(K, seed=1)
    g[::7] = 0
    for eps in (1e-5, 1e-12, 1e3):
        _same(qoq.rmsnorm_quant(dev(X), dev(g), eps), P.rmsnorm_quant(X, g, eps), "degenerate eps=%g" % eps)


@pytest.mark.parametrize("M,I", [(1, 14336), (9, 4096), (65, 11008), (3, 32768), (4, 8), (130, 1024),
                                 (6, 8192), (5, 512), (11, 2048), (2, 20480)])
def test_silu_mul_quant_parity(M, I):
    GU = inputs.make_gate_up(M, I, seed=M * 7 + I)
    _same(qoq.silu_mul_quant(dev(GU)), P.silu_mul_quant(GU), "silu %dx%d" % (M, I))


def test_silu_mul_quant_degenerate_rows():
    I = 2048
    GU = inputs.make_gate_up(8, I, seed=3)
    GU[0] = 0                               # scale 0
    GU[1, :I] = np.float16(-65504)          # e^-g overflows: silu = -0
    GU[2, :I] = np.float16(65504)           # e^-g = 0: silu(g) = g
    GU[3, :I] = np.float16(-87.3)           # around the overflow threshold of e^x
    GU[3, I:] = np.float16(1000)
    GU[4, :I] = np.linspace(-90, 90, I).astype(np.float16)
    GU[5, I:] = 0                           # up half zero
    GU[6] = np.float16(6e-8)
    _same(qoq.silu_mul_quant(dev(GU)), P.silu_mul_quant(GU), "silu degenerate")


def test_exp_matches_oracle_bit_for_bit_on_device():
    """Every representable gate value of a sweep: the device's SiLU-gated
    product equals the oracle's on a row whose up half is 1, so the e^x both
    evaluate agrees bit for bit (the codes alone could hide a 1-ulp slip)."""
    I = 32768
    g = np.linspace(-100, 100, I).astype(np.float16)
    GU = np.concatenate([g, np.ones(I, dtype=np.float16)])[None, :]
    X8, s_x, rs = (host(t) for t in qoq.silu_mul_quant(dev(GU)))
    wX8, ws_x, wrs = P.silu_mul_quant(GU)
    assert np.array_equal(X8, wX8) and np.array_equal(s_x.view(np.uint16), ws_x.view(np.uint16))


def test_producers_at_prefill_size_sampled_rows():
    """M = 16384 in one launch (the prefill token count), rows compared on a
    deterministic sample of 64."""
    M, K, I = 16384, 4096, 14336
    rows = inputs.sample_rows(M, 64)
    X = inputs.make_activations(M, K, seed=11, token_scale_span=(-3, 1))
    g = inputs.make_norm_weight(K, seed=2)
    X8, s_x, rs = (host(t) for t in qoq.rmsnorm_quant(dev(X), dev(g), 1e-5))
    wX8, ws_x, wrs = P.rmsnorm_quant(X[rows], g, 1e-5)
    assert np.array_equal(X8[rows], wX8) and np.array_equal(s_x[rows].view(np.uint16), ws_x.view(np.uint16))
    assert np.array_equal(rs[rows], wrs)
    GU = inputs.make_gate_up(2048, I, seed=12)
    rows = inputs.sample_rows(2048, 64)
    X8, s_x, rs = (host(t) for t in qoq.silu_mul_quant(dev(GU)))
    wX8, ws_x, wrs = P.silu_mul_quant(GU[rows])
    assert np.array_equal(X8[rows], wX8) and np.array_equal(s_x[rows].view(np.uint16), ws_x.view(np.uint16))
    assert np.array_equal(rs[rows], wrs)


def test_producer_feeds_the_gemm():
    """The producer's outputs are the GEMM's activation format: RMSNorm-quant
    -> FP16 GEMM equals the oracle's GEMM on the oracle's producer outputs."""
    import oracle
    M, K, N = 16, 4096, 512
    X = inputs.make_activations(M, K, seed=4)
    g = inputs.make_norm_weight(K, seed=4)
    W = inputs.make_weights(N, K, seed=4)
    X8, s_x, rs = qoq.rmsnorm_quant(dev(X), dev(g), 1e-5)
    blob = qoq.quantize_weights(dev(W), 128)
    ws = qoq.Workspace.for_shape(M, N, K)
    Y = host(qoq.gemm_fp16_out(X8, s_x, blob, N, K, 128, rowsum=rs, ws=ws))
    wX8, ws_x, _ = P.rmsnorm_quant(X, g, 1e-5)
    _, q = oracle.quantize_weights(W, 128)
    acc = oracle.gemm_int(wX8, q["Wint"])
    want = oracle.epilogue_fp16(acc, ws_x, q["s_w"])
    d = oracle.fp16_ulp_distance(Y, want)
    assert d.max() <= 1
