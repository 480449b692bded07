"""CUDA path vs CPU oracle, element by element, through the C ABI.

Bar: bit-exact INT8 codes, FP16 scales, row sums, packed blob bytes and INT32
accumulators; FP16 outputs within 1 ulp of the oracle's FP32 epilogue.
"""
import numpy as np
import pytest

import oracle
from w4a8_quantized_gemm_qoq_b200 import inputs, qoq
from gpu_helpers import check_full, check_sampled, dev, host, assert_fp16_close, sample_tiles, torch

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    t = torch()
    assert t.cuda.is_available(), "GPU tests need a CUDA device"
    from w4a8_quantized_gemm_qoq_b200 import build
    build.build()
    yield


# ----------------------------------------------------------- small, full oracle

def test_config_small_g128():
    """M=16 N=256 K=512, g=128: the small configuration, every intermediate."""
    X = inputs.make_activations(16, 512, seed=0)
    W = inputs.make_weights(256, 512, seed=0)
    check_full(X, W, 128, "C1")


@pytest.mark.parametrize("M", [1, 7, 15, 16, 17, 31, 33, 64, 65, 127, 129, 255, 256, 257, 300])
def test_ragged_tokens_g128(M):
    X = inputs.make_activations(M, 640, seed=M)
    W = inputs.make_weights(384, 640, seed=M)
    check_full(X, W, 128, "M=%d" % M)


@pytest.mark.parametrize("M", [1, 16, 100, 256, 513])
def test_ragged_tokens_per_channel(M):
    X = inputs.make_activations(M, 384, seed=100 + M)
    W = inputs.make_weights(640, 384, seed=100 + M)
    check_full(X, W, 0, "per-channel M=%d" % M)


@pytest.mark.parametrize("M", [513, 600, 700, 1000])
def test_paired_ctas_ragged_tokens(M):
    """Above 512 tokens the GEMM runs 256-token tiles on CTA pairs (one
    256-row MMA across two SMs, each SM staging half of the token tile) when
    the n-tiles pair up (N/128 even). Ragged last tiles whose second half is
    empty (M=513, 600), partly live (700) or nearly full (1000), both
    quantisation modes."""
    X = inputs.make_activations(M, 640, seed=200 + M)
    W = inputs.make_weights(512, 640, seed=200 + M)
    check_full(X, W, 128, "pairs M=%d" % M)
    check_full(X, W, 0, "pairs per-channel M=%d" % M)


@pytest.mark.parametrize("M", [600, 1000])
def test_unpaired_wide_tiles_odd_ntiles(M):
    """256-token tiles whose n-tiles do not pair up (N/128 odd) run on single
    CTAs: two issuers on the two token halves, one dequant and two epilogue
    warpgroups; both quantisation modes."""
    X = inputs.make_activations(M, 640, seed=400 + M)
    W = inputs.make_weights(384, 640, seed=400 + M)
    check_full(X, W, 128, "unpaired M=%d" % M)
    check_full(X, W, 0, "unpaired per-channel M=%d" % M)


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (16, 1024, 1280), (600, 512, 640), (2048, 28672, 4096)])
def test_saturating_decode_ablation_is_bit_identical(M, N, K):
    """The protective-range ablation decodes the weights with per-byte
    saturation. On blobs with the protective range the clamp never acts, so
    the outputs equal the excess-128 decode's bit for bit (both token tiles it
    is built for: 16, and 256 on CTA pairs)."""
    X = inputs.make_activations(M, K, seed=300 + M)
    W = inputs.make_weights(N, K, seed=300 + N)
    blob = qoq.quantize_weights(dev(W), 128)
    X8, s_x, rs = qoq.quantize_act_per_token(dev(X))
    ws = qoq.Workspace.for_shape(M, N, K, 128)
    y = qoq.gemm_fp16_out(X8, s_x, blob, N, K, 128, rowsum=rs, ws=ws)
    y_sat = qoq.gemm_fp16_out_saturating(X8, s_x, blob, N, K, ws=ws)
    torch().cuda.synchronize()
    assert ws.status() == 0
    assert np.array_equal(host(y).view(np.uint16), host(y_sat).view(np.uint16))
    assert ws.control_clear()


@pytest.mark.parametrize("N,K", [(128, 128), (128, 1152), (1152, 128), (896, 2176)])
def test_tile_shapes(N, K):
    X = inputs.make_activations(24, K, seed=N + K)
    W = inputs.make_weights(N, K, seed=N + K)
    check_full(X, W, 128, "N=%d K=%d" % (N, K))
    check_full(X, W, 0, "per-channel N=%d K=%d" % (N, K))


def test_prefill_token_scales():
    X = inputs.make_activations(300, 1024, seed=3, token_scale_span=(-3, 1))
    W = inputs.make_weights(512, 1024, seed=3)
    check_full(X, W, 128, "scaled tokens")


@pytest.mark.parametrize("M,K", [(1, 4096), (100, 14336), (64, 32768), (2000, 4096), (5000, 128), (1000, 14336),
                                 (700, 24576), (300, 32768)])
def test_act_quant_every_row(M, K):
    """Per-token quantisation, every row bit-exact (codes, FP16 scales, row
    sums) with the oracle, in each form the launch picks by shape: 512 threads
    with the row in registers (a few rows), 256 threads in registers, the
    two-pass form with 256 and 128 threads (many rows)."""
    X = inputs.make_activations(M, K, seed=K + M, token_scale_span=(-3, 1))
    X8, s_x, rs = qoq.quantize_act_per_token(dev(X))
    torch().cuda.synchronize()
    X8o, s_xo, rso = oracle.quantize_act_per_token(X)
    assert np.array_equal(host(X8), X8o)
    assert np.array_equal(host(s_x).view(np.uint16), s_xo.view(np.uint16))
    assert np.array_equal(host(rs), rso)


def test_degenerate_inputs():
    """Zero rows and columns, constant rows, one-hot tokens."""
    K, N = 256, 256
    W = inputs.make_weights(N, K, seed=4)
    W[3] = 0
    W[7] = 0.05
    W[9] = -2.0
    W[:, 5] = 0
    X = inputs.make_activations(40, K, seed=4)
    X[0] = 0
    X[1] = 0.25
    X[2] = 0
    X[2, 77] = -3.0
    check_full(X, W, 128, "degenerate")
    check_full(X, W, 0, "degenerate per-channel")


def test_identity_reads_back_dequantised_weights():
    """K one-hot tokens: acc = 127 * Wint^T, i.e. the GEMM returns the whole
    dequantised weight matrix, which pins the packed layout end to end."""
    K, N = 384, 256
    W = inputs.make_weights(N, K, seed=5)
    X = np.zeros((K, K), dtype=np.float16)
    X[np.arange(K), np.arange(K)] = 1.0
    r, g = check_full(X, W, 128, "identity")
    assert np.array_equal(g["acc"], 127 * r["w"]["Wint"].astype(np.int32).T)


def test_workspace_reuse_and_zero_m():
    X = inputs.make_activations(33, 512, seed=6)
    W = inputs.make_weights(256, 512, seed=6)
    Wd, Xd = dev(W), dev(X)
    blob = qoq.quantize_weights(Wd, 128)
    X8, s_x, rs = qoq.quantize_act_per_token(Xd)
    ws = qoq.Workspace.for_shape(33, 256, 512)
    y1 = host(qoq.gemm_fp16_out(X8, s_x, blob, 256, 512, ws=ws))
    y2 = host(qoq.gemm_fp16_out(X8, s_x, blob, 256, 512, ws=ws))
    assert np.array_equal(y1.view(np.uint16), y2.view(np.uint16))
    assert ws.control_clear()
    # M = 0 is a no-op that succeeds
    e = torch().empty((0, 512), dtype=torch().int8, device="cuda")
    out = qoq.gemm_fp16_out(e, s_x[:0], blob, 256, 512, ws=ws)
    assert out.shape == (0, 256)


def test_bad_blob_header_reported_on_device():
    """A blob whose header does not match the arguments: the kernel does no
    work and writes QOQ_ERR_BAD_BLOB to the workspace status word."""
    W = inputs.make_weights(256, 512, seed=7)
    blob = qoq.quantize_weights(dev(W), 128)
    X8 = torch().zeros((16, 512), dtype=torch().int8, device="cuda")
    s_x = torch().ones((16,), dtype=torch().float16, device="cuda")
    ws = qoq.Workspace.for_shape(16, 256, 512)
    Y = torch().full((16, 128), 7.0, dtype=torch().float16, device="cuda")
    # claim N = 128 for a blob built with N = 256
    qoq.gemm_fp16_out(X8, s_x, blob, 128, 512, ws=ws, Y=Y)
    torch().cuda.synchronize()
    assert ws.status() == 5
    assert bool((Y == 7.0).all().item())


# ------------------------------------------------------- full sizes, sampled oracle
# Every (shape, M) of the four full-size configurations. The stream-K split
# (data-parallel waves, tail boundaries, owner and contributor sets) changes
# with every (M, N, K), so no grid point stands in for another. The M values
# of one shape share its weights (seeded per shape).

_L3 = [(K, N) for (K, N, _) in inputs.LLAMA3_8B]
_QW = [(K, N) for (K, N, _) in inputs.QWEN15_72B]
_L2 = [(K, N) for (K, N, _) in inputs.LLAMA2_7B]


@pytest.mark.parametrize("K,N,M", [(K, N, M) for (K, N) in _L3 for M in inputs.DECODE_M])
def test_llama3_8b_decode_shapes(M, K, N):
    check_sampled(M, N, K, 128, seed=M + N, wseed=N + K)


@pytest.mark.parametrize("K,N,M", [(K, N, M) for (K, N) in _L3 for M in inputs.PREFILL_M])
def test_llama3_8b_prefill_shapes(M, K, N):
    check_sampled(M, N, K, 128, seed=M + K, wseed=N + K, token_scale_span=(-3, 1), rows=12)


@pytest.mark.parametrize("K,N,M", [(K, N, M) for (K, N) in _QW for M in inputs.QWEN_M])
def test_qwen15_72b_shapes(M, K, N):
    check_sampled(M, N, K, 128, seed=N + M, wseed=N + K, std=0.01, rows=12)


@pytest.mark.parametrize("K,N,M", [(K, N, M) for (K, N) in _L2 for M in inputs.PER_CHANNEL_M])
def test_llama2_7b_per_channel_shapes(M, K, N):
    check_sampled(M, N, K, 0, seed=K + M, wseed=N + K, rows=12)


# ------------------------------------- saturating decode where the clamp acts

def _saturating_blob(N, K, seed):
    """Codes, integer scales and zero terms drawn so that q*s - z*s leaves
    INT8 in many places (scales up to 40, any int8 zero term), packed by the
    oracle's packer; a quarter of the rows keep protective-range groups."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    s = rng.integers(1, 41, size=(N, K // 128)).astype(np.uint8)
    zs = rng.integers(-128, 128, size=(N, K // 128)).astype(np.int8)
    prot = oracle.quantize_weights_group(inputs.make_weights(N // 4, K, seed=seed))
    q[: N // 4], s[: N // 4], zs[: N // 4] = prot["q"], prot["s"], prot["zs"]
    s_w = (rng.uniform(1e-3, 4e-3, size=N)).astype(np.float16)
    raw = q.astype(np.int64).reshape(N, K // 128, 128) * s.astype(np.int64)[:, :, None] - \
        zs.astype(np.int64)[:, :, None]
    assert (raw > 127).mean() > 0.2, "the fixture must make the clamp act"
    return q, s, zs, s_w, oracle.pack_blob_group(q, s, zs, s_w)


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (16, 384, 640), (600, 512, 640), (1000, 768, 384)])
def test_saturating_decode_matches_oracle_where_the_clamp_acts(M, N, K):
    """The protective-range ablation on a blob whose dequantised weights
    leave INT8: the saturating GEMM equals the oracle's clamp(q*s - z*s,
    -128, 127) decode followed by the exact INT32 product and the epilogue,
    bit for bit, on both token tiles it is built for (16, and 256 on CTA
    pairs)."""
    X = inputs.make_activations(M, K, seed=500 + M)
    q, s, zs, s_w, blob_h = _saturating_blob(N, K, seed=M + N)
    X8o, s_xo, _ = oracle.quantize_act_per_token(X)
    want = oracle.gemm_fp16_saturating(X8o, s_xo, q, s, zs, s_w)
    X8, s_x, rs = qoq.quantize_act_per_token(dev(X))
    ws = qoq.Workspace.for_shape(M, N, K, 128)
    y = qoq.gemm_fp16_out_saturating(X8, s_x, dev(blob_h), N, K, ws=ws)
    torch().cuda.synchronize()
    assert ws.status() == 0
    assert np.array_equal(host(X8), X8o)
    assert np.array_equal(host(y).view(np.uint16), want.view(np.uint16))
    assert ws.control_clear()


# ------------------------------------------ back-to-back graph replays

def test_graph_replays_are_bit_identical():
    """Act quant + GEMM for several shapes captured in one CUDA graph and
    replayed back to back: every replay reproduces the eager outputs bit for
    bit with a clean status word. The shapes cover token tiles whose pipeline
    has an odd stage count (16, 32, 256 tokens) and long per-CTA k ranges,
    where a stage barrier is waited on many times per launch; sampled rows of
    the eager result are checked against the oracle."""
    t = torch()
    cases = [(1, 4096, 28672), (32, 14336, 4096), (8192, 14336, 4096), (2048, 4096, 4096)]
    probs = []
    for i, (M, K, N) in enumerate(cases):
        X = inputs.make_activations(M, K, seed=700 + i, token_scale_span=(-3, 1) if M > 256 else None)
        W = inputs.make_weights(N, K, seed=700 + i)
        Xd = dev(X)
        blob = qoq.quantize_weights(dev(W), 128)
        X8 = t.empty((M, K), dtype=t.int8, device="cuda")
        s_x = t.empty((M,), dtype=t.float16, device="cuda")
        rs = t.empty((M,), dtype=t.int32, device="cuda")
        Y = t.empty((M, N), dtype=t.float16, device="cuda")
        ws = qoq.Workspace.for_shape(M, N, K, 128)
        probs.append(dict(M=M, N=N, K=K, X=X, W=W, Xd=Xd, blob=blob, X8=X8, s_x=s_x, rs=rs, Y=Y, ws=ws))

    def step():
        for p in probs:
            qoq.quantize_act_per_token(p["Xd"], p["X8"], p["s_x"], p["rs"])
            qoq.gemm_fp16_out(p["X8"], p["s_x"], p["blob"], p["N"], p["K"], 128, rowsum=p["rs"], ws=p["ws"], Y=p["Y"])

    stream = t.cuda.Stream()
    stream.wait_stream(t.cuda.current_stream())   # inputs and zeroed workspaces were made on the default stream
    with t.cuda.stream(stream):
        step()
    stream.synchronize()
    ref = [p["Y"].clone() for p in probs]
    for p in probs:
        assert p["ws"].status() == 0
    g = t.cuda.CUDAGraph()
    with t.cuda.graph(g, stream=stream):
        step()
    for r in range(30):
        with t.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        for i, p in enumerate(probs):
            assert p["ws"].status() == 0, "replay %d case %d: status %d %s" % (r, i, p["ws"].status(),
                                                                             p["ws"].timeout_site())
            assert t.equal(p["Y"], ref[i]), "replay %d case %d: output differs from the eager run" % (r, i)
    for i, p in enumerate(probs):
        rows = inputs.sample_rows(p["M"], 6, seed=i)
        X8s, s_xs, _ = oracle.quantize_act_per_token(p["X"][rows])
        Yh = host(ref[i])[rows]
        for nt in sample_tiles(p["N"] // 128, seed=i)[:3]:
            _, d = oracle.quantize_weights(p["W"][nt * 128:(nt + 1) * 128], 128)
            want = oracle.epilogue_fp16(oracle.gemm_int(X8s, d["Wint"]), s_xs, d["s_w"])
            assert_fp16_close(Yh[:, nt * 128:(nt + 1) * 128], want, "graph case %d tile %d" % (i, nt))


# ------------------------------------------------ full matrices at prefill sizes

@pytest.mark.parametrize("M,N,K", [(2048, 4096, 14336), (4096, 28672, 4096)])
def test_full_matrix_against_library_int8_gemm(M, N, K):
    """Every element at a prefill size: X8 against the oracle's activation
    quantiser; the INT32 GEMM against a library INT8 GEMM (torch._int_mm,
    independent of this library's kernels) of the oracle's X8 and Wint; the
    FP16 output against the oracle's epilogue of those sums (<= 1 ulp)."""
    t = torch()
    W = inputs.make_weights(N, K, seed=31)
    X = inputs.make_activations(M, K, seed=31, token_scale_span=(-3, 1))
    d = oracle.quantize_weights_group(W)
    X8o, s_xo, _ = oracle.quantize_act_per_token(X)
    ref = t._int_mm(dev(X8o), dev(d["Wint"]).t())
    t.cuda.synchronize()

    blob = qoq.quantize_weights(dev(W), 128)
    X8, s_x, rs = qoq.quantize_act_per_token(dev(X))
    ws = qoq.Workspace.for_shape(M, N, K, 128)
    acc = qoq.w4a8_gemm(X8, blob, N, K, 128, rowsum=rs, ws=ws)
    Y = qoq.gemm_fp16_out(X8, s_x, blob, N, K, 128, rowsum=rs, ws=ws)
    t.cuda.synchronize()
    assert ws.status() == 0
    assert t.equal(X8, dev(X8o)), "X8 differs from the oracle"
    assert np.array_equal(host(s_x).view(np.uint16), s_xo.view(np.uint16))
    assert t.equal(acc, ref), "INT32 sums differ from the library INT8 GEMM of the oracle's operands"
    want = oracle.epilogue_fp16(host(ref), s_xo, d["s_w"])
    assert_fp16_close(host(Y), want, "full FP16 output")


# ------------------------------------- the whole linear layer in one call

def _oracle_tile_y(X8s, s_xs, rss, W, nt, group):
    _, d = oracle.quantize_weights(W[nt * 128:(nt + 1) * 128], group)
    if group:
        return oracle.epilogue_fp16(oracle.gemm_int(X8s, d["Wint"]), s_xs, d["s_w"])
    return oracle.epilogue_fp16(oracle.w4a8_gemm_per_channel(X8s, rss, d["q"], d["z"]), s_xs, d["s"])


@pytest.mark.parametrize("group", [128, 0])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (7, 384, 640), (16, 6144, 4096), (33, 28672, 4096),
                                   (64, 4096, 14336), (64, 6144, 4096), (100, 512, 640), (256, 4096, 4096),
                                   (300, 512, 640)])
def test_linear_matches_oracle(M, N, K, group):
    """qoq_w4a8_linear (per-token quantisation and GEMM in one call; one
    launch when the token tile is at most 64 tokens): the FP16 output equals
    the two-call path (act quant, then qoq_gemm_fp16_out) bit for bit, and the
    oracle within 1 ulp on every row of sampled n-tiles; the workspace's
    control words (claim counters included) are left zero."""
    t = torch()
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
    assert t.equal(Y.view(t.int16), Y2.view(t.int16)), "one-call and two-call paths differ"
    X8s, s_xs, rss = oracle.quantize_act_per_token(X)
    Yh = host(Y)
    for nt in sample_tiles(N // 128, count=3, seed=M):
        assert_fp16_close(Yh[:, nt * 128:(nt + 1) * 128], _oracle_tile_y(X8s, s_xs, rss, W, nt, group),
                          "linear tile %d" % nt)


def test_linear_graph_replays_are_bit_identical():
    """One-launch linear calls of the four Llama-3-8B decode shapes captured in
    a CUDA graph and replayed back to back (each launch's CTAs start while the
    previous launch runs): every replay reproduces the eager outputs with a
    clean status and cleared claim counters."""
    t = torch()
    probs = []
    for i, (K, N, _) in enumerate(inputs.LLAMA3_8B):
        M = (1, 16, 33, 64)[i]
        X = inputs.make_activations(M, K, seed=950 + i)
        W = inputs.make_weights(N, K, seed=950 + i)
        probs.append(dict(M=M, N=N, K=K, X=X, W=W, Xd=dev(X), blob=qoq.quantize_weights(dev(W), 128),
                          Y=t.empty((M, N), dtype=t.float16, device="cuda"), ws=qoq.Workspace.for_linear(M, N, K)))

    def step():
        for p in probs:
            qoq.linear(p["Xd"], p["blob"], p["N"], p["K"], 128, ws=p["ws"], Y=p["Y"])

    stream = t.cuda.Stream()
    stream.wait_stream(t.cuda.current_stream())
    with t.cuda.stream(stream):
        step()
    stream.synchronize()
    ref = [p["Y"].clone() for p in probs]
    g = t.cuda.CUDAGraph()
    with t.cuda.graph(g, stream=stream):
        step()
    for r in range(30):
        with t.cuda.stream(stream):
            g.replay()
        stream.synchronize()
        for i, p in enumerate(probs):
            assert p["ws"].status() == 0, "replay %d case %d: %d %s" % (r, i, p["ws"].status(), p["ws"].timeout_site())
            assert p["ws"].control_clear(), "replay %d case %d: control words left set" % (r, i)
            assert t.equal(p["Y"], ref[i]), "replay %d case %d differs" % (r, i)
    del g
    for i, p in enumerate(probs):
        X8s, s_xs, rss = oracle.quantize_act_per_token(p["X"])
        for nt in sample_tiles(p["N"] // 128, count=2, seed=i)[:2]:
            assert_fp16_close(host(ref[i])[:, nt * 128:(nt + 1) * 128],
                              _oracle_tile_y(X8s, s_xs, rss, p["W"], nt, 128), "graph linear %d tile %d" % (i, nt))


def test_concurrent_gemms_on_two_streams():
    """Stream-K GEMMs running at the same time on two streams, each with its
    own workspace, 20 launches each, interleaved: decode sizes (decode kernel)
    and prefill sizes (256-token tiles on CTA pairs, 128-token tiles; every
    tile split between CTAs at these sizes). No CTA of either waits for one
    that has not started, so every launch completes with status 0 and the
    outputs of the serial run."""
    t = torch()
    cases = [(16, 28672, 4096), (1, 4096, 14336), (64, 4096, 4096), (2048, 4096, 4096), (1000, 6144, 4096),
             (300, 4096, 4096)]
    probs = []
    for i, (M, N, K) in enumerate(cases):
        X = inputs.make_activations(M, K, seed=970 + i)
        W = inputs.make_weights(N, K, seed=970 + i)
        blob = qoq.quantize_weights(dev(W), 128)
        X8, s_x, rs = qoq.quantize_act_per_token(dev(X))
        probs.append(dict(M=M, N=N, K=K, X=X, W=W, X8=X8, s_x=s_x, rs=rs, blob=blob,
                          ref=qoq.gemm_fp16_out(X8, s_x, blob, N, K, 128, rowsum=rs)))
    t.cuda.synchronize()
    streams = [t.cuda.Stream(), t.cuda.Stream()]
    outs = {}
    for si, s in enumerate(streams):
        s.wait_stream(t.cuda.current_stream())
    for rep in range(20):
        for i, p in enumerate(probs):
            s = streams[(i + rep) % 2]
            key = (i, (i + rep) % 2)
            if key not in outs:
                outs[key] = (qoq.Workspace.for_shape(p["M"], p["N"], p["K"]),
                             t.empty((p["M"], p["N"]), dtype=t.float16, device="cuda"))
                s.wait_stream(t.cuda.current_stream())
            ws, Y = outs[key]
            with t.cuda.stream(s):
                qoq.gemm_fp16_out(p["X8"], p["s_x"], p["blob"], p["N"], p["K"], 128, rowsum=p["rs"], ws=ws, Y=Y,
                                  stream=s)
    t.cuda.synchronize()
    for (i, si), (ws, Y) in outs.items():
        assert ws.status() == 0, "case %d stream %d: status %d %s" % (i, si, ws.status(), ws.timeout_site())
        assert ws.control_clear()
        assert t.equal(Y, probs[i]["ref"]), "case %d stream %d differs from the serial run" % (i, si)
    for i, p in enumerate(probs):
        X8s, s_xs, rss = oracle.quantize_act_per_token(p["X"])
        nt = sample_tiles(p["N"] // 128, seed=i)[1]
        assert_fp16_close(host(p["ref"])[:, nt * 128:(nt + 1) * 128],
                          _oracle_tile_y(X8s, s_xs, rss, p["W"], nt, 128), "concurrent case %d" % i)


@pytest.mark.parametrize("fuse", [0, 1])
def test_linear_both_launch_configurations(fuse):
    """The one-call linear path with the activation quantisation in its own
    launch (fuse=0) and inside the decode GEMM's launch (fuse=1), each in a
    fresh process (the configuration is read once per process): bit for bit
    the two-call path, within 1 ulp of the oracle, and stable over graph
    replays."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, QOQ_FORCE_CONFIG="fuse=%d" % fuse)
    r = subprocess.run([sys.executable, os.path.join(here, "linear_check.py"), str(2 - fuse)], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "linear_check ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]


def test_split_tiles_finished_by_a_late_contributor():
    """Every contributor to a split tile arrives 300 us late (in a process of
    its own: tests/gemm_late_check.py), so every split tile of both GEMM
    kernels is finished by a contributor from the owner's stored partial
    sums: bit-exact INT32 and FP16 within 1 ulp of the oracle, status 0,
    control words clear."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    env = dict(os.environ, QOQ_FORCE_CONFIG="lateck=300")
    r = subprocess.run([sys.executable, os.path.join(here, "gemm_late_check.py")], env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0 and "gemm_late_check ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
