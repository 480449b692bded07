"""Shared pieces of the GPU parity tests: upload inputs, run the CUDA path
through the C ABI, and compare with the CPU oracle."""
from __future__ import annotations

import numpy as np

import oracle
from w4a8_quantized_gemm_qoq_b200 import inputs, qoq

ULP_TOL = 1   # FP16 outputs: at most 1 unit in the last place from the oracle's FP32 epilogue


def torch():
    import torch as _t
    return _t


def dev(a):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    torch().cuda.synchronize()
    return t.cpu().numpy()


def assert_fp16_close(got, want, what=""):
    d = oracle.fp16_ulp_distance(got, want)
    assert d.max(initial=0) <= ULP_TOL, "%s: max ulp distance %d at %s" % (what, d.max(), np.unravel_index(d.argmax(), d.shape))


def gpu_linear(X, W, group):
    """Whole path on the GPU: weight blob, act quant, INT32 GEMM, FP16 GEMM."""
    N, K = W.shape
    Wd, Xd = dev(W), dev(X)
    blob = qoq.quantize_weights(Wd, group)
    X8, s_x, rowsum = qoq.quantize_act_per_token(Xd)
    ws = qoq.Workspace.for_shape(X.shape[0], N, K, group)
    acc = qoq.w4a8_gemm(X8, blob, N, K, group, rowsum=rowsum, ws=ws)
    Y = qoq.gemm_fp16_out(X8, s_x, blob, N, K, group, rowsum=rowsum, ws=ws)
    torch().cuda.synchronize()
    assert ws.status() == 0
    return dict(blob=host(blob), X8=host(X8), s_x=host(s_x), rowsum=host(rowsum), acc=host(acc), Y=host(Y),
                ws=ws)


def check_full(X, W, group, what=""):
    """Element-by-element parity of every intermediate and output."""
    r = oracle.reference_forward(X, W, group)
    g = gpu_linear(X, W, group)
    assert np.array_equal(g["X8"], r["X8"]), what + " X8"
    assert np.array_equal(g["s_x"].view(np.uint16), r["s_x"].view(np.uint16)), what + " s_x"
    assert np.array_equal(g["rowsum"], r["rowsum"]), what + " rowsum"
    assert np.array_equal(g["blob"], r["blob"]), what + " blob"
    assert np.array_equal(g["acc"], r["acc"]), what + " acc"
    assert_fp16_close(g["Y"], r["Y"], what + " Y")
    assert g["ws"].control_clear(), what + " workspace control words not left zero"
    return r, g


def sample_tiles(NT, count=4, seed=0):
    rng = np.random.default_rng(seed)
    pick = {0, NT - 1, NT // 2}
    pick.update(int(x) for x in rng.choice(NT, size=min(NT, count), replace=False))
    return sorted(pick)


_WCACHE = {}


def cached_weights(N, K, group, seed, std):
    """Host weights, their GPU blob and the oracle's per-tile quantisation,
    kept for one (N, K, group, seed, std) at a time so that the M values of a
    shape reuse them (the largest shapes take seconds to draw)."""
    key = (N, K, group, seed, std)
    if key not in _WCACHE:
        _WCACHE.clear()
        W = inputs.make_weights(N, K, seed=seed, std=std)
        blob = qoq.quantize_weights(dev(W), group)
        _WCACHE[key] = dict(W=W, blob=blob, blob_h=host(blob), tiles={})
    return _WCACHE[key]


def check_sampled(M, N, K, group, seed=0, std=0.02, token_scale_span=None, rows=16, wseed=None):
    """Full-size GPU run; oracle on sampled token rows x sampled 128-row n-tiles
    (the oracle quantises only those weight rows, which is exact because both
    weight levels are per output channel). ``wseed`` (default ``seed``) seeds
    the weights, so that the M values of one shape can share them."""
    t = torch()
    wseed = seed if wseed is None else wseed
    c = cached_weights(N, K, group, wseed, std)
    W, blob, blob_h = c["W"], c["blob"], c["blob_h"]
    X = inputs.make_activations(M, K, seed=seed, token_scale_span=token_scale_span)
    Xd = dev(X)
    X8, s_x, rowsum = qoq.quantize_act_per_token(Xd)
    ws = qoq.Workspace.for_shape(M, N, K, group)
    Y = qoq.gemm_fp16_out(X8, s_x, blob, N, K, group, rowsum=rowsum, ws=ws)
    acc = qoq.w4a8_gemm(X8, blob, N, K, group, rowsum=rowsum, ws=ws)
    t.cuda.synchronize()
    assert ws.status() == 0
    del Xd
    mrows = inputs.sample_rows(M, rows, seed=seed)
    tiles = sample_tiles(N // 128, seed=seed)
    ncols = np.concatenate([np.arange(nt * 128, nt * 128 + 128) for nt in tiles])
    X8s, s_xs, rss = oracle.quantize_act_per_token(X[mrows])
    rows_d = t.from_numpy(mrows).cuda()
    assert np.array_equal(host(X8[rows_d]), X8s)
    assert np.array_equal(host(s_x)[mrows].view(np.uint16), s_xs.view(np.uint16))
    assert np.array_equal(host(rowsum)[mrows], rss)
    L = oracle.blob_layout(N, K, group)
    KT = K // 128
    for nt in tiles:
        if nt not in c["tiles"]:
            c["tiles"][nt] = oracle.quantize_weights(W[nt * 128:(nt + 1) * 128], group)
        bt, d = c["tiles"][nt]
        Lt = oracle.blob_layout(128, K, group)
        lo = L["off_codes"] + nt * KT * L["block"]
        assert np.array_equal(blob_h[lo:lo + KT * L["block"]], bt[Lt["off_codes"]:Lt["off_scale"]]), "blob tile %d" % nt
        sc = blob_h[L["off_scale"] + nt * 256: L["off_scale"] + nt * 256 + 256]
        assert np.array_equal(sc, bt[Lt["off_scale"]:Lt["off_scale"] + 256]), "scales tile %d" % nt
        if group:
            ref_acc = oracle.gemm_int(X8s, d["Wint"])
            ref_y = oracle.epilogue_fp16(ref_acc, s_xs, d["s_w"])
        else:
            zc = blob_h[L["off_zero"] + nt * 256: L["off_zero"] + nt * 256 + 256]
            assert np.array_equal(zc, bt[Lt["off_zero"]:Lt["off_zero"] + 256]), "zero points tile %d" % nt
            ref_acc = oracle.w4a8_gemm_per_channel(X8s, rss, d["q"], d["z"])
            ref_y = oracle.epilogue_fp16(ref_acc, s_xs, d["s"])
        cols = t.arange(nt * 128, nt * 128 + 128, device="cuda")
        got_acc = host(acc[rows_d][:, cols])
        got_y = host(Y[rows_d][:, cols])
        assert np.array_equal(got_acc, ref_acc), "acc tile %d" % nt
        assert_fp16_close(got_y, ref_y, "Y tile %d" % nt)
    assert ws.control_clear()
    return ncols
