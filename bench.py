"""Benchmark of the QoQ W4A8 hot path on B200: per-token activation
quantisation + W4A8 GEMM with the fused FP16 epilogue.

One step = every GEMM of the workload once, each preceded by the per-token
quantisation of its activations:
  decode  (default): Llama-3-8B linear shapes (K->N) 4096->6144 (qkv),
                     4096->4096 (o), 4096->28672 (gate+up), 14336->4096 (down)
                     x M in {1, 4, 16, 64, 256}: 20 GEMMs, HBM-bound regime
  prefill:           the same shapes x M in {2048, 8192, 16384}, per-token
                     scales spanning 1e-3..1e1: INT8-tensor-bound regime
Weights are packed once (offline step, not timed); every GEMM of a step reads
its own copy of the packed weights, so the weights a step streams (about
550 MB for decode) exceed the 126 MB L2 and every launch reads from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode|prefill]
    python bench.py --impl reference ...   (the CPU oracle, timed on host cores)

Prints one JSON line. Multi-GPU (torchrun): every rank runs the same step on
its own GPU (independent problems, no collective on the data path; weak
scaling); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from w4a8_quantized_gemm_qoq_b200 import inputs  # noqa: E402

METRIC = "W4A8 GEMM TOPS and % of roofline vs M on Llama-3-8B linear shapes (1 B200)"
GROUP = 128
SHAPES = [(K, N) for (K, N, _) in inputs.LLAMA3_8B]
NAMES = [name for (_, _, name) in inputs.LLAMA3_8B]
WORKLOADS = {
    "decode": dict(M=inputs.DECODE_M, span=None, shapes=inputs.LLAMA3_8B, group=GROUP, std=0.02, bound="hbm",
                   desc="Llama-3-8B decode GEMMs (qkv 4096->6144, o 4096->4096, gate_up 4096->28672, "
                        "down 14336->4096) x M in {1,4,16,64,256}, g128, act-quant + GEMM"),
    "prefill": dict(M=inputs.PREFILL_M, span=(-3, 1), shapes=inputs.LLAMA3_8B, group=GROUP, std=0.02,
                    bound="tensor",
                    desc="Llama-3-8B prefill GEMMs (same four shapes) x M in {2048,8192,16384}, g128, "
                         "per-token scales 1e-3..1e1, act-quant + GEMM"),
    "qwen": dict(M=inputs.QWEN_M, span=None, shapes=inputs.QWEN15_72B, group=GROUP, std=0.01, bound="mixed",
                 desc="Qwen1.5-72B GEMMs (qkv 8192->24576, o 8192->8192, gate_up 8192->49152, "
                      "down 24576->8192) x M in {1,16,128,512,4096}, g128, act-quant + GEMM"),
    "perchannel": dict(M=inputs.PER_CHANNEL_M, span=None, shapes=inputs.LLAMA2_7B, group=0, std=0.02,
                       bound="mixed",
                       desc="per-channel variant (no group level) on Llama-2-7B GEMMs (qkv 4096->12288, "
                            "o 4096->4096, gate_up 4096->22016, down 11008->4096) x M in 1..1024 (powers of 2), "
                            "act-quant + GEMM"),
}


def gemm_bytes(M, N, K, group=GROUP):
    """Algorithmic HBM bytes of one W4A8 GEMM: 4-bit weights, (s, z*s) per
    group and s_w (group 128), or the FP16 s and z per channel plus the row
    sums (per-channel variant); X8, s_x and the FP16 output."""
    if group:
        return 0.5 * N * K + 2 * N * (K // group) + 2 * N + M * K + 2 * M + 2 * M * N
    return 0.5 * N * K + 4 * N + M * K + 2 * M + 4 * M + 2 * M * N


def gemm_ops(M, N, K):
    return 2.0 * M * N * K


def act_bytes(M, K):
    return 2 * M * K + M * K + 2 * M + 4 * M


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def measured_traffic(workload):
    """DRAM bytes per GEMM launch (dram__bytes_read.sum + dram__bytes_write.sum)
    from the committed ncu summary of this workload, or None when there is
    none or the GEMM sources have changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "qoq_gemm_%s_llama3_8b_dram.md" % workload)
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.split(":")[0] in ("kernel_sources_sha256", "traffic_per_launch_bytes"):
                k, v = line.split(":", 1)
                vals[k] = v.strip()
    h = hashlib.sha256()
    for name in ("gemm.cu", "qoq_device.cuh"):
        with open(os.path.join(ROOT, "w4a8_quantized_gemm_qoq_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    if vals.get("kernel_sources_sha256") != h.hexdigest() or "traffic_per_launch_bytes" not in vals:
        return None
    return int(vals["traffic_per_launch_bytes"])


def roof_us(M, N, K, peaks, group=GROUP):
    """Roofline time: the slower of HBM bytes and INT8 tensor work (INT8 peak =
    2 x the measured dense bf16 peak, the nominal 4.5/2.25 PFLOP/s ratio)."""
    t_mem = gemm_bytes(M, N, K, group) / (peaks["hbm"] * 1e9)
    t_tc = gemm_ops(M, N, K) / (2.0 * peaks["bf16"] * 1e12)
    return max(t_mem, t_tc) * 1e6, ("hbm" if t_mem >= t_tc else "tensor")


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Read-only NVML polling (about every 2 ms) of SM clock and clock-event
    reasons while the timed region runs."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, uuid: str | None, period_s: float = 0.002):
        self.uuid, self.period = uuid, period_s
        self.samples = []
        self.max_mhz = None
        self._stop = None
        self._th = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid) if self.uuid else pynvml.nvmlDeviceGetHandleByIndex(0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            return self
        self._stop = threading.Event()

        def poll():
            while not self._stop.is_set():
                try:
                    self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), int(get_reasons(h)),
                                         pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0))
                except Exception:
                    pass
                self._stop.wait(self.period)
        self._th = threading.Thread(target=poll, daemon=True)
        self._th.start()
        return self

    def __exit__(self, *a):
        if self._th is not None:
            self._stop.set()
            self._th.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        mhz = sorted(s[0] for s in self.samples)
        reasons = set()
        for _, r, _ in self.samples:
            for bit, nm in self.REASONS.items():
                if r & bit:
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples), "power_w_max": round(max(s[2] for s in self.samples), 1)}


# ------------------------------------------------------------- ranks

def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (NCCL needs the tensor
    on this rank's GPU; gloo takes a CPU tensor)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------- GPU arm

class Problem:
    def __init__(self, K, N, M, blob, X, span, device, group=GROUP, name=""):
        import torch
        from w4a8_quantized_gemm_qoq_b200 import qoq
        self.K, self.N, self.M = K, N, M
        self.group, self.name = group, name
        self.blob = blob
        self.X = X
        self.X8 = torch.empty((M, K), dtype=torch.int8, device=device)
        self.s_x = torch.empty((M,), dtype=torch.float16, device=device)
        self.rowsum = torch.empty((M,), dtype=torch.int32, device=device)
        self.Y = torch.empty((M, N), dtype=torch.float16, device=device)
        self.ws = qoq.Workspace.for_shape(M, N, K, group, device)

    def run(self, qoq, ev=None):
        if ev is not None:
            ev[0].record()
        qoq.quantize_act_per_token(self.X, self.X8, self.s_x, self.rowsum)
        if ev is not None:
            ev[1].record()
        qoq.gemm_fp16_out(self.X8, self.s_x, self.blob, self.N, self.K, self.group, rowsum=self.rowsum,
                          ws=self.ws, Y=self.Y)
        if ev is not None:
            ev[2].record()

    def run_gemm(self, qoq):
        qoq.gemm_fp16_out(self.X8, self.s_x, self.blob, self.N, self.K, self.group, rowsum=self.rowsum,
                          ws=self.ws, Y=self.Y)


def build_problems(workload, device, seed):
    import torch
    from w4a8_quantized_gemm_qoq_b200 import qoq
    wl = WORKLOADS[workload]
    probs = []
    for si, (K, N, name) in enumerate(wl["shapes"]):
        W = torch.from_numpy(inputs.make_weights(N, K, seed=seed + si, std=wl["std"])).to(device)
        blob0 = qoq.quantize_weights(W, wl["group"])
        del W
        for mi, M in enumerate(wl["M"]):
            blob = blob0 if mi == 0 else blob0.clone()        # one copy per GEMM: no L2 reuse in a step
            X = torch.from_numpy(inputs.make_activations(M, K, seed=seed + 100 * si + mi,
                                                         token_scale_span=wl["span"])).to(device)
            probs.append(Problem(K, N, M, blob, X, wl["span"], device, wl["group"], name))
    torch.cuda.synchronize()
    return probs


def run_gpu(args, rank, world, local_rank):
    import torch
    from w4a8_quantized_gemm_qoq_b200 import build as qbuild, qoq
    qbuild.build()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    peaks = load_peaks()
    wl = WORKLOADS[args.workload]
    probs = build_problems(args.workload, device, seed=rank * 1000)
    stream = torch.cuda.Stream(device)
    nP = len(probs)

    # One CUDA graph per step shape: a plain one, and EV_GRAPHS copies that
    # also record per-launch events (external event nodes) for the last steps
    # of the timed region.
    EV_GRAPHS = 4
    with torch.cuda.stream(stream):
        for p in probs:                      # eager warm-up: library load, attributes, first launch
            p.run(qoq)
    stream.synchronize()
    bad = [(p.K, p.N, p.M, p.ws.status(), p.ws.timeout_site()) for p in probs if p.ws.status() != 0]
    assert not bad, "device status after the eager pass (K, N, M, code, (site, block, detail)): %s" % bad
    ev = [[[torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)] for _ in range(nP)]
          for _ in range(EV_GRAPHS)]
    plain = torch.cuda.CUDAGraph()
    with torch.cuda.graph(plain, stream=stream):
        for p in probs:
            p.run(qoq)
    ev_graphs = []
    for g in range(EV_GRAPHS):
        cg = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cg, stream=stream):
            for p, e in zip(probs, ev[g]):
                p.run(qoq, e)
        ev_graphs.append(cg)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            plain.replay()
    stream.synchronize()
    bad = [(p.K, p.N, p.M, p.ws.status(), p.ws.timeout_site()) for p in probs if p.ws.status() != 0]
    assert not bad, "device status (K, N, M, code, (site, block, detail)): %s" % bad

    K = args.steps
    n_ev = min(EV_GRAPHS, K)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(local_rank).uuid)
    except Exception:
        pass
    with ClockSampler(uuid) as clk:
        with torch.cuda.stream(stream):
            t0.record()
            for k in range(K):
                j = k - (K - n_ev)
                (ev_graphs[j] if j >= 0 else plain).replay()
            t1.record()
        stream.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = max_over_ranks(t0.elapsed_time(t1) / K, device) if world > 1 else t0.elapsed_time(t1) / K
    gemm_ms = [sum(ev[g][i][1].elapsed_time(ev[g][i][2]) for g in range(n_ev)) / n_ev for i in range(nP)]
    act_ms = [sum(ev[g][i][0].elapsed_time(ev[g][i][1]) for g in range(n_ev)) / n_ev for i in range(nP)]
    bad = [(p.K, p.N, p.M, p.ws.status(), p.ws.timeout_site()) for p in probs if p.ws.status() != 0]
    assert not bad, "device status (K, N, M, code, (site, block, detail)): %s" % bad

    # The dominant kernel alone: the step's GEMMs (inputs already quantised by
    # the step) replayed back to back in one graph, CUDA events around the
    # replays only; every GEMM still reads its own weight copy, so the graph
    # streams more than L2 holds. Its per-launch average is the roofline's
    # launch duration (per-launch events inside the step break the overlap of
    # consecutive kernels and overstate each launch).
    gg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gg, stream=stream):
        for p in probs:
            p.run_gemm(qoq)
    with torch.cuda.stream(stream):
        for _ in range(3):
            gg.replay()
    stream.synchronize()
    KG = max(K, 10)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g0.record()
        for _ in range(KG):
            gg.replay()
        g1.record()
    stream.synchronize()
    gemm_only_ms = g0.elapsed_time(g1) / KG
    if world > 1:
        gemm_only_ms = max_over_ranks(gemm_only_ms, device)
    bad = [(p.K, p.N, p.M, p.ws.status(), p.ws.timeout_site()) for p in probs if p.ws.status() != 0]
    assert not bad, "device status (K, N, M, code, (site, block, detail)): %s" % bad
    gemm_only_us = 1000.0 * gemm_only_ms

    ops_step = sum(gemm_ops(p.M, p.N, p.K) for p in probs)
    per = []
    tot_bytes = tot_gemm_us = 0.0
    for i, p in enumerate(probs):
        us = 1000.0 * gemm_ms[i]
        b = gemm_bytes(p.M, p.N, p.K, p.group)
        r_us, bound = roof_us(p.M, p.N, p.K, peaks, p.group)
        aq_us = 1000.0 * act_ms[i]
        per.append({"shape": p.name, "K": p.K, "N": p.N, "M": p.M,
                    "gemm_us_in_step": round(us, 3), "act_quant_us_in_step": round(aq_us, 3),
                    "act_quant_GBps_in_step": round((3.0 * p.M * p.K + 6 * p.M) / aq_us / 1e3, 1),
                    "TOPS": round(gemm_ops(p.M, p.N, p.K) / us / 1e6, 2), "GBps": round(b / us / 1e3, 1),
                    "roof_us": round(r_us, 3), "bound": bound, "frac_of_roofline": round(r_us / us, 3)})
        tot_bytes += b
        tot_gemm_us += us
    timing = {"launch_us": round(gemm_only_us / nP, 3), "launches": nP, "replays": KG,
              "how": "graph of the step's %d GEMM launches replayed back to back; CUDA events around the "
                     "replays on the launching stream" % nP}
    if wl["bound"] == "hbm":
        achieved = tot_bytes / gemm_only_us / 1e3
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
                    "frac": round(achieved / peaks["hbm"], 4), "traffic": measured_traffic("decode"),
                    "algorithmic_bytes_per_launch": round(tot_bytes / nP),
                    "peak_source": peaks["src"], "kernel": "qoq_gemm_kernel",
                    "frac_of_time_roofline": round(sum(x["roof_us"] for x in per) / gemm_only_us, 4),
                    "timing": timing}
    elif wl["bound"] == "tensor":
        achieved = ops_step / gemm_only_us / 1e6
        pk = 2.0 * peaks["bf16"]
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": pk, "unit": "TOPS",
                    "frac": round(achieved / pk, 4), "traffic": None, "peak_source": peaks["src"] +
                    " (INT8 = 2 x measured bf16 burst, nominal ratio)", "kernel": "qoq_gemm_kernel",
                    "frac_of_time_roofline": round(sum(x["roof_us"] for x in per) / gemm_only_us, 4),
                    "timing": timing}
    else:
        # Shapes on both sides of the crossover: the fraction is roofline time
        # (each GEMM's slower bound) over measured time, summed over the step.
        roof = sum(x["roof_us"] for x in per)
        roofline = {"bound": "mixed", "achieved": round(roof / gemm_only_us, 4), "peak": 1.0,
                    "unit": "fraction of each GEMM's roofline time", "frac": round(roof / gemm_only_us, 4),
                    "traffic": None, "peak_source": peaks["src"], "kernel": "qoq_gemm_kernel",
                    "frac_of_time_roofline": round(roof / gemm_only_us, 4), "timing": timing}

    e2e = run_e2e(args, probs, qoq, stream) if rank == 0 else None
    w8a8 = run_w8a8(probs, stream, gemm_only_us, max(K, 10)) if rank == 0 else None
    producers = run_producers(stream, peaks) if rank == 0 and not args.no_context else None
    saturation = run_saturation(stream) if rank == 0 and args.saturation else None
    res = {
        "metric": METRIC, "value": round(world * ops_step / (step_ms * 1e-3) / 1e12, 3), "unit": "TOPS",
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(step_ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic",
        "config": {"workload": wl["desc"], "M": wl["M"], "shapes_K_N": [(K, N) for (K, N, _) in wl["shapes"]],
                   "group_size": wl["group"],
                   "l2": "inputs larger than L2: each GEMM of a step reads its own packed-weight copy "
                         "(%.0f MB per step)" % (sum(0.5 * p.N * p.K + (p.N * p.K / 64 if p.group else 4 * p.N)
                                                     for p in probs) / 1e6),
                   "launch": "CUDA graph replay of the step; per-launch events from the last %d steps" % n_ev,
                   "parallelism": "replicas (one independent step per GPU)" if world > 1 else "single GPU"},
        "roofline": roofline,
        "gpu_launches": 2 * nP * args.steps,
        "clocks": clk.summary(),
        "e2e": e2e,
        "per_gemm": per,
        "w8a8_context": w8a8,
        "producers_context": producers,
        "saturation_context": saturation,
    }
    return res


def run_shape(args):
    """One M x N x K GEMM alone: weights packed and activations quantised
    once, then `steps` launches of qoq_gemm_fp16_out captured back to back in
    one CUDA graph and replayed (after `warmup` eager launches and one
    replay), between CUDA events: the device-side period of a launch, free of
    host launch cost. Weight copies alternate so that no launch finds its
    weights in L2 (enough copies to exceed it)."""
    import torch
    from w4a8_quantized_gemm_qoq_b200 import build as qbuild, qoq
    qbuild.build()
    M, N, K = (int(v) for v in args.shape.lower().split("x"))
    dev = torch.device("cuda", 0)
    W = torch.from_numpy(inputs.make_weights(N, K, seed=1)).to(dev)
    blob = qoq.quantize_weights(W, GROUP)
    del W
    copies = max(2, int(300e6 // blob.numel()) + 1)
    blobs = [blob] + [blob.clone() for _ in range(copies - 1)]
    X = torch.from_numpy(inputs.make_activations(M, K, seed=1)).to(dev)
    X8, s_x, rs = qoq.quantize_act_per_token(X)
    ws = qoq.Workspace.for_shape(M, N, K, GROUP, dev)
    Y = torch.empty((M, N), dtype=torch.float16, device=dev)
    stream = torch.cuda.Stream(dev)
    stream.wait_stream(torch.cuda.current_stream())   # inputs and the zeroed workspace were made on the default stream
    with torch.cuda.stream(stream):
        for i in range(max(1, args.warmup)):
            qoq.gemm_fp16_out(X8, s_x, blobs[i % copies], N, K, GROUP, rowsum=rs, ws=ws, Y=Y)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(args.steps):
            qoq.gemm_fp16_out(X8, s_x, blobs[i % copies], N, K, GROUP, rowsum=rs, ws=ws, Y=Y)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        graph.replay()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    stream.synchronize()
    assert ws.status() == 0, "device status %d" % ws.status()
    us = 1000.0 * e0.elapsed_time(e1) / args.steps
    del graph
    return {"shape": [M, N, K], "launches": args.steps, "us_per_launch": round(us, 3),
            "how": "one CUDA graph of back-to-back launches, replayed",
            "GBps": round(gemm_bytes(M, N, K) / us / 1e3, 1), "TOPS": round(gemm_ops(M, N, K) / us / 1e6, 2)}


def run_saturation(stream, reps=20):
    """Context, not the product: the protective range's point on this GPU.
    The same GEMM with the excess-128 decode (protective range: no saturation
    can occur) and with a decode that saturates every byte (what a kernel
    without the protective range must do), on the gate_up projection at decode
    (M = 16) and prefill (M = 2048) sizes: one graph of back-to-back launches,
    each launch its own weight copy (more than L2 together), events around the
    replays. The two outputs are bit-identical (GPU test)."""
    import torch
    from w4a8_quantized_gemm_qoq_b200 import qoq
    dev = torch.device("cuda", torch.cuda.current_device())
    out = []
    K, N = 4096, 28672
    W = torch.from_numpy(inputs.make_weights(N, K, seed=5)).to(dev)
    blob = qoq.quantize_weights(W, GROUP)
    del W
    blobs = [blob] + [blob.clone() for _ in range(int(300e6 // blob.numel()))]
    for M in (16, 2048):
        X = torch.from_numpy(inputs.make_activations(M, K, seed=5)).to(dev)
        X8, s_x, rs = qoq.quantize_act_per_token(X)
        ws = qoq.Workspace.for_shape(M, N, K, GROUP, dev)
        Y = torch.empty((M, N), dtype=torch.float16, device=dev)
        res = {"M": M, "N": N, "K": K}
        for key, fn in (("protective_us", lambda b: qoq.gemm_fp16_out(X8, s_x, b, N, K, GROUP, rowsum=rs, ws=ws,
                                                                      Y=Y, stream=stream)),
                        ("saturating_us", lambda b: qoq.gemm_fp16_out_saturating(X8, s_x, b, N, K, ws=ws, Y=Y,
                                                                                 stream=stream))):
            stream.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(stream):
                for i in range(3):
                    fn(blobs[i % len(blobs)])
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(reps):
                    fn(blobs[i % len(blobs)])
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                g.replay()
                e0.record(stream)
                g.replay()
                e1.record(stream)
            stream.synchronize()
            assert ws.status() == 0, "device status %d" % ws.status()
            del g
            res[key] = round(1000.0 * e0.elapsed_time(e1) / reps, 3)
        res["saturating_slowdown"] = round(res["saturating_us"] / res["protective_us"], 3)
        out.append(res)
        del X, X8, s_x, rs, ws, Y
    del blobs, blob
    torch.cuda.empty_cache()
    return {"shapes": out, "how": "qoq_gemm_fp16_out vs qoq_gemm_fp16_out_saturating, gate_up 4096->28672; one "
                                  "graph of %d back-to-back launches per variant, own weight copies" % reps}


def run_producers(stream, peaks, reps=20):
    """Context for the fused activation producers (not in the timed step):
    RMSNorm + per-token INT8 on Llama-3-8B hidden rows (K = 4096) and
    SiLU(gate) * up + per-token INT8 on its FFN rows (I = 14336), at decode and
    prefill token counts, next to the stand-alone FP16 activation quantiser on
    the same rows. Each case: `reps` launches back to back in one CUDA graph,
    events around two replays; inputs of 64 MB and more alternate between two
    copies (larger than L2 together), smaller ones stay L2-resident (a latency
    figure). Algorithmic bytes: every input element read once, every code
    written once, plus 6 bytes (scale, row sum) per row."""
    import torch
    from w4a8_quantized_gemm_qoq_b200 import qoq
    dev = torch.device("cuda", torch.cuda.current_device())
    out = []

    def timed(fn, n_in):
        stream.wait_stream(torch.cuda.current_stream())   # inputs were made on the default stream
        with torch.cuda.stream(stream):
            for i in range(max(2, n_in)):
                fn(i)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(reps):
                fn(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            g.replay()
            e0.record(stream)
            g.replay()
            g.replay()
            e1.record(stream)
        stream.synchronize()
        del g
        return 1000.0 * e0.elapsed_time(e1) / (2 * reps)

    for kind, width, Ms in (("rmsnorm_quant", 4096, (16, 2048, 16384)), ("silu_mul_quant", 14336, (16, 2048, 16384))):
        for M in Ms:
            if kind == "rmsnorm_quant":
                x = torch.from_numpy(inputs.make_activations(M, width, seed=M)).to(dev)
                g = torch.from_numpy(inputs.make_norm_weight(width, seed=1)).to(dev)
                nbytes_in = 2 * M * width
            else:
                x = torch.from_numpy(inputs.make_gate_up(M, width, seed=M)).to(dev)
                nbytes_in = 4 * M * width
            xs = [x, x.clone()] if nbytes_in >= 64e6 else [x]
            X8 = torch.empty((M, width), dtype=torch.int8, device=dev)
            s_x = torch.empty((M,), dtype=torch.float16, device=dev)
            rs = torch.empty((M,), dtype=torch.int32, device=dev)
            if kind == "rmsnorm_quant":
                us = timed(lambda i: qoq.rmsnorm_quant(xs[i % len(xs)], g, 1e-5, X8, s_x, rs, stream=stream), len(xs))
                fp16_in = xs
            else:
                us = timed(lambda i: qoq.silu_mul_quant(xs[i % len(xs)], X8, s_x, rs, stream=stream), len(xs))
                fp16_in = [t[:, :width].contiguous() for t in xs]   # an FP16 row of the same width
            aq_us = timed(lambda i: qoq.quantize_act_per_token(fp16_in[i % len(fp16_in)], X8, s_x, rs,
                                                               stream=stream), len(fp16_in))
            b = nbytes_in + M * width + 6 * M
            out.append({"kernel": kind, "M": M, "width": width, "us": round(us, 3),
                        "GBps": round(b / us / 1e3, 1), "frac_of_hbm": round(b / us / 1e3 / peaks["hbm"], 3),
                        "act_quant_alone_us": round(aq_us, 3),
                        "inputs": "two copies, > L2" if len(xs) > 1 else "L2-resident"})
            del xs, fp16_in, x
    torch.cuda.empty_cache()
    return out


def run_w8a8(probs, stream, w4a8_us, reps):
    """Context, not the product: the same GEMM shapes as a W8A8 INT8 GEMM
    through PyTorch (torch._int_mm, cuBLASLt), each problem with its own
    random INT8 weight matrix, replayed back to back in one graph like the
    W4A8 GEMM-only timing. Rows are padded to at least 32 (that routine
    needs more than 16)."""
    import torch
    try:
        dev = probs[0].X8.device
        g = torch.Generator(device=dev)
        g.manual_seed(1234)
        ws, xs, ys = [], [], []
        for p in probs:
            m = max(p.M, 32)
            ws.append(torch.randint(-119, 120, (p.N, p.K), dtype=torch.int8, device=dev, generator=g))
            xs.append(torch.randint(-127, 128, (m, p.K), dtype=torch.int8, device=dev, generator=g))
            ys.append(torch.empty((m, p.N), dtype=torch.int32, device=dev))
        graph = torch.cuda.CUDAGraph()
        stream.wait_stream(torch.cuda.current_stream())   # operands were drawn on the default stream
        with torch.cuda.stream(stream):
            for x, w, y in zip(xs, ws, ys):     # warm-up outside capture (library handles, kernels)
                torch._int_mm(x, w.t(), out=y)
        stream.synchronize()
        with torch.cuda.graph(graph, stream=stream):
            for x, w, y in zip(xs, ws, ys):
                torch._int_mm(x, w.t(), out=y)
        with torch.cuda.stream(stream):
            for _ in range(3):
                graph.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record()
            for _ in range(reps):
                graph.replay()
            e1.record()
        stream.synchronize()
        us = 1000.0 * e0.elapsed_time(e1) / reps
        del graph, ws, xs, ys
        return {"gemm_us_per_step": round(us, 2), "w4a8_gemm_us_per_step": round(w4a8_us, 2),
                "w4a8_speedup": round(us / w4a8_us, 3),
                "how": "torch._int_mm (cuBLASLt INT8) on the same shapes, rows padded to >= 32, one graph "
                       "of the step's GEMMs replayed back to back, events around the replays"}
    except Exception as exc:   # context only: never fails the run
        return {"unavailable": "%s: %s" % (type(exc).__name__, str(exc)[:200])}


def run_e2e(args, probs, qoq, stream):
    """Same metric through the public API with host buffers: every step copies
    each problem's FP16 activations host->device (pinned), runs the two calls,
    and reads the FP16 output back device->host."""
    import torch
    hx = [p.X.cpu().pin_memory() for p in probs]
    hy = [torch.empty(p.Y.shape, dtype=torch.float16).pin_memory() for p in probs]
    dx = [torch.empty_like(p.X) for p in probs]
    h2d = sum(x.numel() * 2 for x in hx)
    d2h = sum(y.numel() * 2 for y in hy)

    def once():
        for p, a, b, c in zip(probs, hx, dx, hy):
            b.copy_(a, non_blocking=True)
            X8, s_x, rs = qoq.quantize_act_per_token(b, p.X8, p.s_x, p.rowsum)
            qoq.gemm_fp16_out(X8, s_x, p.blob, p.N, p.K, p.group, rowsum=rs, ws=p.ws, Y=p.Y)
            c.copy_(p.Y, non_blocking=True)

    steps = max(1, args.steps)
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for _ in range(3):
            once()
        stream.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            once()
        e1.record()
    stream.synchronize()
    ms = e0.elapsed_time(e1) / steps
    ops = sum(gemm_ops(p.M, p.N, p.K) for p in probs)
    return {"value": round(ops / (ms * 1e-3) / 1e12, 3), "unit": "TOPS", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 4),
            "launch": "eager calls through the C ABI, pinned host buffers"}


# ------------------------------------------------------------- CPU oracle

def oracle_sample(workload, seed=0):
    """A bounded sample of the workload for the CPU oracle: the o-projection
    GEMM (K=N=4096) at M=16 (decode-sized workloads) or M=64 (prefill), weights
    quantised beforehand (offline), act-quant + int64 GEMM + FP16 epilogue
    timed; the per-channel workload uses the per-channel scheme."""
    import oracle
    K, N = 4096, 4096
    M = 64 if workload == "prefill" else 16
    wl = WORKLOADS[workload]
    W = inputs.make_weights(N, K, seed=seed, std=wl["std"])
    X = inputs.make_activations(M, K, seed=seed, token_scale_span=wl["span"])
    if wl["group"]:
        d = oracle.quantize_weights_group(W)

        def once():
            X8, s_x, rowsum = oracle.quantize_act_per_token(X)
            acc = oracle.gemm_int(X8, d["Wint"])
            oracle.epilogue_fp16(acc, s_x, d["s_w"])
    else:
        d = oracle.quantize_weights_per_channel(W)

        def once():
            X8, s_x, rowsum = oracle.quantize_act_per_token(X)
            t = oracle.w4a8_gemm_per_channel(X8, rowsum, d["q"], d["z"])
            oracle.epilogue_fp16(t, s_x, d["s"])
    desc = "o-proj GEMM K=N=4096, M=%d: act quant + int64 triple-loop GEMM + FP16 epilogue " \
           "(weights pre-quantised%s)" % (M, "" if wl["group"] else ", per-channel variant")
    return once, gemm_ops(M, N, K), desc


def time_oracle(workload, budget_s=10.0, min_runs=1):
    once, ops, desc = oracle_sample(workload)
    once()   # compile/load the C part outside the timing
    n, t0 = 0, time.perf_counter()
    while True:
        once()
        n += 1
        el = time.perf_counter() - t0
        if n >= min_runs and el >= budget_s:
            break
    return {"value": round(ops * n / el / 1e12, 6), "unit": "TOPS", "cores": 1, "kind": "oracle",
            "sample": "%s; %d runs in %.1f s" % (desc, n, el)}


def run_reference(args):
    """--impl reference: the CPU oracle, as it stands, on the host cores."""
    cb_steps = []
    once, ops, desc = oracle_sample(args.workload)
    once()
    for _ in range(max(0, args.warmup)):
        once()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        s = time.perf_counter()
        once()
        cb_steps.append(time.perf_counter() - s)
    el = time.perf_counter() - t0
    val = ops * args.steps / el / 1e12
    return {"impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": "TOPS", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1000 * el / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
            "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload]["desc"], "sample": desc},
            "cpu_baseline": {"value": round(val, 6), "unit": "TOPS", "cores": 1, "kind": "oracle",
                             "sample": "%s; one sample GEMM per step" % desc},
            "e2e": {"value": round(val, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="decode")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--saturation", action="store_true",
                    help="also time the protective-range ablation (saturating weight decode) as context")
    ap.add_argument("--no-context", action="store_true",
                    help="skip the fused-producer context measurements (not part of the timed step)")
    ap.add_argument("--shape", default=None,
                    help="MxNxK: one GEMM shape alone (act quant once, then --steps GEMM launches back to back); "
                         "small footprint for profiling")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)))
        return
    if args.shape:
        print(json.dumps(run_shape(args)))
        return

    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        cpu = time_oracle(args.workload, budget_s=args.cpu_budget)
    res = run_gpu(args, rank, world, local_rank)
    if rank == 0:
        res["cpu_baseline"] = cpu
        print(json.dumps(res))
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
