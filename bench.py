"""Benchmark of the QoQ W4A8 hot path on B200: the linear layer (per-token
activation quantisation + W4A8 GEMM with the fused FP16 epilogue) through the
library's one-call entry point, qoq_w4a8_linear (the quantiser, then the
GEMM; decode batches run on the decode-regime GEMM kernel, prefill batches on
256-token tiles of CTA pairs).

One step = every GEMM of the workload once:
  llama3_8b (default): Llama-3-8B linear shapes (K->N) 4096->6144 (qkv),
                     4096->4096 (o), 4096->28672 (gate+up), 14336->4096 (down)
                     x M in {1, 4, 16, 64, 256} (decode: HBM-bound) and
                     M in {2048, 8192, 16384} (prefill, per-token scales
                     spanning 1e-3..1e1: INT8-tensor-bound): 32 GEMMs
  decode, prefill:   the two halves of it
  qwen, perchannel:  Qwen1.5-72B shapes; the per-channel variant on
                     Llama-2-7B shapes
Weights are packed once (offline step, not timed); every GEMM of a step reads
its own copy of the packed weights, so the weights a step streams exceed the
126 MB L2 and every launch reads from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
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
    "llama3_8b": dict(M=inputs.DECODE_M + inputs.PREFILL_M, span_from=2048, shapes=inputs.LLAMA3_8B, group=GROUP,
                      std=0.02,
                      desc="Llama-3-8B linear layers (qkv 4096->6144, o 4096->4096, gate_up 4096->28672, "
                           "down 14336->4096) x M in {1,4,16,64,256} (decode) and {2048,8192,16384} (prefill, "
                           "per-token scales 1e-3..1e1), g128, act-quant + W4A8 GEMM + FP16 epilogue"),
    "decode": dict(M=inputs.DECODE_M, span_from=None, shapes=inputs.LLAMA3_8B, group=GROUP, std=0.02,
                   desc="Llama-3-8B decode GEMMs (qkv 4096->6144, o 4096->4096, gate_up 4096->28672, "
                        "down 14336->4096) x M in {1,4,16,64,256}, g128, act-quant + GEMM"),
    "prefill": dict(M=inputs.PREFILL_M, span_from=0, shapes=inputs.LLAMA3_8B, group=GROUP, std=0.02,
                    desc="Llama-3-8B prefill GEMMs (same four shapes) x M in {2048,8192,16384}, g128, "
                         "per-token scales 1e-3..1e1, act-quant + GEMM"),
    "qwen": dict(M=inputs.QWEN_M, span_from=None, shapes=inputs.QWEN15_72B, group=GROUP, std=0.01,
                 desc="Qwen1.5-72B GEMMs (qkv 8192->24576, o 8192->8192, gate_up 8192->49152, "
                      "down 24576->8192) x M in {1,16,128,512,4096}, g128, act-quant + GEMM"),
    "perchannel": dict(M=inputs.PER_CHANNEL_M, span_from=None, shapes=inputs.LLAMA2_7B, group=0, std=0.02,
                       desc="per-channel variant (no group level) on Llama-2-7B GEMMs (qkv 4096->12288, "
                            "o 4096->4096, gate_up 4096->22016, down 11008->4096) x M in 1..1024 (powers of 2), "
                            "act-quant + GEMM"),
}
# Regimes the roofline is graded in: HBM-bound decode batches, INT8-tensor-bound prefill batches.
DECODE_HBM_MAX_M = 64
PREFILL_TENSOR_MIN_M = 2048


def token_span(wl, M):
    """Per-token scale span of the workload's M (prefill batches: 1e-3..1e1)."""
    return (-3, 1) if wl["span_from"] is not None and M >= wl["span_from"] else None


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


def measured_traffic(name, sources):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)
    from the committed ncu summary profiles/<name>.md, or None when there is
    none or the kernel's sources have changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", name + ".md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.split(":")[0] in ("kernel_sources_sha256", "traffic_per_launch_bytes"):
                k, v = line.split(":", 1)
                vals[k] = v.strip()
    h = hashlib.sha256()
    for src in sources:
        with open(os.path.join(ROOT, "w4a8_quantized_gemm_qoq_b200", "csrc", src), "rb") as f:
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
    """One linear layer of the step: FP16 X [M][K], its own packed-weight copy,
    FP16 Y [M][N] and the workspace of the one-call path; plus the buffers of
    the two-call path (X8, s_x, row sums, GEMM workspace) for the GEMM-only
    roofline timing."""

    def __init__(self, K, N, M, blob, X, device, group=GROUP, name=""):
        import torch
        from w4a8_quantized_gemm_qoq_b200 import qoq
        self.K, self.N, self.M = K, N, M
        self.group, self.name = group, name
        self.blob = blob
        self.X = X
        self.tok, self.launches = qoq.plan(M, N, K)
        self.Y = torch.empty((M, N), dtype=torch.float16, device=device)
        self.ws_lin = qoq.Workspace.for_linear(M, N, K, group, device)
        self.X8 = torch.empty((M, K), dtype=torch.int8, device=device)
        self.s_x = torch.empty((M,), dtype=torch.float16, device=device)
        self.rowsum = torch.empty((M,), dtype=torch.int32, device=device)
        self.ws = qoq.Workspace.for_shape(M, N, K, group, device)

    def run(self, qoq, stream=None):
        qoq.linear(self.X, self.blob, self.N, self.K, self.group, ws=self.ws_lin, Y=self.Y, stream=stream)

    def quantize(self, qoq, stream=None):
        qoq.quantize_act_per_token(self.X, self.X8, self.s_x, self.rowsum, stream=stream)

    def run_gemm(self, qoq, stream=None):
        qoq.gemm_fp16_out(self.X8, self.s_x, self.blob, self.N, self.K, self.group, rowsum=self.rowsum,
                          ws=self.ws, Y=self.Y, stream=stream)

    def status(self):
        return self.ws_lin.status() or self.ws.status()


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
                                                         token_scale_span=token_span(wl, M))).to(device)
            probs.append(Problem(K, N, M, blob, X, device, wl["group"], name))
    torch.cuda.synchronize()
    return probs


def graph_time_us(fn, stream, reps):
    """Capture fn() in a CUDA graph, replay it 3 times untimed, then `reps`
    times between CUDA events on `stream`; returns microseconds per replay."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    stream.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
    stream.synchronize()
    del g
    return 1000.0 * e0.elapsed_time(e1) / reps


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
    stream.wait_stream(torch.cuda.current_stream())   # inputs and zeroed workspaces were made on the default stream
    nP = len(probs)

    def check(where):
        bad = [(p.K, p.N, p.M, p.status(), p.ws_lin.timeout_site()) for p in probs if p.status() != 0]
        assert not bad, "device status %s (K, N, M, code, (site, block, detail)): %s" % (where, bad)

    with torch.cuda.stream(stream):
        for p in probs:                      # eager pass: library load, attributes, first launch
            p.run(qoq)
    stream.synchronize()
    check("after the eager pass")
    step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(step, stream=stream):
        for p in probs:
            p.run(qoq)
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step.replay()
    stream.synchronize()
    check("after warm-up")

    # ---- the timed region: K replays of the step, nothing else.
    K = args.steps
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
            for _ in range(K):
                step.replay()
            t1.record()
        stream.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    step_ms = max_over_ranks(t0.elapsed_time(t1) / K, device) if world > 1 else t0.elapsed_time(t1) / K
    check("after the timed steps")
    del step

    analysis = analyse(args, probs, qoq, stream, peaks, wl, world, device)
    ops_step = sum(gemm_ops(p.M, p.N, p.K) for p in probs)
    res = {
        "metric": METRIC, "value": round(world * ops_step / (step_ms * 1e-3) / 1e12, 3), "unit": "TOPS",
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": round(step_ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic",
        "gpu_launches": sum(p.launches for p in probs) * args.steps,
        "clocks": clk.summary(),
    }
    res["config"] = {
        "workload": wl["desc"], "M": wl["M"], "shapes_K_N": [(K_, N_) for (K_, N_, _) in wl["shapes"]],
        "group_size": wl["group"],
        "l2": "inputs larger than L2: each GEMM of a step reads its own packed-weight copy (%.0f MB per step)"
              % (sum(0.5 * p.N * p.K + (p.N * p.K / 64 if p.group else 4 * p.N) for p in probs) / 1e6),
        "launch": "CUDA graph replay of the step (qoq_w4a8_linear per GEMM: %d launches per step)"
                  % sum(p.launches for p in probs),
        "parallelism": "replicas (one independent step per GPU)" if world > 1 else "single GPU"}
    res.update(analysis)
    res["e2e"] = run_e2e(args, probs, qoq, stream) if rank == 0 else None
    res["w8a8_context"] = run_w8a8(probs, stream, res["gemm_us_per_step"], max(K, 10)) if rank == 0 else None
    res["producers_context"] = run_producers(stream, peaks) if rank == 0 and not args.no_context else None
    res["kv4_attention_context"] = run_kv4(stream, peaks) if rank == 0 and not args.no_context else None
    res["saturation_context"] = run_saturation(stream) if rank == 0 and args.saturation else None
    return res


def linear_bytes(p):
    """Algorithmic HBM bytes of one qoq_w4a8_linear call: the GEMM's (packed
    weights, scales, X8, s_x, Y) with the FP16 activations read in place of
    X8 (2 M K instead of M K)."""
    return gemm_bytes(p.M, p.N, p.K, p.group) + p.M * p.K


def analyse(args, probs, qoq, stream, peaks, wl, world, device):
    """Everything measured after the timed steps: per-launch durations inside
    the step (external event nodes between the calls: they break the overlap
    of consecutive launches, so they overstate each one), and the roofline of
    each regime from graphs of that regime's launches alone, back to back,
    with CUDA events around the replays only."""
    import torch
    reps = max(args.steps, 10)
    nP = len(probs)
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in probs]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for p, e in zip(probs, ev):
            e[0].record()
            p.run(qoq)
            e[1].record()
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    stream.synchronize()
    in_step = [1000.0 * e[0].elapsed_time(e[1]) for e in ev]
    del g

    out = {}
    regimes = {}
    # Decode batches (HBM-bound): the one-call launches (GEMM quantising its
    # own activations) back to back.
    dec = [p for p in probs if p.M <= DECODE_HBM_MAX_M]
    if dec:
        us = graph_time_us(lambda: [p.run(qoq) for p in dec], stream, reps)
        b = sum(linear_bytes(p) for p in dec)
        ach = b / us / 1e3
        regimes["decode"] = {
            "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm"], 4),
            "traffic": measured_traffic("qoq_decode_linear_llama3_8b_dram", ("gemm_decode.cu", "gemm_common.cuh",
                                                                            "qoq_device.cuh", "quant_math.cuh")),
            "algorithmic_bytes_per_launch": round(b / len(dec)), "peak_source": peaks["src"] + " (HBM copy)",
            "kernel": "act_quant_kernel + qoq_decode_kernel (the linear call's two launches)",
            "frac_of_time_roofline": round(sum(roof_us(p.M, p.N, p.K, peaks, p.group)[0] for p in dec) / us, 4),
            "timing": {"launch_us": round(us / len(dec), 3), "launches": len(dec), "replays": reps,
                       "M": sorted({p.M for p in dec}),
                       "how": "graph of the step's M <= %d linear calls replayed back to back; CUDA events around "
                              "the replays on the launching stream" % DECODE_HBM_MAX_M}}
    # Every GEMM alone on pre-quantised activations (the two-call path).
    with torch.cuda.stream(stream):
        for p in probs:
            p.quantize(qoq)
    stream.synchronize()
    out["gemm_us_per_step"] = round(graph_time_us(lambda: [p.run_gemm(qoq) for p in probs], stream, reps), 2)
    pre = [p for p in probs if p.M >= PREFILL_TENSOR_MIN_M]
    if pre:
        us = graph_time_us(lambda: [p.run_gemm(qoq) for p in pre], stream, reps)
        ops = sum(gemm_ops(p.M, p.N, p.K) for p in pre)
        ach = ops / us / 1e6
        pk = 2.0 * peaks["bf16"]
        regimes["prefill"] = {
            "bound": "tensor", "achieved": round(ach, 1), "peak": pk, "unit": "TOPS", "frac": round(ach / pk, 4),
            "traffic": measured_traffic("qoq_gemm_prefill_llama3_8b_dram", ("gemm.cu", "gemm_common.cuh",
                                                                           "qoq_device.cuh")),
            "algorithmic_ops_per_launch": round(ops / len(pre)),
            "peak_source": peaks["src"] + " (INT8 = 2 x measured bf16 burst, the nominal 4.5/2.25 ratio)",
            "kernel": "qoq_gemm_kernel (256-token tiles on CTA pairs)",
            "frac_of_time_roofline": round(sum(roof_us(p.M, p.N, p.K, peaks, p.group)[0] for p in pre) / us, 4),
            "timing": {"launch_us": round(us / len(pre), 3), "launches": len(pre), "replays": reps,
                       "M": sorted({p.M for p in pre}),
                       "how": "graph of the step's M >= %d GEMM launches (activations quantised beforehand) "
                              "replayed back to back; CUDA events around the replays" % PREFILL_TENSOR_MIN_M}}
    # The dominant kernel: the regime with the larger share of the step.
    share = {k: sum(t for p, t in zip(probs, in_step) if (p.M <= DECODE_HBM_MAX_M if k == "decode"
                                                             else p.M >= PREFILL_TENSOR_MIN_M))
             for k in regimes}
    if regimes:
        dom = max(share, key=share.get)
        out["roofline"] = dict(regimes[dom], regime=dom)
        for k, v in regimes.items():
            if k != dom:
                out["roofline_" + k] = dict(v, regime=k)
    else:
        roof = sum(roof_us(p.M, p.N, p.K, peaks, p.group)[0] for p in probs)
        us = graph_time_us(lambda: [p.run(qoq) for p in probs], stream, reps)
        out["roofline"] = {"bound": "mixed", "achieved": round(roof / us, 4), "peak": 1.0,
                           "unit": "fraction of each GEMM's roofline time", "frac": round(roof / us, 4),
                           "traffic": None, "peak_source": peaks["src"], "kernel": "qoq_w4a8_linear"}
    per, by_m = [], {}
    for p, us in zip(probs, in_step):
        r_us, bound = roof_us(p.M, p.N, p.K, peaks, p.group)
        per.append({"shape": p.name, "K": p.K, "N": p.N, "M": p.M, "token_tile": p.tok, "launches": p.launches,
                    "us_in_step": round(us, 3), "TOPS": round(gemm_ops(p.M, p.N, p.K) / us / 1e6, 2),
                    "GBps": round(linear_bytes(p) / us / 1e3, 1), "roof_us": round(r_us, 3), "bound": bound,
                    "frac_of_roofline": round(r_us / us, 3)})
        d = by_m.setdefault(p.M, {"M": p.M, "us_in_step": 0.0, "roof_us": 0.0, "ops": 0.0})
        d["us_in_step"] += us
        d["roof_us"] += r_us
        d["ops"] += gemm_ops(p.M, p.N, p.K)
    out["per_gemm"] = per
    out["by_M"] = [{"M": d["M"], "us_in_step": round(d["us_in_step"], 2), "TOPS": round(d["ops"] / d["us_in_step"]
                                                                                       / 1e6, 2),
                    "frac_of_roofline": round(d["roof_us"] / d["us_in_step"], 3)} for d in by_m.values()]
    return out


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


def run_kv4(stream, peaks, reps=20):
    """KV4 decode attention (context, not in the timed step): batch 64 x 1024
    cached tokens, Llama-3-8B heads (32 query heads over 8 KV heads, D = 128),
    the pages' attention measurement shape. One graph of `reps` launches,
    alternating between two copies of the 4-bit cache (142 MB together, more
    than L2), events around the replays. Algorithmic bytes per launch: K and V
    codes (D/2 bytes per token and head) with their FP16 scale and zero, the
    FP16 queries and outputs. Beside it, the same attention over FP16 K/V
    through PyTorch's scaled_dot_product_attention (the library's kernel,
    context for the pages' KV4-over-FP16 argument)."""
    import torch
    from w4a8_quantized_gemm_qoq_b200 import qoq
    dev = torch.device("cuda", torch.cuda.current_device())
    a = inputs.LLAMA3_8B_ATTN
    B, T, Hq, Hkv, D = 64, 1024, a["Hq"], a["Hkv"], a["D"]
    q, K, V = inputs.make_decode_attention(B, T, Hq, Hkv, D, seed=21)
    qd = torch.from_numpy(q).to(dev)
    Kd, Vd = torch.from_numpy(K).to(dev), torch.from_numpy(V).to(dev)
    caches = []
    for _ in range(2):
        caches.append((qoq.KV4Cache(B, Hkv, T, D).write(Kd), qoq.KV4Cache(B, Hkv, T, D).write(Vd)))
    ws = qoq.Workspace(qoq.kv4_workspace_bytes(B, Hq, Hkv, T, D))
    out = torch.empty((B, Hq, D), dtype=torch.float16, device=dev)
    torch.cuda.synchronize()
    stream.wait_stream(torch.cuda.current_stream())
    us = graph_time_us(lambda: [qoq.kv4_decode_attention(qd, *caches[i % 2], ws=ws, out=out) for i in range(reps)],
                       stream, 2) / reps
    nbytes = 2 * B * Hkv * T * (D // 2 + 4) + 2 * B * Hq * D * 2
    res = {"B": B, "T": T, "Hq": Hq, "Hkv": Hkv, "D": D, "us": round(us, 3), "GBps": round(nbytes / us / 1e3, 1),
           "frac_of_hbm": round(nbytes / us / 1e3 / peaks["hbm"], 3), "bytes_per_launch": nbytes,
           "kernel": "kv4_attn_kernel (one launch)"}
    try:
        import torch.nn.functional as F
        q4 = qd.view(B, Hq, 1, D)
        kv16 = [(Kd, Vd), (Kd.clone(), Vd.clone())]
        with torch.cuda.stream(stream):   # eager first call: kernel selection and workspace outside capture
            F.scaled_dot_product_attention(q4, Kd, Vd, enable_gqa=True)
        stream.synchronize()
        us16 = graph_time_us(lambda: [F.scaled_dot_product_attention(q4, *kv16[i % 2], enable_gqa=True)
                                      for i in range(reps)], stream, 2) / reps
        res["fp16_kv_sdpa_us"] = round(us16, 3)
        res["kv4_speedup_over_fp16_kv"] = round(us16 / us, 3)
    except Exception as exc:   # context only
        res["fp16_kv_sdpa"] = "unavailable: %s" % str(exc)[:120]
    del caches, Kd, Vd
    torch.cuda.empty_cache()
    return res


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
    each problem's FP16 activations host->device (pinned), makes the one
    linear call (qoq_w4a8_linear), and reads the FP16 output back
    device->host, all eager on one stream."""
    import torch
    hx = [p.X.cpu().pin_memory() for p in probs]
    hy = [torch.empty(p.Y.shape, dtype=torch.float16).pin_memory() for p in probs]
    h2d = sum(x.numel() * 2 for x in hx)
    d2h = sum(y.numel() * 2 for y in hy)

    def once():
        for p, a, c in zip(probs, hx, hy):
            p.X.copy_(a, non_blocking=True)
            p.run(qoq)
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
    """A bounded sample of the workload for the CPU oracle: every shape of the
    workload, its first 1024 weight rows (8 of the n-tiles) and all of K, at
    the workload's M values up to 256 (larger M: a 64-row slab, whose rate
    stands for the rest); weights quantised beforehand (the offline step),
    then per GEMM the oracle's act quant + int64 GEMM (OpenMP over the output
    elements) + FP16 epilogue, timed. Returns (run, ops per run, description)."""
    import oracle
    wl = WORKLOADS[workload]
    rows = 1024
    jobs = []
    for si, (K, N, name) in enumerate(wl["shapes"]):
        W = inputs.make_weights(rows, K, seed=seed + si, std=wl["std"])
        d = oracle.quantize_weights_group(W) if wl["group"] else oracle.quantize_weights_per_channel(W)
        for M in sorted({min(M, 256) if M <= 256 else 64 for M in wl["M"]}):
            X = inputs.make_activations(M, K, seed=seed + si, token_scale_span=token_span(wl, M))
            jobs.append((X, d))

    def once():
        for X, d in jobs:
            X8, s_x, rowsum = oracle.quantize_act_per_token(X)
            if wl["group"]:
                oracle.epilogue_fp16(oracle.gemm_int(X8, d["Wint"]), s_x, d["s_w"])
            else:
                oracle.epilogue_fp16(oracle.w4a8_gemm_per_channel(X8, rowsum, d["q"], d["z"]), s_x, d["s"])
    ops = sum(gemm_ops(X.shape[0], rows, X.shape[1]) for X, _ in jobs)
    Ms = sorted({X.shape[0] for X, _ in jobs})
    desc = ("every shape of the workload, first %d weight rows, full K, M in %s (M > 256 as a 64-row slab): act "
            "quant + int64 GEMM (OpenMP, %d threads) + FP16 epilogue; weights pre-quantised"
            % (rows, Ms, oracle.gemm_threads()))
    return once, ops, desc


def time_oracle(workload, budget_s=10.0, min_runs=1):
    import oracle
    once, ops, desc = oracle_sample(workload)
    once()   # compile/load the C part outside the timing
    n, t0 = 0, time.perf_counter()
    while True:
        once()
        n += 1
        el = time.perf_counter() - t0
        if n >= min_runs and el >= budget_s:
            break
    return {"value": round(ops * n / el / 1e12, 6), "unit": "TOPS", "cores": oracle.gemm_threads(),
            "kind": "oracle", "sample": "%s; %d runs in %.1f s" % (desc, n, el)}


def run_reference(args):
    """--impl reference: the CPU oracle, as it stands, on the host cores."""
    import oracle
    once, ops, desc = oracle_sample(args.workload)
    once()
    for _ in range(max(0, args.warmup)):
        once()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        once()
    el = time.perf_counter() - t0
    val = ops * args.steps / el / 1e12
    return {"impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": "TOPS", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1000 * el / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
            "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload]["desc"], "sample": desc},
            "cpu_baseline": {"value": round(val, 6), "unit": "TOPS", "cores": oracle.gemm_threads(),
                             "kind": "oracle", "sample": "%s; one sample per step" % desc},
            "e2e": {"value": round(val, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="llama3_8b")
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
