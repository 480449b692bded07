"""Host-side checks of the measurement harness and of the binding's failure
behaviour that need no GPU: the reference arm's JSON line keeps the bench
contract, the roofline arithmetic counts the bytes the workload defines, and
the product calls refuse host tensors instead of falling back to the CPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    """`bench.py --impl reference` times the CPU oracle and prints one JSON
    line with the contract's keys; its end-to-end figure moves no bytes
    between host and device."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=300, check=True)
    d = json.loads(out.stdout.strip().splitlines()[-1])
    import bench
    # The contract's metric string, spelled out here independently of the
    # constant bench.py prints, so that a drift in either is caught.
    contract = "W4A8 GEMM TOPS and % of roofline vs M on Llama-3-8B linear shapes (1 B200)"
    assert bench.METRIC == contract
    assert d["impl"] == "reference" and d["metric"] == contract
    for k in ("value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config"):
        assert k in d, k
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["steps"] == 1 and d["warmup"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_roofline_byte_and_op_counts():
    """Bytes per GEMM: 4-bit codes, one (s, z*s) byte pair per 128 weights,
    FP16 s_w, INT8 X8, FP16 s_x, FP16 Y; ops: 2*M*N*K. Counted by hand for
    two decode shapes."""
    import bench
    # M=1, K=4096 -> N=6144: 12582912 + 393216 + 12288 + 4096 + 2 + 12288
    assert bench.gemm_bytes(1, 6144, 4096) == 13004802
    # M=256, K=14336 -> N=4096: 29360128 + 917504 + 8192 + 3670016 + 512 + 2097152
    assert bench.gemm_bytes(256, 4096, 14336) == 36053504
    assert bench.gemm_ops(2048, 28672, 4096) == 2 * 2048 * 28672 * 4096
    peaks = {"hbm": 6550.1, "bf16": 1589.5}
    us, bound = bench.roof_us(1, 28672, 4096, peaks)
    assert bound == "hbm" and abs(us - bench.gemm_bytes(1, 28672, 4096) / 6550.1e3) < 1e-6
    us, bound = bench.roof_us(16384, 4096, 14336, peaks)
    assert bound == "tensor" and abs(us - 2 * 16384 * 4096 * 14336 / (2 * 1589.5e6)) < 1e-3


def test_product_calls_refuse_host_tensors():
    """No CPU fallback: the binding accepts device tensors only."""
    import torch
    from w4a8_quantized_gemm_qoq_b200 import qoq
    X = torch.zeros((4, 128), dtype=torch.float16)
    with pytest.raises(TypeError):
        qoq.quantize_act_per_token(X)
    with pytest.raises(TypeError):
        qoq.gemm_fp16_out(torch.zeros((4, 128), dtype=torch.int8), torch.ones(4, dtype=torch.float16),
                          torch.zeros(16, dtype=torch.uint8), 128, 128)
    with pytest.raises(TypeError):
        qoq.rmsnorm_quant(X, torch.ones(128, dtype=torch.float16), 1e-5)
