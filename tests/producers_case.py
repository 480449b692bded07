"""One launch of each fused producer on Llama-3-8B rows, for profiling:
RMSNorm + per-token INT8 on 16384 x 4096 hidden rows and SiLU(gate) * up +
per-token INT8 on 4096 x 14336 FFN rows (inputs of 134 MB and 235 MB, larger
than L2). Run as `python tests/producers_case.py`; prints "ok"."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import torch  # noqa: E402

from w4a8_quantized_gemm_qoq_b200 import inputs, qoq  # noqa: E402


def main():
    dev = torch.device("cuda", 0)
    x = torch.from_numpy(inputs.make_activations(16384, 4096, seed=1)).to(dev)
    g = torch.from_numpy(inputs.make_norm_weight(4096, seed=1)).to(dev)
    gu = torch.from_numpy(inputs.make_gate_up(4096, 14336, seed=2)).to(dev)
    torch.cuda.synchronize()
    qoq.rmsnorm_quant(x, g, 1e-5)
    qoq.silu_mul_quant(gu)
    torch.cuda.synchronize()
    print("ok")


if __name__ == "__main__":
    main()
