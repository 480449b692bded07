"""Both GEMM kernels' stream-K fix-up when the owner of a split tile is not
the last to arrive, run in a process of its own with every
contributor's arrival delayed (QOQ_FORCE_CONFIG=lateck=<us>, read once per
process): owners then store their partial tiles and set the owner bit, and
the last contributor writes the tile from their sums. Decode-size problems
(the decode kernel), prefill-size and ragged ones (the general kernel;
every tile split at these sizes), group and per-channel variants; INT32 and
FP16 outputs against the CPU oracle on sampled tiles, status words zero,
control words left clear.

    QOQ_FORCE_CONFIG=lateck=300 python tests/gemm_late_check.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

from gpu_helpers import check_sampled  # noqa: E402
from w4a8_quantized_gemm_qoq_b200 import build  # noqa: E402


def main():
    build.build()
    cases = [(1, 4096, 4096, 128), (16, 28672, 4096, 128), (64, 4096, 14336, 128), (33, 4096, 4096, 0),
             (2048, 4096, 4096, 128), (300, 4096, 4096, 128), (1000, 6144, 4096, 128), (600, 512, 640, 128),
             (700, 4096, 4096, 0), (2048, 1024, 14336, 128)]
    for M, N, K, group in cases:
        check_sampled(M, N, K, group, seed=M + N, token_scale_span=(-3, 1) if M >= 2048 else None)
    print("gemm_late_check ok")


if __name__ == "__main__":
    main()
