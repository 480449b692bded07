"""CPU reference ("oracle") for the QoQ W4A8 GEMM -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import, call, link or execute anything in this package. The
product path (the CUDA library and its Python binding) never does, and nothing
here imports the product package: the two share no code.

Contents
  qoq_ref.py   quantisers, packer, integer GEMM driver and FP32 epilogue in
               plain numpy, each step written from the QServe pages.
  qoq_gemm.c   the integer GEMM as a plain int64 triple loop (gcc, no tiling).
  producers.py the fused activation producers (RMSNorm or SiLU-gated product,
               then per-token INT8 quantisation) in plain numpy and Python
               integers.
  kv4.py       KV4 decode attention (per-head dynamic asymmetric INT4 K/V,
               grouped-query softmax attention) in plain numpy; no kernel
               implements it yet.

Pinning: every function here is checked in ``tests/test_oracle_*.py`` against
something other than itself -- exact rational arithmetic (``fractions``),
closed forms, an exhaustive enumeration of the second quantisation level,
brute force with Python integers and hand-worked fixtures in
``tests/golden/``. The pages print no worked numeric example, so no pin comes
from a printed value.
"""
from .qoq_ref import *  # noqa: F401,F403
from . import producers  # noqa: F401
from . import kv4  # noqa: F401
