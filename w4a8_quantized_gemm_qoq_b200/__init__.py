"""QoQ W4A8 GEMM for NVIDIA B200 (sm_100a).

The compute path lives in the CUDA library ``libqoq.so`` (sources in
``csrc/``, C-ABI declared in ``include/qoq.h``); ``qoq`` is its thin ctypes
binding. Importing this package loads nothing: the library is opened on first
use of ``w4a8_quantized_gemm_qoq_b200.qoq``.
"""
__all__ = ["inputs", "qoq"]
