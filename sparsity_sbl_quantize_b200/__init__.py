"""B200-native Sparse-BitLinear: mask + ternarise + pack, per-token int8
activation quantisation, masked ternary x int8 GEMM with dequantisation, and
the Dual-STE backward, as hand-written sm_100a CUDA kernels behind a small
C ABI (``include/sbl.h``).

``sparsity_sbl_quantize_b200.sbl`` is the Python binding of that ABI; it loads
``libsbl.so`` from this directory and raises if it is missing.  There is no
CPU fallback.
"""

__all__ = ["sbl", "workloads"]
