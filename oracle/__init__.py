"""CPU oracle for the SVDQuant W4A4 linear and the AWQ W4A16 linear.

ORACLE -- TEST INFRASTRUCTURE ONLY. Plain, slow, float64 code that states what
the hot path computes. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import it. It shares no code with the
CUDA library (``bit_quantized_diffusion_b200``) and imports nothing from it;
the two meet only in the seeded input module ``workloads``.

Modules:
    formats  E2M1 / UE4M3 / FP16 / BF16 rounding from the format definitions
    svdq     smoothing, group quantization, packing, down/up projection, GEMM
    layout   the tiled storage formats the kernels read, as index formulas
    prep     offline smoothing factors, SVD split and residual (weights)
    awq      AWQ W4A16 weight quantization and linear
"""

from . import awq, formats, layout, prep, svdq  # noqa: F401
