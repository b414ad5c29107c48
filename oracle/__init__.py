"""CPU oracle for the 4-bit weight-only linear layer (TEST INFRASTRUCTURE).

This package is the plain, slow, obviously-correct definition that the CUDA
library is checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it; the library itself never
does, and there is no CPU fallback that routes through it.

It shares no code with the CUDA path: no kernels, headers, tables, constant
generators or pre/post-processing.  The only common module is the seeded input
generator (``weight_only_bit_gemm_b200.synthetic``), which draws random numbers
and holds none of the quantization arithmetic.
"""
from .w4_oracle import *  # noqa: F401,F403
