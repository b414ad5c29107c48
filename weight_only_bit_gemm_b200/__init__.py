"""Group-wise 4-bit weight-only linear layer for NVIDIA B200 (sm_100a).

The compute path lives in the CUDA library ``libw4b200.so`` (sources under
``csrc/``) behind the C ABI declared in ``include/w4.h``; ``w4`` is its thin
ctypes binding.  ``synthetic`` draws the seeded test/benchmark inputs.
"""
