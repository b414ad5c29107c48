"""Host-side checks of the C ABI library (no GPU needed): it loads, exports
every function include/w4.h declares, and rejects bad arguments on the host
before launching anything."""
import ctypes

import pytest

from weight_only_bit_gemm_b200 import build

build.build()
from weight_only_bit_gemm_b200 import w4  # noqa: E402

import oracle as O  # noqa: E402


def test_exports_every_declared_function():
    names = w4.header_functions()
    assert "w4a16_gemm" in names and "nf4_gemm" in names and len(names) >= 18
    missing = [n for n in names if not hasattr(w4.lib, n)]
    assert missing == []


def test_status_strings_and_version():
    assert w4.lib.w4_status_string(0) == b"ok"
    for s in range(1, 6):
        assert len(w4.lib.w4_status_string(s)) > 3
    assert w4.lib.w4_status_string(99) == b"unknown status"
    assert w4.lib.w4_version() == 100


def test_size_functions():
    # canonical storage: codes + fp16 scale + 4-bit zero per group
    assert w4.lib.w4_weight_bytes(12288, 4096, 128) == O.weight_bytes(12288, 4096, 128)
    assert w4.lib.w4_weight_bytes(5120, 13824, 32) == O.weight_bytes(5120, 13824, 32)
    assert w4.lib.w4_weight_bytes(1, 100, 128) == 0.0          # K < G
    # prepacked: 128-row tiles x 128-channel stages (+ permutation)
    stage = 8192 + 128 * 1 * 2 + 128 // 2
    assert w4.prepacked_bytes(4096, 4096, 128) == 32 * 32 * stage
    stage32 = 8192 + 128 * 4 * 2 + 128 * 4 // 2
    assert w4.prepacked_bytes(200, 192, 32, True) == 2 * 2 * stage32 + 192 * 4
    assert w4.prepacked_bytes(0, 4096, 128) == 0
    assert w4.prepacked_bytes(16, 4096, 96) == 0                # unsupported group
    assert w4.lib.nf4_prepacked_bytes(4096, 14336) == 32 * 112 * (8192 + 256)
    assert w4.lib.nf4_prepacked_bytes(16, 100) == 0             # K % 64 != 0
    assert w4.workspace_bytes(1, 4096, 4096, 128) > 0
    assert w4.workspace_bytes(0, 4096, 4096, 128) == 0


def test_nf4_levels_equal_oracle_table():
    got = w4.nf4_levels()
    want = O.nf4_table().tolist()
    assert got == want


@pytest.mark.parametrize("call", [
    lambda: w4.lib.w4_quantize_rtn(None, 4, 128, 128, None, None, None, None, None),
    lambda: w4.lib.w4_dequant(None, None, None, None, 4, 128, 128, None, None),
    lambda: w4.lib.w4_prepack(None, None, None, None, 4, 128, 128, None, None),
    lambda: w4.lib.w4a16_gemm(None, None, 1, 4, 128, 128, 0, None, None, 0, None),
    lambda: w4.lib.nf4_quantize(None, 4, 128, 64, 256, None, None, None, None),
    lambda: w4.lib.nf4_gemm(None, None, None, 1, 4, 128, 256, None, None, 0, None),
])
def test_null_pointers_rejected_on_host(call):
    assert call() == w4.W4_ERR_INVALID_ARG


def test_bad_shapes_rejected_on_host():
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: shape checks come first
    assert w4.lib.w4_quantize_rtn(fake, 4, 100, 128, None, fake, fake, fake, None) == \
        w4.W4_ERR_INVALID_ARG
    assert w4.lib.w4_quantize_rtn(fake, 4, 256, 48, None, fake, fake, fake, None) == \
        w4.W4_ERR_INVALID_ARG
    assert w4.lib.nf4_quantize(fake, 4, 96, 64, 256, fake, fake, fake, None) == \
        w4.W4_ERR_INVALID_ARG
    assert w4.lib.nf4_quantize(fake, 4, 128, 32, 256, fake, fake, fake, None) == \
        w4.W4_ERR_INVALID_ARG
    # misaligned X for the tensor-memory path
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert w4.lib.w4a16_gemm(odd, fake, 1, 4, 128, 128, 0, fake, fake, 1 << 20, None) == \
        w4.W4_ERR_INVALID_ARG
