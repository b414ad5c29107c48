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


def test_fp4_levels_equal_oracle_table():
    got = w4.fp4_levels()
    want = O.fp4_table()
    import numpy as np
    assert np.array_equal(np.array(got, np.float32).view(np.uint32), want.view(np.uint32))


def test_prefill_tail_split_workspace():
    # 148 SMs (the planner's count without a device).  (40, 19000, 2560):
    # 149 tiles of 64 tokens x 128 rows, 20 stages; one full wave of whole
    # tiles (cost 21.5) and the remaining tile in 5 K ranges (4 + 13.5) beats
    # two waves of whole tiles (43): partials for 5 ranges of one 64 x 128
    # tile after the 65536 arrival counters.
    assert w4.workspace_bytes(40, 19000, 2560, 128) == 65536 * 4 + 5 * 64 * 128 * 4
    # (512, 28672, 8192): 448 tiles of 256 tokens, 64 stages; three full
    # waves (196.5) and 4 tail tiles in 4 K ranges each (16 + 1.5 + 12; more
    # ranges cost more reduction round trips than they save) against 262 for
    # four waves of whole tiles
    assert w4.workspace_bytes(512, 28672, 8192, 128) == 65536 * 4 + 4 * 4 * 256 * 128 * 4
    # (2048, 8192, 28672): 512 tiles, 224 stages; 3 waves whole and 68 tiles in
    # 2 ranges (802) against every tile in 2 ranges (878)
    assert w4.workspace_bytes(2048, 8192, 28672, 128) == 65536 * 4 + 68 * 2 * 256 * 128 * 4
    # one partial wave (128 tiles): whole tiles, no partials
    assert w4.workspace_bytes(512, 8192, 28672, 128) == 65536 * 4


def test_workspace_sizes_of_the_variants():
    r256 = lambda v: (v + 255) // 256 * 256
    # the AWQ call adds the rewritten activations, M x K bf16, to the plain plan
    for (M, N, K) in [(1, 4096, 4096), (16, 12288, 4096), (512, 8192, 28672)]:
        plain = w4.workspace_bytes(M, N, K, 128)
        assert w4.awq_workspace_bytes(M, N, K, 128) == plain + r256(2 * M * K)
        assert w4.awq_workspace_bytes(M, N, K, 128, True) == w4.workspace_bytes(M, N, K, 128, True)
    # GPTQ: two fp64 and one fp32 K x K matrices, the fp32 working weights, the
    # block errors, the codes and per-channel vectors
    N, K = 13824, 5120
    got = w4.lib.w4_gptq_workspace_bytes(N, K, 32)
    floor = 20 * K * K + 4 * N * K + 4 * 128 * N + N * K + 17 * K
    assert floor <= got <= floor + 12 * 256
    assert w4.lib.w4_gptq_workspace_bytes(N, 5120 + 16, 16) == 0   # unsupported group
    assert w4.lib.w4_gptq_workspace_bytes(N, 131072, 128) == 0     # K above 65536
    # LLM.int8: row-tile counters, int32 accumulator, flags, per-scan-CTA
    # lists / counts / per-token maxima, the outlier list, q_x, s_x
    M, N, K = 16, 22016, 4096
    got = w4.lib.llm_int8_workspace_bytes(M, N, K)
    nscan = K // 32                                   # scan CTAs of 32 channels
    extra = N // 4 + 9 * K + 4 * nscan * (M + 1) + 4 * M + 12 * 256
    assert M * K + 4 * M * N <= got <= M * K + 4 * M * N + extra
    assert w4.lib.llm_int8_workspace_bytes(M, N, 4000) == 0         # K % 64 != 0


@pytest.mark.parametrize("call", [
    lambda: w4.lib.w4_quantize_sym(None, 4, 128, 128, None, None, None, None, None),
    lambda: w4.lib.w4_awq_scale_weights(None, None, 4, 128, None, None),
    lambda: w4.lib.w4_awq_scale_activations(None, None, 1, 128, None, None),
    lambda: w4.lib.w4a16_awq_gemm(None, None, None, 1, 4, 128, 128, 0, None, None, 0, None),
    lambda: w4.lib.fp4_quantize(None, 4, 128, 64, 256, None, None, None, None),
    lambda: w4.lib.fp4_dequant(None, None, None, 4, 128, 64, 256, None, None),
    lambda: w4.lib.fp4_gemm(None, None, None, 1, 4, 128, 256, None, None, 0, None),
    lambda: w4.lib.w4_gptq_hessian(None, 16, 128, None, None),
    lambda: w4.lib.w4_gptq_quantize(None, None, 4, 128, 32, 0, 0.01, None, None, None, None,
                                    None, 0, None),
    lambda: w4.lib.llm_int8_quantize_weights(None, 4, 128, None, None, None),
    lambda: w4.lib.llm_int8_gemm(None, None, None, 1, 4, 128, 6.0, None, None, 0, None),
])
def test_null_pointers_rejected_on_host_variants(call):
    assert call() == w4.W4_ERR_INVALID_ARG


def test_variant_bad_arguments_rejected_on_host():
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: argument checks come first
    # act-order GPTQ needs somewhere to put g_idx
    assert w4.lib.w4_gptq_quantize(fake, fake, 4, 128, 32, 1, 0.01, fake, fake, fake, None,
                                   fake, 1 << 30, None) == w4.W4_ERR_INVALID_ARG
    # negative damping, too small a workspace
    assert w4.lib.w4_gptq_quantize(fake, fake, 4, 128, 32, 0, -1.0, fake, fake, fake, None,
                                   fake, 1 << 30, None) == w4.W4_ERR_INVALID_ARG
    assert w4.lib.w4_gptq_quantize(fake, fake, 4, 128, 32, 0, 0.01, fake, fake, fake, None,
                                   fake, 256, None) == w4.W4_ERR_INVALID_ARG
    # LLM.int8: K % 64, negative threshold, weights not 16-byte aligned
    assert w4.lib.llm_int8_gemm(fake, fake, fake, 1, 4, 96, 6.0, fake, fake, 1 << 30, None) == \
        w4.W4_ERR_INVALID_ARG
    assert w4.lib.llm_int8_gemm(fake, fake, fake, 1, 4, 128, -1.0, fake, fake, 1 << 30, None) == \
        w4.W4_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert w4.lib.llm_int8_gemm(fake, odd, fake, 1, 4, 128, 6.0, fake, fake, 1 << 30, None) == \
        w4.W4_ERR_INVALID_ARG
    # AWQ: the factor must be 16-byte aligned; activations need K % 8 == 0
    assert w4.lib.w4a16_awq_gemm(fake, odd, fake, 1, 4, 128, 128, 0, fake, fake, 1 << 30,
                                 None) == w4.W4_ERR_INVALID_ARG
    assert w4.lib.w4_awq_scale_activations(fake, fake, 1, 12, fake, None) == \
        w4.W4_ERR_INVALID_ARG


def test_decode_row_limit_rejected_on_host():
    # the decode kernel keeps one arrival counter per 32-row group in a fixed
    # region of 65536 counters: N = 2097152 is the largest decode N; one row
    # more is reported unsupported (workspace size 0, the call refused before
    # any launch, so fake device pointers do) instead of aliasing the counters
    limit = 65536 * 32
    for M in (1, 16, 32):
        assert w4.lib.w4_workspace_bytes(M, limit, 256, 128, 0) > 0
        assert w4.lib.w4_workspace_bytes(M, limit + 1, 256, 128, 0) == 0
        assert w4.lib.w4_awq_workspace_bytes(M, limit + 1, 256, 128, 0) == 0
        assert w4.lib.nf4_workspace_bytes(M, limit + 1, 256) == 0
    # above the decode range the tensor-core kernel has no such limit
    assert w4.lib.w4_workspace_bytes(33, limit + 1, 256, 128, 0) > 0
    fake = ctypes.c_void_p(1 << 20)
    ws = ctypes.c_void_p(1 << 24)
    st = w4.lib.w4a16_gemm(fake, fake, 1, limit + 32, 256, 128, 0, fake, ws, 1 << 30, None)
    assert st == w4.W4_ERR_UNSUPPORTED
    st = w4.lib.nf4_gemm(fake, fake, fake, 4, limit + 32, 256, 256, fake, ws, 1 << 30, None)
    assert st == w4.W4_ERR_UNSUPPORTED
    st = w4.lib.w4a16_gemm_static_scratch(fake, fake, 1, limit + 32, 256, 128, 0, fake, None)
    assert st == w4.W4_ERR_UNSUPPORTED


def test_meandq_entry_points_reject_missing_means():
    fake = ctypes.c_void_p(1 << 20)
    assert w4.lib.nf4_quantize_meandq(fake, 4, 128, 64, 256, fake, fake, None, fake,
                                      None) == w4.W4_ERR_INVALID_ARG
    assert w4.lib.nf4_dequant_meandq(fake, fake, None, fake, 4, 128, 64, 256, fake,
                                     None) == w4.W4_ERR_INVALID_ARG
    assert w4.lib.nf4_gemm_meandq(fake, fake, None, fake, 1, 4, 128, 256, fake, fake, 1 << 20,
                                  None) == w4.W4_ERR_INVALID_ARG
    # misaligned means
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert w4.lib.nf4_quantize_meandq(fake, 4, 128, 64, 256, fake, fake, odd, fake,
                                      None) == w4.W4_ERR_INVALID_ARG


def test_checked_build_exports_the_same_functions():
    # the bounds-checked twin of the library: same C ABI, reports itself
    build.build(checked=True)
    chk = w4.checked_library()
    assert chk.w4_checked_build() == 1
    assert w4.lib.w4_checked_build() == 0
    missing = [n for n in w4.header_functions() if not hasattr(chk, n)]
    assert missing == []
    assert b"bounds" in w4.lib.w4_status_string(w4.W4_ERR_BOUNDS)
