"""w4a16_gemm_static_scratch: the GEMM with the library's static device
scratch as workspace, called through the C ABI, against the existing
w4a16_gemm entry point on the same inputs and against the oracle's fp64
product, both within the matmul tolerance.

Collected last (file name), so it runs after every other test has used the
library, and it passes alone too.  Two calls in a row per case: the second
one reuses the counters that the first left behind."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from weight_only_bit_gemm_b200 import synthetic as S


def _lib():
    from weight_only_bit_gemm_b200 import build
    build.build()
    from weight_only_bit_gemm_b200 import w4 as mod
    return mod


def test_static_scratch_rejects_oversized_shape_on_host():
    # split-K partial sums of 2 x 32 tiles of 256 x 128: more than 16 MiB of
    # workspace; rejected on the host before any device work, so fake device
    # pointers do
    w4 = _lib()
    M, N, K, G = 512, 4096, 4096, 128
    assert w4.lib.w4_workspace_bytes(M, N, K, G, 0) > w4.W4_STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)
    st = w4.lib.w4a16_gemm_static_scratch(fake, fake, M, N, K, G, 0, fake, None)
    assert st == w4.W4_ERR_SCRATCH_LIMIT
    assert b"static scratch" in w4.lib.w4_status_string(st)


def _host_u16(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


CASES = [
    # (M, N, K, G, act)
    (1, 4096, 4096, 128, False),    # decode: row groups split over warps
    (16, 1000, 2048, 64, False),    # ragged N, two token blocks
    (4, 1024, 5120, 32, True),      # act-order: X gathered into the scratch
    (128, 512, 4096, 128, False),   # tensor-core path, split K
]


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,G,act", CASES)
def test_static_scratch_matches_w4a16_gemm(M, N, K, G, act):
    w4 = _lib()
    assert w4.lib.w4_workspace_bytes(M, N, K, G, int(act)) <= w4.W4_STATIC_SCRATCH_BYTES
    W = S.draw_w(N, K, 0.02, seed=M, tag=2)
    g_idx = S.act_order_g_idx(S.draw_perm(K, seed=M, tag=2, N=N), G) if act else None
    q, s, z = O.quantize_rtn(W, G, g_idx)
    Wq = O.pack_nibbles(q)
    what = O.dequant_rtn(Wq, s, z, G, g_idx)
    Wp = w4.prepack(_dev(Wq), _dev(s.view(np.int16), torch.float16), _dev(z), G,
                    _dev(g_idx) if act else None)
    xb = S.draw_x(M, K, seed=M, tag=2, N=N, outlier_frac=0.001, outlier_scale=50.0)
    X = _dev(xb.view(np.int16), torch.bfloat16)
    y_entry = w4.w4a16_gemm(X, Wp, N, K, G, act)
    assert w4.device_status() == w4.W4_OK
    y_via_entry = O.bf16_bits_to_f64(_host_u16(y_entry))
    y_oracle, abs_ref = O.matmul_ref(xb, what)
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        w4.w4a16_gemm_static_scratch(X, Wp, N, K, G, act, out=y)
        assert w4.device_status() == w4.W4_OK
        yh = _host_u16(y)
        ok, ratio = O.check_matmul(yh, y_via_entry, abs_ref)
        assert ok, f"against w4a16_gemm: worst difference / tolerance = {ratio}"
        ok, ratio = O.check_matmul(yh, y_oracle, abs_ref)
        assert ok, f"against the oracle: worst error / tolerance = {ratio}"


@pytest.mark.gpu
def test_static_scratch_limit_leaves_output_untouched():
    w4 = _lib()
    M, N, K, G = 512, 4096, 4096, 128
    assert w4.lib.w4_workspace_bytes(M, N, K, G, 0) > w4.W4_STATIC_SCRATCH_BYTES
    X = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    Wp = torch.zeros(w4.lib.w4_prepacked_bytes(N, K, G, 0), dtype=torch.uint8, device="cuda")
    y = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4Error) as e:
        w4.w4a16_gemm_static_scratch(X, Wp, N, K, G, out=y)
    assert e.value.status == w4.W4_ERR_SCRATCH_LIMIT
    assert w4.device_status() == w4.W4_OK
    assert bool((y == 3.0).all())
