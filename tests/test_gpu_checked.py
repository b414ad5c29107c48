"""The bounds-checked build (libw4b200_checked.so, compiled with W4_CHECKED)
on ragged cases of every entry point: no kernel index may fall outside its
buffer (the device status stays W4_OK, never W4_ERR_BOUNDS), and the results
are bit-identical to the normal build's (every kernel here is deterministic;
the checks only skip accesses that would be out of bounds)."""
import numpy as np
import pytest
import torch

from weight_only_bit_gemm_b200 import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    from weight_only_bit_gemm_b200 import build
    build.build()
    build.build(checked=True)
    from weight_only_bit_gemm_b200 import w4
    chk = w4.checked_library()
    assert chk.w4_checked_build() == 1
    return w4, chk


def _x(M, K, N, seed):
    xb = S.draw_x(M, K, seed=seed, tag=60, N=N, outlier_frac=0.002, outlier_scale=50.0)
    return torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()


def _both(w4, chk, fn):
    """fn() through the normal and the checked build; both must report OK."""
    a = fn()
    assert w4.device_status() == w4.W4_OK
    with w4.using(chk):
        b = fn()
        st = w4.device_status()
    assert st == w4.W4_OK, f"checked build reported status {st}"
    return a, b


def _same(a, b):
    if isinstance(a, (tuple, list)):
        for x, y in zip(a, b):
            _same(x, y)
    elif a is not None:
        assert torch.equal(a.view(torch.uint8) if a.dtype != torch.uint8 else a,
                           b.view(torch.uint8) if b.dtype != torch.uint8 else b)


INT4_CASES = [
    # (M, N, K, G, act)
    (1, 77, 320, 32, False),
    (5, 300, 4160, 64, False),
    (16, 1000, 2048, 64, False),
    (32, 200, 1536, 128, False),
    (4, 300, 1280, 64, True),
    (16, 130, 2560, 128, True),
    (33, 128, 192, 64, False),
    (100, 640, 2048, 128, False),
    (300, 384, 1024, 128, False),
    (256, 256, 2048, 32, True),
    # CTA pairs: ragged token halves, K-split partials, head and tail tiles
    (129, 512, 2048, 128, False),
    (520, 2304, 4096, 64, False),
    (300, 9728, 4096, 128, False),
]


@pytest.mark.parametrize("M,N,K,G,act", INT4_CASES)
def test_checked_int4_path(libs, M, N, K, G, act):
    w4, chk = libs
    W = torch.from_numpy(S.draw_w(N, K, 0.02, seed=M, tag=61)).cuda()
    gi = (torch.from_numpy(S.act_order_g_idx(S.draw_perm(K, seed=M, tag=61, N=N), G)).cuda()
          if act else None)
    q = _both(w4, chk, lambda: w4.quantize_rtn(W, G, gi))
    _same(*q)
    Wq, sc, zr = q[0]
    _same(*_both(w4, chk, lambda: w4.quantize_sym(W, G, gi)))
    _same(*_both(w4, chk, lambda: w4.dequant(Wq, sc, zr, G, gi)))
    wp = _both(w4, chk, lambda: w4.prepack(Wq, sc, zr, G, gi))
    _same(*wp)
    _same(*_both(w4, chk, lambda: w4.unprepack(wp[0], N, K, G, act)))
    X = _x(M, K, N, seed=M)
    _same(*_both(w4, chk, lambda: w4.w4a16_gemm(X, wp[0], N, K, G, act)))
    s = torch.from_numpy(S.draw_awq_s(K, seed=M, tag=61, N=N)).cuda()
    _same(*_both(w4, chk, lambda: w4.w4a16_awq_gemm(X, s, wp[0], N, K, G, act)))


@pytest.mark.parametrize("M,N,K", [(1, 40, 64), (8, 300, 1024), (32, 200, 1536), (48, 256, 512),
                                   (300, 256, 512), (260, 1024, 4096)])
def test_checked_blockwise_path(libs, M, N, K):
    w4, chk = libs
    W = torch.from_numpy(S.draw_w(N, K, 0.02, seed=M, tag=62)).cuda()
    X = _x(M, K, N, seed=M)
    for quant, deq, gemm in ((w4.nf4_quantize, w4.nf4_dequant, w4.nf4_gemm),
                             (w4.fp4_quantize, w4.fp4_dequant, w4.fp4_gemm)):
        q = _both(w4, chk, lambda: quant(W))
        _same(*q)
        Wq, c, s2 = q[0]
        _same(*_both(w4, chk, lambda: deq(Wq, c, s2)))
        wp = _both(w4, chk, lambda: w4.nf4_prepack(Wq, c))
        _same(*wp)
        _same(*_both(w4, chk, lambda: gemm(X, wp[0], s2, N, K)))
    q = _both(w4, chk, lambda: w4.nf4_quantize_meandq(W))
    _same(*q)
    Wq, c, m, s2 = q[0]
    _same(*_both(w4, chk, lambda: w4.nf4_dequant_meandq(Wq, c, m, s2)))
    wp = w4.nf4_prepack(Wq, c.view(torch.uint8))
    _same(*_both(w4, chk, lambda: w4.nf4_gemm_meandq(X, wp, m, s2, N, K)))


@pytest.mark.parametrize("M,N,K", [(1, 100, 256), (16, 300, 1024), (40, 64, 512),
                                   (130, 300, 1088)])
def test_checked_llm_int8(libs, M, N, K):
    w4, chk = libs
    W = torch.from_numpy(S.draw_w(N, K, 0.02, seed=M, tag=63)).cuda()
    q = _both(w4, chk, lambda: w4.llm_int8_quantize_weights(W))
    _same(*q)
    X = _x(M, K, N, seed=M)
    _same(*_both(w4, chk, lambda: w4.llm_int8_gemm(X, q[0][0], q[0][1])))


def test_checked_gptq(libs):
    w4, chk = libs
    N, K, G = 130, 512, 32
    xc = torch.from_numpy(S.draw_calib_x(384, K, seed=1, tag=64).view(np.int16)).view(
        torch.bfloat16).cuda()
    H = _both(w4, chk, lambda: w4.gptq_hessian(xc))
    _same(*H)
    W = torch.from_numpy(S.draw_w(N, K, 0.02, seed=1, tag=64)).cuda()
    _same(*_both(w4, chk, lambda: w4.gptq_quantize(W, H[0], G, True)))
