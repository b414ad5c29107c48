"""GPU parity for the symmetric INT4 quantizer and the AWQ per-input-channel
factor, through the C ABI, against the CPU oracle on the same seeded inputs.

Bit-exact: symmetric quantize (codes, fp16 scales, zero points, with and
without act-order), the weight product W * s and the activation division
bf16(x / s).  The AWQ GEMM within |y - y_ref| <= 1e-3 * sum_k |x' w_hat| +
ulp_bf16(y_ref), where x' = bf16(x / s) and w_hat dequantizes the codes of
W * s; and bit-identical to the two-call form (scale X, then w4a16_gemm)."""
import numpy as np
import pytest
import torch

import oracle as O
from weight_only_bit_gemm_b200 import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    from weight_only_bit_gemm_b200 import build
    build.build()
    from weight_only_bit_gemm_b200 import w4 as mod
    return mod


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def host_u16(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def x_dev(xbits):
    return dev(xbits.view(np.int16), torch.bfloat16)


def status_ok(w4):
    assert w4.device_status() == w4.W4_OK


# ----------------------------------------------------------------- symmetric quantize

SYM_CASES = [
    (512, 512, 128, False),
    (200, 384, 64, False),        # ragged N
    (64, 5120, 32, False),
    (96, 512, 32, True),          # act-order
    (33, 1024, 128, True),
    (7, 256, 32, False),
]


@pytest.mark.parametrize("N,K,G,act", SYM_CASES)
def test_quantize_sym_bit_exact(w4, N, K, G, act):
    W = S.draw_w(N, K, 0.02, seed=1, tag=20 + G)
    W[0, :G] = 0.0                           # all-zero group: scale 1, codes 8
    W[1, :G] = -0.25                         # constant negative group
    W[2, :8] = np.array([-1.75, 0, 3.5, 0.5, -0.25, 1.75, -3.5, 1.25], np.float32)  # ties
    W[3, :G] = 80.0 * np.sign(W[3, :G])      # every weight at +-max|w|
    g_idx = S.act_order_g_idx(S.draw_perm(K, seed=1, tag=6, N=N), G) if act else None
    q, s, z = O.quantize_sym(W, G, g_idx)
    Wq_ref = O.pack_nibbles(q)
    gi = dev(g_idx) if act else None
    Wq, sc, zr = w4.quantize_sym(dev(W), G, gi)
    status_ok(w4)
    assert np.array_equal(Wq.cpu().numpy(), Wq_ref)
    assert np.array_equal(host_u16(sc), s.view(np.uint16))
    assert np.array_equal(zr.cpu().numpy(), z)
    what = w4.dequant(Wq, sc, zr, G, gi)
    status_ok(w4)
    assert np.array_equal(host_u16(what), O.dequant_rtn(Wq_ref, s, z, G, g_idx))


# ----------------------------------------------------------------- AWQ factor

# (64, 4096), (300, 1028), (5, 8): the float4 row kernel (K % 4 == 0; 257
# float4 per row leave a ragged last trip, 2 per row fewer than one trip);
# (3, 10), (1000, 777): the element kernel
@pytest.mark.parametrize("N,K", [(64, 4096), (300, 1028), (5, 8), (3, 10), (1000, 777)])
def test_awq_scale_weights_bit_exact(w4, N, K):
    W = S.draw_w(N, K, 0.02, seed=2, tag=21)
    s = S.draw_awq_s(K, seed=2, tag=21, lo=0.25, hi=4.0)
    ref = O.awq_scale_weights(W, s)
    out = w4.awq_scale_weights(dev(W), dev(s))
    status_ok(w4)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    Wd = dev(W)                               # in place
    w4.awq_scale_weights(Wd, dev(s), out=Wd)
    assert np.array_equal(Wd.cpu().numpy().view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("M,K,lo,hi", [(1, 4096, 0.95, 1.05), (16, 11008, 0.95, 1.05),
                                       (300, 1024, 0.1, 10.0), (5, 8, 0.5, 2.0)])
def test_awq_scale_activations_bit_exact(w4, M, K, lo, hi):
    xb = S.draw_x(M, K, seed=3, tag=22, outlier_frac=0.01, outlier_scale=50.0)
    s = S.draw_awq_s(K, seed=3, tag=22, lo=lo, hi=hi)
    ref = O.awq_scale_activations(xb, s)
    out = w4.awq_scale_activations(x_dev(xb), dev(s))
    status_ok(w4)
    assert np.array_equal(host_u16(out), ref)
    Xd = x_dev(xb)                            # in place
    w4.awq_scale_activations(Xd, dev(s), out=Xd)
    assert np.array_equal(host_u16(Xd), ref)


def _awq_layer(w4, N, K, G, act, sym, seed, lo=0.95, hi=1.05):
    """Oracle w_hat of the AWQ-scaled weights, the device-prepacked weights
    (quantized on the device, checked bit-exact) and the factor s."""
    W = S.draw_w(N, K, 0.02, seed=seed, tag=23)
    s = S.draw_awq_s(K, seed=seed, tag=23, N=N, lo=lo, hi=hi)
    g_idx = S.act_order_g_idx(S.draw_perm(K, seed=seed, tag=23, N=N), G) if act else None
    Ws = O.awq_scale_weights(W, s)
    q, sc, z = (O.quantize_sym if sym else O.quantize_rtn)(Ws, G, g_idx)
    Wq_ref = O.pack_nibbles(q)
    what = O.dequant_rtn(Wq_ref, sc, z, G, g_idx)
    gi = dev(g_idx) if act else None
    Wsd = w4.awq_scale_weights(dev(W), dev(s))
    Wq, scd, zd = (w4.quantize_sym if sym else w4.quantize_rtn)(Wsd, G, gi)
    status_ok(w4)
    assert np.array_equal(Wq.cpu().numpy(), Wq_ref)
    assert np.array_equal(host_u16(scd), sc.view(np.uint16))
    Wp = w4.prepack(Wq, scd, zd, G, gi)
    return what, Wp, s


AWQ_GEMM_CASES = [
    # (M, N, K, G, act, sym)
    (1, 512, 512, 128, False, True),
    (4, 1000, 4096, 128, False, True),      # ragged N, split row groups
    (16, 384, 1024, 64, False, False),      # AWQ's own format: zero point, G = 128/64
    (32, 256, 2048, 32, True, True),        # act-order: gather and divide in one pass
    (40, 200, 768, 64, False, True),        # tensor-core path, ragged
    (256, 256, 4096, 128, False, False),
    (300, 384, 1024, 32, True, True),
]


@pytest.mark.parametrize("M,N,K,G,act,sym", AWQ_GEMM_CASES)
def test_awq_gemm_tolerance_and_two_call_identity(w4, M, N, K, G, act, sym):
    what, Wp, s = _awq_layer(w4, N, K, G, act, sym, seed=M)
    xb = S.draw_x(M, K, seed=4, tag=23, N=N, outlier_frac=0.001, outlier_scale=50.0)
    sd = dev(s)
    y = w4.w4a16_awq_gemm(x_dev(xb), sd, Wp, N, K, G, act)
    status_ok(w4)
    xs = O.awq_scale_activations(xb, s)
    y_ref, ab = O.matmul_ref(xs, what)
    ok, ratio = O.check_matmul(host_u16(y), y_ref, ab)
    assert ok, f"worst error / tolerance = {ratio}"
    # the fused prologue is the standalone division followed by the same GEMM
    y2 = w4.w4a16_gemm(w4.awq_scale_activations(x_dev(xb), sd), Wp, N, K, G, act)
    status_ok(w4)
    assert torch.equal(y, y2)


def test_awq_gemm_unit_factor_equals_plain_gemm(w4):
    # s = 1: X / s = X bit for bit, so the AWQ call must equal w4a16_gemm
    M, N, K, G = 8, 512, 2048, 128
    W = S.draw_w(N, K, 0.02, seed=5, tag=24)
    Wq, sc, zr = w4.quantize_sym(dev(W), G)
    Wp = w4.prepack(Wq, sc, zr, G)
    xb = S.draw_x(M, K, seed=5, tag=24, N=N)
    one = torch.ones(K, dtype=torch.float32, device="cuda")
    y1 = w4.w4a16_awq_gemm(x_dev(xb), one, Wp, N, K, G)
    y2 = w4.w4a16_gemm(x_dev(xb), Wp, N, K, G)
    status_ok(w4)
    assert torch.equal(y1, y2)


def test_awq_argument_errors(w4):
    N, K, G = 64, 512, 128
    W = S.draw_w(N, K, 0.02, seed=6, tag=25)
    Wq, sc, zr = w4.quantize_sym(dev(W), G)
    Wp = w4.prepack(Wq, sc, zr, G)
    X = torch.zeros((2, K), dtype=torch.bfloat16, device="cuda")
    s = torch.ones(K + 4, dtype=torch.float32, device="cuda")
    with pytest.raises(w4.W4Error) as e:       # s not 16-byte aligned
        w4.w4a16_awq_gemm(X, s[1:K + 1], Wp, N, K, G)
    assert e.value.status == w4.W4_ERR_INVALID_ARG
    with pytest.raises(w4.W4Error) as e:       # K % 8 != 0
        w4.awq_scale_activations(torch.zeros((2, 12), dtype=torch.bfloat16, device="cuda"),
                                 torch.ones(12, dtype=torch.float32, device="cuda"))
    assert e.value.status == w4.W4_ERR_INVALID_ARG
    status_ok(w4)
