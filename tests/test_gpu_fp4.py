"""GPU parity for FP4 (E2M1 codes over 6) in the block-wise NF4 scheme,
through the C ABI, against the CPU oracle on the same seeded inputs.

Bit-exact: the level table, quantize (codes, absmax codes, s2) and dequant.
The GEMM (decode and tensor-core kernels, the NF4 kernels with the FP4 table)
exactly on unit-vector X and within |y - y_ref| <= 1e-3 * sum_k |x w_hat| +
ulp_bf16(y_ref) otherwise."""
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


def test_fp4_levels_match_oracle(w4):
    lv = np.array(w4.fp4_levels(), np.float32)
    assert np.array_equal(lv.view(np.uint32), O.fp4_table().view(np.uint32))


@pytest.mark.parametrize("N,K,dq", [(256, 512, 256), (100, 4096, 256), (33, 640, 7)])
def test_fp4_quantize_dequant_bit_exact(w4, N, K, dq):
    W = S.draw_w(N, K, 0.02, seed=0, tag=7)
    W[0, :64] = 0.0                                         # zero block
    W[3, 64:128] = 0.01                                     # constant block
    W[4, :8] = [6, -3, 0.25, 0.3, -0.74, 2.2, -4.9, 1.1]    # midpoint tie, signs
    W[4, 8:64] = 0.0
    W[5, :64] = -np.abs(W[5, :64])                          # one-signed block
    Wq_r, c_r, s2_r = O.fp4_quantize(W, 64, dq)
    Wq, c, s2 = w4.fp4_quantize(dev(W), 64, dq)
    status_ok(w4)
    assert np.array_equal(Wq.cpu().numpy(), Wq_r)
    assert np.array_equal(c.cpu().numpy(), c_r)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), s2_r.view(np.uint32))
    what = w4.fp4_dequant(Wq, c, s2, dq)
    status_ok(w4)
    assert np.array_equal(host_u16(what), O.fp4_dequant(Wq_r, c_r, s2_r, 64, dq))


@pytest.mark.parametrize("M", [32, 256])
def test_fp4_gemm_unit_vectors_exact(w4, M):
    N, K = 256, 1024
    W = S.draw_w(N, K, 0.02, seed=4, tag=7)
    Wq_r, c_r, s2_r = O.fp4_quantize(W)
    what = O.fp4_dequant(Wq_r, c_r, s2_r)
    Wp = w4.nf4_prepack(dev(Wq_r), dev(c_r))
    ks = (np.arange(M) * 37 + 3) % K
    x = np.zeros((M, K), np.float32)
    x[np.arange(M), ks] = 1.0
    xb = S.to_bf16_bits(x)
    y = w4.fp4_gemm(x_dev(xb), Wp, dev(s2_r), N, K)
    status_ok(w4)
    assert np.array_equal(host_u16(y), what[:, ks].T)


@pytest.mark.parametrize("M,N,K", [(1, 512, 4096), (8, 384, 1024), (32, 200, 1536),
                                   (300, 256, 512), (1, 40, 64), (3, 4096, 14336)])
def test_fp4_gemm_tolerance(w4, M, N, K):
    W = S.draw_w(N, K, 0.02, seed=M, tag=7)
    Wq_r, c_r, s2_r = O.fp4_quantize(W)
    what = O.fp4_dequant(Wq_r, c_r, s2_r)
    Wp = w4.nf4_prepack(dev(Wq_r), dev(c_r))
    xb = S.draw_x(M, K, seed=M, tag=7, N=N)
    y = w4.fp4_gemm(x_dev(xb), Wp, dev(s2_r), N, K)
    status_ok(w4)
    y_ref, ab = O.matmul_ref(xb, what)
    ok, ratio = O.check_matmul(host_u16(y), y_ref, ab)
    assert ok, f"worst error / tolerance = {ratio}"


def test_fp4_and_nf4_calls_interleave(w4):
    # the level table is chosen per call: NF4 and FP4 GEMMs back to back on
    # one stream each see their own table
    N, K, M = 384, 2048, 4
    W = S.draw_w(N, K, 0.02, seed=8, tag=7)
    qf, cf, sf = O.fp4_quantize(W)
    qn, cn, sn = O.nf4_quantize(W)
    Wpf = w4.nf4_prepack(dev(qf), dev(cf))
    Wpn = w4.nf4_prepack(dev(qn), dev(cn))
    xb = S.draw_x(M, K, seed=8, tag=7, N=N)
    X = x_dev(xb)
    yf = w4.fp4_gemm(X, Wpf, dev(sf), N, K)
    yn = w4.nf4_gemm(X, Wpn, dev(sn), N, K)
    status_ok(w4)
    for y, what in ((yf, O.fp4_dequant(qf, cf, sf)), (yn, O.nf4_dequant(qn, cn, sn))):
        y_ref, ab = O.matmul_ref(xb, what)
        ok, ratio = O.check_matmul(host_u16(y), y_ref, ab)
        assert ok, f"worst error / tolerance = {ratio}"
