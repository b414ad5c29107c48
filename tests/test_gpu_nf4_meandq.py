"""GPU parity for NF4 with mean-offset double quantization of the block
constants (the oracle's R20 reading): quantize and dequant bit-exact, the
GEMM exact on unit-vector activations (decode and tensor-core kernels) and
within |y - y_ref| <= 1e-3 * sum_k |x w_hat| + ulp_bf16(y_ref) otherwise."""
import math

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


def _u16(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _x(xb):
    return torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()


def _layer(w4, N, K, dq, seed, tag=12):
    W = S.draw_w(N, K, 0.02, seed=seed, tag=tag)
    W[0, :64] = 0.0                               # a zero block
    Wq_r, c_r, m_r, s2_r = O.nf4_quantize_meandq(W, 64, dq)
    Wq, c, m, s2 = w4.nf4_quantize_meandq(torch.from_numpy(W).cuda(), 64, dq)
    assert w4.device_status() == w4.W4_OK
    assert np.array_equal(Wq.cpu().numpy(), Wq_r)
    assert np.array_equal(c.cpu().numpy(), c_r)
    assert np.array_equal(m.cpu().numpy().view(np.uint32), m_r.view(np.uint32))
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), s2_r.view(np.uint32))
    what = O.nf4_dequant_meandq(Wq_r, c_r, m_r, s2_r, 64, dq)
    return what, (Wq, c, m, s2)


@pytest.mark.parametrize("N,K,dq", [(256, 512, 256), (100, 4096, 256), (37, 1024, 256),
                                    (64, 1024, 64), (33, 192, 7)])
def test_meandq_quantize_dequant_bit_exact(w4, N, K, dq):
    what, (Wq, c, m, s2) = _layer(w4, N, K, dq, seed=N)
    got = w4.nf4_dequant_meandq(Wq, c, m, s2, dq)
    assert w4.device_status() == w4.W4_OK
    assert np.array_equal(_u16(got), what)


@pytest.mark.parametrize("M", [32, 48, 300])
def test_meandq_gemm_unit_vectors_exact(w4, M):
    # decode kernel (M = 32), tensor-core kernel (M = 48) and its CTA pairs
    # (M = 300: two 256-token tiles over the two 128-row tiles): each output
    # is one w_hat, so the in-kernel reconstruction of the constants is exact
    N, K = 256, 1024
    what, (Wq, c, m, s2) = _layer(w4, N, K, 256, seed=5)
    Wp = w4.nf4_prepack(Wq, c.view(torch.uint8))
    ks = (np.arange(M) * 37 + 3) % K
    x = np.zeros((M, K), np.float32)
    x[np.arange(M), ks] = 1.0
    y = w4.nf4_gemm_meandq(_x(S.to_bf16_bits(x)), Wp, m, s2, N, K)
    assert w4.device_status() == w4.W4_OK
    assert np.array_equal(_u16(y), what[:, ks].T)


@pytest.mark.parametrize("M,N,K", [(1, 512, 4096), (8, 384, 1024), (32, 200, 1536),
                                   (300, 256, 512), (3, 4096, 14336 // 4)])
def test_meandq_gemm_tolerance(w4, M, N, K):
    what, (Wq, c, m, s2) = _layer(w4, N, K, 256, seed=M + 1)
    Wp = w4.nf4_prepack(Wq, c.view(torch.uint8))
    xb = S.draw_x(M, K, seed=M, tag=12, N=N)
    y = w4.nf4_gemm_meandq(_x(xb), Wp, m, s2, N, K)
    assert w4.device_status() == w4.W4_OK
    y_ref, ab = O.matmul_ref(xb, what)
    ok, ratio = O.check_matmul(_u16(y), y_ref, ab)
    assert ok, f"worst error / tolerance = {ratio}"


@pytest.mark.parametrize("K,N", S.NF4_DECODE["shapes"])
def test_fullsize_meandq_decode(w4, K, N):
    # the NF4 decode workload at full size: device quantization of whole
    # double-quantization windows around sampled rows bit-exact, sampled
    # outputs within tolerance at every M
    wl = S.NF4_DECODE
    dq = wl["dq_group"]
    W = S.layer_w(wl, K, N)
    Wq, c, m, s2 = w4.nf4_quantize_meandq(torch.from_numpy(W).cuda(), 64, dq)
    Wp = w4.nf4_prepack(Wq, c.view(torch.uint8))
    kb64 = K // 64
    step = dq // math.gcd(kb64, dq)
    rng = np.random.default_rng([K, N, 12])
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 20, replace=False)]))
    Wq_h, c_h, m_h, s2_h = Wq.cpu().numpy(), c.cpu().numpy(), m.cpu().numpy(), s2.cpu().numpy()
    what_rows = []
    for r in rows:
        r0 = (r // step) * step
        r1 = min(N, r0 + step)
        wq_w, c_w, m_w, s2_w = O.nf4_quantize_meandq(W[r0:r1], 64, dq)
        if r1 - r0 == step:
            b0, b1 = r0 * kb64, r1 * kb64
            assert np.array_equal(Wq_h[r0:r1], wq_w)
            assert np.array_equal(c_h[b0:b1], c_w)
            assert np.array_equal(m_h[b0 // dq:b0 // dq + m_w.size].view(np.uint32),
                                  m_w.view(np.uint32))
            assert np.array_equal(s2_h[b0 // dq:b0 // dq + s2_w.size].view(np.uint32),
                                  s2_w.view(np.uint32))
        what_rows.append(O.nf4_dequant_meandq(wq_w, c_w, m_w, s2_w, 64, dq)[r - r0])
    what = np.stack(what_rows)
    del W
    for M in wl["Ms"]:
        xb = S.layer_x(wl, M, K, N)
        Y = w4.nf4_gemm_meandq(_x(xb), Wp, m, s2, N, K, dq)
        assert w4.device_status() == w4.W4_OK
        y = _u16(Y)[:, rows]
        y_ref, ab = O.matmul_ref(xb, what)
        ok, ratio = O.check_matmul(y, y_ref, ab)
        assert ok, f"worst error / tolerance = {ratio}"
