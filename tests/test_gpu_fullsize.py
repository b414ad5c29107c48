"""Full-size parity: every workload at its full layer shapes and token counts,
through the same C-ABI calls (and so the same kernels and launch
configurations) that bench.py times, checked against the oracle on sampled
outputs.

The oracle quantizes only the sampled output rows (INT4 RTN is per row; for
NF4 the window of rows whose double-quantization runs cover the sampled rows)
and computes their fp64 products.  Checked per workload: the device
quantization of the sampled rows is bit-exact, and every sampled output is
within |y - y_ref| <= 1e-3 * sum_k |x w_hat| + ulp_bf16(y_ref)."""
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


def _host_u16(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _sample_rows(N, n, seed):
    rng = np.random.default_rng([seed, N, 99])
    rows = set(rng.choice(N, size=min(n, N), replace=False).tolist())
    rows.update({0, N - 1, (N // 128) * 128 - 1 if N >= 128 else 0})  # ends and a tile edge
    return np.array(sorted(rows), dtype=np.int64)


def _check(y_dev, xbits, what_rows, rows, tokens=None):
    y = _host_u16(y_dev)[:, rows]
    xb = xbits
    if tokens is not None:
        y = y[tokens]
        xb = xbits[tokens]
    y_ref, ab = O.matmul_ref(xb, what_rows)
    ok, ratio = O.check_matmul(y, y_ref, ab)
    assert ok, f"worst error / tolerance = {ratio}"


def _int4_case(w4, wl, K, N, Ms, act, n_rows=48, n_tokens=None):
    G = wl["G"]
    W = S.layer_w(wl, K, N)
    g_idx = S.act_order_g_idx(S.draw_perm(K, tag=wl["tag"], N=N), G) if act else None
    gi = torch.from_numpy(g_idx).cuda() if act else None
    Wq, sc, zr = w4.quantize_rtn(torch.from_numpy(W).cuda(), G, gi)
    Wp = w4.prepack(Wq, sc, zr, G, gi)
    rows = _sample_rows(N, n_rows, K)
    q, s, z = O.quantize_rtn(W[rows], G, g_idx)
    Wq_r = O.pack_nibbles(q)
    assert np.array_equal(Wq.cpu().numpy()[rows], Wq_r)
    assert np.array_equal(_host_u16(sc)[rows], s.view(np.uint16))
    assert np.array_equal(zr.cpu().numpy()[rows], z)
    what = O.dequant_rtn(Wq_r, s, z, G, g_idx)
    del W
    for M in Ms:
        xb = S.layer_x(wl, M, K, N)
        X = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
        Y = w4.w4a16_gemm(X, Wp, N, K, G, act)
        assert w4.device_status() == w4.W4_OK
        tokens = None
        if n_tokens is not None and M > n_tokens:
            rng = np.random.default_rng([M, K, 7])
            tokens = np.sort(np.concatenate([[0, M - 1], rng.choice(M, n_tokens, replace=False)]))
        _check(Y, xb, what, rows, tokens)
        del X, Y


@pytest.mark.parametrize("K,N", S.LLAMA7B_DECODE["shapes"])
def test_fullsize_llama7b_decode(w4, K, N):
    _int4_case(w4, S.LLAMA7B_DECODE, K, N, S.LLAMA7B_DECODE["Ms"], False)


@pytest.mark.parametrize("G", [S.ACT_ORDER_13B["G"], *S.ACT_ORDER_13B["G_sweep"]])
@pytest.mark.parametrize("K,N", S.ACT_ORDER_13B["shapes"])
def test_fullsize_act_order_13b(w4, K, N, G):
    # group 32 and the 64 / 128 sweep, each with its own g_idx of the same
    # seeded permutation
    _int4_case(w4, dict(S.ACT_ORDER_13B, G=G), K, N, S.ACT_ORDER_13B["Ms"], True, n_tokens=24)


@pytest.mark.parametrize("K,N", S.PREFILL_70B["shapes"])
def test_fullsize_prefill_70b(w4, K, N):
    _int4_case(w4, S.PREFILL_70B, K, N, S.PREFILL_70B["Ms"], False, n_rows=24, n_tokens=24)


@pytest.mark.parametrize("K,N", S.NF4_DECODE["shapes"])
def test_fullsize_nf4_decode(w4, K, N):
    wl = S.NF4_DECODE
    dq = wl["dq_group"]
    W = S.layer_w(wl, K, N)
    Wq, c, s2 = w4.nf4_quantize(torch.from_numpy(W).cuda(), 64, dq)
    Wp = w4.nf4_prepack(Wq, c)
    # windows of whole double-quantization runs around the sampled rows:
    # rows per window a multiple of `step`, starting on a run boundary
    kb64 = K // 64
    step = dq // math.gcd(kb64, dq)
    rows = _sample_rows(N, 24, K)
    Wq_h, c_h, s2_h = Wq.cpu().numpy(), c.cpu().numpy(), s2.cpu().numpy()
    what_rows = []
    for r in rows:
        r0 = (r // step) * step
        r1 = min(N, r0 + step)
        wq_w, c_w, s2_w = O.nf4_quantize(W[r0:r1], 64, dq)
        if r1 - r0 == step:     # a whole window: the device values of its rows must agree
            b0, b1 = r0 * kb64, r1 * kb64
            assert np.array_equal(Wq_h[r0:r1], wq_w)
            assert np.array_equal(c_h[b0:b1], c_w)
            assert np.array_equal(s2_h[b0 // dq:b0 // dq + s2_w.size].view(np.uint32),
                                  s2_w.view(np.uint32))
        what_w = O.nf4_dequant(wq_w, c_w, s2_w, 64, dq)
        what_rows.append(what_w[r - r0])
    what = np.stack(what_rows)
    del W
    for M in wl["Ms"]:
        xb = S.layer_x(wl, M, K, N)
        X = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
        Y = w4.nf4_gemm(X, Wp, s2, N, K, dq)
        assert w4.device_status() == w4.W4_OK
        _check(Y, xb, what, rows)
        del X, Y


@pytest.mark.parametrize("K,N", S.AWQ_SYM_DECODE["shapes"])
def test_fullsize_awq_sym_decode(w4, K, N):
    wl = S.AWQ_SYM_DECODE
    G = wl["G"]
    W = S.layer_w(wl, K, N)
    s = S.layer_awq_s(wl, K, N)
    sd = torch.from_numpy(s).cuda()
    Wsd = w4.awq_scale_weights(torch.from_numpy(W).cuda(), sd)
    Wq, sc, zr = w4.quantize_sym(Wsd, G)
    del Wsd
    Wp = w4.prepack(Wq, sc, zr, G)
    rows = _sample_rows(N, 48, K)
    q, sr, z = O.quantize_sym(O.awq_scale_weights(W[rows], s), G)
    Wq_r = O.pack_nibbles(q)
    assert np.array_equal(Wq.cpu().numpy()[rows], Wq_r)
    assert np.array_equal(_host_u16(sc)[rows], sr.view(np.uint16))
    assert np.array_equal(zr.cpu().numpy()[rows], z)
    what = O.dequant_rtn(Wq_r, sr, z, G)
    del W
    for M in wl["Ms"]:
        xb = S.layer_x(wl, M, K, N)
        X = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
        Y = w4.w4a16_awq_gemm(X, sd, Wp, N, K, G)
        assert w4.device_status() == w4.W4_OK
        _check(Y, O.awq_scale_activations(xb, s), what, rows)
        del X, Y


@pytest.mark.parametrize("K,N", S.FP4_DECODE["shapes"])
def test_fullsize_fp4_decode(w4, K, N):
    wl = S.FP4_DECODE
    dq = wl["dq_group"]
    W = S.layer_w(wl, K, N)
    Wq, c, s2 = w4.fp4_quantize(torch.from_numpy(W).cuda(), 64, dq)
    Wp = w4.nf4_prepack(Wq, c)
    kb64 = K // 64
    step = dq // math.gcd(kb64, dq)
    rows = _sample_rows(N, 24, K)
    Wq_h, c_h, s2_h = Wq.cpu().numpy(), c.cpu().numpy(), s2.cpu().numpy()
    what_rows = []
    for r in rows:
        r0 = (r // step) * step
        r1 = min(N, r0 + step)
        wq_w, c_w, s2_w = O.fp4_quantize(W[r0:r1], 64, dq)
        if r1 - r0 == step:
            b0, b1 = r0 * kb64, r1 * kb64
            assert np.array_equal(Wq_h[r0:r1], wq_w)
            assert np.array_equal(c_h[b0:b1], c_w)
            assert np.array_equal(s2_h[b0 // dq:b0 // dq + s2_w.size].view(np.uint32),
                                  s2_w.view(np.uint32))
        what_rows.append(O.fp4_dequant(wq_w, c_w, s2_w, 64, dq)[r - r0])
    what = np.stack(what_rows)
    del W
    for M in wl["Ms"]:
        xb = S.layer_x(wl, M, K, N)
        X = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).cuda()
        Y = w4.fp4_gemm(X, Wp, s2, N, K, dq)
        assert w4.device_status() == w4.W4_OK
        _check(Y, xb, what, rows)
        del X, Y
