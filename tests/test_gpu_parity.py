"""GPU parity: the CUDA library, called through its C ABI, against the CPU
oracle on the same seeded inputs.

Bit-exact for quantize / pack / prepack / dequant (INT4 and NF4); the matmul
within |y - y_ref| <= 1e-3 * sum_k |x w_hat| + ulp_bf16(y_ref).  A unit-vector
X makes every output a single product x * w_hat = w_hat, so there the matmul
is checked bit-exactly as well (it proves the in-kernel dequant equals the
oracle's w_hat)."""
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


# ----------------------------------------------------------------- quantize

QUANT_CASES = [
    (512, 512, 128, False),
    (4096, 1024, 128, False),
    (200, 384, 64, False),        # ragged N
    (64, 5120, 32, False),
    (96, 512, 32, True),          # act-order
    (40, 13824, 32, True),
    (33, 1024, 128, True),
]


@pytest.mark.parametrize("N,K,G,act", QUANT_CASES)
def test_quantize_dequant_bit_exact(w4, N, K, G, act):
    W = S.draw_w(N, K, 0.02, seed=0, tag=10 + G)
    W[0, :G] = 0.0                           # all-zero group
    W[1, :G] = 0.25                          # constant group
    W[2, :8] = np.array([-1.5, 0, 0.75, 6, 3.25, -0.25, 1, 2.5], np.float32)  # RNE ties
    g_idx = S.act_order_g_idx(S.draw_perm(K, seed=0, tag=5, N=N), G) if act else None
    q, s, z = O.quantize_rtn(W, G, g_idx)
    Wq_ref = O.pack_nibbles(q)
    gi = dev(g_idx) if act else None
    Wq, sc, zr = w4.quantize_rtn(dev(W), G, gi)
    status_ok(w4)
    assert np.array_equal(Wq.cpu().numpy(), Wq_ref)
    assert np.array_equal(host_u16(sc), s.view(np.uint16))
    assert np.array_equal(zr.cpu().numpy(), z)
    what = w4.dequant(Wq, sc, zr, G, gi)
    status_ok(w4)
    assert np.array_equal(host_u16(what), O.dequant_rtn(Wq_ref, s, z, G, g_idx))


def test_quantize_bad_g_idx_reported(w4):
    N, K, G = 8, 256, 64
    W = S.draw_w(N, K, 0.02, seed=1, tag=3)
    g = np.zeros(K, np.int32)
    g[5] = 99                                 # out of range
    w4.quantize_rtn(dev(W), G, dev(g))
    assert w4.device_status() == w4.W4_ERR_DEVICE_INPUT
    assert w4.device_status() == w4.W4_OK     # cleared


@pytest.mark.parametrize("N,K", [(256, 512), (100, 4096), (4096, 14336 // 8)])
def test_nf4_quantize_dequant_bit_exact(w4, N, K):
    W = S.draw_w(N, K, 0.02, seed=0, tag=3)
    W[0, :64] = 0.0
    W[3, 64:128] = 0.01
    Wq_r, c_r, s2_r = O.nf4_quantize(W)
    Wq, c, s2 = w4.nf4_quantize(dev(W))
    status_ok(w4)
    assert np.array_equal(Wq.cpu().numpy(), Wq_r)
    assert np.array_equal(c.cpu().numpy(), c_r)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), s2_r.view(np.uint32))
    what = w4.nf4_dequant(Wq, c, s2)
    assert np.array_equal(host_u16(what), O.nf4_dequant(Wq_r, c_r, s2_r))


@pytest.mark.parametrize("table", ["nf4", "fp4"])
@pytest.mark.parametrize("N,K,dq", [(37, 1024, 300), (64, 4096, 1024), (20, 640, 3)])
def test_blockwise_quantize_dq_group_bit_exact(w4, table, N, K, dq):
    # runs longer than one pass of the kernel (256 blocks), a last run
    # shorter than the others, and very short runs
    W = S.draw_w(N, K, 0.02, seed=N, tag=3)
    W[1, 64:128] = 0.0
    oq, odq = (O.nf4_quantize, O.nf4_dequant) if table == "nf4" else (O.fp4_quantize,
                                                                      O.fp4_dequant)
    dq_dev = w4.nf4_dequant if table == "nf4" else w4.fp4_dequant
    Wq_r, c_r, s2_r = oq(W, 64, dq)
    Wq, c, s2 = (w4.nf4_quantize if table == "nf4" else w4.fp4_quantize)(dev(W), 64, dq)
    status_ok(w4)
    assert np.array_equal(Wq.cpu().numpy(), Wq_r)
    assert np.array_equal(c.cpu().numpy(), c_r)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), s2_r.view(np.uint32))
    assert np.array_equal(host_u16(dq_dev(Wq, c, s2, dq)), odq(Wq_r, c_r, s2_r, 64, dq))


@pytest.mark.parametrize("table", ["nf4", "fp4"])
def test_blockwise_codes_at_decision_thresholds(w4, table):
    # weights whose quotient w / absmax falls on a decision threshold or a few
    # ulps to either side (the codes' exact-division path), for several block
    # scales, both signs
    mids = O.nf4_midpoints() if table == "nf4" else O.fp4_midpoints()
    vals = []
    for t in mids.astype(np.float32):
        for sgn in ((1.0, -1.0) if table == "fp4" else (1.0,)):
            v = t
            for _ in range(2):
                v = np.nextafter(v, np.float32(-np.inf))
            for _ in range(5):                            # t - 2 ulps .. t + 2 ulps
                vals.append(np.float32(sgn) * v)
                v = np.nextafter(v, np.float32(np.inf))
    vals = np.array(vals, np.float32)
    rows = []
    for a in (1.0, 0.7, 0.013, 3.1e-5, 1234.5):
        a = np.float32(a)
        body = (vals * a).astype(np.float32)              # w / a rounds to within ulps of vals
        body = body[np.abs(body) <= a]
        blk = np.concatenate([[a], body])                 # a: the absmax of every block
        blk = np.resize(blk, ((blk.size + 127) // 128) * 128).astype(np.float32)
        rows.append(blk)
    W = np.ascontiguousarray(np.concatenate(rows).reshape(-1, 128).astype(np.float32))
    oq = O.nf4_quantize if table == "nf4" else O.fp4_quantize
    Wq_r, c_r, s2_r = oq(W)
    Wq, c, s2 = (w4.nf4_quantize if table == "nf4" else w4.fp4_quantize)(dev(W))
    status_ok(w4)
    assert np.array_equal(Wq.cpu().numpy(), Wq_r)
    assert np.array_equal(c.cpu().numpy(), c_r)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), s2_r.view(np.uint32))


# ----------------------------------------------------------------- prepack

@pytest.mark.parametrize("N,K,G,act", [(300, 320, 64, False), (256, 1024, 32, True),
                                       (128, 512, 128, False)])
def test_prepack_round_trip(w4, N, K, G, act):
    W = S.draw_w(N, K, 0.02, seed=2, tag=7)
    g_idx = S.act_order_g_idx(S.draw_perm(K, seed=2, tag=5, N=N), G) if act else None
    q, s, z = O.quantize_rtn(W, G, g_idx)
    Wq = O.pack_nibbles(q)
    Wp = w4.prepack(dev(Wq), dev(s.view(np.int16), torch.float16), dev(z), G,
                    dev(g_idx) if act else None)
    status_ok(w4)
    uq, us, uz, up = w4.unprepack(Wp, N, K, G, act)
    if act:
        perm = up.cpu().numpy()
        # stable sort of channels by group
        assert np.array_equal(perm, np.argsort(g_idx, kind="stable"))
        q = q[:, perm]
    assert np.array_equal(uq.cpu().numpy(), O.pack_nibbles(q))
    assert np.array_equal(host_u16(us), s.view(np.uint16))
    assert np.array_equal(uz.cpu().numpy(), z)


def test_prepack_bad_group_sizes_reported(w4):
    N, K, G = 128, 256, 64
    q = np.zeros((N, K // 2), np.uint8)
    s = np.ones((N, K // G), np.float16)
    z = np.zeros((N, K // G), np.uint8)
    g = (np.arange(K) // G).astype(np.int32)
    g[0] = 1                                  # group 0 short, group 1 long
    w4.prepack(dev(q), dev(s.view(np.int16), torch.float16), dev(z), G, dev(g))
    assert w4.device_status() == w4.W4_ERR_DEVICE_INPUT


# ----------------------------------------------------------------- matmul

def _int4_layer(w4, N, K, G, act, seed=0, tag=2, sigma=0.02):
    W = S.draw_w(N, K, sigma, seed=seed, tag=tag)
    g_idx = S.act_order_g_idx(S.draw_perm(K, seed=seed, tag=tag, N=N), G) if act else None
    q, s, z = O.quantize_rtn(W, G, g_idx)
    Wq = O.pack_nibbles(q)
    what = O.dequant_rtn(Wq, s, z, G, g_idx)
    Wp = w4.prepack(dev(Wq), dev(s.view(np.int16), torch.float16), dev(z), G,
                    dev(g_idx) if act else None)
    return what, Wp


def _check(y_dev, xbits, what, rows=None):
    y = host_u16(y_dev)
    if rows is not None:
        xbits = xbits[rows]
        y = y[rows]
    y_ref, ab = O.matmul_ref(xbits, what)
    ok, ratio = O.check_matmul(y, y_ref, ab)
    assert ok, f"worst error / tolerance = {ratio}"
    return ratio


@pytest.mark.parametrize("G,act", [(128, False), (64, False), (32, False), (32, True),
                                   (64, True), (128, True)])
def test_gemm_unit_vectors_exact(w4, G, act):
    # X rows are unit vectors e_k: Y[m, :] = w_hat[:, k_m] exactly
    N, K = 256, 1024
    what, Wp = _int4_layer(w4, N, K, G, act, seed=3)
    for M in (16, 256):
        ks = (np.arange(M) * 61 + 5) % K
        x = np.zeros((M, K), np.float32)
        x[np.arange(M), ks] = 1.0
        xb = S.to_bf16_bits(x)
        y = w4.w4a16_gemm(x_dev(xb), Wp, N, K, G, act)
        status_ok(w4)
        assert np.array_equal(host_u16(y), what[:, ks].T)


GEMM_CASES = [
    # (M, N, K, G, act)
    (1, 512, 512, 128, False),       # tiny single linear
    (4, 512, 512, 128, False),
    (16, 384, 1024, 128, False),
    (17, 200, 768, 64, False),       # ragged N, M just over a tile
    (33, 128, 192, 64, False),       # K not a multiple of 128
    (100, 640, 2048, 128, False),
    (256, 256, 4096, 32, False),
    (300, 384, 1024, 128, False),
    (1, 1024, 5120, 32, True),
    (16, 512, 13824, 32, True),
    (256, 256, 2048, 32, True),
    # act-order group-size sweep ([Survey] §3.2 desc_act with group 64 / 128)
    (1, 300, 1280, 64, True),        # ragged N, K = 10 stages
    (7, 77, 768, 128, True),
    (16, 512, 5120, 64, True),
    (24, 200, 2560, 128, True),      # three token blocks
    (33, 128, 1024, 64, True),       # just over the decode range: tensor-core path
    (256, 384, 2048, 128, True),
    (300, 256, 1536, 64, True),      # ragged M tile
    # decode work-split edge cases
    (1, 16, 64, 64, False),          # one unit: a single warp does everything
    (2, 1, 128, 128, False),         # one output row
    (8, 77, 320, 32, False),         # last stage has no second half, ragged N
    (32, 1000, 4096, 128, False),    # four token blocks, ragged N
    # prefill work split: one full wave of whole tiles, then the last partial
    # wave's tiles split in K (149 and 150 tiles on 148 SMs)
    (40, 19000, 2560, 128, False),   # ragged N, one tail tile in 5 K ranges
    (300, 9550, 2560, 64, True),     # two token tiles, act-order, two tail tiles
    (5, 4096, 4160, 64, False),      # K = 32.5 stages: last stage half, G = 64
    # CTA pairs (256-token tiles over an even number of 128-row tiles): the
    # odd CTA holds tokens 128..255 of a tile, its 128 rows the pair's second
    (129, 512, 2048, 128, False),    # the odd CTA's token half holds one token
    (520, 2304, 4096, 64, False),    # every tile in 2 K ranges, third token tile 8 tokens
    (700, 1536, 8192, 128, False),   # 4 K ranges, ragged third token tile
    (260, 1024, 4096, 32, True),     # act-order, 4 K ranges
    (300, 9728, 4096, 128, False),   # one wave of 74 pairs whole, 2 tail pairs in 4 K ranges
]


@pytest.mark.parametrize("M,N,K,G,act", GEMM_CASES)
def test_gemm_tolerance(w4, M, N, K, G, act):
    what, Wp = _int4_layer(w4, N, K, G, act, seed=M)
    xb = S.draw_x(M, K, seed=0, tag=2, N=N, outlier_frac=0.001, outlier_scale=50.0)
    y = w4.w4a16_gemm(x_dev(xb), Wp, N, K, G, act)
    status_ok(w4)
    _check(y, xb, what)


def test_gemm_repeat_deterministic_and_workspace_clean(w4):
    M, N, K, G = 4, 1024, 8192, 128      # split-K path
    what, Wp = _int4_layer(w4, N, K, G, False, seed=9)
    xb = S.draw_x(M, K, seed=9, tag=2, N=N)
    y1 = w4.w4a16_gemm(x_dev(xb), Wp, N, K, G)
    y2 = w4.w4a16_gemm(x_dev(xb), Wp, N, K, G)
    status_ok(w4)
    assert torch.equal(y1, y2)
    _check(y1, xb, what)


def test_nf4_gemm_unit_vectors_exact(w4):
    N, K = 256, 1024
    W = S.draw_w(N, K, 0.02, seed=4, tag=3)
    Wq_r, c_r, s2_r = O.nf4_quantize(W)
    what = O.nf4_dequant(Wq_r, c_r, s2_r)
    Wp = w4.nf4_prepack(dev(Wq_r), dev(c_r))
    M = 32
    ks = (np.arange(M) * 37 + 3) % K
    x = np.zeros((M, K), np.float32)
    x[np.arange(M), ks] = 1.0
    xb = S.to_bf16_bits(x)
    y = w4.nf4_gemm(x_dev(xb), Wp, dev(s2_r), N, K)
    status_ok(w4)
    assert np.array_equal(host_u16(y), what[:, ks].T)


@pytest.mark.parametrize("M,N,K", [(1, 512, 4096), (8, 384, 1024), (32, 200, 1536),
                                   (300, 256, 512), (1, 40, 64), (3, 4096, 14336),
                                   (260, 1024, 4096)])   # CTA pairs, 4 K ranges
def test_nf4_gemm_tolerance(w4, M, N, K):
    W = S.draw_w(N, K, 0.02, seed=M, tag=3)
    Wq_r, c_r, s2_r = O.nf4_quantize(W)
    what = O.nf4_dequant(Wq_r, c_r, s2_r)
    Wp = w4.nf4_prepack(dev(Wq_r), dev(c_r))
    xb = S.draw_x(M, K, seed=M, tag=3, N=N)
    y = w4.nf4_gemm(x_dev(xb), Wp, dev(s2_r), N, K)
    status_ok(w4)
    _check(y, xb, what)


def test_workspace_shared_across_shapes(w4):
    # split-K calls of different tile counts share one workspace: the counters
    # of one call must never be overwritten by another call's partial sums
    ws = torch.zeros(64 << 20, dtype=torch.uint8, device="cuda")
    layers = [(4, 256, 8192, 128), (1, 4096, 4096, 128), (16, 1024, 2048, 64),
              (3, 2048, 6144, 128)]
    built = [(M, N, K, G, *_int4_layer(w4, N, K, G, False, seed=20 + i))
             for i, (M, N, K, G) in enumerate(layers)]
    for _ in range(2):
        for M, N, K, G, what, Wp in built:
            xb = S.draw_x(M, K, seed=M, tag=2, N=N)
            y = w4.w4a16_gemm(x_dev(xb), Wp, N, K, G, workspace=ws)
            status_ok(w4)
            _check(y, xb, what)
    # the counter region is left zeroed
    assert int(ws[: 65536 * 4].count_nonzero()) == 0


def test_bounded_wait_times_out_and_context_survives(w4):
    # a pipeline wait on a barrier that nothing arrives on gives up, reports
    # W4_ERR_TIMEOUT through the device error word, and leaves the context usable
    w4.selftest_wait_timeout()
    assert w4.device_status() == w4.W4_ERR_TIMEOUT
    assert w4.device_status() == w4.W4_OK          # the word was cleared
    what, Wp = _int4_layer(w4, 256, 512, 128, False, seed=4)
    xb = S.draw_x(4, 512, seed=4, tag=2, N=256)
    y = w4.w4a16_gemm(x_dev(xb), Wp, 256, 512, 128)
    status_ok(w4)
    _check(y, xb, what)
