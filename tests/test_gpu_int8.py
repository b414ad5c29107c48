"""GPU parity for the LLM.int8 mixed decomposition, through the C ABI,
against the CPU oracle on the same seeded inputs.

Bit-exact: the INT8 weights and their per-row scales.  The product within
|y - y_ref| <= 1e-3 * sum |terms| + ulp_bf16(y_ref) (the INT8 part is an
exact integer sum on both sides; the scaling and the 16-bit outlier part are
fp32 on the device), and bit-exact on inputs whose quantization and products
are exact."""
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


@pytest.mark.parametrize("N,K", [(64, 4096), (1000, 777), (3, 64)])
def test_int8_weights_bit_exact(w4, N, K):
    W = S.draw_w(N, K, 0.02, seed=1, tag=60, outlier_frac=0.01, outlier_scale=8.0)
    W[0] = 0.0                                   # zero row -> scale 1, codes 0
    qw, sw = w4.llm_int8_quantize_weights(dev(W))
    status_ok(w4)
    q_r, s_r = O.int8_quantize_weights(W)
    assert np.array_equal(qw.cpu().numpy(), q_r)
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), s_r.view(np.uint32))


INT8_CASES = [
    # (M, N, K, threshold, outlier_frac)
    (1, 4096, 4096, 6.0, 0.001),       # Llama-7B decode inputs: 0.1% of channels x50
    (4, 1000, 2048, 6.0, 0.001),       # ragged N
    (16, 512, 11008, 6.0, 0.001),
    (40, 256, 1024, 6.0, 0.01),        # more than 32 tokens: the tensor-core (kind::i8) product
    (64, 4096, 4096, 6.0, 0.001),      # prefill-sized LLM.int8, split K
    (256, 512, 2048, 6.0, 0.001),
    (300, 200, 1088, 6.0, 0.002),      # ragged token tile and rows, K = 8.5 stages
    (7, 33, 64, 6.0, 0.05),            # tiny, ragged
    (5, 300, 512, 1e30, 0.0),          # no outliers
    (3, 128, 256, 0.0, 0.0),           # every nonzero channel an outlier
    # tensor-core product: ~120 outlier channels gathered into shared memory
    # for the epilogue, and 2048 (more than fit) read from global memory
    (100, 300, 4096, 6.0, 0.03),
    (48, 256, 2048, 0.0, 0.0),
]


@pytest.mark.parametrize("M,N,K,thr,frac", INT8_CASES)
def test_int8_gemm_tolerance(w4, M, N, K, thr, frac):
    W = S.draw_w(N, K, 0.02, seed=M, tag=61)
    xb = S.draw_x(M, K, seed=M, tag=61, N=N, outlier_frac=frac, outlier_scale=50.0)
    qw, sw = w4.llm_int8_quantize_weights(dev(W))
    y = w4.llm_int8_gemm(x_dev(xb), qw, sw, thr)
    status_ok(w4)
    q_r, s_r = O.int8_quantize_weights(W)
    y_ref, ab = O.int8_mixed_ref(xb, q_r, s_r, thr)
    ok, ratio = O.check_matmul(host_u16(y), y_ref, ab)
    assert ok, f"worst error / tolerance = {ratio}"


@pytest.mark.parametrize("M,N,K", [(3, 48, 128), (64, 256, 1024), (256, 130, 512)])
def test_int8_gemm_exact_on_exact_inputs(w4, M, N, K):
    # weights k/32 with a row maximum of 127/32 and activations k/64 with a
    # token maximum of 127/64 (plus one outlier channel of 8): every scale is
    # a power of two, every code exact, every sum exact in fp32 (warp-level
    # and, above 32 tokens, tensor-core INT8 products)
    rng = np.random.default_rng(7)
    W = rng.integers(-127, 128, (N, K)).astype(np.float32) / 32
    W[:, 0] = 127.0 / 32
    x = rng.integers(-127, 128, (M, K)).astype(np.float32) / 64
    x[:, 1] = 127.0 / 64
    x[:, 5] = 8.0
    xb = S.to_bf16_bits(x)
    qw, sw = w4.llm_int8_quantize_weights(dev(W))
    y = w4.llm_int8_gemm(x_dev(xb), qw, sw)
    status_ok(w4)
    exact = x.astype(np.float64) @ W.astype(np.float64).T
    assert np.array_equal(host_u16(y), S.to_bf16_bits(exact.astype(np.float32)))


def test_int8_argument_errors(w4):
    qw = torch.zeros((8, 96), dtype=torch.int8, device="cuda")      # K % 64 != 0
    sw = torch.ones(8, dtype=torch.float32, device="cuda")
    X = torch.zeros((2, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(w4.W4Error) as e:
        w4.llm_int8_gemm(X, qw, sw)
    assert e.value.status == w4.W4_ERR_INVALID_ARG
    status_ok(w4)


def test_int8_call_leaves_the_w4a16_workspace_clean(w4):
    # the LLM.int8 call runs on its own scratch: a W4A16 GEMM after it (split
    # row groups, so arrival counters in use) still sees a zeroed workspace
    N, K, G, M = 1024, 8192, 128, 4
    W = S.draw_w(N, K, 0.02, seed=9, tag=62)
    q, s, z = O.quantize_rtn(W, G)
    Wq = O.pack_nibbles(q)
    Wp = w4.prepack(dev(Wq), dev(s.view(np.int16), torch.float16), dev(z), G)
    xb = S.draw_x(M, K, seed=9, tag=62, N=N)
    qw, sw = w4.llm_int8_quantize_weights(dev(W))
    w4.llm_int8_gemm(x_dev(xb), qw, sw)
    y = w4.w4a16_gemm(x_dev(xb), Wp, N, K, G)
    status_ok(w4)
    y_ref, ab = O.matmul_ref(xb, O.dequant_rtn(Wq, s, z, G))
    ok, ratio = O.check_matmul(host_u16(y), y_ref, ab)
    assert ok, ratio


def test_int8_calls_share_one_workspace(w4):
    # the workspace's regions move with the shape, so each call clears the
    # counters and the accumulator it uses: calls of different shapes in turn
    # on one (initially garbage) workspace stay right, and the same call
    # twice gives the same bits
    ws = torch.randint(0, 255, (w4.lib.llm_int8_workspace_bytes(16, 1000, 11008) + 256,),
                       dtype=torch.uint8, device="cuda")
    shapes = [(16, 1000, 11008), (1, 4096, 4096), (3, 77, 320), (16, 1000, 11008)]
    for i, (M, N, K) in enumerate(shapes * 2):
        W = S.draw_w(N, K, 0.02, seed=i % 4, tag=64)
        xb = S.draw_x(M, K, seed=i % 4, tag=64, N=N, outlier_frac=0.003, outlier_scale=50.0)
        qw, sw = w4.llm_int8_quantize_weights(dev(W))
        y1 = w4.llm_int8_gemm(x_dev(xb), qw, sw, workspace=ws)
        y2 = w4.llm_int8_gemm(x_dev(xb), qw, sw, workspace=ws)
        status_ok(w4)
        assert torch.equal(y1, y2)
        q_r, s_r = O.int8_quantize_weights(W)
        y_ref, ab = O.int8_mixed_ref(xb, q_r, s_r)
        ok, ratio = O.check_matmul(host_u16(y1), y_ref, ab)
        assert ok, f"call {i}: worst error / tolerance = {ratio}"
