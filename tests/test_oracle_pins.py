"""Pins for the CPU oracle: what the pages and the mathematics fix, checked
against the oracle without re-typing its formulas.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, truncation instead of round-half-even, swapped nibbles, a
transposed operand) fails at least one of them; ``test_planted_mistakes``
checks exactly that by planting such slips in copies of oracle functions.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from weight_only_bit_gemm_b200 import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse_worked(path):
    cases, cur = [], None
    for line in open(path, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        if key == "name":
            cur = {"name": vals[0]}
            cases.append(cur)
        else:
            cur[key] = vals
    return cases


WORKED = _parse_worked(os.path.join(GOLDEN, "int4_rtn_worked.txt"))


# ---------------------------------------------------------------- worked examples

@pytest.mark.parametrize("case", WORKED, ids=lambda c: c["name"])
def test_int4_worked_examples(case):
    G = int(case["G"][0])
    w = np.array([float(v) for v in case["w"]], np.float32)[None, :]
    codes, s16, zp = O.quantize_rtn(w, G)
    assert s16.view(np.uint16)[0, 0] == int(case["scale_f16_bits"][0], 16)
    assert zp[0, 0] == int(case["zero"][0])
    assert codes[0].tolist() == [int(v) for v in case["codes"]]
    packed = O.pack_nibbles(codes)
    assert packed[0].tolist() == [int(v, 16) for v in case["packed_hex"]]
    if "what_f32" in case:
        f = O.dequant_rtn_f32(packed, s16, zp, G)
        assert f[0].tolist() == [float(v) for v in case["what_f32"]]
    what = O.bf16_bits_to_f32(O.dequant_rtn(packed, s16, zp, G))
    assert what[0].tolist() == [float(v) for v in case["what"]]


def test_sizes_closed_forms():
    # primer: 7B fp16 ~14 GB, 4-bit ~3.5 GB; survey / comparison: 70B 140 -> 35 GB
    assert 7_000_000_000 * 2 == 14_000_000_000
    assert O.code_bytes(7_000_000_000) == 3_500_000_000
    assert O.code_bytes(70_000_000_000) == 35_000_000_000
    # handbook §4.1: 1.5e9 params, group 128.  Codes (1.5e9*4)/8 B divided by
    # 1024^2 is 715.3 (MiB), printed "0.71GB"; scales 1.5e9/128*2 B = 23.4 MB,
    # printed "0.023GB".  The byte counts are exact; the printed figures carry
    # a unit slip, so they are matched to their printed digits only.
    p = 1_500_000_000
    assert O.code_bytes(p) == 750_000_000
    assert abs(O.code_bytes(p) / 1024 ** 2 / 1000 - 0.71) < 0.01
    scale_total = O.weight_bytes(1, p, 128, zero_bytes=0) - O.code_bytes(p)
    assert scale_total == 23_437_500
    assert abs(scale_total / 1e9 - 0.023) < 0.001
    # the handbook counts a 2-byte zero point per group; this library stores 4 bits
    pages = O.weight_bytes(1, p, 128, zero_bytes=2.0)
    ours = O.weight_bytes(1, p, 128)
    assert pages - ours == (p // 128) * 1.5
    # a Llama-7B-shaped layer: K=4096, N=12288 at G=128
    assert O.weight_bytes(12288, 4096, 128) == 12288 * 2048 + 12288 * 32 * 2.5


# ---------------------------------------------------------------- library agreement

def test_bf16_rounding_matches_torch_cast():
    rng = np.random.default_rng(11)
    vals = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(20_000) * 1e-30).astype(np.float32),
        (rng.standard_normal(20_000) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -3.0e38], np.float32),
    ])
    # exact ties: low 16 bits 0x8000 with even and odd kept LSB
    u = rng.integers(0, 2 ** 31 - 2 ** 24, 50_000, dtype=np.uint64).astype(np.uint32)
    ties = ((u & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    vals = np.concatenate([vals, ties[np.isfinite(ties)]])
    ours = O.bf16_round_bits(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_fp16_scale_rounding_matches_torch_cast():
    rng = np.random.default_rng(12)
    s = np.abs(rng.standard_normal(100_000)).astype(np.float32) * np.float32(0.01)
    s = np.concatenate([s, np.float32(2.0) ** np.arange(-30, 16, dtype=np.float32)])
    ref = torch.from_numpy(s).to(torch.float16).numpy()
    assert np.array_equal(s.astype(np.float16).view(np.uint16), ref.view(np.uint16))


# ---------------------------------------------------------------- INT4 invariants

def _rand_w(N, K, seed, sigma=0.02):
    return S.draw_w(N, K, sigma, seed=seed, tag=99)


@pytest.mark.parametrize("G", [32, 64, 128])
def test_int4_codes_and_error_bound(G):
    W = _rand_w(64, 1024, G)
    W[3, :G] = 0.0                     # all-zero group
    W[4, G:2 * G] = 0.0173             # constant positive group
    W[5, :G] = -0.0311                 # constant negative group
    q, s16, zp = O.quantize_rtn(W, G)
    assert q.min() >= 0 and q.max() <= 15
    assert zp.min() >= 0 and zp.max() <= 15
    sf = s16.astype(np.float32)
    gk = np.arange(W.shape[1]) // G
    what = O.dequant_rtn_f32(O.pack_nibbles(q), s16, zp, G)
    err = np.abs(W.astype(np.float64) - what)
    bound = sf[:, gk].astype(np.float64)
    unclamped = (q > 0) & (q < 15)
    assert np.all(err[unclamped] <= bound[unclamped] / 2)
    # clamped codes: fp16 rounding of the scale can push the end of the range
    # by at most 15 * 2^-11 * scale
    clamped = ~unclamped
    assert np.all(err[clamped] <= bound[clamped] * (0.5 + 15 * 2.0 ** -11))
    # group min -> code near 0, group max -> code near 15 (for mixed-sign groups)
    Wg = W.reshape(64, -1, G)
    qg = q.reshape(64, -1, G)
    mixed = (Wg.min(-1) < 0) & (Wg.max(-1) > 0)
    qmin = np.take_along_axis(qg, Wg.argmin(-1)[..., None], -1)[..., 0]
    qmax = np.take_along_axis(qg, Wg.argmax(-1)[..., None], -1)[..., 0]
    assert np.all(qmin[mixed] <= 1) and np.all(qmax[mixed] >= 14)
    # constant and zero groups dequantize without error beyond bf16 rounding
    w_bf = O.bf16_bits_to_f32(O.dequant_rtn(O.pack_nibbles(q), s16, zp, G))
    assert np.all(w_bf[3, :G] == 0)
    assert np.allclose(w_bf[4, G:2 * G], 0.0173, rtol=2 ** -8)
    assert np.allclose(w_bf[5, :G], -0.0311, rtol=2 ** -8)


def test_int4_brute_force_nearest_level():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((40, 16)) * 0.05).astype(np.float32)
    W[0, :4] = np.array([-0.1, 0.05, 0.0, 0.2], np.float32)
    G = 4
    q, s16, zp = O.quantize_rtn(W, G)
    sf = s16.astype(np.float64)
    for n in range(W.shape[0]):
        for k in range(W.shape[1]):
            g = k // G
            # the code picked by round(w/s)+zp is a nearest of the 16 levels,
            # measured in units of the scale (no clamping happens here)
            t = float(np.float32(W[n, k]) / np.float32(sf[n, g]))
            dist = [abs(t - (lv - int(zp[n, g]))) for lv in range(16)]
            best = min(dist)
            assert abs(dist[int(q[n, k])] - best) < 1e-12


def test_int4_requantize_round_trip():
    W = _rand_w(32, 512, 3)
    q, s16, zp = O.quantize_rtn(W, 128)
    f = O.dequant_rtn_f32(O.pack_nibbles(q), s16, zp, 128)
    sk = s16.astype(np.float32)[:, np.arange(512) // 128]
    zk = zp.astype(np.float32)[:, np.arange(512) // 128]
    q2 = np.clip(np.rint(f.astype(np.float32) / sk) + zk, 0, 15)
    assert np.array_equal(q2.astype(np.uint8), q)


def test_pack_unpack_bijective():
    rng = np.random.default_rng(2)
    q = rng.integers(0, 16, (7, 64), dtype=np.uint8)
    p = O.pack_nibbles(q)
    assert p.shape == (7, 32)
    assert np.array_equal(O.unpack_nibbles(p), q)
    assert np.array_equal(p & 0xF, q[:, 0::2])


# ---------------------------------------------------------------- act-order

def test_act_order_identity_equals_contiguous():
    W = _rand_w(16, 512, 4)
    g_id = (np.arange(512) // 64).astype(np.int32)
    a = O.quantize_rtn(W, 64)
    b = O.quantize_rtn(W, 64, g_id)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    assert np.array_equal(O.dequant_rtn(O.pack_nibbles(a[0]), a[1], a[2], 64),
                          O.dequant_rtn(O.pack_nibbles(b[0]), b[1], b[2], 64, g_id))


def test_act_order_equals_permuted_contiguous():
    # quantizing with g_idx[perm[j]] = j // G is the same as quantizing the
    # column-permuted matrix W[:, perm] with contiguous groups
    K, G = 256, 32
    W = _rand_w(12, K, 6)
    perm = S.draw_perm(K, seed=1, tag=5, N=12)
    g_idx = S.act_order_g_idx(perm, G)
    q, s, z = O.quantize_rtn(W, G, g_idx)
    qp, sp, zpp = O.quantize_rtn(W[:, perm], G)
    assert np.array_equal(q[:, perm], qp)
    assert np.array_equal(s, sp) and np.array_equal(z, zpp)
    d = O.dequant_rtn(O.pack_nibbles(q), s, z, G, g_idx)
    dp = O.dequant_rtn(O.pack_nibbles(qp), sp, zpp, G)
    assert np.array_equal(d[:, perm], dp)


def test_g_idx_validation():
    W = _rand_w(2, 64, 1)
    with pytest.raises(ValueError):
        O.quantize_rtn(W, 32, np.full(64, 2, np.int32))
    with pytest.raises(ValueError):
        O.quantize_rtn(W, 32, np.full(64, -1, np.int32))


# ---------------------------------------------------------------- symmetric INT4

SYM_WORKED = _parse_worked(os.path.join(GOLDEN, "int4_sym_worked.txt"))


def test_sym_page_worked_example():
    # [Survey] §1: a largest magnitude of 80 gives an 8-bit symmetric scale of
    # 80/127, about 0.63; the sign of the extreme does not matter (absmax)
    for ext in (80.0, -80.0):
        w = np.array([[ext, 3.0, -1.0, 0.5]], np.float32)
        s32, _ = O.sym_params(w, 4, bits=8)
        assert abs(float(s32[0, 0]) - 0.63) < 0.005
        assert float(s32[0, 0]) == float(np.float32(80.0) / np.float32(127.0))


@pytest.mark.parametrize("case", SYM_WORKED, ids=lambda c: c["name"])
def test_sym_worked_examples(case):
    G = int(case["G"][0])
    w = np.array([float(v) for v in case["w"]], np.float32)[None, :]
    codes, s16, zp = O.quantize_sym(w, G)
    assert s16.view(np.uint16)[0, 0] == int(case["scale_f16_bits"][0], 16)
    assert np.all(zp == 8)
    assert codes[0].tolist() == [int(v) for v in case["codes"]]
    packed = O.pack_nibbles(codes)
    assert packed[0].tolist() == [int(v, 16) for v in case["packed_hex"]]
    what = O.bf16_bits_to_f32(O.dequant_rtn(packed, s16, zp, G))
    assert what[0].tolist() == [float(v) for v in case["what"]]


@pytest.mark.parametrize("G", [32, 128])
def test_sym_bound_symmetry_and_nearest_level(G):
    W = _rand_w(48, 512, 40 + G)
    W[2, :G] = 0.0
    q, s16, zp = O.quantize_sym(W, G)
    assert q.min() >= 1 and q.max() <= 15 and np.all(zp == 8)
    gk = np.arange(W.shape[1]) // G
    sf = s16.astype(np.float64)[:, gk]
    # max|w| of each group lands on code 1 or 15; every weight is within half
    # a step (fp16 rounding of the scale moves the ends by at most 7 * 2^-11)
    what = O.dequant_rtn_f32(O.pack_nibbles(q), s16, zp, G)
    err = np.abs(W.astype(np.float64) - what)
    assert np.all(err <= sf * (0.5 + 7 * 2.0 ** -11))
    Wg, qg = W.reshape(48, -1, G), q.reshape(48, -1, G)
    amax_at = np.abs(Wg).argmax(-1)[..., None]
    qa = np.take_along_axis(qg, amax_at, -1)[..., 0]
    nz = np.abs(Wg).max(-1) > 0
    assert np.all((qa[nz] == 1) | (qa[nz] == 15))
    # zero group -> scale 1.0 and every code 8
    assert s16[2, 0] == np.float16(1.0) and np.all(q[2, :G] == 8)
    # negating W mirrors every code about the zero point: rint(-t) = -rint(t)
    qn, sn, _ = O.quantize_sym(-W, G)
    assert np.array_equal(sn, s16) and np.array_equal(qn.astype(int), 16 - q.astype(int))
    # brute force on a slice: the code is a nearest of the 15 levels in units
    # of the scale, ties to the even integer
    for n in range(4):
        for k in range(0, 512, 7):
            t = float(np.float32(W[n, k]) / np.float32(sf[n, k]))
            dist = [abs(t - (lv - 8)) for lv in range(1, 16)]
            best = min(dist)
            cands = [lv for lv, d in zip(range(1, 16), dist) if abs(d - best) < 1e-12]
            pick = cands[0] if len(cands) == 1 else [c for c in cands if (c - 8) % 2 == 0][0]
            assert int(q[n, k]) == pick


def test_sym_act_order_equals_permuted_contiguous():
    K, G = 256, 64
    W = _rand_w(10, K, 41)
    perm = S.draw_perm(K, seed=2, tag=5, N=10)
    g_idx = S.act_order_g_idx(perm, G)
    q, s, z = O.quantize_sym(W, G, g_idx)
    qp, sp, zpp = O.quantize_sym(W[:, perm], G)
    assert np.array_equal(q[:, perm], qp)
    assert np.array_equal(s, sp) and np.array_equal(z, zpp)


# ---------------------------------------------------------------- AWQ factor

def test_awq_identity_and_powers_of_two():
    W = _rand_w(8, 256, 42)
    xb = S.draw_x(4, 256, seed=3)
    one = np.ones(256, np.float32)
    assert np.array_equal(O.awq_scale_weights(W, one), W)
    assert np.array_equal(O.awq_scale_activations(xb, one), xb)
    # a power of two changes only the exponent: exact on both sides
    s = np.where(np.arange(256) % 3 == 0, 2.0, 0.5).astype(np.float32)
    ws = O.awq_scale_weights(W, s)
    assert np.array_equal(ws, W * s[None, :])
    xs = O.bf16_bits_to_f32(O.awq_scale_activations(xb, s))
    assert np.array_equal(xs, O.bf16_bits_to_f32(xb) / s[None, :])


def test_awq_product_invariance():
    # [Survey] §4.1: (W s)(X / s) leaves the product unchanged; with bf16
    # activations the only change is one bf16 rounding of each x / s
    rng = np.random.default_rng(7)
    M, N, K = 3, 5, 192
    W = _rand_w(N, K, 43)
    s = rng.uniform(0.5, 2.0, K).astype(np.float32)   # not a power of two
    xb = S.draw_x(M, K, seed=4)
    x = O.bf16_bits_to_f32(xb).astype(np.float64)
    xs = O.bf16_bits_to_f32(O.awq_scale_activations(xb, s)).astype(np.float64)
    ws = O.awq_scale_weights(W, s).astype(np.float64)
    y0 = x @ W.astype(np.float64).T
    y1 = xs @ ws.T
    bound = (np.abs(x) @ np.abs(W.astype(np.float64)).T) * (2.0 ** -8 + 2.0 ** -22)
    assert np.all(np.abs(y1 - y0) <= bound)


def test_awq_effective_weight_follows_page_formula():
    # [Comparison] §4.1: the weight X sees is round(W s / scale) scale / s,
    # so its error is at most half a step of the scaled group, divided by s_k
    rng = np.random.default_rng(8)
    N, K, G = 16, 256, 64
    W = _rand_w(N, K, 44)
    s = rng.uniform(0.95, 1.05, K).astype(np.float32)
    q, s16, zp = O.quantize_rtn(O.awq_scale_weights(W, s), G)
    f = O.dequant_rtn_f32(O.pack_nibbles(q), s16, zp, G)
    eff = f / s[None, :].astype(np.float64)
    step = s16.astype(np.float64)[:, np.arange(K) // G]
    bound = step * (0.5 + 15 * 2.0 ** -11) / s[None, :] + np.abs(W) * 2.0 ** -22
    assert np.all(np.abs(eff - W.astype(np.float64)) <= bound)


# ---------------------------------------------------------------- NF4

def test_nf4_table_invariants():
    T = O.nf4_table().astype(np.float64)
    assert T.shape == (16,)
    assert np.all(np.diff(T) > 0)                      # 16 distinct increasing levels
    assert T[0] == -1.0 and T[15] == 1.0               # normalised to [-1, 1]
    assert T[7] == 0.0 and np.count_nonzero(T == 0) == 1
    assert np.count_nonzero(T < 0) == 7 and np.count_nonzero(T > 0) == 8
    gaps = np.diff(T)
    # denser near zero: gaps grow monotonically away from zero on each side
    assert np.all(np.diff(gaps[7:]) > 0) and np.all(np.diff(gaps[:7]) < 0)
    # quantile spacing: the positive levels sit at equally spaced probabilities
    # of the standard normal (a property, checked through the normal CDF)
    top = math.sqrt(2) * _erfinv_pos(2 * (1 - 0.5 * (1 / 30 + 1 / 32)) - 1)
    p = [0.5 * (1 + math.erf(t * top / math.sqrt(2))) for t in T[8:]]
    d = np.diff(p)
    assert np.allclose(d, d[0], rtol=1e-5)


def _erfinv_pos(y):
    # bisection on math.erf (independent of statistics.NormalDist.inv_cdf)
    lo, hi = 0.0, 6.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if math.erf(mid) < y:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def _normal_quantile_bisect(p):
    """x with Phi(x) = p, Phi(x) = erfc(-x / sqrt 2) / 2, by 300 bisection
    steps in fp64 (converges to the last bit; no library inverse CDF)."""
    lo, hi = -12.0, 12.0
    for _ in range(300):
        mid = 0.5 * (lo + hi)
        if 0.5 * math.erfc(-mid / math.sqrt(2.0)) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def _nf4_levels_independent():
    """The R6 construction evaluated independently of the oracle: the QLoRA
    offset delta = 1 - (1/30 + 1/32)/2; quantiles at the first 8 of 9 equally
    spaced probabilities from delta down to 1/2 (positive side) and the first
    7 of 8 (negative side, mirrored); an exact zero; all divided by the
    largest quantile; fp64 throughout, one rounding to fp32 at the end
    ([Survey] §6.1: levels are normal quantiles, denser near zero, with an
    exact zero; §6.2 and [Primer] §七: NF4 spans [-1, 1] under the absmax)."""
    delta = 1.0 - (Fraction(1, 30) + Fraction(1, 32)) / 2
    steps_p = [delta + (Fraction(1, 2) - delta) * i / 8 for i in range(8)]
    steps_n = [delta + (Fraction(1, 2) - delta) * i / 7 for i in range(7)]
    top = _normal_quantile_bisect(float(delta))
    vals = [_normal_quantile_bisect(float(p)) / top for p in steps_p]
    vals += [-_normal_quantile_bisect(float(p)) / top for p in steps_n]
    vals.append(0.0)
    return np.array(sorted(vals), np.float64).astype(np.float32)


def test_nf4_table_digits_pinned():
    # every level within one fp32 ulp of the independent evaluation (they
    # agree bit for bit on this machine); a wrong delta, a wrong split of the
    # quantiles between the two signs or a wrong normaliser moves several
    # levels by thousands of ulps
    T = O.nf4_table()
    ref = _nf4_levels_independent()
    assert T.dtype == np.float32 and T.shape == (16,)
    assert np.all(np.abs(T.view(np.int32).astype(np.int64) - ref.view(np.int32)) <= 1)


def test_planted_mistakes_nf4_table(monkeypatch):
    import statistics
    import oracle.w4_oracle as M
    nd = statistics.NormalDist()

    def built(delta, n_pos_steps, n_neg_steps, n_pos, n_neg, norm="top"):
        pos = [nd.inv_cdf(delta + (0.5 - delta) * i / n_pos_steps) for i in range(n_pos)]
        neg = [-nd.inv_cdf(delta + (0.5 - delta) * i / n_neg_steps) for i in range(n_neg)]
        lv = sorted(neg + [0.0] + pos)
        d = nd.inv_cdf(delta) if norm == "top" else max(abs(v) for v in lv[1:-1])
        return np.array([v / d for v in lv], np.float64).astype(np.float32)

    good = 1.0 - 0.5 * (1 / 30 + 1 / 32)
    mistakes = {
        "delta from 1/30 only": built(1.0 - 0.5 * (2 / 30), 8, 7, 8, 7),
        "delta from 1/32 only": built(1.0 - 0.5 * (2 / 32), 8, 7, 8, 7),
        "negatives on the positive grid": built(good, 8, 8, 8, 7),
        "positives on the negative grid": built(good, 7, 7, 8, 7),
        "normalised by the second level": built(good, 8, 7, 8, 7, norm="second"),
    }
    for name, table in mistakes.items():
        monkeypatch.setattr(M, "nf4_table", lambda t=table: t)
        monkeypatch.setattr(O, "nf4_table", lambda t=table: t)
        with pytest.raises(AssertionError):
            test_nf4_table_digits_pinned()
        monkeypatch.undo()
    test_nf4_table_digits_pinned()


def test_nf4_codes_brute_force_nearest():
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((6, 128)) * 0.02).astype(np.float32)
    W[1, :64] = 0.0                                    # all-zero block
    q = O.nf4_codes(W)
    T = O.nf4_table().astype(np.float64)
    a = O.nf4_absmax(W)
    for b in range(a.size):
        n, j = divmod(b * 64, 128)
        for i in range(64):
            w = W[n, j + i]
            v = float(np.float32(w) / np.float32(a[b])) if a[b] > 0 else 0.0
            dist = np.abs(v - T)
            qq = int(q[n, j + i])
            assert dist[qq] <= dist.min() + 1e-7
    assert np.all(q[1, :64] == 7)
    # the block maximum magnitude maps to an end level
    for b in range(a.size):
        n, j = divmod(b * 64, 128)
        blk = W[n, j:j + 64]
        if a[b] > 0:
            i = int(np.argmax(np.abs(blk)))
            assert int(q[n, j + i]) in (0, 15)


def test_nf4_double_quant_bound_and_zero_block():
    W = S.draw_w(40, 1024, 0.02, seed=3, tag=3)
    W[0, :64] = 0.0
    Wq, c, s2 = O.nf4_quantize(W)
    a = O.nf4_absmax(W).astype(np.float64)
    nb = a.size
    assert c.shape == (nb,) and s2.shape == ((nb + 255) // 256,)
    s = s2.astype(np.float64)[np.arange(nb) // 256]
    a_dq = c.astype(np.float64) * s
    assert np.all(np.abs(a - a_dq) <= s / 2 * (1 + 1e-6))
    # the largest absmax of each run is reproduced by code 255 (up to fp32)
    for r in range(s2.size):
        run = slice(r * 256, (r + 1) * 256)
        assert c[run].max() == 255
    what = O.bf16_bits_to_f32(O.nf4_dequant(Wq, c, s2))
    assert np.all(what[0, :64] == 0.0)
    # dequantized values are T[q] * absmax' up to one bf16 rounding
    q = O.unpack_nibbles(Wq).reshape(-1, 64)
    ref = O.nf4_table()[q].astype(np.float64) * a_dq[:, None]
    assert np.allclose(what.reshape(-1, 64), ref, rtol=2 ** -8, atol=0)


# ---------------------------------------------------------------- matmul

def test_matmul_exact_small_brute_force():
    wl = S.TINY
    K, N = 64, 24
    W = S.draw_w(N, K, 0.02, seed=0, tag=wl["tag"])
    q, s, z = O.quantize_rtn(W, 32)
    what = O.dequant_rtn(O.pack_nibbles(q), s, z, 32)
    x = S.draw_x(3, K, seed=0, tag=1, N=N)
    y, ab = O.matmul_ref(x, what)
    exact = O.matmul_exact_small(x, what)
    for m in range(3):
        for n in range(N):
            # fp64 accumulation of exact bf16 x bf16 products: relative error
            # is far below the 1e-3 tolerance of the GPU check
            assert abs(Fraction(float(y[m, n])) - exact[m][n]) <= Fraction(1, 10 ** 12) * \
                Fraction(float(ab[m, n]) + 1e-30)


def test_matmul_unit_vector_picks_column():
    K, N = 256, 16
    W = _rand_w(N, K, 9)
    q, s, z = O.quantize_rtn(W, 128)
    what = O.dequant_rtn(O.pack_nibbles(q), s, z, 128)
    for k in (0, 1, 77, 255):
        e = np.zeros((1, K), np.float32)
        e[0, k] = 1.0
        y, ab = O.matmul_ref(S.to_bf16_bits(e), what)
        assert np.array_equal(y[0], O.bf16_bits_to_f64(what[:, k]))


def test_matmul_constant_group_closed_form():
    # W constant c on a group: every code dequantizes to the same bf16 value v,
    # so y = v * sum(x) over the group
    K, G = 128, 128
    W = np.full((1, K), 0.0123, np.float32)
    q, s, z = O.quantize_rtn(W, G)
    what = O.dequant_rtn(O.pack_nibbles(q), s, z, G)
    v = O.bf16_bits_to_f64(what[0, 0])
    assert np.all(O.bf16_bits_to_f64(what) == v)
    x = S.draw_x(2, K, seed=4, tag=1)
    y, _ = O.matmul_ref(x, what)
    assert np.allclose(y[:, 0], v * O.bf16_bits_to_f64(x).sum(1), rtol=1e-14)


def test_matmul_ref_matches_float64_numpy_layer():
    wl = S.LLAMA7B_DECODE
    K, N = 1024, 512
    W = S.draw_w(N, K, 0.02, seed=0, tag=wl["tag"])
    q, s, z = O.quantize_rtn(W, 128)
    what = O.dequant_rtn(O.pack_nibbles(q), s, z, 128)
    x = S.draw_x(4, K, seed=0, tag=2, N=N, outlier_frac=0.001, outlier_scale=50.0)
    y, ab = O.matmul_ref(x, what)
    xf = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).double()
    wf = torch.from_numpy(what.view(np.int16)).view(torch.bfloat16).double()
    yt = (xf @ wf.T).numpy()
    assert np.allclose(y, yt, rtol=1e-12, atol=1e-12)
    assert np.all(ab >= np.abs(y))


def test_tolerance_ulp():
    assert O.ulp_bf16(np.array([1.0]))[0] == 2.0 ** -7
    assert O.ulp_bf16(np.array([1.5]))[0] == 2.0 ** -7
    assert O.ulp_bf16(np.array([-2.0]))[0] == 2.0 ** -6
    assert O.ulp_bf16(np.array([0.0]))[0] == 2.0 ** -133
    ok, r = O.check_matmul(S.to_bf16_bits(np.array([[1.0]], np.float32)),
                           np.array([[1.0 + 2 ** -8]]), np.array([[0.0]]))
    assert ok and r <= 0.5


# ------------------------------------------------- NF4 mean-offset double quant (R20)

def test_meandq_worked_example():
    # two runs of dq_group = 4 constants (the second one partial):
    # run 0 = (1, 2, 3, 6): mean 12 / 4 = 3 exactly; residuals (-2, -1, 0, 3);
    #   scale = 3 / 127; codes -2 / (3/127) = -84.67 -> -85, -1 -> -42.33 -> -42,
    #   0 -> 0 and 3 -> 127; the residual 0 comes back as the mean itself
    # run 1 = (10, 10, 10): equal constants, residuals 0, scale 1 (the zero
    #   rule), codes 0, every constant back exactly
    a = np.array([1, 2, 3, 6, 10, 10, 10], np.float32)
    c, mean, s2 = O.nf4_double_quant_mean(a, 4)
    assert c.dtype == np.int8 and c.tolist() == [-85, -42, 0, 127, 0, 0, 0]
    assert mean.tolist() == [3.0, 10.0]
    assert s2[0] == np.float32(3.0) / np.float32(127.0) and s2[1] == 1.0
    back = O.nf4_absmax_mean_dequant(c, mean, s2, 4)
    assert back[2] == 3.0 and back[4:].tolist() == [10.0, 10.0, 10.0]
    assert np.all(np.abs(back[:4].astype(np.float64) - a[:4]) <= float(s2[0]) / 2)
    # an all-zero run stays zero
    c0, m0, s0 = O.nf4_double_quant_mean(np.zeros(5, np.float32), 256)
    assert c0.tolist() == [0] * 5 and m0[0] == 0 and s0[0] == 1.0
    assert np.all(O.nf4_absmax_mean_dequant(c0, m0, s0, 256) == 0)


@pytest.mark.parametrize("dq_group", [256, 64])
def test_meandq_bound_nearest_and_centring(dq_group):
    W = _rand_w(40, 4096 + 64, 51)
    W[3, :64] = 0.0                                   # one zero block
    a = O.nf4_absmax(W)
    c, mean, s2 = O.nf4_double_quant_mean(a, dq_group)
    back = O.nf4_absmax_mean_dequant(c, mean, s2, dq_group).astype(np.float64)
    run = np.arange(a.size) // dq_group
    s = s2.astype(np.float64)[run]
    # each code is the nearest of the 255 levels c * s2 to the residual
    d = (a - mean[run]).astype(np.float32).astype(np.float64)
    assert np.all(np.abs(c.astype(np.float64) - d / s) <= 0.5 + 1e-6)
    # reconstruction within half a level plus fp32 rounding of the steps
    amax = a.astype(np.float64).max()
    assert np.all(np.abs(back - a) <= s / 2 + 4 * amax * 2.0 ** -24)
    for r in range(mean.size):
        blk = a[r * dq_group:(r + 1) * dq_group].astype(np.float64)
        # the mean is the run's mean (against an exactly rounded sum)
        exact = math.fsum(blk) / blk.size
        assert abs(float(mean[r]) - exact) <= abs(exact) * 2.0 ** -23
        # residuals centred: they sum to ~0, the largest maps to +-127
        dr = d[r * dq_group:(r + 1) * dq_group]
        assert abs(dr.sum()) <= blk.size * abs(exact) * 2.0 ** -22
        assert np.abs(c[r * dq_group:(r + 1) * dq_group]).max() == 127


def test_meandq_keeps_the_4bit_codes_and_bounds_w_hat():
    # the second quantization touches only the constants: the 4-bit codes are
    # those of the plain scheme; the dequantized weight stays within half a
    # table gap of the block plus the constant's error and bf16 rounding
    W = _rand_w(24, 1024, 52)
    W[1, 64:128] = 0.0
    Wq_plain, _, _ = O.nf4_quantize(W)
    Wq, c, mean, s2 = O.nf4_quantize_meandq(W)
    assert np.array_equal(Wq, Wq_plain)
    what = O.bf16_bits_to_f32(O.nf4_dequant_meandq(Wq, c, mean, s2)).astype(np.float64)
    B = W.reshape(-1, 64).astype(np.float64)
    a = np.abs(B).max(axis=1, keepdims=True)
    back = O.nf4_absmax_mean_dequant(c, mean, s2)[:, None].astype(np.float64)
    half_gap = np.diff(O.nf4_table().astype(np.float64)).max() / 2
    err = np.abs(what.reshape(B.shape) - B)
    assert np.all(err <= a * half_gap + np.abs(back - a) + np.abs(B) * 2.0 ** -8 + 1e-12)
    assert np.all(what.reshape(B.shape)[(1 * 1024 + 64) // 64] == 0)   # the zero block


def test_planted_mistakes_meandq(monkeypatch):
    import oracle.w4_oracle as M
    checks = [test_meandq_worked_example,
              lambda: test_meandq_bound_nearest_and_centring(256),
              lambda: test_meandq_bound_nearest_and_centring(64)]

    def caught(name, fn):
        monkeypatch.setattr(M, name, fn)
        monkeypatch.setattr(O, name, fn)
        try:
            for chk in checks:
                try:
                    chk()
                except AssertionError:
                    return True
            return False
        finally:
            monkeypatch.undo()

    orig_dq = M.nf4_double_quant_mean
    orig_back = M.nf4_absmax_mean_dequant

    def no_centring(absmax, dq_group=256):          # plain symmetric 8-bit, mean 0
        a = np.asarray(absmax, np.float32)
        c, mean, s2 = orig_dq(a, dq_group)
        n = (a.size + dq_group - 1) // dq_group
        s = np.array([max(a[r * dq_group:(r + 1) * dq_group].max() / np.float32(127), 1e-30)
                      for r in range(n)], np.float32)
        cc = np.clip(np.rint(a / s[np.arange(a.size) // dq_group]), -127, 127).astype(np.int8)
        return cc, np.zeros(n, np.float32), s
    assert caught("nf4_double_quant_mean", no_centring)

    def global_mean(absmax, dq_group=256):          # one mean for every run
        a = np.asarray(absmax, np.float32)
        c, mean, s2 = orig_dq(a, dq_group)
        mu = np.float32(a.astype(np.float64).mean())
        d = (a - mu).astype(np.float32)
        run = np.arange(a.size) // dq_group
        s = np.array([np.abs(d[run == r]).max() / np.float32(127) for r in range(mean.size)],
                     np.float32)
        s[s == 0] = 1
        cc = np.clip(np.rint(d / s[run]), -127, 127).astype(np.int8)
        return cc, np.full(mean.size, mu, np.float32), s
    assert caught("nf4_double_quant_mean", global_mean)

    def over_255(absmax, dq_group=256):             # the unsigned 8-bit range
        c, mean, s2 = orig_dq(absmax, dq_group)
        s = (s2 * np.float32(127) / np.float32(255)).astype(np.float32)
        a = np.asarray(absmax, np.float32)
        run = np.arange(a.size) // dq_group
        cc = np.clip(np.rint((a - mean[run]) / s[run]), -127, 127).astype(np.int8)
        return cc, mean, s
    assert caught("nf4_double_quant_mean", over_255)

    def mean_dropped(c, mean, s2, dq_group=256):    # reconstruction without the mean
        return orig_back(c, np.zeros_like(np.asarray(mean, np.float32)), s2, dq_group)
    assert caught("nf4_absmax_mean_dequant", mean_dropped)


# ---------------------------------------------------------------- planted mistakes

# ---------------------------------------------------------------- FP4 (E2M1)

FP4_WORKED = _parse_worked(os.path.join(GOLDEN, "fp4_worked.txt"))


def test_fp4_table_is_e2m1():
    # the E2M1 magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6 (one sign, two
    # exponent, one mantissa bit); the table is them over 6, sign in bit 3
    T = O.fp4_table()
    assert T.dtype == np.float32 and T.shape == (16,)
    e2m1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(8):
        exact = Fraction(e2m1[c]) / 6
        assert abs(Fraction(float(T[c])) - exact) <= exact * Fraction(1, 2 ** 24)
        assert T[c + 8] == -T[c]
    assert np.signbit(T[8]) and T[8] == 0
    assert T[7] == 1.0 and T[15] == -1.0
    assert np.all(np.diff(T[:8]) > 0)
    # spacing doubles with each exponent step above the subnormal pair
    gaps = np.diff(T[:8].astype(np.float64)) * 6
    assert np.allclose(gaps, [0.5, 0.5, 0.5, 0.5, 1, 1, 2])


@pytest.mark.parametrize("case", FP4_WORKED, ids=lambda c: c["name"])
def test_fp4_worked_example(case):
    w = np.zeros((1, 64), np.float32)
    vals = [float(v) for v in case["w"]]
    w[0, :len(vals)] = vals
    Wq, c, s2 = O.fp4_quantize(w)
    codes = O.unpack_nibbles(Wq)[0]
    assert codes[:len(vals)].tolist() == [int(v) for v in case["codes"]]
    assert np.all(codes[len(vals):] == 0)
    assert Wq[0, :4].tolist() == [int(v, 16) for v in case["packed_hex"]]
    assert np.all(Wq[0, 4:] == 0)
    assert int(c[0]) == int(case["absmax_code"][0])
    what = O.bf16_bits_to_f32(O.fp4_dequant(Wq, c, s2))[0]
    assert what[:len(vals)].tolist() == [float(v) for v in case["what"]]


def test_fp4_brute_force_nearest_and_sign():
    W = _rand_w(16, 256, 45, sigma=1.0)
    W[0, :64] = 0.0                                   # zero block -> all code 0
    W[1, 1:64] = np.linspace(-1, 1, 63, dtype=np.float32) * np.float32(0.9)
    W[1, 0] = 1.0                                     # absmax 1: v = w exactly
    q = O.fp4_codes(W)
    assert np.all(q[0, :64] == 0)
    T = O.fp4_table().astype(np.float64)
    B = W.reshape(-1, 64)
    a = np.abs(B).max(axis=1)
    qb = q.reshape(-1, 64)
    for b in range(B.shape[0]):
        for k in range(64):
            if a[b] == 0:
                continue
            v = float(np.float32(B[b, k]) / np.float32(a[b]))
            dist = [abs(abs(v) - T[m]) for m in range(8)]
            best = min(dist)
            mag = min(m for m in range(8) if dist[m] - best <= 1e-15)   # lower on a tie
            want = mag + 8 if (v < 0 and mag > 0) else mag
            assert int(qb[b, k]) == want
    # negating W flips the sign bit of every nonzero magnitude
    qn = O.fp4_codes(-W)
    nz = (q & 7) > 0
    assert np.array_equal(qn[nz], q[nz] ^ 8) and np.array_equal(qn[~nz], q[~nz])


def test_fp4_dequant_error_bound():
    W = _rand_w(32, 512, 46)
    Wq, c, s2 = O.fp4_quantize(W)
    what = O.bf16_bits_to_f32(O.fp4_dequant(Wq, c, s2)).astype(np.float64)
    B = W.reshape(-1, 64).astype(np.float64)
    a = np.abs(B).max(axis=1, keepdims=True)
    s = s2.astype(np.float64)[np.arange(B.shape[0]) // 256][:, None]
    # largest half-gap of the table is (6 - 4) / 2 / 6 = 1/6 of the absmax;
    # the 8-bit absmax adds at most s2 / 2; bf16 rounding 2^-9 relative
    err = np.abs(what.reshape(B.shape) - B)
    assert np.all(err <= a / 6 + s / 2 + np.abs(B) * 2.0 ** -8 + 1e-12)
    # a weight at +-absmax comes back within the absmax quantization step
    top = np.abs(B).argmax(axis=1)
    wt = what.reshape(B.shape)[np.arange(B.shape[0]), top]
    bt = B[np.arange(B.shape[0]), top]
    assert np.all(np.abs(wt - bt) <= s[:, 0] / 2 + np.abs(bt) * 2.0 ** -8)


def test_planted_mistakes_fp4(monkeypatch):
    import oracle.w4_oracle as M
    checks = [test_fp4_table_is_e2m1, lambda: [test_fp4_worked_example(c) for c in FP4_WORKED],
              test_fp4_brute_force_nearest_and_sign]

    def caught(name, fn):
        monkeypatch.setattr(M, name, fn)
        monkeypatch.setattr(O, name, fn)
        try:
            for chk in checks:
                try:
                    chk()
                except AssertionError:
                    return True
            return False
        finally:
            monkeypatch.undo()

    orig_table = M.fp4_table

    def bias_off_by_one():                 # 2^e instead of 2^(e-1)
        T = orig_table() * np.float32(6)
        T = np.where(np.abs(T) >= 1, T * 2, T).astype(np.float32)
        return (T / np.float32(12)).astype(np.float32)
    assert caught("fp4_table", bias_off_by_one)

    orig_codes = M.fp4_codes

    def negative_zero_code(W, blocksize=64):  # sign bit set on zero magnitudes
        q = orig_codes(W, blocksize)
        neg = np.asarray(W, np.float32) < 0
        return np.where(neg, q | 8, q).astype(np.uint8)
    assert caught("fp4_codes", negative_zero_code)

    def ties_up(W, blocksize=64):             # upper magnitude on a midpoint
        B = M._blocks(W, blocksize)
        a = np.abs(B).max(axis=1)
        safe = np.where(a > 0, a, np.float32(1.0)).astype(np.float32)
        v = np.where(a[:, None] > 0, B / safe[:, None], np.float32(0.0)).astype(np.float32)
        mag = np.searchsorted(M.fp4_midpoints(), np.abs(v), side="right")
        q = np.where((v < 0) & (mag > 0), mag + 8, mag)
        return q.astype(np.uint8).reshape(np.shape(W))
    assert caught("fp4_codes", ties_up)


# ---------------------------------------------------------------- GPTQ

def _calib_h(K, n, seed, rank=4):
    # correlated synthetic calibration activations: noise plus a few shared factors
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, K)) + rng.standard_normal((n, rank)) @ rng.standard_normal((rank, K))
    return O.gptq_hessian(S.to_bf16_bits(x.astype(np.float32)))


def _rtn_code(w, s, z):
    return int(np.clip(np.rint(np.float32(w) / np.float32(s)) + z, 0, 15))


@pytest.mark.parametrize("act", [False, True])
def test_gptq_identity_hessian_is_rtn(act):
    # H = c I: the inverse Hessian has no off-diagonal entries, nothing is
    # spread, and (equal diagonal) act-order keeps the natural order
    W = _rand_w(24, 256, 47)
    q, s, z, gi = O.gptq_quantize(W, 3.5 * np.eye(256), 64, act)
    qr, sr, zr = O.quantize_rtn(W, 64)
    assert np.array_equal(q, qr) and np.array_equal(s, sr) and np.array_equal(z, zr)
    if act:
        assert np.array_equal(gi, np.arange(256) // 64)


def test_gptq_two_columns_closed_form():
    # K = 2, one group: column 0 is quantized as RTN; column 1 then carries
    # the value u minimising the 2x2 quadratic (e0, w1 - u) H' (e0, w1 - u)^T,
    # u = w1 + e0 * b' / c' for H' = [[a', b'], [b', c']] (damped), and is
    # quantized with the group's RTN parameters
    rng = np.random.default_rng(48)
    changed = 0
    for _ in range(200):
        w = rng.uniform(-1, 1, 2).astype(np.float32)
        a, c = rng.uniform(0.5, 2.0, 2)
        b = rng.uniform(-0.9, 0.9) * np.sqrt(a * c)
        H = np.array([[a, b], [b, c]])
        q, s, z, _ = O.gptq_quantize(w[None, :], H, 2)
        sr_, zr_ = O.rtn_params(w[None, :], 2)
        sf, zf = float(sr_[0, 0]), int(zr_[0, 0])
        assert s[0, 0] == sr_[0, 0] and z[0, 0] == zf
        q0 = _rtn_code(w[0], sf, zf)
        e0 = float(w[0]) - float(np.float32((q0 - zf) * np.float32(sf)))
        lam = 0.01 * (a + c) / 2
        u = float(w[1]) + e0 * b / (c + lam)
        assert q[0, 0] == q0 and q[0, 1] == _rtn_code(u, sf, zf)
        changed += q[0, 1] != _rtn_code(w[1], sf, zf)
    assert changed > 3           # the compensation does move codes


def test_gptq_elimination_is_inverse_of_remaining_block():
    rng = np.random.default_rng(49)
    A = rng.standard_normal((12, 12))
    H = A @ A.T + 12 * np.eye(12)
    Hi = np.linalg.inv(H)
    for j in range(3):
        Hi = O.gptq_eliminate(Hi, 0)
        assert np.allclose(Hi, np.linalg.inv(H[j + 1:, j + 1:]), rtol=1e-10, atol=1e-12)


def test_gptq_lowers_layer_error_and_handles_dead_channels():
    K, N, G = 256, 32, 32
    H = _calib_h(K, 384, 50)
    H[7, :] = 0.0
    H[:, 7] = 0.0                       # channel 7 never activated
    W = _rand_w(N, K, 51)
    for act in (False, True):
        q, s, z, gi = O.gptq_quantize(W, H, G, act)
        gk = O.group_index(K, G, gi)
        assert q.max() <= 15
        # dead channel: weight treated as 0 -> code = zero point -> w_hat = 0
        assert np.array_equal(q[:, 7], z[np.arange(N), gk[7]])
        what = O.dequant_rtn(O.pack_nibbles(q), s, z, G, gi)
        assert np.all(what[:, 7] == 0)
        qr, sr, zr = O.quantize_rtn(W, G)
        Wl = W.copy()
        Wl[:, 7] = 0.0
        l_g = O.gptq_loss(Wl, what, H)
        l_r = O.gptq_loss(Wl, O.dequant_rtn(O.pack_nibbles(qr), sr, zr, G), H)
        assert l_g < 0.5 * l_r
        if act:
            # processing order: decreasing diag(H), each group exactly G channels
            d = np.diag(H).copy()
            d[7] = 1.0
            ng = K // G
            assert all(d[gi == g].min() >= d[gi == g + 1].max() for g in range(ng - 1))
            assert np.all(np.bincount(gi) == G)


def test_planted_mistakes_gptq(monkeypatch):
    import oracle.w4_oracle as M
    checks = [test_gptq_two_columns_closed_form,
              test_gptq_lowers_layer_error_and_handles_dead_channels,
              test_gptq_elimination_is_inverse_of_remaining_block]

    def caught(name, fn):
        monkeypatch.setattr(M, name, fn)
        monkeypatch.setattr(O, name, fn)
        try:
            for chk in checks:
                try:
                    chk()
                except (AssertionError, np.linalg.LinAlgError):
                    return True
            return False
        finally:
            monkeypatch.undo()

    def no_elimination(Hi, j):                # keep the first inverse: drop the row/col only
        return Hi[j + 1:, j + 1:].copy()
    assert caught("gptq_eliminate", no_elimination)

    def elim_sign(Hi, j):                     # + instead of -
        r = Hi[j, j + 1:]
        return Hi[j + 1:, j + 1:] + np.outer(Hi[j + 1:, j], r) / Hi[j, j]
    assert caught("gptq_eliminate", elim_sign)

    orig_prep = M.gptq_prepare

    def undamped_as_hessian(H, act_order, damp=0.01):   # H where H^-1 belongs
        Hp, perm, dead = orig_prep(H, act_order, damp)
        return np.linalg.inv(Hp), perm, dead
    assert caught("gptq_prepare", undamped_as_hessian)


# ---------------------------------------------------------------- LLM.int8

INT8_WORKED = _parse_worked(os.path.join(GOLDEN, "int8_mixed_worked.txt"))


@pytest.mark.parametrize("case", INT8_WORKED, ids=lambda c: c["name"])
def test_int8_worked_example(case):
    f = lambda key: np.array([float(v) for v in case[key]], np.float32)
    xb = S.to_bf16_bits(f("x")[None, :])
    W = np.stack([f("w0"), f("w1")])
    qw, sw = O.int8_quantize_weights(W)
    assert qw[0].tolist() == [int(v) for v in case["qw0"]] and np.all(qw[1] == 0)
    assert sw.tolist() == [float(v) for v in case["sw"]]
    Ol = O.int8_outliers(xb)
    assert np.flatnonzero(Ol).tolist() == [int(v) for v in case["outliers"]]
    qx, sx = O.int8_quantize_activations(xb, Ol)
    assert qx[0].tolist() == [int(v) for v in case["qx"]]
    assert sx.tolist() == [float(v) for v in case["sx"]]
    y, _ = O.int8_mixed_ref(xb, qw, sw)
    assert y[0].tolist() == [float(v) for v in case["y"]]


def test_int8_threshold_is_strict_and_all_outliers_is_16bit():
    xb = S.to_bf16_bits(np.array([[6.0, -6.0, 6.03125, 1.0]], np.float32))
    assert np.flatnonzero(O.int8_outliers(xb)).tolist() == [2]
    # every channel an outlier: the INT8 part vanishes, y = x . bf16(q_w s_w)
    W = _rand_w(8, 64, 52)
    xb = S.draw_x(3, 64, seed=5)
    qw, sw = O.int8_quantize_weights(W)
    y, _ = O.int8_mixed_ref(xb, qw, sw, threshold=0.0)
    w16 = O.bf16_bits_to_f64(O.bf16_round_bits((qw.astype(np.float32) * sw[:, None]).astype(np.float32)))
    assert np.allclose(y, O.bf16_bits_to_f64(xb) @ w16.T, rtol=1e-12, atol=0)


def test_int8_error_bound_against_exact_product():
    # |y - x W| <= sum_k |x| s_w / 2 + |w| s_x / 2 + s_x s_w / 4 over the INT8
    # channels, plus the outlier channels' bf16 weight rounding
    W = _rand_w(32, 1024, 53)
    xb = S.draw_x(5, 1024, seed=6, outlier_frac=0.005, outlier_scale=40.0)
    qw, sw = O.int8_quantize_weights(W)
    y, _ = O.int8_mixed_ref(xb, qw, sw)
    x = O.bf16_bits_to_f64(xb)
    Ol = O.int8_outliers(xb)
    assert Ol.sum() >= 3
    _, sx = O.int8_quantize_activations(xb, Ol)
    Wd = W.astype(np.float64)
    keep = ~Ol
    b = (np.abs(x[:, keep]) @ np.ones((keep.sum(), 1))) * sw[None, :] / 2 \
        + sx[:, None].astype(np.float64) * (np.abs(Wd[:, keep]).sum(axis=1)[None, :] / 2) \
        + keep.sum() * sx[:, None] * sw[None, :] / 4
    b += np.abs(x[:, Ol]) @ (np.abs(Wd[:, Ol]).T * (2.0 ** -8) + sw[None, :] / 2)
    assert np.all(np.abs(y - x @ Wd.T) <= b * 1.0001)


def test_planted_mistakes_int8(monkeypatch):
    import oracle.w4_oracle as M
    checks = [lambda: [test_int8_worked_example(c) for c in INT8_WORKED],
              test_int8_threshold_is_strict_and_all_outliers_is_16bit,
              test_int8_error_bound_against_exact_product]

    def caught(name, fn):
        monkeypatch.setattr(M, name, fn)
        monkeypatch.setattr(O, name, fn)
        try:
            for chk in checks:
                try:
                    chk()
                except AssertionError:
                    return True
            return False
        finally:
            monkeypatch.undo()

    def per_column_scale(W):                  # one scale per input channel
        W = np.ascontiguousarray(W, np.float32)
        s = (np.abs(W).max(axis=0) / np.float32(127.0)).astype(np.float32)
        s[s == 0] = np.float32(1.0)
        q = np.clip(np.rint(W / s[None, :]), -127, 127).astype(np.int8)
        return q, np.ones(W.shape[0], np.float32) * s.mean()
    assert caught("int8_quantize_weights", per_column_scale)

    def inclusive(x_bits, threshold=6.0):    # >= instead of >
        return np.any(np.abs(M.bf16_bits_to_f32(x_bits)) >= np.float32(threshold), axis=0)
    assert caught("int8_outliers", inclusive)

    orig_qa = M.int8_quantize_activations

    def outliers_counted_twice(x_bits, outliers):
        q, s = orig_qa(x_bits, np.zeros_like(np.asarray(outliers, bool)))
        return q, s
    assert caught("int8_quantize_activations", outliers_counted_twice)


def _pins_fail(monkeypatch, name, fn):
    """Replace one oracle function by a mutated copy and report whether any
    of the core pins catches it."""
    import oracle.w4_oracle as M
    monkeypatch.setattr(M, name, fn)
    monkeypatch.setattr(O, name, fn)
    checks = [
        lambda: [test_int4_worked_examples(c) for c in WORKED],
        lambda: test_int4_codes_and_error_bound(32),
        lambda: test_nf4_codes_brute_force_nearest(),
        lambda: test_nf4_double_quant_bound_and_zero_block(),
    ]
    for chk in checks:
        try:
            chk()
        except AssertionError:
            return True
    return False


def test_planted_mistakes(monkeypatch):
    import oracle.w4_oracle as M
    orig_pack = M.pack_nibbles

    def swapped_nibbles(codes):
        p = orig_pack(codes)
        return ((p >> 4) | (p << 4)).astype(np.uint8)
    assert _pins_fail(monkeypatch, "pack_nibbles", swapped_nibbles)
    monkeypatch.undo()

    orig_round = M.bf16_round_bits

    def truncating(f):
        return (np.ascontiguousarray(f, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert _pins_fail(monkeypatch, "bf16_round_bits", truncating)
    monkeypatch.undo()
    assert M.bf16_round_bits is orig_round

    def half_up_quant(W, G, g_idx=None):
        W = np.ascontiguousarray(W, np.float32)
        gk = M.group_index(W.shape[1], G, g_idx)
        s16, zp = M.rtn_params(W, G, g_idx)
        sk = s16.astype(np.float32)[:, gk]
        q = np.clip(np.floor(W / sk + np.float32(0.5)) + zp.astype(np.float32)[:, gk], 0, 15)
        return q.astype(np.uint8), s16, zp
    assert _pins_fail(monkeypatch, "quantize_rtn", half_up_quant)
    monkeypatch.undo()

    def zero_sign_flipped(W, G, g_idx=None):
        s16, zp = rtn_orig(W, G, g_idx)
        return s16, np.clip(15 - zp.astype(np.int32), 0, 15).astype(np.uint8)
    rtn_orig = M.rtn_params
    assert _pins_fail(monkeypatch, "rtn_params", zero_sign_flipped)
    monkeypatch.undo()

    orig_dq = M.nf4_double_quant

    def dq_truncating(absmax, dq_group=256):
        c, s2 = orig_dq(absmax, dq_group)
        a = np.asarray(absmax, np.float32)
        s = s2[np.arange(a.size) // dq_group]
        return np.floor(a / s).astype(np.uint8), s2
    assert _pins_fail(monkeypatch, "nf4_double_quant", dq_truncating)
    monkeypatch.undo()


def test_planted_mistakes_sym_and_awq(monkeypatch):
    import oracle.w4_oracle as M

    def caught(name, fn, checks):
        monkeypatch.setattr(M, name, fn)
        monkeypatch.setattr(O, name, fn)
        try:
            for chk in checks:
                try:
                    chk()
                except AssertionError:
                    return True
            return False
        finally:
            monkeypatch.undo()

    sym_checks = [
        lambda: [test_sym_worked_examples(c) for c in SYM_WORKED],
        lambda: test_sym_bound_symmetry_and_nearest_level(32),
        test_sym_page_worked_example,
    ]
    orig_params = M.sym_params

    def over_eight(W, G, g_idx=None, bits=4):      # 2^(b-1) instead of 2^(b-1) - 1
        s32, _ = orig_params(W, G, g_idx, bits)
        q = 2.0 ** (bits - 1)
        s32 = (s32 * np.float32(2 ** (bits - 1) - 1) / np.float32(q)).astype(np.float32)
        s16 = s32.astype(np.float16)
        s16[s16 == 0] = np.float16(1.0)
        return s32, s16
    assert caught("sym_params", over_eight, sym_checks)

    def signed_max(W, G, g_idx=None, bits=4):      # max(w) instead of max|w|
        W = np.ascontiguousarray(W, np.float32)
        gk = M.group_index(W.shape[1], G, g_idx)
        _, mx = M._group_minmax(W, G, gk, g_idx is None)
        s32 = (mx / np.float32(2 ** (bits - 1) - 1)).astype(np.float32)
        s16 = s32.astype(np.float16)
        s16[s16 == 0] = np.float16(1.0)
        return s32, s16
    assert caught("sym_params", signed_max, sym_checks)

    def sym_floor(W, G, g_idx=None):
        W = np.ascontiguousarray(W, np.float32)
        gk = M.group_index(W.shape[1], G, g_idx)
        _, s16 = M.sym_params(W, G, g_idx, 4)
        q = np.clip(np.floor(W / s16.astype(np.float32)[:, gk] + np.float32(0.5)), -7, 7) + 8
        return q.astype(np.uint8), s16, np.full(s16.shape, 8, np.uint8)
    assert caught("quantize_sym", sym_floor, sym_checks)

    awq_checks = [test_awq_identity_and_powers_of_two, test_awq_product_invariance,
                  test_awq_effective_weight_follows_page_formula]

    def x_times_s(x_bits, s):
        x = M.bf16_bits_to_f32(x_bits)
        return M.bf16_round_bits((x * np.asarray(s, np.float32)[None, :]).astype(np.float32))
    assert caught("awq_scale_activations", x_times_s, awq_checks)

    def w_over_s(W, s):
        return (np.asarray(W, np.float32) / np.asarray(s, np.float32)[None, :]).astype(np.float32)
    assert caught("awq_scale_weights", w_over_s, awq_checks)
