"""Host-side replay of the tensor-core GEMM's work split (no GPU needed).

The planner (csrc/w4_gemm_host.inc, make_plan) picks the token tile, whether
256-token tiles run on CTA pairs, and the K split: uniform `splits`, or the
first head_tiles work tiles whole and the rest in tail_splits K ranges.  The
kernel (csrc/w4_gemm_kernel.cuh) maps blockIdx.x to (token tile, 128-row
tile, K range, partial slot, arrival counter).  Both are re-derived here; the
planner copy is pinned to the library through w4_workspace_bytes (which
encodes the partial-slot count), and the decode copy is checked to cover
every (token tile, row tile, K stage) exactly once with both CTAs of a pair
on the same token tile and K range, partial slots and counters in bounds.
On a host without a GPU the library plans for 148 SMs."""
import pytest

from weight_only_bit_gemm_b200 import build

build.build()
from weight_only_bit_gemm_b200 import w4  # noqa: E402

SMS = 148
COUNTERS = 65536          # arrival counters at the start of every workspace
X_GROUP_BYTES = 48 << 20  # L2 budget of one group of token tiles


def ceil_div(a, b):
    return -(-a // b)


def plan(M, N, K):
    """make_plan for M > 32 (tcgen05 path), without act-order."""
    tiles_n, KS = ceil_div(N, 128), ceil_div(K, 128)
    MT = 64 if M <= 64 else 128 if M <= 128 else 256
    tiles_m = ceil_div(M, MT)
    pair = MT == 256 and tiles_n % 2 == 0
    unit = 2 if pair else 1
    slots_at_once = SMS // unit
    base = (tiles_n // unit) * tiles_m
    max_s = 1 if base * unit > COUNTERS else min(KS, 64)

    def split_cost(s):
        return max(12.0, 4.0 + 0.5 * (MT / 16) * ((s + 3) // 4))

    best, splits = 1e30, 1
    for s in range(1, max_s + 1):
        cost = ceil_div(base * s, slots_at_once) * (ceil_div(KS, s) + 1.5 +
                                                    (split_cost(s) if s > 1 else 0.0))
        if cost < best - 1e-9:
            best, splits = cost, s
    head = tail = 0
    if base > slots_at_once:
        waves, rem = divmod(base, slots_at_once)
        smax = min(slots_at_once // rem if rem else 0, KS // 4, 16)
        for st in range(2, smax + 1):
            cost = waves * (KS + 1.5) + (ceil_div(KS, st) + 1.5 + split_cost(st))
            if cost < best - 1e-9:
                best, splits, head, tail = cost, 1, waves * slots_at_once, st
    slots = ((base - head) * tail if tail else (base * splits if splits > 1 else 0)) * unit
    group_m = max(1, min(tiles_m, X_GROUP_BYTES // (MT * K * 2)))
    work_n = tiles_n // unit
    grid = unit * (head + (work_n * tiles_m - head) * tail if tail else work_n * splits * tiles_m)
    return dict(tiles_n=tiles_n, KS=KS, MT=MT, tiles_m=tiles_m, pair=pair, splits=splits,
                head=head, tail=tail, slots=slots, group_m=group_m, grid=grid)


def decode(P, bx):
    """The kernel's blockIdx.x -> (token tile, row tile, K range, slot, counter)."""
    pair = P["pair"]
    rank = bx & 1 if pair else 0
    b = bx >> 1 if pair else bx
    tn = P["tiles_n"] >> 1 if pair else P["tiles_n"]
    ns = tn * P["splits"] if P["tail"] == 0 else tn
    lt = b
    if P["tail"] == 0:
        nsplit = P["splits"]
    elif b < P["head"]:
        nsplit = 1
    else:
        nsplit = P["tail"]
        lt = P["head"] + (b - P["head"]) // nsplit
    gsize = P["group_m"] * ns
    grp = lt // gsize
    gm = min(P["group_m"], P["tiles_m"] - grp * P["group_m"])
    lin = lt - grp * gsize
    mtile, nts = grp * P["group_m"] + lin % gm, lin // gm
    if P["tail"] == 0:
        nt, split = nts // nsplit, nts % nsplit
        if pair:
            nt = 2 * nt + rank
        cidx = mtile * P["tiles_n"] + nt
    else:
        nt = 2 * nts + rank if pair else nts
        split = 0 if b < P["head"] else (b - P["head"]) % nsplit
        cidx = 2 * (lt - P["head"]) + rank if pair else lt - P["head"]
    s0 = split * P["KS"] // nsplit
    s1 = (split + 1) * P["KS"] // nsplit
    return mtile, nt, split, nsplit, cidx, cidx * nsplit, s0, s1


SHAPES = [(M, N, K) for M in (40, 100, 129, 256, 300, 520, 2048, 8192)
          for (N, K) in ((8192, 28672), (28672, 8192), (4096, 4096), (22016, 4096),
                         (4096, 11008), (256, 128), (19000, 2560), (9728, 4096),
                         (13824, 5120), (5120, 13824), (384, 1024))]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_planner_copy_matches_library(M, N, K):
    P = plan(M, N, K)
    want = COUNTERS * 4 + ceil_div(P["slots"] * P["MT"] * 128 * 4, 256) * 256
    assert w4.workspace_bytes(M, N, K, 128, False) == want


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_work_decode_covers_each_tile_stage_once(M, N, K):
    P = plan(M, N, K)
    if P["pair"]:
        assert P["grid"] % 2 == 0
    floats = P["slots"] * P["MT"] * 128
    seen = set()
    for bx in range(P["grid"]):
        mt, nt, sp, ns, cidx, pbase, s0, s1 = decode(P, bx)
        assert 0 <= mt < P["tiles_m"] and 0 <= nt < P["tiles_n"] and s0 < s1
        if P["pair"] and bx & 1:
            prev = decode(P, bx - 1)
            assert (prev[0], prev[1] + 1, prev[2], prev[3], prev[6], prev[7]) == \
                (mt, nt, sp, ns, s0, s1)
        for k in range(s0, s1):
            assert (mt, nt, k) not in seen
            seen.add((mt, nt, k))
        if ns > 1:
            assert 0 <= cidx < COUNTERS
            assert (pbase + sp + 1) * P["MT"] * 128 <= floats
    assert len(seen) == P["tiles_m"] * P["tiles_n"] * P["KS"]


def test_pairs_where_expected():
    assert plan(2048, 8192, 28672)["pair"] and plan(512, 28672, 8192)["pair"]
    assert not plan(300, 9550, 2560)["pair"]      # 75 row tiles: single CTAs
    assert not plan(100, 8192, 4096)["pair"]      # 128-token tiles
