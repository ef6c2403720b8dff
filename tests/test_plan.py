"""Work partitioning of the two attention kernels (host logic, no GPU).

Replays, in Python, the integer arithmetic by which the kernels turn a plan
(alspec_query_plan / alspec_query_chunks) into tiles of cache rows, and checks
that for every (sequence, KV head) each cache row [0, L) is read exactly once:
by the sink-set kernel when it is one of the first S or last W rows, by the
exact-path kernel otherwise.  Also checks the completion counts the kernels
use for their tickets.
"""
import random

import pytest

import speculative_flash_decoding_b200 as sfd
from speculative_flash_decoding_b200 import alspec as ab


def cdiv(a, b):
    return (a + b - 1) // b


def geom(L, S, W):
    ns = min(S, L)
    ws = max(ns, L - W)
    return ns, ws


def tiles_of(B, Hq, Hkv, d, Lmax, dtype, S, W, lens, split=0, engine="auto"):
    desc = sfd.make_desc(B, Hq, Hkv, d, Lmax, dtype, split, 0, engine)
    st, plan = sfd.alspec_query_plan(desc, S, W)
    assert st == 0
    st, fq, TT = sfd.alspec_query_chunks(desc, S, W)
    assert st == 0 and len(fq) == plan["n2"] + 1 and TT == (32 if plan["engine"] == 2 else 16)
    assert fq[0] == 0 and (plan["n2"] == 0 or fq[-1] == 1 << 24)
    assert all(a <= b for a, b in zip(fq, fq[1:]))
    c1, n1, n2 = plan["c1"], plan["n1"], plan["n2"]
    assert c1 % TT == 0
    seen = {}
    pieces = {}
    for spec in (True, False):
        per = n1 if spec else n2
        for item in range(B * Hkv * per):
            # Sink-set CTAs of one head are consecutive (one cluster); middle
            # items are chunk-major across heads.
            if spec:
                bh, chunk = item // n1, item % n1
            else:
                bh, chunk = item % (B * Hkv), item // (B * Hkv)
            b, kvh = bh // Hkv, bh % Hkv
            L = lens[b]
            ns, ws = geom(L, S, W)
            tiles = []
            if spec:
                tpi = c1 // TT
                t0 = chunk * tpi
                T = cdiv(ns, TT) + cdiv(L - ws, TT)
                for t in range(t0, min(t0 + tpi, T)):
                    tsink = cdiv(ns, TT)
                    if t < tsink:
                        start = t * TT
                        nvalid = min(TT, ns - start)
                    else:
                        start = ws + (t - tsink) * TT
                        nvalid = min(TT, L - start)
                    tiles.append((start, nvalid))
            else:
                mt = cdiv(ws - ns, TT)
                tlo, thi = (mt * fq[chunk]) >> 24, (mt * fq[chunk + 1]) >> 24
                lo, hi = ns + tlo * TT, min(ns + thi * TT, ws)
                for t in range(max(0, thi - tlo)):
                    tiles.append((lo + t * TT, min(TT, hi - lo - t * TT)))
            if tiles and not spec:
                pieces[(b, kvh)] = pieces.get((b, kvh), 0) + 1
            for start, nvalid in tiles:
                assert 1 <= nvalid <= TT and 0 <= start and start + nvalid <= L
                row = (b * Hkv + kvh) * Lmax + start
                assert 0 <= row < 2 ** 31
                for j in range(start, start + nvalid):
                    assert (b, kvh, j) not in seen, ("read twice", b, kvh, j)
                    seen[(b, kvh, j)] = spec
    for b in range(B):
        L = lens[b]
        ns, ws = geom(L, S, W)
        mt = cdiv(ws - ns, TT)
        nonempty = sum(1 for c in range(n2) if (mt * fq[c + 1]) >> 24 > (mt * fq[c]) >> 24)
        for kvh in range(Hkv):
            # The completion ticket of (b, kvh) expects 1 + nonempty pieces.
            assert pieces.get((b, kvh), 0) == nonempty
            for j in range(L):
                assert (b, kvh, j) in seen, ("never read", b, kvh, j)
                assert seen[(b, kvh, j)] == (j < S or j >= L - W)
    return plan


CASES = [
    # B, Hq, Hkv, d, Lmax, dtype, S, W
    (1, 4, 1, 64, 1024, "f32", 4, 128),
    (1, 32, 8, 128, 8197, "bf16", 4, 1024),
    (8, 32, 8, 128, 9000, "bf16", 4, 512),
    (4, 64, 8, 128, 8199, "bf16", 4, 1024),
    (5, 8, 2, 64, 777, "bf16", 40, 70),
    (3, 4, 4, 128, 300, "f32", 0, 16),
    (3, 4, 4, 128, 300, "bf16", 7, 0),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("engine", ["auto", "cuda_cores"])
def test_every_row_read_exactly_once(case, engine):
    B, Hq, Hkv, d, Lmax, dtype, S, W = case
    rng = random.Random(hash(case) & 0xffff)
    for _ in range(3):
        lens = [rng.randint(1, Lmax) for _ in range(B)]
        lens[0] = Lmax
        tiles_of(B, Hq, Hkv, d, Lmax, dtype, S, W, lens, engine=engine)


@pytest.mark.parametrize("split", [16, 112, 1024, 100000])
def test_fixed_split_sizes(split):
    tiles_of(8, 32, 8, 128, 9000, "bf16", 4, 512, [9000, 2000, 4500, 1, 3000, 8999, 530, 6000],
             split=split)


def test_guided_chunks_shrink_and_fill_the_grid():
    desc = sfd.make_desc(1, 32, 8, 128, 131072, "bf16")
    st, plan = sfd.alspec_query_plan(desc, 4, 1024)
    st2, fq, TT = sfd.alspec_query_chunks(desc, 4, 1024)
    assert st == st2 == 0
    sizes = [b - a for a, b in zip(fq, fq[1:])]
    assert sizes[0] >= sizes[-1] * 4          # large chunks first, small at the end
    assert all(x >= y - 2 for x, y in zip(sizes, sizes[1:]))  # non-increasing (rounding)
    # The sink-set kernel runs as a cluster of a few CTAs per head (8 heads
    # here) within half of the GPU; the middle kernel takes every SM.
    assert 1 < plan["n1"] <= 8 and 8 * plan["n1"] <= 74 and plan["grid2"] == 148


def test_query_chunks_rejects_small_buffer():
    desc = sfd.make_desc(1, 32, 8, 128, 131072, "bf16")
    import ctypes
    fq = (ctypes.c_uint32 * 2)()
    n2, tile = ctypes.c_int(0), ctypes.c_int(0)
    st = ab._lib.alspec_query_chunks(ctypes.byref(desc), 4, 1024, fq, 2, ctypes.byref(n2),
                                     ctypes.byref(tile))
    assert st == ab.ALSPEC_ERR_INVALID_ARG
