"""Work partitioning of the two attention kernels (host logic, no GPU).

Replays, in Python, the integer arithmetic by which the kernels turn a plan
(alspec_query_plan / alspec_query_chunks) into tiles of cache rows, and checks
that for every (sequence, KV head) each cache row [0, L) is read exactly once:
by a sink-set item when it is one of the first S or last W rows, by an
exact-path item otherwise -- for both schedules (two streams: separate
kernels; one launch: one queue, sink-set items first).  Also checks the
completion counts the kernels use for their tickets.
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


def decode_index(item, B, Hkv, n1, n2, fused):
    """(is sink-set item, (b, kv head) index, chunk) of a queue index."""
    heads = B * Hkv
    if fused:
        if item < heads * n1:
            return True, item // n1, item % n1
        item -= heads * n1
        return False, item % heads, item // heads
    raise AssertionError("two-stream indices are per kernel")


def tiles_of(B, Hq, Hkv, d, Lmax, dtype, S, W, lens, split=0, engine="auto", schedule="auto"):
    desc = sfd.make_desc(B, Hq, Hkv, d, Lmax, dtype, split, 0, engine, schedule)
    st, plan = sfd.alspec_query_plan(desc, S, W)
    assert st == 0
    fused = plan["schedule"] == ab.ALSPEC_SCHEDULE_FUSED
    assert fused == (schedule == "fused")
    st, fq, TT = sfd.alspec_query_chunks(desc, S, W)
    assert st == 0 and len(fq) == plan["n2"] + 1 and TT == (32 if plan["engine"] == 2 else 16)
    assert fq[0] == 0 and (plan["n2"] == 0 or fq[-1] == 1 << 24)
    assert all(a <= b for a, b in zip(fq, fq[1:]))
    c1, n1, n2 = plan["c1"], plan["n1"], plan["n2"]
    assert c1 % TT == 0
    seen = {}
    pieces = {}
    spec_tile_sum, mid_tile_sum, spec_items = {}, {}, {}
    if fused:
        # One queue: B * Hkv * n1 sink-set items, then the middle items.
        queue = [decode_index(i, B, Hkv, n1, n2, True) for i in range(B * Hkv * (n1 + n2))]
        assert plan["grid2"] == min(148, len(queue))
    else:
        # Sink-set CTAs of one head are consecutive (one cluster); middle
        # items are chunk-major across heads.
        queue = [(True, i // n1, i % n1) for i in range(B * Hkv * n1)]
        queue += [(False, i % (B * Hkv), i // (B * Hkv)) for i in range(B * Hkv * n2)]
    for spec, bh, chunk in queue:
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
        # Tile tickets of the one-launch schedule: each item adds its
        # tile count (items without tiles never reach a consumer).
        acc = spec_tile_sum if spec else mid_tile_sum
        acc[(b, kvh)] = acc.get((b, kvh), 0) + len(tiles)
        if tiles and spec:
            spec_items.setdefault((b, kvh), []).append(chunk)
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
        T = cdiv(ns, TT) + cdiv(L - ws, TT)
        for kvh in range(Hkv):
            # The completion ticket of (b, kvh) expects 1 + nonempty pieces.
            assert pieces.get((b, kvh), 0) == nonempty
            # One launch: the sink-set ticket completes at the sink set's
            # tile count, the head ticket at the middle's plus one; the
            # items with rows are exactly the first cdiv(T, tiles per item).
            assert spec_tile_sum.get((b, kvh), 0) == T
            assert mid_tile_sum.get((b, kvh), 0) == mt
            assert sorted(spec_items[(b, kvh)]) == list(range(cdiv(T, c1 // TT)))
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
@pytest.mark.parametrize("schedule", ["streams", "fused", "sink_first"])
def test_every_row_read_exactly_once(case, engine, schedule):
    B, Hq, Hkv, d, Lmax, dtype, S, W = case
    rng = random.Random(hash(case) & 0xffff)
    for _ in range(3):
        lens = [rng.randint(1, Lmax) for _ in range(B)]
        lens[0] = Lmax
        tiles_of(B, Hq, Hkv, d, Lmax, dtype, S, W, lens, engine=engine, schedule=schedule)


def test_sink_first_plan_takes_every_sm_for_the_sink_set():
    """SINK_FIRST runs the sink-set kernel alone, so its clusters may cover
    every SM; the concurrent schedule keeps them within 3/4 of the SMs."""
    for B, Hkv, W in [(8, 8, 2048), (4, 8, 4096), (1, 8, 1024)]:
        plans = {}
        for sch in ("streams", "sink_first"):
            desc = sfd.make_desc(B, 4 * Hkv, Hkv, 128, 65536, "bf16", schedule=sch)
            st, plans[sch] = sfd.alspec_query_plan(desc, 4, W)
            assert st == 0
        assert plans["sink_first"]["schedule"] == ab.ALSPEC_SCHEDULE_SINK_FIRST
        heads = B * Hkv
        assert plans["streams"]["n1"] * heads <= 148 * 3 // 4
        assert plans["sink_first"]["n1"] * heads <= 148
        assert plans["sink_first"]["n1"] >= plans["streams"]["n1"]
        assert plans["sink_first"]["n2"] == plans["streams"]["n2"]


@pytest.mark.parametrize("split", [16, 112, 1024, 100000])
@pytest.mark.parametrize("schedule", ["streams", "fused"])
def test_fixed_split_sizes(split, schedule):
    tiles_of(8, 32, 8, 128, 9000, "bf16", 4, 512, [9000, 2000, 4500, 1, 3000, 8999, 530, 6000],
             split=split, schedule=schedule)


def test_fused_plan_shapes():
    """One launch: at most one sink-set item per 4 tiles, about one per CTA of the first wave."""
    for B, Hkv, L, W, want_n1 in [(1, 8, 131072, 1024, 9), (8, 8, 65536, 2048, 2),
                                  (4, 8, 131072, 4096, 4), (1, 1, 1024, 128, 2)]:
        desc = sfd.make_desc(B, 8 * Hkv if Hkv == 8 else 4, Hkv, 128 if Hkv == 8 else 64, L,
                             "bf16", schedule="fused")
        st, plan = sfd.alspec_query_plan(desc, 4, W)
        assert st == 0 and plan["schedule"] == ab.ALSPEC_SCHEDULE_FUSED
        assert plan["n1"] == want_n1, (B, Hkv, L, W, plan)
        tiles = cdiv(4, 32) + cdiv(W, 32)
        assert plan["n1"] <= cdiv(tiles, 4)
        assert plan["c1"] // 32 * plan["n1"] >= tiles


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


@pytest.mark.parametrize("shape", [(1, 32, 8, 128, 131072, 4, 1024), (1, 32, 8, 128, 32768, 4, 1024),
                                   (8, 32, 8, 128, 65536, 4, 2048), (4, 64, 8, 128, 131072, 4, 4096),
                                   (1, 4, 1, 64, 1024, 4, 128), (64, 32, 8, 128, 4096, 4, 64)])
def test_sink_set_ctas_and_middle_grid(shape):
    """The sink-set kernel has n1 CTAs (one cluster) per (sequence, KV head),
    together within 3/4 of the SMs unless one per head already exceeds it
    (all SMs with SINK_FIRST); the persistent middle kernel takes every SM
    (148 without a GPU), or one CTA per item when there are fewer."""
    import speculative_flash_decoding_b200 as sfd
    B, Hq, Hkv, d, L, S, W = shape
    sms = 148
    tiles = -(-min(S, L) // 32) + -(-min(W, L) // 32)
    heads = B * Hkv
    n1_of = {}
    for sched in ("streams", "sink_first", "auto"):
        desc = sfd.make_desc(B, Hq, Hkv, d, L, "bf16", schedule=sched)
        st, plan = sfd.alspec_query_plan(desc, S, W)
        assert st == 0
        assert plan["grid1"] == heads * plan["n1"]
        share = sms if sched in ("sink_first", "auto") else sms * 3 // 4
        assert plan["n1"] == 1 or plan["grid1"] <= share
        if plan["n2"]:
            assert plan["grid2"] == min(sms, heads * plan["n2"])
        n1_of[sched] = plan["n1"]
    # The automatic schedule widens the sink set only when 3/4 of the SMs
    # would leave a sink-set CTA more than 24 tiles.
    per_cta = -(-tiles // n1_of["streams"])
    if per_cta > 24:
        assert n1_of["auto"] >= n1_of["streams"]
        assert n1_of["auto"] == max(1, min(8, sms // heads, -(-tiles // 5)))
    else:
        assert n1_of["auto"] == n1_of["streams"]
