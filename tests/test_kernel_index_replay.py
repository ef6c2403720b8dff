"""Index arithmetic of two warp-parallel steps in the kernels, replayed in
Python on the CPU (host logic, no GPU):

* the ring's first fill on the tensor-core engine (fill_fresh): lane l of the
  producer warp issues copy l % OPS of stage l / OPS in rounds of 32 / OPS
  stages.  Every (stage, copy) pair is issued exactly once, every stage's
  expected bytes are set once (by its copy-0 lane, before the copies of its
  round), and in each round a lower stage's copies all come from lower lanes
  than a higher stage's (one copy instruction issues lanes in order, so
  stage 0 leaves first);
* the merge kernel's list of non-empty middle chunks (warp 0, 32 chunks per
  ballot): equal to the list a single thread builds by walking the chunk
  table, chunk c holding tiles [mt * fq[c] >> 24, mt * fq[c + 1] >> 24), for
  the plan's own tables over many middle lengths.
"""
import random

import pytest

import speculative_flash_decoding_b200 as sfd

FRAC_BITS = 24


def fresh_fill_issue_order(fresh, d):
    """(round, lane, stage, copy) in issue order, and the expect-tx setters."""
    ops = 2 * (d // 64)
    per = 32 // ops
    issued, expect = [], []
    for s0 in range(0, fresh, per):
        for lane in range(32):
            s, op = s0 + lane // ops, lane % ops
            if s < fresh and op == 0:
                expect.append((s0, s))
        for lane in range(32):            # one copy instruction, lanes in order
            s, op = s0 + lane // ops, lane % ops
            if s < fresh:
                issued.append((s0, lane, s, op))
    return issued, expect, ops


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("fresh", [1, 3, 4, 5, 8, 9, 12, 13, 16, 24])
def test_first_fill_issues_every_copy_once_in_stage_order(d, fresh):
    issued, expect, ops = fresh_fill_issue_order(fresh, d)
    pairs = [(s, op) for _, _, s, op in issued]
    assert sorted(pairs) == [(s, op) for s in range(fresh) for op in range(ops)]
    assert sorted(s for _, s in expect) == list(range(fresh))
    # Within a round the copies leave in stage order; the expected bytes of
    # every stage of the round are set before the round's copy instruction.
    rounds = {}
    for r, lane, s, op in issued:
        rounds.setdefault(r, []).append(s)
    for r, stages in rounds.items():
        assert stages == sorted(stages)
        assert {s for rr, s in expect if rr == r} == set(stages)
    assert issued[0][2] == 0 and all(s == 0 for _, _, s, _ in issued[:ops])


def chunk_table(mid_tiles_max, heads):
    """The plan's guided self-scheduling table (chunk boundaries as 24-bit
    fractions), from the library's own planner."""
    desc = sfd.make_desc(1, 4 * heads, heads, 128, mid_tiles_max * 32 + 1028, "bf16")
    st, fq, _ = sfd.alspec_query_chunks(desc, 4, 1024)
    assert st == sfd.ALSPEC_OK
    return fq, len(fq) - 1


def list_one_thread(mt, fq, n2):
    out, prev = [], 0
    for c in range(n2):
        t = (mt * fq[c + 1]) >> FRAC_BITS
        if t > prev:
            out.append(c)
        prev = t
    return out


def list_ballot(mt, fq, n2):
    """Warp 0's rounds: a ballot of the non-empty chunks among 32, each lane
    writing its chunk at count + (set bits of the lanes below it)."""
    out = [None] * 256
    count = 0
    for c0 in range(0, n2, 32):
        ballot = 0
        for lane in range(32):
            c = c0 + lane
            if c < n2:
                lo = (mt * fq[c]) >> FRAC_BITS
                hi = (mt * fq[c + 1]) >> FRAC_BITS
                if hi > lo:
                    ballot |= 1 << lane
        for lane in range(32):
            if ballot >> lane & 1:
                out[count + bin(ballot & ((1 << lane) - 1)).count("1")] = c0 + lane
        count += bin(ballot).count("1")
    assert all(x is None for x in out[count:])
    return out[:count]


@pytest.mark.parametrize("heads", [1, 8])
def test_merge_chunk_list_matches_the_table_walk(heads):
    rng = random.Random(heads)
    for mid_max in (16, 300, 992, 4064, 16000):
        fq, n2 = chunk_table(mid_max, heads)
        assert fq[0] == 0 and all(a <= b for a, b in zip(fq, fq[1:]))
        for mt in sorted({0, 1, 2, mid_max - 1, mid_max} |
                         {rng.randint(0, mid_max) for _ in range(40)}):
            mt = max(mt, 0)
            assert list_ballot(mt, fq, n2) == list_one_thread(mt, fq, n2), (mid_max, mt)
