"""The seeded input generator (workloads.py), on CPU: the recipe the design
notes state -- reproducibility, ragged lengths, where the needles go and how
many, the sink bias and the needle bump as seen by the query heads, and the
NaN tails past each length.
"""
import math

import pytest
import torch

import workloads


def _small(i, **kw):
    wl = workloads.CONFIGS[i]
    base = dict(L=min(wl.L, 4096), W=min(wl.W, 512))
    if wl.ragged:
        base["ragged"] = (1024, 4096)
    base.update(kw)
    return wl.replace(**base)


def test_same_seed_same_bits_other_layer_other_bits():
    wl = _small(2)
    a = workloads.make_layer(wl, layer=3)
    b = workloads.make_layer(wl, layer=3)
    c = workloads.make_layer(wl, layer=4)
    for key in ("q", "k", "v"):
        assert torch.equal(a[key].view(torch.int16), b[key].view(torch.int16))
        assert not torch.equal(a[key].view(torch.int16), c[key].view(torch.int16))
    assert a["needles"] == b["needles"]


def test_ragged_lengths_in_range_and_seeded():
    wl = workloads.CONFIGS[3]
    lens = workloads.seq_lens_for(wl, 0)
    assert len(lens) == wl.B and all(16384 <= L <= 65536 for L in lens)
    assert lens == workloads.seq_lens_for(wl, 0) and lens != workloads.seq_lens_for(wl, 1)
    assert workloads.seq_lens_for(workloads.CONFIGS[2]) == [131072]


@pytest.mark.parametrize("i", [0, 1, 3, 4])
def test_needles_lie_outside_the_sink_set(i):
    wl = _small(i)
    data = workloads.make_layer(wl)
    assert data["needles"], "every workload but the commit variant plants needles"
    seen = set()
    for b, kv, h, p in data["needles"]:
        assert 0 <= b < wl.B and 0 <= kv < wl.Hkv and 0 <= h < wl.g
        assert wl.S <= p < data["lens"][b] - wl.W
        assert (b, kv, p) not in seen     # distinct positions within a head
        seen.add((b, kv, p))


def test_needle_counts_per_recipe():
    # Head 3 of the tiny workload (group of 4 on one KV head).
    n0 = workloads.make_layer(_small(0))["needles"]
    assert [(b, kv, h) for b, kv, h, _ in n0] == [(0, 0, 3)]
    # 25% of the KV heads of the 32K layer: 2 of 8.
    assert len(workloads.make_layer(_small(1))["needles"]) == round(0.25 * 8)
    # 12.5% of the (sequence, KV head) pairs of the ragged batch: 8 of 64.
    n3 = workloads.make_layer(_small(3))["needles"]
    assert len({(b, kv) for b, kv, _, _ in n3}) == round(0.125 * 8 * 8)
    # Poisson(1), at most 3, per KV head of the 70B batch.
    n4 = workloads.make_layer(_small(4))["needles"]
    per = {}
    for b, kv, _, _ in n4:
        per[(b, kv)] = per.get((b, kv), 0) + 1
    assert max(per.values()) <= 3


def test_sink_bias_and_needle_bump_as_logits():
    """Every query head sees its sink keys about sink_bump above the others
    (the bias is the group's sum of unit query directions), and its needle
    key about needle_bump above them."""
    wl = _small(1, L=2048, W=256)
    data = workloads.make_layer(wl)
    q = data["q"].float()
    qhat = q / q.norm(dim=-1, keepdim=True)
    k = data["k"].float()
    B, Hkv, g = wl.B, wl.Hkv, wl.g
    sink_gap, needle_gap = [], []
    for b in range(B):
        for kv in range(Hkv):
            keys = k[b, kv]                                  # [L, d]
            for h in range(g):
                logit = keys @ qhat[b, kv * g + h]           # q_hat . k_j
                sink_gap.append(float(logit[: wl.S].mean() - logit[wl.S:].mean()))
    for b, kv, h, p in data["needles"]:
        logit = k[b, kv] @ qhat[b, kv * g + h]
        needle_gap.append(float(logit[p] - logit[wl.S:].mean()))
    assert abs(sum(sink_gap) / len(sink_gap) - wl.sink_bump) < 1.5
    assert needle_gap and min(needle_gap) > wl.needle_bump - 4.5


def test_poisoned_tail_is_nan_past_each_length():
    wl = _small(3)
    data = workloads.make_layer(wl, poison_tail=True)
    for b, L in enumerate(data["lens"]):
        assert torch.isfinite(data["k"][b, :, :L].float()).all()
        assert torch.isfinite(data["v"][b, :, :L].float()).all()
        if L < wl.L:
            assert torch.isnan(data["k"][b, :, L:].float()).all()
            assert torch.isnan(data["v"][b, :, L:].float()).all()


def test_dtypes_and_kv_bytes():
    wl0, wl2 = _small(0), _small(2)
    assert workloads.make_layer(wl0)["k"].dtype == torch.float32
    assert workloads.make_layer(wl2)["k"].dtype == torch.bfloat16
    assert workloads.kv_bytes(workloads.CONFIGS[2]) == 131072 * 8 * 128 * 2 * 2
    assert workloads.kv_bytes(wl0) == 1024 * 1 * 64 * 2 * 4
    lens = workloads.seq_lens_for(workloads.CONFIGS[3])
    assert workloads.kv_bytes(workloads.CONFIGS[3], lens) == sum(lens) * 8 * 128 * 4
    assert math.isclose(workloads.kv_bytes(workloads.CONFIGS[2]) / 2 ** 20, 512.0)
