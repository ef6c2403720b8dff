"""Randomised GPU parity: seeded shapes across every supported dimension.

Each case draws a batch, KV head count, group size, head size, dtype and
engine, a ragged set of lengths (1 token and up), a sink and a window (either
may be 0), a split size and a threshold, and compares the CUDA path with the
fp64 oracle on the same bits, under each launch schedule.
"""
import numpy as np
import pytest
import torch

import workloads
from parity import assert_parity, gpu_decode, oracle_decode

pytestmark = pytest.mark.gpu


def _case(seed):
    rng = np.random.default_rng(seed)
    dtype = "bf16" if rng.random() < 0.75 else "f32"
    engine = "cuda_cores" if dtype == "f32" else ("tensor_cores" if rng.random() < 0.7
                                                  else "cuda_cores")
    g = int(rng.choice([1, 2, 4, 8]))
    hkv = int(rng.integers(1, 5))
    d = int(rng.choice([64, 128]))
    B = int(rng.integers(1, 7))
    Lmax = int(rng.integers(1, 6000))
    S = int(rng.integers(0, 41))
    W = int(rng.integers(0, 700))
    if S + W == 0:
        W = 1
    lens = sorted(int(x) for x in rng.integers(1, Lmax + 1, size=B))
    lens[-1] = Lmax
    split = 0 if rng.random() < 0.5 else int(rng.integers(16, 2500))
    lam = float(rng.choice([0.0, 0.05, 0.3, 2.0]))
    wl = workloads.Workload(f"random-{seed}", B=B, Hq=g * hkv, Hkv=hkv, d=d, L=Lmax, S=S, W=W,
                            lam=lam, dtype=dtype, seed=90000 + seed)
    return wl, lens, engine, split


@pytest.mark.parametrize("schedule", ["streams", "fused", "sink_first"])
@pytest.mark.parametrize("seed", range(24))
def test_random_shapes_match_oracle(cuda_device, seed, schedule):
    wl, lens, engine, split = _case(seed)
    data = workloads.make_layer(wl, device=cuda_device, poison_tail=True)
    data["lens"] = lens
    data["seq_lens"] = torch.tensor(lens, dtype=torch.int32, device=cuda_device)
    # Rows past each sequence's length hold NaN: reading one would show.
    for b, L in enumerate(lens):
        data["k"][b, :, L:, :] = float("nan")
        data["v"][b, :, L:, :] = float("nan")
    dec, out = gpu_decode(wl, data, cuda_device, engine=engine, split_tokens=split,
                          schedule=schedule)
    what = (f"{schedule} seed {seed}: B{wl.B} Hkv{wl.Hkv} g{wl.g} d{wl.d} {wl.dtype} {engine} "
            f"L{lens} S{wl.S} W{wl.W} split {split} lam {wl.lam}")
    assert_parity(out, oracle_decode(wl, data), wl.lam, what=what)
    for b, L in enumerate(lens):
        if L <= wl.S + wl.W:
            assert torch.equal(out["out_spec"][b], out["out_exact"][b]), what
            assert out["rel_l2"][b].item() == 0.0, what
    assert dec.device_error() == (0, 0), what
