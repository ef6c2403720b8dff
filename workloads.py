"""Seeded synthetic decode workloads for the speculative flash-decode path.

This module only makes inputs.  It holds none of the attention arithmetic:
the CUDA path and the oracle both read the tensors it returns, bit for bit.

Every workload is a Llama-shaped grouped-query decode layer (or a stack of
independent layers): one query row per sequence, a bf16 (or fp32) KV cache in
[B, H_kv, L_max, d] layout (token-major, d contiguous) and per-sequence
lengths.  The value distributions follow the structure the method is about:
  - q, K and V entries are i.i.d. N(0, 1), rounded once to the cache dtype;
  - the first S ("sink") keys of every KV head are biased along the unit query
    directions of the query heads that share that KV head (sum over the group
    of bump * q_h / ||q_h||), so attention mass concentrates on the sinks;
  - "needles" are planted outside the sink set: at a position in
    [S, L_b - W), the key gets needle_bump * q_h / ||q_h|| for one query head
    h of the group, and the value gets 4 * N(0, I) added, so exact attention
    differs from the sink approximation there.
The planted needles stand in for the needle-in-a-haystack structure of the
evaluation suite named on the pages; no dataset item is reproduced.

Seeds: workload i uses seed 20250 + i; layer l of it uses seed * 1000 + l.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape, thresholds and input recipe of one decode workload."""

    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    L: int                      # cache capacity L_max (and the length when not ragged)
    S: int                      # sink tokens
    W: int                      # recent-window tokens
    lam: float                  # relative-L2 threshold
    dtype: str = "bf16"         # "bf16" or "f32" (q, K and V share it)
    n_layers: int = 1
    seed: int = 20250
    ragged: Optional[tuple] = None      # (lo, hi): L_b ~ U[lo, hi] per sequence
    sink_bump: float = 8.0
    needle_bump: float = 8.0
    needle_v_scale: float = 4.0
    # Needle recipe, one of:
    #   ("head", h)         : query head h of KV head 0 of every sequence
    #   ("kv_frac", f)      : round(f * H_kv) KV heads per sequence
    #   ("kv_frac_layer", fs): per layer, f drawn uniformly from fs
    #   ("pair_frac", f)    : round(f * B * H_kv) (b, kv) pairs overall
    #   ("poisson", mean, cap): per KV head, min(Poisson(mean), cap) needles
    #   ("none",)
    needles: tuple = ("none",)

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny fp32 layer, a Llama-3.1-8B-shaped 32K layer, a
# 32-layer 128K decode step, a ragged batch and a Llama-70B-shaped 128K layer.
CONFIGS = {
    0: Workload("tiny-fp32-1k", B=1, Hq=4, Hkv=1, d=64, L=1024, S=4, W=128,
                lam=0.10, dtype="f32", seed=20250, needles=("head", 3)),
    1: Workload("llama8b-layer-32k", B=1, Hq=32, Hkv=8, d=128, L=32768, S=4,
                W=1024, lam=0.10, seed=20251, needles=("kv_frac", 0.25)),
    2: Workload("llama8b-32layers-128k", B=1, Hq=32, Hkv=8, d=128, L=131072,
                S=4, W=1024, lam=0.10, n_layers=32, seed=20252,
                needles=("kv_frac_layer", (0.0, 0.125, 0.5))),
    3: Workload("ragged-b8-16k-64k", B=8, Hq=32, Hkv=8, d=128, L=65536, S=4,
                W=2048, lam=0.10, seed=20253, ragged=(16384, 65536),
                needles=("pair_frac", 0.125)),
    4: Workload("llama70b-b4-128k", B=4, Hq=64, Hkv=8, d=128, L=131072, S=4,
                W=4096, lam=0.05, seed=20254, needles=("poisson", 1.0, 3)),
}

# Supplementary variant (not one of the five): stronger sinks so that the
# approximation is accurate where no needle is present, and needles in only
# 1/16 of the (sequence, KV head) pairs, so a batch mixes commit and discard.
# Llama-3.1-8B head shapes, batch 8, ragged 24K-32K.
COMMIT_VARIANT = CONFIGS[1].replace(name="llama8b-b8-32k-commit", B=8, seed=20259,
                                    ragged=(24576, 32768), sink_bump=24.0, needle_bump=32.0,
                                    needles=("pair_frac", 0.0625))


def layer_seed(wl: Workload, layer: int) -> int:
    return wl.seed * 1000 + layer


def seq_lens_for(wl: Workload, layer: int = 0) -> List[int]:
    """Per-sequence lengths (host list).  Ragged lengths come from the seed."""
    if wl.ragged is None:
        return [wl.L] * wl.B
    lo, hi = wl.ragged
    g = torch.Generator().manual_seed(layer_seed(wl, layer) + 7)
    return [int(x) for x in torch.randint(lo, hi + 1, (wl.B,), generator=g)]


def _needle_plan(wl: Workload, layer: int, lens: List[int]):
    """List of (b, kv_head, q_head_in_group, position) needles, from the seed."""
    g = torch.Generator().manual_seed(layer_seed(wl, layer) + 13)
    kind = wl.needles[0]
    pairs = []  # (b, kv) pairs that get needles, with counts
    if kind == "none":
        return []
    if kind == "head":
        h = wl.needles[1]
        pairs = [(b, h // wl.g, 1, h % wl.g) for b in range(wl.B)]
    elif kind in ("kv_frac", "kv_frac_layer"):
        if kind == "kv_frac":
            frac = wl.needles[1]
        else:
            choices = wl.needles[1]
            frac = choices[int(torch.randint(len(choices), (1,), generator=g))]
        n = int(round(frac * wl.Hkv))
        for b in range(wl.B):
            heads = torch.randperm(wl.Hkv, generator=g)[:n].tolist()
            pairs += [(b, kv, 1, None) for kv in sorted(heads)]
    elif kind == "pair_frac":
        n = int(round(wl.needles[1] * wl.B * wl.Hkv))
        flat = torch.randperm(wl.B * wl.Hkv, generator=g)[:n].tolist()
        pairs = [(f // wl.Hkv, f % wl.Hkv, 1, None) for f in sorted(flat)]
    elif kind == "poisson":
        mean, cap = wl.needles[1], wl.needles[2]
        counts = torch.poisson(torch.full((wl.B * wl.Hkv,), float(mean)), generator=g)
        for f, c in enumerate(counts.tolist()):
            c = min(int(c), cap)
            if c:
                pairs.append((f // wl.Hkv, f % wl.Hkv, c, None))
    else:
        raise ValueError(f"unknown needle recipe {wl.needles}")

    plan = []
    for b, kv, count, fixed_h in pairs:
        lo, hi = wl.S, lens[b] - wl.W          # outside the sink set
        if hi - lo < count:
            continue
        pos = (torch.randperm(hi - lo, generator=g)[:count] + lo).tolist()
        for p in pos:
            h = fixed_h if fixed_h is not None else int(torch.randint(wl.g, (1,), generator=g))
            plan.append((b, kv, h, int(p)))
    return plan


def make_layer(wl: Workload, layer: int = 0, device="cpu", poison_tail: bool = False):
    """Generate one layer's inputs.

    Returns a dict with
      q        [B, Hq, d]          cache dtype
      k, v     [B, Hkv, L_max, d]  cache dtype
      seq_lens [B] int32 (on ``device``) and ``lens`` (host list)
      needles  list of (b, kv_head, head_in_group, position)
    With ``poison_tail`` the cache rows at positions >= L_b are NaN, so that
    any read past a sequence's end shows up in the outputs.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(layer_seed(wl, layer))
    B, Hq, Hkv, d, L = wl.B, wl.Hq, wl.Hkv, wl.d, wl.L
    td = wl.torch_dtype
    lens = seq_lens_for(wl, layer)

    q = torch.randn(B, Hq, d, generator=gen, device=dev, dtype=torch.float32).to(td)
    qf = q.float()
    qhat = qf / qf.norm(dim=-1, keepdim=True)                       # [B, Hq, d]
    qhat_g = qhat.view(B, Hkv, wl.g, d)

    k = torch.empty(B, Hkv, L, d, device=dev, dtype=td)
    v = torch.empty(B, Hkv, L, d, device=dev, dtype=td)
    # Generate per sequence to bound the fp32 temporaries.
    for b in range(B):
        kb = torch.randn(Hkv, L, d, generator=gen, device=dev, dtype=torch.float32)
        if wl.S > 0:
            kb[:, : wl.S, :] += wl.sink_bump * qhat_g[b].sum(dim=1, keepdim=True)
        k[b] = kb.to(td)
        del kb
        v[b] = torch.randn(Hkv, L, d, generator=gen, device=dev, dtype=torch.float32).to(td)

    plan = _needle_plan(wl, layer, lens)
    if plan:
        ng = torch.Generator().manual_seed(layer_seed(wl, layer) + 29)
        for b, kv, h, p in plan:
            kf = k[b, kv, p].float() + wl.needle_bump * qhat_g[b, kv, h].to(k.device)
            k[b, kv, p] = kf.to(td)
            noise = torch.randn(d, generator=ng).to(dev)
            v[b, kv, p] = (v[b, kv, p].float() + wl.needle_v_scale * noise).to(td)

    if poison_tail:
        for b in range(B):
            if lens[b] < L:
                k[b, :, lens[b]:, :] = float("nan")
                v[b, :, lens[b]:, :] = float("nan")

    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    return dict(q=q, k=k, v=v, seq_lens=seq, lens=lens, needles=plan)


def kv_bytes(wl: Workload, lens: Optional[List[int]] = None) -> int:
    """Algorithmic KV bytes of one layer: sum_b L_b * H_kv * d * 2 (K and V) * elem."""
    lens = lens if lens is not None else seq_lens_for(wl)
    return sum(lens) * wl.Hkv * wl.d * 2 * wl.elem_bytes


def to_numpy_bits(t: torch.Tensor):
    """CPU numpy view of a tensor for the oracle: bfloat16 as uint16 bit patterns."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()


__all__ = ["Workload", "CONFIGS", "COMMIT_VARIANT", "make_layer", "seq_lens_for",
           "kv_bytes", "to_numpy_bits", "layer_seed"]

