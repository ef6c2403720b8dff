"""GPU parity of the one-launch schedule (ALSPEC_SCHEDULE_FUSED) against the
fp64 oracle: the sink-set items share the exact path's work queue, and the
merges of O_spec, O_exact, rel_l2 and the flag happen inside the launch,
done by whichever CTA takes a head's (or a sequence's) last tile ticket.
"""
import numpy as np
import pytest
import torch

import workloads
from parity import assert_parity, gpu_decode, oracle_decode, per_head_rel
from test_gpu_parity import EDGE, _small

pytestmark = pytest.mark.gpu

FUSED = dict(schedule="fused")


@pytest.mark.parametrize("cfg,engine", [(0, "auto"), (1, "auto"), (2, "auto"), (3, "auto"),
                                        (4, "auto"), (1, "cuda_cores"), (4, "cuda_cores")])
def test_small_configs(cuda_device, cfg, engine):
    wl = _small(cfg)
    for layer in range(3 if cfg == 2 else 1):
        data = workloads.make_layer(wl, layer=layer, device=cuda_device, poison_tail=True)
        dec, out = gpu_decode(wl, data, cuda_device, engine=engine, **FUSED)
        assert dec.plan()["schedule"] == 2
        assert_parity(out, oracle_decode(wl, data), wl.lam,
                      what=f"fused cfg{cfg} layer{layer} {engine}")
        assert dec.device_error() == (0, 0)


def test_schedules_agree(cuda_device):
    """Both schedules on the same inputs: the same values up to the fp32
    summation order of the merges."""
    for cfg in (1, 3, 4):
        wl = _small(cfg)
        data = workloads.make_layer(wl, device=cuda_device)
        _, a = gpu_decode(wl, data, cuda_device, schedule="streams")
        _, b = gpu_decode(wl, data, cuda_device, **FUSED)
        for name in ("out_spec", "out_exact"):
            assert per_head_rel(a[name].double().numpy(), b[name].double().numpy()).max() < 1e-5
        assert np.allclose(a["rel_l2"].numpy(), b["rel_l2"].numpy(), rtol=1e-5, atol=0)


@pytest.mark.parametrize("dtype,d,g,engine", EDGE)
def test_edge_lengths(cuda_device, dtype, d, g, engine):
    """L = 1, L < S, L = S + W, L = S + W + 1, W = 0, S = 0, ragged tails."""
    Hkv = 2
    for S, W in ((4, 16), (0, 16), (4, 0), (1, 1), (40, 70)):
        lens = sorted({1, 3, S + W, S + W + 1, 37, 250, 16 * 9 + 5})
        lens = [L for L in lens if L >= 1]
        wl = workloads.Workload("edge", B=len(lens), Hq=g * Hkv, Hkv=Hkv, d=d, L=max(lens), S=S,
                                W=W, lam=0.3, dtype=dtype, seed=777 + g + d)
        data = workloads.make_layer(wl, device=cuda_device)
        data["lens"] = lens
        data["seq_lens"] = torch.tensor(lens, dtype=torch.int32, device=cuda_device)
        dec, out = gpu_decode(wl, data, cuda_device, engine=engine, **FUSED)
        assert_parity(out, oracle_decode(wl, data), wl.lam,
                      what=f"fused {dtype} d{d} g{g} S{S} W{W} {engine}")
        for b, L in enumerate(lens):
            if L <= S + W:
                assert torch.equal(out["out_spec"][b], out["out_exact"][b])
                assert out["rel_l2"][b].item() == 0.0 and out["commit"][b].item() == 1
        assert dec.device_error() == (0, 0)


def test_only_sink_set_items(cuda_device):
    """Every sequence within S + W: the queue holds no middle item at all and
    each head's merges are done by the CTA that completes its sink set."""
    lens = [1, 5, 100, 200]
    wl = workloads.Workload("no-middle", B=4, Hq=8, Hkv=2, d=128, L=200, S=8, W=192, lam=0.0,
                            dtype="bf16", seed=31)
    data = workloads.make_layer(wl, device=cuda_device)
    data["lens"] = lens
    data["seq_lens"] = torch.tensor(lens, dtype=torch.int32, device=cuda_device)
    dec, out = gpu_decode(wl, data, cuda_device, **FUSED)
    assert dec.plan()["n2"] == 0
    assert_parity(out, oracle_decode(wl, data), wl.lam, what="no middle")
    assert torch.equal(out["out_spec"], out["out_exact"])
    assert (out["rel_l2"] == 0).all() and (out["commit"] == 1).all()


def test_deterministic_and_reusable_workspace(cuda_device):
    """Repeated calls on one workspace: the tickets reset themselves and the
    results are bit-identical whichever CTAs did the merges."""
    wl = _small(3)
    data = workloads.make_layer(wl, device=cuda_device)
    dec, a = gpu_decode(wl, data, cuda_device, **FUSED)
    for _ in range(5):
        _, b = gpu_decode(wl, data, cuda_device, dec=dec)
        for k in a:
            assert torch.equal(a[k], b[k]), k
    # Counters are back at zero after each call.
    nwords = 4 + wl.B + wl.B * wl.Hkv
    assert (dec.workspace[: 4 * nwords].view(torch.int32)[[0, 1, 3]] == 0).all()
    assert (dec.workspace[: 4 * nwords].view(torch.int32)[4:] == 0).all()


def test_split_sizes_agree(cuda_device):
    wl = _small(3)
    data = workloads.make_layer(wl, device=cuda_device)
    ref = oracle_decode(wl, data)
    for engine in ("tensor_cores", "cuda_cores"):
        for split in (16, 112, 1024, 100000):
            _, out = gpu_decode(wl, data, cuda_device, split_tokens=split, engine=engine,
                                **FUSED)
            assert_parity(out, ref, wl.lam, what=f"fused split {split} {engine}")


def test_bad_seq_lens_are_clamped_and_flagged(cuda_device):
    wl = _small(1).replace(B=3, L=600, W=64)
    data = workloads.make_layer(wl, device=cuda_device)
    data["seq_lens"] = torch.tensor([0, 600, 9999], dtype=torch.int32, device=cuda_device)
    dec, out = gpu_decode(wl, data, cuda_device, **FUSED)
    st, err = dec.device_error()
    assert err & 1 and st != 0
    assert_parity(out, oracle_decode(wl, data, lens=[1, 600, 600]), wl.lam, what="fused clamped")


def test_traced_stamps_and_spec_event(cuda_device):
    """O_spec is published inside the launch, no later than O_exact;
    spec_event fires at the launch's end with O_spec complete."""
    wl = _small(2)
    data = workloads.make_layer(wl, device=cuda_device)
    import speculative_flash_decoding_b200 as sfd
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device,
                      **FUSED)
    trace = torch.zeros(2, dtype=torch.int64, device=cuda_device)
    plain = {k: v.clone() for k, v in dec.decode(data["q"], data["k"], data["v"],
                                                  data["seq_lens"], wl.lam).items()}
    traced = dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam, trace=trace)
    torch.cuda.synchronize()
    for k in plain:
        assert torch.equal(plain[k], traced[k]), k
    t = trace.cpu().numpy()
    assert (t > 0).all() and t[0] <= t[1], t
    ev = torch.cuda.Event()
    ev.record()
    out = dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam, spec_event=ev)
    ev.synchronize()
    assert torch.equal(out["out_spec"].cpu(), plain["out_spec"].cpu())


def test_graph_replay_matches_direct_calls(cuda_device):
    import speculative_flash_decoding_b200 as sfd
    wl = _small(2)
    layers = [workloads.make_layer(wl, layer=i, device=cuda_device) for i in range(3)]
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device,
                      **FUSED)
    outs = [dec.alloc_outputs() for _ in layers]
    direct = []
    for data, o in zip(layers, outs):
        dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam, out=o)
        torch.cuda.synchronize()
        direct.append({k: v.clone() for k, v in o.items()})
        for v in o.values():
            v.zero_()
    stream = torch.cuda.Stream(cuda_device)
    with torch.cuda.stream(stream):
        assert sfd.alspec_graph_begin(stream.cuda_stream) == 0
        for data, o in zip(layers, outs):
            dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam, out=o,
                       stream=stream)
        st, graph = sfd.alspec_graph_end(stream.cuda_stream)
        assert st == 0 and graph
        for _ in range(3):
            assert sfd.alspec_graph_launch(graph, stream.cuda_stream) == 0
        stream.synchronize()
        assert sfd.alspec_graph_destroy(graph) == 0
    for d, o in zip(direct, outs):
        for k in d:
            assert torch.equal(d[k], o[k]), k


def test_speculative_projection_is_not_offered(cuda_device):
    import speculative_flash_decoding_b200 as sfd
    wl = _small(1)
    data = workloads.make_layer(wl, device=cuda_device)
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device,
                      **FUSED)
    w = torch.zeros(64, wl.Hq * wl.d, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(sfd.AlspecError) as e:
        dec.decode_oproj(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam, w)
    assert e.value.status == sfd.ALSPEC_ERR_UNSUPPORTED


def test_one_millisecond_limit_does_not_fire_on_normal_work(cuda_device):
    wl = _small(2)
    data = workloads.make_layer(wl, device=cuda_device)
    dec, out = gpu_decode(wl, data, cuda_device, timeout_ms=1, **FUSED)
    assert dec.device_error() == (0, 0)
    assert_parity(out, oracle_decode(wl, data), wl.lam, what="fused 1 ms wait limit")


# --------------------------------------------------------------- full size

def test_full_size_128k_layer(cuda_device):
    wl = workloads.CONFIGS[2]
    data = workloads.make_layer(wl, layer=0, device=cuda_device)
    _, out = gpu_decode(wl, data, cuda_device, **FUSED)
    assert_parity(out, oracle_decode(wl, data), wl.lam, what="fused cfg2 layer0 full")


def test_full_size_32k_layer(cuda_device):
    wl = workloads.CONFIGS[1]
    data = workloads.make_layer(wl, device=cuda_device)
    _, out = gpu_decode(wl, data, cuda_device, **FUSED)
    assert_parity(out, oracle_decode(wl, data), wl.lam, what="fused cfg1 full")


def test_full_size_ragged_batch(cuda_device):
    wl = workloads.CONFIGS[3]
    data = workloads.make_layer(wl, device=cuda_device, poison_tail=True)
    _, out = gpu_decode(wl, data, cuda_device, **FUSED)
    lens = np.array(data["lens"])
    pick = [int(lens.argmin()), int(lens.argmax())]
    assert_parity(out, oracle_decode(wl, data, batch=pick), wl.lam, batch=pick,
                  what="fused cfg3 full")
    assert torch.isfinite(out["out_exact"]).all()


def test_full_size_70b_layer(cuda_device):
    wl = workloads.CONFIGS[4]
    data = workloads.make_layer(wl, device=cuda_device)
    _, out = gpu_decode(wl, data, cuda_device, **FUSED)
    assert_parity(out, oracle_decode(wl, data, batch=[0]), wl.lam, batch=[0],
                  what="fused cfg4 full b0")
