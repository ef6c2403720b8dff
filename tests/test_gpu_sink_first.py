"""GPU parity of the SINK_FIRST schedule (the sink-set kernel alone first on
the caller's stream, with clusters that may cover every SM, then the
exact-path and merge kernels) against the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import workloads
from parity import assert_parity, gpu_decode, oracle_decode
from test_gpu_parity import _small

pytestmark = pytest.mark.gpu

SF = dict(schedule="sink_first")


@pytest.mark.parametrize("cfg,engine", [(0, "auto"), (1, "auto"), (2, "auto"), (3, "auto"),
                                        (4, "auto"), (3, "cuda_cores")])
def test_small_configs(cuda_device, cfg, engine):
    wl = _small(cfg)
    data = workloads.make_layer(wl, device=cuda_device, poison_tail=True)
    dec, out = gpu_decode(wl, data, cuda_device, engine=engine, **SF)
    assert dec.plan()["schedule"] == 3
    assert_parity(out, oracle_decode(wl, data), wl.lam, what=f"sink-first cfg{cfg} {engine}")
    assert dec.device_error() == (0, 0)


def test_short_sequences_in_wide_clusters(cuda_device):
    """Every SM for the sink set: 7-CTA clusters (33 tiles at about 5 per
    CTA), most CTAs of short sequences without rows."""
    lens = [1, 3, 40, 1000, 1028, 1029, 2100, 4096]
    wl = workloads.Workload("short-sf", B=len(lens), Hq=8, Hkv=2, d=128, L=4096, S=4, W=1024,
                            lam=0.3, dtype="bf16", seed=4343)
    data = workloads.make_layer(wl, device=cuda_device)
    data["lens"] = lens
    data["seq_lens"] = torch.tensor(lens, dtype=torch.int32, device=cuda_device)
    dec, out = gpu_decode(wl, data, cuda_device, **SF)
    assert dec.plan()["n1"] == 7
    assert_parity(out, oracle_decode(wl, data), wl.lam, what="short in wide clusters")
    for b, L in enumerate(lens):
        if L <= wl.S + wl.W:
            assert torch.equal(out["out_spec"][b], out["out_exact"][b])
            assert out["rel_l2"][b].item() == 0.0


def test_spec_event_and_graph(cuda_device):
    """spec_event marks O_spec complete; a captured graph of two layers gives
    the eager results bit for bit."""
    import speculative_flash_decoding_b200 as sfd
    wl = _small(3)
    layers = [workloads.make_layer(wl, layer=i, device=cuda_device) for i in range(2)]
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device,
                      **SF)
    ev = torch.cuda.Event()
    ev.record()
    d0 = layers[0]
    out = dec.decode(d0["q"], d0["k"], d0["v"], d0["seq_lens"], wl.lam, spec_event=ev)
    ev.synchronize()
    spec = out["out_spec"].cpu()
    torch.cuda.synchronize()
    assert torch.equal(spec, out["out_spec"].cpu())
    outs = [dec.alloc_outputs() for _ in layers]
    direct = []
    for d, o in zip(layers, outs):
        dec.decode(d["q"], d["k"], d["v"], d["seq_lens"], wl.lam, out=o)
        torch.cuda.synchronize()
        direct.append({k: v.clone() for k, v in o.items()})
    stream = torch.cuda.Stream(cuda_device)
    with torch.cuda.stream(stream):
        assert sfd.alspec_graph_begin(stream.cuda_stream) == 0
        for d, o in zip(layers, outs):
            dec.decode(d["q"], d["k"], d["v"], d["seq_lens"], wl.lam, out=o, stream=stream)
        st, graph = sfd.alspec_graph_end(stream.cuda_stream)
        assert st == 0 and graph
        for o in outs:
            for v in o.values():
                v.zero_()
        assert sfd.alspec_graph_launch(graph, stream.cuda_stream) == 0
        stream.synchronize()
        assert sfd.alspec_graph_destroy(graph) == 0
    for d, o in zip(direct, outs):
        for k in d:
            assert torch.equal(d[k], o[k]), k


def test_speculative_projection(cuda_device):
    """The speculative output projection waits for O_spec from the caller's
    stream; y equals the oracle's gated projection."""
    import oracle
    wl = _small(1).replace(B=3, L=3000)
    data = workloads.make_layer(wl, device=cuda_device)
    import speculative_flash_decoding_b200 as sfd
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device,
                      **SF)
    g = torch.Generator(device="cpu").manual_seed(5)
    w = (torch.randn(96, wl.Hq * wl.d, generator=g) / 64).to(torch.bfloat16).to(cuda_device)
    out = dec.decode_oproj(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam, w)
    torch.cuda.synchronize()
    ref = oracle_decode(wl, data)
    assert_parity({k: v.cpu() for k, v in out.items() if k != "y"}, ref, wl.lam, what="sf oproj")
    want = oracle.oproj_gated(out["out_spec"].cpu().numpy().reshape(wl.B, -1),
                              out["out_exact"].cpu().numpy().reshape(wl.B, -1),
                              out["commit"].cpu().numpy(), workloads.to_numpy_bits(w))
    got = out["y"].cpu().double().numpy()
    rel = np.linalg.norm(got - want, axis=1) / np.linalg.norm(want, axis=1)
    assert rel.max() < 1e-5, rel  # fp32 sums of 4096 products against fp64


def test_full_size_ragged_batch(cuda_device):
    wl = workloads.CONFIGS[3]
    data = workloads.make_layer(wl, device=cuda_device, poison_tail=True)
    _, out = gpu_decode(wl, data, cuda_device, **SF)
    lens = np.array(data["lens"])
    pick = [int(lens.argmin()), int(lens.argmax())]
    assert_parity(out, oracle_decode(wl, data, batch=pick), wl.lam, batch=pick,
                  what="sink-first cfg3 full")
    assert torch.isfinite(out["out_exact"]).all()


def test_full_size_70b_layer(cuda_device):
    wl = workloads.CONFIGS[4]
    data = workloads.make_layer(wl, device=cuda_device)
    _, out = gpu_decode(wl, data, cuda_device, **SF)
    assert_parity(out, oracle_decode(wl, data, batch=[0]), wl.lam, batch=[0],
                  what="sink-first cfg4 full b0")
