"""GPU parity of the output projection that follows attention and of the
speculative decode + projection with commit gating, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import FLAG_BAND, oracle_decode

pytestmark = pytest.mark.gpu

ROW_TOL = 1e-4   # per-row relative L2 of y (fp32 accumulation over K terms)


def _row_rel(got, want):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    return np.linalg.norm(got - want, axis=-1) / np.maximum(np.linalg.norm(want, axis=-1), 1e-30)


def _bf16_weights(n, k, seed, device):
    g = torch.Generator(device="cpu").manual_seed(seed)
    w = (torch.randn(n, k, generator=g) / np.sqrt(k)).to(torch.bfloat16)
    return w.to(device)


# K = 8192 (Llama-70B-shaped, 64 heads x 128) and 12296 give rows of several
# bulk-copy pieces, so consecutive fills of a stage go to different warps.
@pytest.mark.parametrize("B,K,N", [(1, 4096, 4096), (3, 520, 77), (8, 1024, 300), (2, 8, 5),
                                   (4, 8192, 8192), (2, 12296, 1000)])
def test_oproj_matches_oracle(cuda_device, B, K, N):
    import speculative_flash_decoding_b200 as sfd
    g = torch.Generator(device="cpu").manual_seed(B * 1000 + K + N)
    x = torch.randn(B, K, generator=g).to(cuda_device)
    w = _bf16_weights(N, K, K + N, cuda_device)
    y = torch.full((B, N), 7.0, device=cuda_device)
    assert sfd.alspec_oproj(x.data_ptr(), w.data_ptr(), y.data_ptr(), 0, B, K, N,
                            torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    ref = oracle.oproj(x.cpu().numpy(), workloads.to_numpy_bits(w))
    assert _row_rel(y.cpu().numpy(), ref).max() < ROW_TOL
    # Masked rows are left exactly as they were.
    skip = torch.tensor([b % 2 for b in range(B)], dtype=torch.uint8, device=cuda_device)
    y2 = torch.full((B, N), 7.0, device=cuda_device)
    assert sfd.alspec_oproj(x.data_ptr(), w.data_ptr(), y2.data_ptr(), skip.data_ptr(), B, K, N,
                            torch.cuda.current_stream().cuda_stream) == 0
    torch.cuda.synchronize()
    for b in range(B):
        if b % 2:
            assert torch.all(y2[b] == 7.0)
        else:
            assert torch.equal(y2[b], y[b])


def _pipeline(wl, data, w, lam, device, graph=False, gate="kernel"):
    import speculative_flash_decoding_b200 as sfd
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=device)
    trace = torch.zeros(3, dtype=torch.int64, device=device)
    if not graph:
        out = dec.decode_oproj(data["q"], data["k"], data["v"], data["seq_lens"], lam, w,
                               trace=trace, gate=gate)
        torch.cuda.synchronize()
        return {k: v.cpu() for k, v in out.items()}, trace.cpu().numpy()
    # A first call outside the capture creates the library's stream and events.
    dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], lam)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream(device)
    out = dec.alloc_outputs()
    out["y"] = torch.full((wl.B, w.shape[0]), 7.0, device=device)
    with torch.cuda.stream(stream):
        assert sfd.alspec_graph_begin(stream.cuda_stream) == 0
        dec.decode_oproj(data["q"], data["k"], data["v"], data["seq_lens"], lam, w, out=out,
                         stream=stream, trace=trace, gate=gate)
        st, g = sfd.alspec_graph_end(stream.cuda_stream)
        assert st == 0 and g
        for _ in range(2):
            trace.zero_()
            out["y"].fill_(7.0)
            assert sfd.alspec_graph_launch(g, stream.cuda_stream) == 0
        stream.synchronize()
        assert sfd.alspec_graph_destroy(g) == 0
    return {k: v.cpu() for k, v in out.items()}, trace.cpu().numpy()


@pytest.mark.parametrize("graph,gate", [(False, "kernel"), (True, "kernel"),
                                        (True, "graph_conditional")])
@pytest.mark.parametrize("lam", [0.1, 1.0])
def test_speculative_projection_with_gating(cuda_device, graph, gate, lam):
    """y = o_proj(commit ? O_spec : O_exact): against the oracle's chain, and
    exactly the projection of the device's own O_spec / O_exact rows."""
    wl = workloads.COMMIT_VARIANT.replace(L=8192, ragged=(6000, 8192))
    data = workloads.make_layer(wl, device=cuda_device)
    hidden = 1000
    w = _bf16_weights(hidden, wl.Hq * wl.d, 99, cuda_device)
    out, tr = _pipeline(wl, data, w, lam, cuda_device, graph=graph, gate=gate)
    commit = out["commit"].numpy()
    if lam == 1.0:
        assert commit.all()
    else:
        assert 0 < commit.sum() < wl.B
    w_bits = workloads.to_numpy_bits(w)
    # The device's own attention outputs, gated by its own flags.
    mine = oracle.oproj_gated(out["out_spec"].numpy().reshape(wl.B, -1),
                              out["out_exact"].numpy().reshape(wl.B, -1), commit, w_bits)
    assert _row_rel(out["y"].numpy(), mine).max() < ROW_TOL
    # The oracle's chain, for tokens whose flag is clear of the band.
    ref = oracle_decode(wl.replace(lam=lam), data)
    chain = oracle.oproj_gated(ref["out_spec"].reshape(wl.B, -1),
                               ref["out_exact"].reshape(wl.B, -1), ref["commit"], w_bits)
    clear = np.abs(ref["rel_l2"] - lam) > FLAG_BAND
    assert (commit[clear] == ref["commit"][clear]).all()
    assert _row_rel(out["y"].numpy()[clear], chain[clear]).max() < 2e-3
    # Time stamps: O_spec before O_exact; the projection's stamp is set.
    assert tr[0] > 0 and tr[1] > tr[0] and tr[2] > 0


@pytest.mark.parametrize("gate", ["kernel", "graph_conditional"])
def test_graph_with_all_committed_skips_the_recomputation(cuda_device, gate):
    """With every token committed the recomputation writes nothing: y is the
    projection of O_spec (bit-identical to the eager result)."""
    wl = workloads.COMMIT_VARIANT.replace(L=8192, ragged=(6000, 8192))
    data = workloads.make_layer(wl, device=cuda_device)
    w = _bf16_weights(512, wl.Hq * wl.d, 5, cuda_device)
    eager, _ = _pipeline(wl, data, w, 1.0, cuda_device)
    graph, _ = _pipeline(wl, data, w, 1.0, cuda_device, graph=True, gate=gate)
    for k in ("out_spec", "out_exact", "rel_l2", "commit", "y"):
        assert torch.equal(eager[k], graph[k]), k


def test_read_probe_streams_without_error(cuda_device):
    import bench
    buf = torch.empty(256 << 20, dtype=torch.uint8, device=cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    s = torch.cuda.current_stream()
    assert bench.read_probe_fn()(buf.data_ptr(), buf.numel() - 48, s.cuda_stream,
                                 err.data_ptr()) == 0
    torch.cuda.synchronize()
    assert err.item() == 0


def test_speculative_projection_over_layers_in_one_graph(cuda_device):
    """Three layers of decode + speculative projection captured in one graph
    (each layer's own weights), replayed: every layer's y is the gated
    projection of its own attention outputs."""
    import speculative_flash_decoding_b200 as sfd
    wl = workloads.COMMIT_VARIANT.replace(L=8192, ragged=(6000, 8192))
    layers = [workloads.make_layer(wl, layer=i, device=cuda_device) for i in range(3)]
    ws = [_bf16_weights(768, wl.Hq * wl.d, 50 + i, cuda_device) for i in range(3)]
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device)
    dec.decode(layers[0]["q"], layers[0]["k"], layers[0]["v"], layers[0]["seq_lens"], wl.lam)
    torch.cuda.synchronize()
    outs = []
    for _ in layers:
        o = dec.alloc_outputs()
        o["y"] = torch.full((wl.B, 768), 7.0, device=cuda_device)
        outs.append(o)
    stream = torch.cuda.Stream(cuda_device)
    with torch.cuda.stream(stream):
        assert sfd.alspec_graph_begin(stream.cuda_stream) == 0
        for d, o, w in zip(layers, outs, ws):
            dec.decode_oproj(d["q"], d["k"], d["v"], d["seq_lens"], wl.lam, w, out=o,
                             stream=stream)
        st, g = sfd.alspec_graph_end(stream.cuda_stream)
        assert st == 0 and g
        for _ in range(2):
            assert sfd.alspec_graph_launch(g, stream.cuda_stream) == 0
        stream.synchronize()
        assert sfd.alspec_graph_destroy(g) == 0
    for d, o, w in zip(layers, outs, ws):
        commit = o["commit"].cpu().numpy()
        mine = oracle.oproj_gated(o["out_spec"].cpu().numpy().reshape(wl.B, -1),
                                  o["out_exact"].cpu().numpy().reshape(wl.B, -1), commit,
                                  workloads.to_numpy_bits(w))
        assert _row_rel(o["y"].cpu().numpy(), mine).max() < ROW_TOL
    assert dec.device_error() == (0, 0)


def test_projection_behind_the_merge_reads_fresh_outputs(cuda_device):
    """The projection is launched programmatically and the merge lets its
    dependents launch early: captured right behind two decodes that write
    the same O_exact buffer, each projection must see its own layer's
    O_exact (x is read only once the merge has completed), never the
    previous layer's."""
    import speculative_flash_decoding_b200 as sfd
    wl = workloads.CONFIGS[1].replace(L=16384)
    layers = [workloads.make_layer(wl, layer=i, device=cuda_device) for i in range(2)]
    kdim = wl.Hq * wl.d
    hidden = 4096
    w = _bf16_weights(hidden, kdim, 77, cuda_device)
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device)
    exact = []
    for d in layers:
        o = dec.decode(d["q"], d["k"], d["v"], d["seq_lens"], wl.lam)
        torch.cuda.synchronize()
        exact.append(o["out_exact"].cpu().numpy().reshape(wl.B, -1))
    assert _row_rel(exact[0], exact[1]).min() > 0.5
    out = dec.alloc_outputs()
    ys = [torch.full((wl.B, hidden), 7.0, device=cuda_device) for _ in layers]
    stream = torch.cuda.Stream(cuda_device)
    with torch.cuda.stream(stream):
        assert sfd.alspec_graph_begin(stream.cuda_stream) == 0
        for d, y in zip(layers, ys):
            dec.decode(d["q"], d["k"], d["v"], d["seq_lens"], wl.lam, out=out, stream=stream)
            assert sfd.alspec_oproj(out["out_exact"].data_ptr(), w.data_ptr(), y.data_ptr(), 0,
                                    wl.B, kdim, hidden, stream.cuda_stream) == 0
        st, g = sfd.alspec_graph_end(stream.cuda_stream)
        assert st == 0 and g
        w_bits = workloads.to_numpy_bits(w)
        for _ in range(3):
            for y in ys:
                y.fill_(7.0)
            assert sfd.alspec_graph_launch(g, stream.cuda_stream) == 0
            stream.synchronize()
            for y, x in zip(ys, exact):
                assert _row_rel(y.cpu().numpy(), oracle.oproj(x, w_bits)).max() < ROW_TOL
        assert sfd.alspec_graph_destroy(g) == 0
    assert dec.device_error() == (0, 0)
