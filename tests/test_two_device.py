"""Two-device speculation protocol (speculative_flash_decoding_b200.two_device)
on CPU ranks: gloo, world size 2, the attention rank's decode computed by the
fp64 oracle and the projection rank's projection by a plain matrix product,
both injected.  Checks what the protocol owns -- which tensors cross, in
which order, and that the projection rank keeps the speculative rows of
committed tokens and recomputes the discarded ones on O_exact.  (The CUDA
entry points are the defaults of the two roles; the two-GPU path itself
needs two GPUs and is not run by these tests; the default projection is
checked on one GPU below.)
"""
import json
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LAYERS = 3
HIDDEN = 48


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload():
    import workloads
    # Strong sinks, occasional needles: the flags mix commit and discard.
    return workloads.COMMIT_VARIANT.replace(B=6, L=3000, ragged=(2000, 3000), lam=0.01)


def _weights(kdim):
    import torch
    g = torch.Generator().manual_seed(77)
    return torch.randn(HIDDEN, kdim, generator=g, dtype=torch.float32) / 16


def _rank_main(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=2)
    from speculative_flash_decoding_b200 import two_device
    import oracle
    import workloads
    wl = _workload()
    kdim = wl.Hq * wl.d
    w = _weights(kdim)
    record = []
    if rank == 0:
        def decode_fn(q, k, v, seq_lens, lam):
            r = oracle.decode(workloads.to_numpy_bits(q), workloads.to_numpy_bits(k),
                              workloads.to_numpy_bits(v), seq_lens.numpy(), wl.S, wl.W, lam)
            return dict(out_spec=torch.from_numpy(r["out_spec"]).float(),
                        out_exact=torch.from_numpy(r["out_exact"]).float(),
                        rel_l2=torch.from_numpy(r["rel_l2"]).float(),
                        commit=torch.from_numpy(r["commit"].astype(np.uint8)))
        side = two_device.AttentionRank(None, peer=1, decode_fn=decode_fn)
        for layer in range(LAYERS):
            data = workloads.make_layer(wl, layer=layer)
            out, works = side.step(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam)
            for wk in works:
                wk.wait()
            os_ = out["out_spec"].reshape(wl.B, -1).double()
            oe = out["out_exact"].reshape(wl.B, -1).double()
            c = out["commit"].bool()
            expect = torch.where(c[:, None], os_ @ w.double().T, oe @ w.double().T)
            record.append(dict(commit=out["commit"].tolist(), y=expect.tolist(),
                               o_spec=os_.tolist()))
    else:
        calls = []

        def project_fn(x, wt, y, skip):
            calls.append(None if skip is None else skip.tolist())
            full = (x.double() @ wt.double().T).float()
            if skip is None:
                y.copy_(full)
            else:
                keep = skip.bool()
                y.copy_(torch.where(keep[:, None], y, full))

        side = two_device.ProjectionRank(w, wl.B, kdim, peer=0, project_fn=project_fn)
        for layer in range(LAYERS):
            y, o_spec, commit, o_exact = side.step()
            record.append(dict(commit=commit.tolist(), y=y.double().tolist(),
                               o_spec=o_spec.double().tolist(), calls=calls[-2:]))
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(record, f)


def test_speculative_projection_across_two_ranks(tmp_path):
    import torch.multiprocessing as mp
    mp.spawn(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=2, join=True)
    att = json.load(open(tmp_path / "rank0.json"))
    proj = json.load(open(tmp_path / "rank1.json"))
    assert len(att) == len(proj) == LAYERS
    mixed = False
    for a, p in zip(att, proj):
        # The flags and O_spec arrived as sent.
        assert a["commit"] == p["commit"]
        assert np.array_equal(np.float32(a["o_spec"]), np.float32(p["o_spec"]))
        # First the speculative projection of every row, then the
        # recomputation gated by the flags.
        assert p["calls"][0] is None and p["calls"][1] == a["commit"]
        # y: committed rows from O_spec, discarded rows from O_exact.
        assert np.allclose(p["y"], a["y"], rtol=1e-5, atol=1e-5)
        mixed |= 0 < sum(a["commit"]) < len(a["commit"])
    assert mixed, "the workload should mix commit and discard"


@pytest.mark.gpu
def test_default_projection_on_one_gpu(cuda_device):
    """The projection rank's default projection (alspec_oproj): every row,
    then only the rows whose skip flag is 0."""
    import torch
    from speculative_flash_decoding_b200 import two_device
    g = torch.Generator().manual_seed(3)
    B, K, N = 5, 512, 96
    x = torch.randn(B, K, generator=g).to(cuda_device)
    x2 = torch.randn(B, K, generator=g).to(cuda_device)
    w = (torch.randn(N, K, generator=g) / 16).to(torch.bfloat16).to(cuda_device)
    y = torch.empty(B, N, device=cuda_device)
    two_device._default_project(x, w, y, None)
    skip = torch.tensor([1, 0, 1, 0, 0], dtype=torch.uint8, device=cuda_device)
    two_device._default_project(x2, w, y, skip)
    torch.cuda.synchronize()
    wf = w.double()
    want = torch.where(skip.bool()[:, None], x.double() @ wf.T, x2.double() @ wf.T)
    assert torch.allclose(y.double(), want, rtol=1e-4, atol=1e-4)


class _LocalLink:
    """Same-GPU stand-in for the NCCL transport: a send copies its tensor
    with a small kernel, on the CUDA stream current at the send (the
    attention rank's side stream for O_spec), into a buffer of its own and
    records a timing event after the copy; a receive waits for that event
    and takes the oldest message.  Point-to-point messages of a pair arrive in issue order, as
    with NCCL."""

    class _Done:
        def wait(self):
            return True

    def __init__(self):
        import collections
        self.pending = collections.deque()
        self.sent = []

    def send(self, tensor, peer, group=None):
        import torch
        buf = torch.empty_like(tensor)
        # A copy kernel on the SMs (as a send kernel would be), rather than a
        # memcpy, which the driver may hand to a copy engine.
        torch.add(tensor, 0, out=buf)
        ev = torch.cuda.Event(enable_timing=True)
        ev.record()
        self.pending.append((buf, ev))
        self.sent.append((buf, ev))
        return self._Done()

    def recv(self, tensor, peer, group=None):
        import torch
        buf, ev = self.pending.popleft()
        torch.cuda.current_stream(tensor.device).wait_event(ev)
        tensor.copy_(buf)


class _EventDecoder:
    """The library's Decoder, with timing events on every call (events [0]
    at the call's start and [4] when all of its work is complete)."""

    def __init__(self, dec):
        self.dec = dec
        self.events = None

    def decode(self, q, k, v, seq_lens, lam, spec_event=None):
        import torch
        import speculative_flash_decoding_b200 as sfd
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(sfd.ALSPEC_PROF_EVENTS)]
        for e in self.events:
            e.record()  # gives each event its CUDA handle
        return self.dec.decode(q, k, v, seq_lens, lam, spec_event=spec_event,
                               prof_events=self.events)


@pytest.mark.gpu
def test_spec_event_branch_on_one_gpu(cuda_device):
    """The attention rank with the real CUDA decoder (no decode_fn): O_spec
    leaves from the side stream at spec_event while the exact path runs.
    The received O_spec is the decoder's bit for bit, it was sent before the
    decode's work completed, and the projection rank's y follows the
    oracle's chain (project O_spec, redo discarded rows on O_exact)."""
    import torch
    import oracle
    import workloads
    import speculative_flash_decoding_b200 as sfd
    from speculative_flash_decoding_b200 import two_device
    from parity import FLAG_BAND, oracle_decode

    # Long caches (so the exact path runs well past O_spec), strong sinks and
    # a few needles (so the flags mix commit and discard).
    wl = workloads.COMMIT_VARIANT.replace(L=65536, ragged=(49152, 65536))
    hidden = 1024
    kdim = wl.Hq * wl.d
    g = torch.Generator().manual_seed(11)
    w = (torch.randn(hidden, kdim, generator=g) / 64).to(torch.bfloat16).to(cuda_device)
    link = _LocalLink()
    dec = _EventDecoder(sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W,
                                    device=cuda_device))
    att = two_device.AttentionRank(dec, peer=1, send_fn=link.send)
    proj = two_device.ProjectionRank(w, wl.B, kdim, peer=0, recv_fn=link.recv)
    # A first step outside the checked ones: the first launch of each kernel
    # loads it, and the side stream and its first buffers are created then,
    # which holds up the host, not the GPU's order of work.
    warm = workloads.make_layer(wl, layer=2, device=cuda_device)
    att.step(warm["q"], warm["k"], warm["v"], warm["seq_lens"], wl.lam)
    proj.step()
    torch.cuda.synchronize(cuda_device)
    del warm
    for layer in range(2):
        data = workloads.make_layer(wl, layer=layer, device=cuda_device)
        torch.cuda.synchronize(cuda_device)
        # Hold the stream (a bounded spin of ~10 ms) while the host enqueues
        # the step, so that the GPU's order of events, not the host's
        # enqueue latency, decides when O_spec leaves.
        torch.cuda._sleep(20_000_000)
        out, works = att.step(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam)
        for wk in works:
            wk.wait()
        (spec_buf, spec_ev), (commit_buf, _), (exact_buf, _) = link.sent[-3:]
        y, o_spec, commit, o_exact = proj.step()
        torch.cuda.synchronize(cuda_device)
        # What crossed is what the decoder wrote.
        assert torch.equal(spec_buf, out["out_spec"].reshape(wl.B, -1))
        assert torch.equal(o_spec, out["out_spec"].reshape(wl.B, -1))
        assert torch.equal(commit, out["commit"])
        assert torch.equal(o_exact, out["out_exact"].reshape(wl.B, -1))
        # O_spec was on its way before the decode's work (exact path, merge,
        # flags) was complete -- well before, with these cache lengths.
        start, spec_done, done = dec.events[0], dec.events[1], dec.events[4]
        t_spec = start.elapsed_time(spec_ev)
        t_done = start.elapsed_time(done)
        assert 0 < t_spec < 0.5 * t_done, (t_spec, start.elapsed_time(spec_done), t_done)
        # The projection rank's result against the oracle's chain.
        ref = oracle_decode(wl, data)
        assert not (np.abs(ref["rel_l2"] - wl.lam) <= FLAG_BAND).any()
        assert (commit.cpu().numpy() == ref["commit"]).all()
        assert 0 < ref["commit"].sum() < wl.B, "the flags should mix commit and discard"
        chain = oracle.oproj_gated(ref["out_spec"].reshape(wl.B, -1),
                                   ref["out_exact"].reshape(wl.B, -1), ref["commit"],
                                   workloads.to_numpy_bits(w))
        got = y.double().cpu().numpy()
        rel = np.linalg.norm(got - chain, axis=-1) / np.linalg.norm(chain, axis=-1)
        assert rel.max() < 2e-3, rel
