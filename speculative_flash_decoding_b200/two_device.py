"""Attention-level speculation across two devices.

The pages run ALSpec on several devices: the device computing attention
publishes the speculative result, another device starts the post-attention
ops on it at once, and the verification flag later commits or discards that
work (Attention-Level Speculation, atlas.scime.ai summary, "Approach":
"static-graph dynamic-concurrency runtime with priority gating"; ICML 2025
poster page, abstract).  Here the post-attention op is the output
projection, and the two roles are two ranks of a torch.distributed group:

* the attention rank decodes (``Decoder.decode``) and, from a side stream
  that waits on the decode's ``spec_event``, sends O_spec to the projection
  rank while the exact path still runs; after the decode it sends the
  commit flags and O_exact;
* the projection rank receives O_spec and projects it at once
  (y = O_spec W^T, the speculative result), then receives the flags and
  O_exact and recomputes y on O_exact for the discarded tokens only.

Messages per layer, in this order on the pair's process group (NCCL over
NVLink between GPUs; point-to-point operations of a pair complete in issue
order): O_spec [B, H_q * d] fp32, commit [B] uint8, O_exact [B, H_q * d]
fp32.  O_exact is always sent -- B * H_q * d * 4 bytes, 16 KB per token for
Llama-3.1-8B shapes, tens of nanoseconds on NVLink 5 -- so both ranks post
the same messages without reading the flags on the host.

The decode and projection calls are parameters (``decode_fn``,
``project_fn``); by default they are this library's CUDA entry points.  So
is the transport (``send_fn`` on the attention rank, ``recv_fn`` on the
projection rank): by default torch.distributed's point-to-point ``isend``
and ``recv``.  A send is issued on the CUDA stream current at the call -- the
side stream for O_spec -- and returns a handle with ``wait()``.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import alspec as ab


def _default_project(x, w, y, skip):
    """y[b] = x[b] @ w.T for every row (skip None) or the rows with skip[b] == 0
    (alspec_oproj on the current stream)."""
    if x.device.type != "cuda":
        raise RuntimeError("the default projection needs CUDA tensors")
    B, K = x.shape
    N = w.shape[0]
    st = ab.alspec_oproj(x.data_ptr(), w.data_ptr(), y.data_ptr(),
                         skip.data_ptr() if skip is not None else 0, B, K, N,
                         torch.cuda.current_stream(x.device).cuda_stream)
    if st != ab.ALSPEC_OK:
        raise ab.AlspecError(st, "alspec_oproj")


def _isend(tensor, peer, group):
    return dist.isend(tensor, peer, group=group)


def _recv(tensor, peer, group):
    dist.recv(tensor, peer, group=group)


class AttentionRank:
    """The rank that owns the KV cache: decode, then stream the results to
    the projection rank ``peer``."""

    def __init__(self, decoder, peer: int, group=None, decode_fn=None, send_fn=None):
        self.decoder = decoder
        self.peer = peer
        self.group = group
        self.decode_fn = decode_fn
        self.send = send_fn or _isend
        self._side = None

    def step(self, q, k, v, seq_lens, lam):
        """One layer: returns the decode's outputs (device tensors) and the
        pending send handles (wait on them before reusing the outputs)."""
        cuda = q.device.type == "cuda"
        if self.decode_fn is not None:
            out = self.decode_fn(q, k, v, seq_lens, lam)
            spec_ready = None
        else:
            spec_ready = torch.cuda.Event()
            spec_ready.record()  # gives the event its CUDA handle
            out = self.decoder.decode(q, k, v, seq_lens, lam, spec_event=spec_ready)
        B = out["out_spec"].shape[0]
        works = []
        if cuda and spec_ready is not None:
            # O_spec leaves as soon as the sink-set kernel has written it.
            if self._side is None:
                self._side = torch.cuda.Stream(q.device, priority=-1)
            self._side.wait_event(spec_ready)
            with torch.cuda.stream(self._side):
                works.append(self.send(out["out_spec"].reshape(B, -1), self.peer, self.group))
            # The messages of a pair complete in issue order; the flags and
            # O_exact follow on the caller's stream, after the decode.
            torch.cuda.current_stream(q.device).wait_stream(self._side)
        else:
            works.append(self.send(out["out_spec"].reshape(B, -1).contiguous(), self.peer,
                                   self.group))
        works.append(self.send(out["commit"].contiguous(), self.peer, self.group))
        works.append(self.send(out["out_exact"].reshape(B, -1).contiguous(), self.peer,
                               self.group))
        return out, works


class ProjectionRank:
    """The rank that runs the post-attention projection speculatively."""

    def __init__(self, w_o, batch: int, kdim: int, peer: int, group=None, project_fn=None,
                 recv_fn=None):
        self.w = w_o
        self.batch = batch
        self.kdim = kdim
        self.peer = peer
        self.group = group
        self.project_fn = project_fn or _default_project
        self.recv = recv_fn or _recv

    def step(self):
        """One layer: returns (y, o_spec, commit, o_exact) as received and
        computed on this rank; y is the committed or recomputed projection."""
        dev = self.w.device
        B, K, N = self.batch, self.kdim, self.w.shape[0]
        o_spec = torch.empty(B, K, dtype=torch.float32, device=dev)
        commit = torch.empty(B, dtype=torch.uint8, device=dev)
        o_exact = torch.empty(B, K, dtype=torch.float32, device=dev)
        y = torch.empty(B, N, dtype=torch.float32, device=dev)
        self.recv(o_spec, self.peer, self.group)
        # Speculative: project O_spec for every token at once.
        self.project_fn(o_spec, self.w, y, None)
        self.recv(commit, self.peer, self.group)
        self.recv(o_exact, self.peer, self.group)
        # Verified: redo the discarded tokens' rows on O_exact.
        self.project_fn(o_exact, self.w, y, commit)
        return y, o_spec, commit, o_exact
