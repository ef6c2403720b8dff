"""The allocation-free entry point against the regular one.

alspec_decode_noalloc serves callers that cannot allocate device memory (so
cannot hand the library a workspace): it runs the same plan and the same
kernels on a fixed scratch array inside the library.  These tests call both
entry points through the C ABI on the same inputs, twice in a row (the
second call finds the scratch holding the first call's leftovers), under
each launch schedule, and require the outputs to be bit for bit the same:
the kernels reduce in fixed orders, so any difference would mean stale
scratch (counters, tickets, partials) leaking into a result.  The file is
named so that pytest collects it last.
"""
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


def _noalloc(sfd, desc, wl, data, out, stream):
    return sfd.alspec_decode_noalloc(
        desc, data["q"].data_ptr(), data["k"].data_ptr(), data["v"].data_ptr(),
        data["seq_lens"].data_ptr(), wl.S, wl.W, wl.lam, out["out_spec"].data_ptr(),
        out["out_exact"].data_ptr(), out["rel_l2"].data_ptr(), out["commit"].data_ptr(),
        stream.cuda_stream)


@pytest.mark.parametrize("schedule", ["streams", "fused", "sink_first"])
@pytest.mark.parametrize("cfg", [1, 3])
def test_noalloc_matches_decode_twice(cuda_device, cfg, schedule):
    import speculative_flash_decoding_b200 as sfd
    wl = workloads.CONFIGS[cfg].replace(L=8192 + 5, W=1024 if cfg == 1 else 512,
                                        ragged=None if cfg == 1 else (2000, 8192))
    desc = sfd.make_desc(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, schedule=schedule)
    assert 0 < sfd.alspec_workspace_size(desc, wl.S, wl.W) <= sfd.ALSPEC_NOALLOC_SCRATCH_BYTES
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device,
                      schedule=schedule)
    stream = torch.cuda.current_stream(cuda_device)
    for call in range(2):
        data = workloads.make_layer(wl, layer=call, device=cuda_device)
        ref = dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam)
        out = dec.alloc_outputs()
        for t in out.values():
            t.fill_(7)  # anything left unwritten would show
        st = _noalloc(sfd, desc, wl, data, out, stream)
        assert st == 0, sfd.alspec_status_string(st)
        torch.cuda.synchronize(cuda_device)
        for name in ("out_spec", "out_exact", "rel_l2", "commit"):
            assert torch.equal(out[name], ref[name]), (call, schedule, name)
    assert sfd.alspec_noalloc_device_error(stream.cuda_stream) == (0, 0)


def test_noalloc_device_error_word(cuda_device):
    """Lengths outside [1, max_seq_len] are clamped by the kernels and
    flagged in the scratch's error word, which the getter reads and clears."""
    import speculative_flash_decoding_b200 as sfd
    wl = workloads.CONFIGS[1].replace(B=3, L=600, W=64)
    data = workloads.make_layer(wl, device=cuda_device)
    data["seq_lens"] = torch.tensor([0, 600, 9999], dtype=torch.int32, device=cuda_device)
    desc = sfd.make_desc(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype)
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device)
    out = dec.alloc_outputs()
    stream = torch.cuda.current_stream(cuda_device)
    assert _noalloc(sfd, desc, wl, data, out, stream) == 0
    st, err = sfd.alspec_noalloc_device_error(stream.cuda_stream)
    assert st == sfd.ALSPEC_ERR_DEVICE_DATA and err == sfd.ALSPEC_DEVERR_SEQ_LEN
    assert sfd.alspec_noalloc_device_error(stream.cuda_stream) == (0, 0)  # read clears it
    # The clamped call's outputs equal the regular entry point's.
    ref = dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam)
    torch.cuda.synchronize(cuda_device)
    for name in ref:
        assert torch.equal(out[name], ref[name]), name


def test_noalloc_rejects_oversized_problem(cuda_device):
    import speculative_flash_decoding_b200 as sfd
    from speculative_flash_decoding_b200 import alspec as ab
    # 4096 sequences x 8 KV heads of 32K tokens need far more than 8 MiB of
    # partials; nothing is launched, so the pointers are never used.
    desc = sfd.make_desc(4096, 32, 8, 128, 32768 // 512, "bf16", split_tokens=16)
    need = sfd.alspec_workspace_size(desc, 4, 16)
    assert need > sfd.ALSPEC_NOALLOC_SCRATCH_BYTES
    fake = 1 << 20
    st = sfd.alspec_decode_noalloc(desc, fake, fake, fake, fake, 4, 16, 0.1, fake, fake, fake,
                                   fake, 0)
    assert st == ab.ALSPEC_ERR_WORKSPACE


def test_noalloc_rejected_call_queues_nothing(cuda_device):
    """A call refused on the host (a misaligned query here) must not touch
    the shared scratch: a correct call right after it still matches."""
    import speculative_flash_decoding_b200 as sfd
    from speculative_flash_decoding_b200 import alspec as ab
    wl = workloads.CONFIGS[1].replace(L=4096, W=256)
    data = workloads.make_layer(wl, device=cuda_device)
    desc = sfd.make_desc(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype)
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device)
    out = dec.alloc_outputs()
    stream = torch.cuda.current_stream(cuda_device)
    st = sfd.alspec_decode_noalloc(
        desc, data["q"].data_ptr() + 2, data["k"].data_ptr(), data["v"].data_ptr(),
        data["seq_lens"].data_ptr(), wl.S, wl.W, wl.lam, out["out_spec"].data_ptr(),
        out["out_exact"].data_ptr(), out["rel_l2"].data_ptr(), out["commit"].data_ptr(),
        stream.cuda_stream)
    assert st == ab.ALSPEC_ERR_INVALID_ARG
    assert _noalloc(sfd, desc, wl, data, out, stream) == 0
    ref = dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam)
    torch.cuda.synchronize(cuda_device)
    for name in ref:
        assert torch.equal(out[name], ref[name]), name
