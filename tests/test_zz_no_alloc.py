"""The allocation-free entry point against the regular one.

alspec_decode_noalloc serves callers that cannot allocate device memory (so
cannot hand the library a workspace): it runs the same kernels on a fixed
scratch array inside the library.  This test calls both entry points
through the C ABI on the same inputs, twice in a row (the second call finds
the scratch holding the first call's leftovers), and checks that the
outputs agree within the parity tolerance the other GPU tests use.  The
file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu

TOL = 1e-3  # per-head relative L2, as in the oracle parity tests


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    num = np.linalg.norm(a - b, axis=-1)
    den = np.linalg.norm(b, axis=-1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


@pytest.mark.parametrize("cfg", [1, 3])
def test_noalloc_matches_decode_twice(cuda_device, cfg):
    import speculative_flash_decoding_b200 as sfd
    wl = workloads.CONFIGS[cfg].replace(L=8192 + 5, W=1024 if cfg == 1 else 512,
                                        ragged=None if cfg == 1 else (2000, 8192))
    desc = sfd.make_desc(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype)
    assert 0 < sfd.alspec_workspace_size(desc, wl.S, wl.W) <= sfd.ALSPEC_NOALLOC_SCRATCH_BYTES
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device)
    stream = torch.cuda.current_stream(cuda_device)
    for call in range(2):
        data = workloads.make_layer(wl, layer=call, device=cuda_device)
        ref = dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam)
        out = dec.alloc_outputs()
        for t in out.values():
            t.fill_(7)  # anything left unwritten would show
        st = sfd.alspec_decode_noalloc(
            desc, data["q"].data_ptr(), data["k"].data_ptr(), data["v"].data_ptr(),
            data["seq_lens"].data_ptr(), wl.S, wl.W, wl.lam, out["out_spec"].data_ptr(),
            out["out_exact"].data_ptr(), out["rel_l2"].data_ptr(), out["commit"].data_ptr(),
            stream.cuda_stream)
        assert st == 0, sfd.alspec_status_string(st)
        torch.cuda.synchronize(cuda_device)
        for name in ("out_spec", "out_exact"):
            assert _rel(out[name], ref[name]).max() <= TOL, (call, name)
        r, r0 = out["rel_l2"].double().cpu().numpy(), ref["rel_l2"].double().cpu().numpy()
        assert np.all(np.abs(r - r0) <= TOL * (1 + r0)), (call, r, r0)
        band = np.abs(r0 - wl.lam) <= TOL
        assert (out["commit"].cpu().numpy()[~band] == ref["commit"].cpu().numpy()[~band]).all()


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
