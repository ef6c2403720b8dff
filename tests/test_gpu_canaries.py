"""Guard canaries: every buffer the library writes -- out_spec, out_exact,
rel_l2, commit and the workspace -- is a view into a larger buffer whose
bytes before and after it hold a known pattern; after each call the
patterns must be intact (a write out of bounds would change them).  Run
for the three schedules on shapes with ragged lengths, tails that are not a
multiple of a tile and several cluster sizes.
"""
import pytest
import torch

import workloads
from parity import assert_parity, oracle_decode

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side (keeps 256-byte alignment)
PATTERN = 0xA5


def _guarded(nbytes, device):
    buf = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device=device)
    return buf, buf[GUARD:GUARD + nbytes]


def _intact(buf, nbytes):
    return bool((buf[:GUARD] == PATTERN).all()) and bool((buf[GUARD + nbytes:] == PATTERN).all())


CASES = [
    # name, workload, lens
    ("ragged-g4", workloads.Workload("c1", B=5, Hq=16, Hkv=4, d=128, L=3001, S=4, W=300,
                                     lam=0.2, dtype="bf16", seed=11), [3001, 1, 77, 2049, 304]),
    ("fp32-g8-d64", workloads.Workload("c2", B=3, Hq=8, Hkv=1, d=64, L=1500, S=7, W=100,
                                       lam=0.2, dtype="f32", seed=12), [1500, 999, 107]),
    ("batch-12", workloads.Workload("c3", B=12, Hq=32, Hkv=8, d=128, L=1800, S=4, W=256,
                                    lam=0.2, dtype="bf16", seed=13),
     [1800, 5, 900, 1799, 261, 1024, 33, 1500, 640, 1700, 1, 1234]),
]


@pytest.mark.parametrize("schedule", ["streams", "fused", "sink_first"])
@pytest.mark.parametrize("name,wl,lens", CASES, ids=[c[0] for c in CASES])
def test_writes_stay_in_bounds(cuda_device, schedule, name, wl, lens):
    import speculative_flash_decoding_b200 as sfd
    data = workloads.make_layer(wl, device=cuda_device)
    data["lens"] = lens
    data["seq_lens"] = torch.tensor(lens, dtype=torch.int32, device=cuda_device)
    dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=cuda_device,
                      schedule=schedule)
    # The workspace: zeroed, with guards on both sides.
    ws_buf, ws = _guarded(dec.workspace_bytes, cuda_device)
    ws.zero_()
    dec.workspace = ws
    assert ws.data_ptr() % 256 == 0
    B, Hq, d = wl.B, wl.Hq, wl.d
    bufs = {}
    out = {}
    for key, shape, dtype in (("out_spec", (B, Hq, d), torch.float32),
                              ("out_exact", (B, Hq, d), torch.float32),
                              ("rel_l2", (B,), torch.float32),
                              ("commit", (B,), torch.uint8)):
        n = torch.Size(shape).numel() * torch.tensor([], dtype=dtype).element_size()
        buf, view = _guarded(n, cuda_device)
        bufs[key] = (buf, n)
        out[key] = view.view(dtype).view(shape)
    for _ in range(2):  # the second call reuses the workspace's counters
        dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam, out=out)
        torch.cuda.synchronize()
        assert _intact(ws_buf, dec.workspace_bytes), "workspace guard overwritten"
        for key, (buf, n) in bufs.items():
            assert _intact(buf, n), f"{key} guard overwritten"
    assert dec.device_error() == (0, 0)
    assert_parity({k: v.cpu() for k, v in out.items()}, oracle_decode(wl, data), wl.lam,
                  what=f"canaries {name} {schedule}")
