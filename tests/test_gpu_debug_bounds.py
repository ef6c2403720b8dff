"""The bounds-checked debug build (libalspec_debug.so: the same sources with
ALSPEC_DEBUG_BOUNDS, where an index outside its buffer sets
ALSPEC_DEVERR_BOUNDS and the access is skipped).  On valid inputs spanning
the kernels' configurations -- both engines, head sizes 64 and 128, every
schedule, ragged batches with sequences shorter than the sink set, a batch
wide enough for the cluster merge and one of more than 32 sequences -- no
check fires, and the outputs are bit-identical to the normal build's.

Each build runs in its own process (ALSPEC_LIBRARY selects the library)."""
import os
import subprocess
import sys
import textwrap

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = textwrap.dedent('''
    import sys
    import torch
    import workloads
    import speculative_flash_decoding_b200 as sfd

    assert sfd.LIB_PATH.endswith(sys.argv[2]), sfd.LIB_PATH
    dev = torch.device("cuda:0")
    C = workloads.CONFIGS
    cases = {
        "tiny_f32_cuda_cores": (C[0], "auto", "auto"),
        "bf16_d64_tensor_cores": (C[1].replace(d=64, L=8192, Hq=16, Hkv=4), "auto", "auto"),
        "bf16_d128_cuda_cores": (C[1].replace(L=6144), "auto", "cuda_cores"),
        "l8k_auto": (C[1].replace(L=8192), "auto", "auto"),
        "l8k_fused": (C[1].replace(L=8192), "fused", "auto"),
        "l8k_sink_first": (C[1].replace(L=8192), "sink_first", "auto"),
        "ragged_short_cluster_merge": (C[3].replace(L=12288, ragged=(600, 12288)), "auto", "auto"),
        "ragged_fused": (C[3].replace(L=12288, ragged=(600, 12288)), "fused", "auto"),
        "batch40": (C[1].replace(B=40, Hq=8, Hkv=2, L=3072, ragged=(900, 3072),
                                  needles=("pair_frac", 0.1)), "auto", "auto"),
        "gqa8_70b_shape": (C[4].replace(B=2, L=16384), "auto", "auto"),
    }
    out = {}
    for name, (wl, schedule, engine) in cases.items():
        data = workloads.make_layer(wl, device=dev)
        dec = sfd.Decoder(wl.B, wl.Hq, wl.Hkv, wl.d, wl.L, wl.dtype, wl.S, wl.W, device=dev,
                          schedule=schedule, engine=engine)
        res = {}
        for rep in range(2):
            o = dec.decode(data["q"], data["k"], data["v"], data["seq_lens"], wl.lam)
            torch.cuda.synchronize()
            res = {k: v.cpu() for k, v in o.items()}
        st, err = dec.device_error()
        res["device_error"] = torch.tensor([st, err])
        out[name] = res
    torch.save(out, sys.argv[1])
''')


def _run(tmp_path, library):
    script = tmp_path / "run_cases.py"
    script.write_text(SCRIPT)
    dst = tmp_path / f"{library}.pt"
    env = dict(os.environ, ALSPEC_LIBRARY=library,
               PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    lib = "libalspec_debug.so" if library == "debug" else "libalspec.so"
    subprocess.run([sys.executable, str(script), str(dst), lib], check=True, env=env, cwd=ROOT,
                   timeout=600)
    return torch.load(dst)


def test_debug_build_reports_nothing_and_matches_the_normal_build(tmp_path):
    debug = _run(tmp_path, "debug")
    normal = _run(tmp_path, "default")
    assert debug.keys() == normal.keys()
    for name in debug:
        st, err = debug[name]["device_error"].tolist()
        assert (st, err) == (0, 0), f"{name}: device error word {err:#x}"
        assert normal[name]["device_error"].tolist() == [0, 0], name
        for k in ("out_spec", "out_exact", "rel_l2", "commit"):
            assert torch.equal(debug[name][k], normal[name][k]), f"{name}: {k}"
