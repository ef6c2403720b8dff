"""The C ABI: the library loads, exports every declared symbol, and rejects
bad arguments on the host without launching anything (no GPU needed)."""
import ctypes
import math
import os
import re

import pytest

import speculative_flash_decoding_b200 as sfd
from speculative_flash_decoding_b200 import alspec as ab

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.join(ROOT, "speculative_flash_decoding_b200")
HEADER = os.path.join(INCLUDE, "alspec.h")
# Every header under include/ and the library that implements it.
LIBRARY_OF = {"alspec.h": os.path.join(PKG, "libalspec.so"),
              "alspec_read_probe.h": os.path.join(PKG, "libalspec_read_probe.so")}


def declared_functions(header=HEADER):
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(alspec_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_surface():
    names = declared_functions()
    assert "alspec_decode" in names and "alspec_workspace_size" in names
    assert set(names) == set(ab.SIGNATURES), "binding and header disagree"


def test_every_header_has_its_library():
    assert sorted(f for f in os.listdir(INCLUDE) if f.endswith(".h")) == sorted(LIBRARY_OF)


@pytest.mark.parametrize("header", sorted(LIBRARY_OF))
def test_library_exports_every_declared_symbol(header):
    names = declared_functions(os.path.join(INCLUDE, header))
    assert names
    lib = ctypes.CDLL(LIBRARY_OF[header])
    for name in names:
        assert hasattr(lib, name), f"{os.path.basename(LIBRARY_OF[header])} does not export {name}"


def test_debug_library_exports_the_decode_surface():
    """The bounds-checked build exports exactly the decode library's symbols."""
    debug = ctypes.CDLL(os.path.join(PKG, "libalspec_debug.so"))
    for name in declared_functions():
        assert hasattr(debug, name), f"libalspec_debug.so does not export {name}"
    assert not hasattr(debug, "alspec_read_probe")


@pytest.mark.parametrize("value,library", [("debug", "libalspec_debug.so"),
                                           ("default", "libalspec.so"), ("", "libalspec.so")])
def test_library_switch(value, library):
    """ALSPEC_LIBRARY picks the library the binding loads; there is no
    fallback to another one."""
    import subprocess
    import sys
    env = dict(os.environ, ALSPEC_LIBRARY=value, PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", "import speculative_flash_decoding_b200 as s; "
                          "print(s.LIB_PATH)"], env=env, capture_output=True, text=True,
                         check=True, timeout=120)
    assert out.stdout.strip() == os.path.join(PKG, library)


def test_library_switch_rejects_unknown_values():
    import subprocess
    import sys
    env = dict(os.environ, ALSPEC_LIBRARY="cpu", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", "import speculative_flash_decoding_b200"],
                         env=env, capture_output=True, text=True, timeout=120)
    assert out.returncode != 0 and "ALSPEC_LIBRARY" in out.stderr


def test_debug_bounds_bit_is_declared():
    text = open(HEADER).read()
    assert "#define ALSPEC_DEVERR_BOUNDS 0x4u" in text
    assert sfd.ALSPEC_DEVERR_BOUNDS == 0x4


def test_decode_library_has_no_benchmark_probe():
    """The read-bandwidth probe is a measurement aid in its own library."""
    assert not hasattr(ctypes.CDLL(sfd.LIB_PATH), "alspec_read_probe")


def test_version_and_status_strings():
    assert sfd.alspec_version() == 301
    for st in range(7):
        assert sfd.alspec_status_string(st) and "unknown" not in sfd.alspec_status_string(st)
    assert "unknown" in sfd.alspec_status_string(99)


DESC = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, max_seq_len=131072, dtype="bf16")


def desc(**kw):
    d = dict(DESC)
    d.update(kw)
    return sfd.make_desc(**d)


def test_workspace_size_and_plan():
    d = desc()
    n = sfd.alspec_workspace_size(d, 4, 1024)
    assert n > 0 and n % 256 == 0
    st, plan = sfd.alspec_query_plan(d, 4, 1024)
    assert st == 0
    assert plan["c1"] % 16 == 0 and plan["c2"] % 16 == 0
    # The sink set is tiled as a sink run (1 tile) and a window run (32
    # tiles of 32 rows); n1 CTAs of c1 / 32 tiles each cover it exactly.
    tiles, per = 1 + 1024 // 32, plan["c1"] // 32
    assert plan["n1"] * per >= tiles > (plan["n1"] - 1) * per
    # Middle chunks shrink along the queue (their coverage is checked in
    # test_plan.py); the first one is the largest.
    assert 1 <= plan["n2"] <= 256 and plan["c2"] % 32 == 0
    assert 0 < plan["smem"] <= 227 * 1024 and plan["threads"] % 32 == 0
    # A fixed split size is honoured, rounded up to the engine's tile:
    # 32 tokens for the tensor-core engine, 16 for the CUDA-core engine.
    st, plan = sfd.alspec_query_plan(desc(split_tokens=1000), 4, 1024)
    assert st == 0 and plan["engine"] == ab.ALSPEC_ENGINE_TENSOR_CORES and plan["c2"] == 1024
    st, plan = sfd.alspec_query_plan(desc(split_tokens=1000, engine="cuda_cores"), 4, 1024)
    assert st == 0 and plan["engine"] == ab.ALSPEC_ENGINE_CUDA_CORES and plan["c2"] == 1008
    # fp32 caches have no tensor-core engine.
    st, _ = sfd.alspec_query_plan(desc(dtype="f32", engine="tensor_cores"), 4, 1024)
    assert st == ab.ALSPEC_ERR_UNSUPPORTED
    st, plan = sfd.alspec_query_plan(desc(dtype="f32"), 4, 1024)
    assert st == 0 and plan["engine"] == ab.ALSPEC_ENGINE_CUDA_CORES
    # Whole cache inside the sink set: no middle items at all.
    st, plan = sfd.alspec_query_plan(desc(max_seq_len=1000), 4, 1024)
    assert st == 0 and plan["n2"] == 0


@pytest.mark.parametrize("kw,S,W,code", [
    (dict(n_q_heads=30), 4, 8, ab.ALSPEC_ERR_INVALID_ARG),      # Hq % Hkv != 0
    (dict(head_dim=96), 4, 8, ab.ALSPEC_ERR_UNSUPPORTED),
    (dict(n_q_heads=96, n_kv_heads=8), 4, 8, ab.ALSPEC_ERR_UNSUPPORTED),  # g = 12
    (dict(batch=0), 4, 8, ab.ALSPEC_ERR_INVALID_ARG),
    (dict(max_seq_len=0), 4, 8, ab.ALSPEC_ERR_INVALID_ARG),
    (dict(dtype=7), 4, 8, ab.ALSPEC_ERR_INVALID_ARG),
    (dict(engine=3), 4, 8, ab.ALSPEC_ERR_INVALID_ARG),
    (dict(schedule=4), 4, 8, ab.ALSPEC_ERR_INVALID_ARG),
    (dict(schedule=-1), 4, 8, ab.ALSPEC_ERR_INVALID_ARG),
    (dict(max_seq_len=1 << 29), 4, 8, ab.ALSPEC_ERR_UNSUPPORTED),  # rows >= 2^31
    (dict(), 0, 0, ab.ALSPEC_ERR_INVALID_ARG),                  # empty sink set
    (dict(), -1, 8, ab.ALSPEC_ERR_INVALID_ARG),
])
def test_bad_descriptions(kw, S, W, code):
    d = desc(**kw)
    assert sfd.alspec_workspace_size(d, S, W) == 0
    st, _ = sfd.alspec_query_plan(d, S, W)
    assert st == code
    # alspec_decode rejects it before touching any pointer.
    fake = 1 << 20
    st = sfd.alspec_decode(d, fake, fake, fake, fake, S, W, 0.1, fake, fake, fake, fake, fake,
                           1 << 30, 0, 0, None)
    assert st == code


def test_schedules_in_the_plan_and_workspace():
    """AUTO resolves to STREAMS; each schedule reports itself; the one-launch
    schedule needs room for its sink-set item partials."""
    sizes = {}
    for name, code in (("auto", 1), ("streams", 1), ("fused", 2), ("sink_first", 3)):
        d = desc(schedule=name)
        st, plan = sfd.alspec_query_plan(d, 4, 1024)
        assert st == 0 and plan["schedule"] == code
        sizes[name] = sfd.alspec_workspace_size(d, 4, 1024)
        assert sizes[name] > 0
    assert sizes["auto"] == sizes["streams"] == sizes["sink_first"] < sizes["fused"]
    # The fused schedule merges inside its kernel: no separate merge kernel.
    assert sfd.alspec_query_plan(desc(schedule="fused"), 4, 1024)[1]["merge_c"] == 0


def _decode_with(**over):
    d = desc(max_seq_len=4096)
    fake = 1 << 20
    args = dict(q=fake, k=fake, v=fake, seq=fake, S=4, W=64, lam=0.1, os_=fake, oe=fake, r=fake,
                c=fake, ws=fake, wsb=sfd.alspec_workspace_size(d, 4, 64))
    args.update(over)
    return sfd.alspec_decode(d, args["q"], args["k"], args["v"], args["seq"], args["S"], args["W"],
                             args["lam"], args["os_"], args["oe"], args["r"], args["c"], args["ws"],
                             args["wsb"], 0)


@pytest.mark.parametrize("over,code", [
    (dict(q=0), ab.ALSPEC_ERR_INVALID_ARG),
    (dict(k=0), ab.ALSPEC_ERR_INVALID_ARG),
    (dict(seq=0), ab.ALSPEC_ERR_INVALID_ARG),
    (dict(c=0), ab.ALSPEC_ERR_INVALID_ARG),
    (dict(k=(1 << 20) + 8), ab.ALSPEC_ERR_INVALID_ARG),          # not 16-byte aligned
    (dict(lam=-0.5), ab.ALSPEC_ERR_INVALID_ARG),
    (dict(lam=math.nan), ab.ALSPEC_ERR_INVALID_ARG),
    (dict(lam=math.inf), ab.ALSPEC_ERR_INVALID_ARG),
    (dict(ws=0), ab.ALSPEC_ERR_WORKSPACE),
    (dict(wsb=256), ab.ALSPEC_ERR_WORKSPACE),
])
def test_bad_arguments_return_codes(over, code):
    assert _decode_with(**over) == code


def test_null_handles():
    assert sfd.alspec_graph_launch(0, 0) == ab.ALSPEC_ERR_INVALID_ARG
    assert sfd.alspec_graph_destroy(0) == ab.ALSPEC_ERR_INVALID_ARG
    assert sfd.alspec_workspace_init(0, 16, 0) == ab.ALSPEC_ERR_INVALID_ARG
    st, err = sfd.alspec_get_device_error(0, 1024, 0)
    assert st == ab.ALSPEC_ERR_INVALID_ARG


@pytest.mark.parametrize("trace,code", [(0, ab.ALSPEC_ERR_INVALID_ARG),
                                        ((1 << 20) + 4, ab.ALSPEC_ERR_INVALID_ARG)])
def test_traced_decode_rejects_bad_trace_buffer(trace, code):
    """A missing or misaligned time-stamp buffer is refused before any launch."""
    d = desc(max_seq_len=4096)
    fake = 1 << 20
    st = sfd.alspec_decode_traced(d, fake, fake, fake, fake, 4, 64, 0.1, fake, fake, fake, fake,
                                  fake, sfd.alspec_workspace_size(d, 4, 64), 0, trace)
    assert st == code


@pytest.mark.parametrize("buf,nbytes", [(0, 1024), ((1 << 20) + 8, 1024), (1 << 20, 1000),
                                        (1 << 20, 0)])
def test_read_probe_rejects_bad_buffers(buf, nbytes):
    import bench
    assert bench.read_probe_fn()(buf, nbytes, 0) == ab.ALSPEC_ERR_INVALID_ARG


@pytest.mark.parametrize("kw", [dict(max_seq_len=0), dict(head_dim=96), dict(n_kv_heads=3)])
def test_noalloc_rejects_bad_descriptions_before_launching(kw):
    d = desc(**kw)
    fake = 1 << 20
    st = sfd.alspec_decode_noalloc(d, fake, fake, fake, fake, 4, 64, 0.1, fake, fake, fake, fake,
                                   0)
    assert st in (ab.ALSPEC_ERR_INVALID_ARG, ab.ALSPEC_ERR_UNSUPPORTED)


def test_noalloc_error_getter_needs_an_output():
    from speculative_flash_decoding_b200 import alspec as abm
    assert abm._lib.alspec_noalloc_device_error(None, None) == ab.ALSPEC_ERR_INVALID_ARG


@pytest.mark.parametrize("ws,nbytes,ms", [(0, 4096, 1), (1 << 20, 4096, 0), (1 << 20, 4096, 20000),
                                          (1 << 20, 4, 1), ((1 << 20) + 4, 4096, 1)])
def test_wait_timeout_hook_rejects_bad_arguments(ws, nbytes, ms):
    assert sfd.alspec_test_wait_timeout(ws, nbytes, ms, 0) == ab.ALSPEC_ERR_INVALID_ARG
