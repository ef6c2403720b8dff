"""The C ABI from C: tests/c/abi_host.c is compiled against include/alspec.h
with gcc and linked to the in-tree libalspec.so; its view of the descriptor
size, the plans of the four schedules, the argument checks and a status
string must equal the ctypes binding's (host-only calls: no GPU needed)."""
import ctypes
import os
import shutil
import subprocess

import pytest

import speculative_flash_decoding_b200 as sfd
from speculative_flash_decoding_b200 import alspec as ab

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c_program_sees_the_same_abi(tmp_path):
    lib_dir = os.path.dirname(sfd.LIB_PATH)
    exe = tmp_path / "abi_host"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"), "-L", lib_dir, "-lalspec",
                    f"-Wl,-rpath,{lib_dir}", "-o", str(exe)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr
    lines = dict(l.split(" ", 1) for l in res.stdout.strip().splitlines() if " " in l)
    assert int(lines["sizeof_desc"]) == ctypes.sizeof(ab.alspec_desc)
    assert int(lines["version"]) == sfd.alspec_version()
    got = [l for l in res.stdout.splitlines() if l.startswith("schedule ")]
    assert len(got) == 4
    for line, name in zip(got, ("auto", "streams", "fused", "sink_first")):
        parts = line.split()
        assert parts[3] == "0"                               # status
        desc = sfd.make_desc(1, 32, 8, 128, 131072, "bf16", schedule=name)
        assert int(parts[5]) == sfd.alspec_workspace_size(desc, 4, 1024)
        st, plan = sfd.alspec_query_plan(desc, 4, 1024)
        assert st == 0
        assert [int(x) for x in parts[7:]] == list(plan.values())
    assert int(lines["bad_schedule"]) == ab.ALSPEC_ERR_INVALID_ARG
    assert int(lines["bad_heads"]) == ab.ALSPEC_ERR_INVALID_ARG
    assert lines["status_string"] == sfd.alspec_status_string(ab.ALSPEC_ERR_WORKSPACE)
