"""Host-side rules of the benchmark (no GPU): when a stored ncu traffic
figure may be reported beside a measurement."""
import hashlib

import bench


def _summary(tmp_path, workload, digest, nbytes=123456):
    p = tmp_path / "summary.md"
    p.write_text(f"text\ntraffic_workload: {workload}\ndram_bytes_per_launch: {nbytes}\n"
                 f"source_sha256: {digest}\n")
    return str(p)


def _digest(paths):
    h = hashlib.sha256()
    for f in paths:
        h.update(open(f, "rb").read())
    return h.hexdigest()


def test_stored_traffic_needs_the_same_sources_and_workload(tmp_path, monkeypatch):
    a = tmp_path / "a.cuh"
    b = tmp_path / "b.cu"
    a.write_text("kernel v1")
    b.write_text("planner v1")
    monkeypatch.setattr(bench, "KERNEL_SRCS", [str(a), str(b)])
    path = _summary(tmp_path, "w128k", _digest([a, b]))
    assert bench.stored_traffic(path, "w128k") == 123456
    # Another workload's line does not get it.
    assert bench.stored_traffic(path, "ragged") is None
    # A changed planner (or kernel) makes it stale.
    b.write_text("planner v2")
    assert bench.stored_traffic(path, "w128k") is None
    # Order matters: the digest is over the kernel file, then the planner.
    b.write_text("planner v1")
    assert bench.stored_traffic(_summary(tmp_path, "w128k", _digest([b, a])), "w128k") is None


def test_stored_traffic_missing_fields(tmp_path, monkeypatch):
    a = tmp_path / "a.cuh"
    a.write_text("k")
    monkeypatch.setattr(bench, "KERNEL_SRCS", [str(a)])
    p = tmp_path / "s.md"
    p.write_text("dram_bytes_per_launch: 5\nsource_sha256: " + _digest([a]) + "\n")
    assert bench.stored_traffic(str(p), "w") is None       # no workload line
    assert bench.stored_traffic(str(tmp_path / "none.md"), "w") is None

