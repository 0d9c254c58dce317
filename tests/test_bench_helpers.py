"""bench.py's host-side helpers on CPU: the kernel-source hash that keeps a
recorded DRAM-traffic figure tied to the code it was measured on, the lookup of
that figure, and the algorithmic throughput formula."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _hash_of(tmp_path, texts, monkeypatch):
    paths = []
    for i, t in enumerate(texts):
        p = tmp_path / f"src{i}.cuh"
        p.write_text(t)
        paths.append(str(p))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", paths)
    return bench.kernel_source_hash()


def test_source_hash_ignores_comments_and_layout(tmp_path, monkeypatch):
    a = _hash_of(tmp_path, ["int f(int x) {\n  return x + 1;  // one more\n}\n", "/* two */ int g;"], monkeypatch)
    b = _hash_of(tmp_path, ["// a comment\nint f(int x)   {\n\n  return x + 1;\n}", "int g;"], monkeypatch)
    c = _hash_of(tmp_path, ["int f(int x) {\n  return x + 2;\n}\n", "int g;"], monkeypatch)
    assert a == b
    assert a != c


def test_recorded_traffic_is_tied_to_workload_and_code(monkeypatch):
    got = bench.recorded_traffic("long_context_1x32x16384x128_causal")
    assert got is None or got > 0
    assert bench.recorded_traffic("sweep_2x32x8192x128_causal") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0000000000000000")
    assert bench.recorded_traffic("long_context_1x32x16384x128_causal") is None


def test_recorded_traffic_matches_the_committed_kernels():
    """The committed record was taken on the committed backward kernel code."""
    assert bench.recorded_traffic("long_context_1x32x16384x128_causal") is not None


def test_job_throughput():
    # 2 ranks x 3 steps x 1e12 flop in 1.5 s = 4 TFLOP/s for the whole job
    assert abs(bench.job_throughput(2, 1e12, 3, 1500.0) - 4.0) < 1e-12
