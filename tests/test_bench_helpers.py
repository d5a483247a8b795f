"""Host helpers of bench.py (CPU): the source hash that ties a committed ncu
summary to the kernel it was taken on, and the max-over-ranks aggregation."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_code_only_drops_comments_and_blank_lines(bench):
    src = "int a; // note\n\n/* block\n   comment */ int b;\n  // whole line\nint c;  \n"
    assert bench._code_only(src) == "int a;\n int b;\nint c;"


def test_source_hash_follows_code_not_comments(bench, tmp_path, monkeypatch):
    f = tmp_path / "k.cu"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ("k.cu",))
    f.write_text("__global__ void k() { int x = 1; }  // one\n")
    h0 = bench.kernel_source_hash()
    f.write_text("// a new header comment\n__global__ void k() { int x = 1; }  /* two */\n")
    assert bench.kernel_source_hash() == h0
    f.write_text("__global__ void k() { int x = 2; }\n")
    assert bench.kernel_source_hash() != h0


def test_profiled_traffic_needs_matching_hash_and_sparsity(bench, tmp_path, monkeypatch):
    (tmp_path / "k.cu").write_text("__global__ void k() {}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ("k.cu",))
    monkeypatch.setattr(bench, "PROFILE_SUMMARIES", {"kern": "p.md"})
    h = bench.kernel_source_hash()
    (tmp_path / "p.md").write_text(
        "- `kernel`: kern\n- `sparsity`: 0.5\n- `traffic_bytes_per_launch`: 1234\n"
        f"- `kernel_source_sha256_16`: {h}\n")
    assert bench.profiled_traffic("kern", 0.5)[0] == 1234
    assert bench.profiled_traffic("kern", 0.7)[0] is None
    (tmp_path / "k.cu").write_text("__global__ void k() { return; }\n")
    assert bench.profiled_traffic("kern", 0.5) == (None, "kernel changed since the ncu capture")
    assert bench.profiled_traffic("other", 0.5)[0] is None


def test_replica_throughput_uses_the_slowest_rank(bench):
    # every rank processed bytes_per_step each step; time = the slowest rank's
    assert bench.replica_gbs(1e9, 10, 4, 1000.0) == pytest.approx(4 * 10 * 1e9 / 1.0 / 1e9)
