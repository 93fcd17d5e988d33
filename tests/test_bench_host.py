"""Host logic of bench.py that ties a recorded ncu figure to the code it was
taken on: the source hash ignores comments and nothing else, and a traffic
record is returned only for its own kernel, workload and hash. No GPU."""

import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_host_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_strip_comments_keeps_code_only():
    b = _bench()
    src = "int a = 1; // one\n/* block\n comment */ int b = 2;\n\n   \nint c = a + b;  /* tail */\n"
    assert b._strip_comments(src) == "int a = 1;\n int b = 2;\nint c = a + b;"


def test_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    b = _bench()
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    (tmp_path / "k.cu").write_text("__global__ void k(float* x) { x[0] = 1.f; }  // first\n")
    h0 = b.kernel_source_hash(["k.cu"])
    (tmp_path / "k.cu").write_text("// a new header\n__global__ void k(float* x) { x[0] = 1.f; }  /* second */\n")
    assert b.kernel_source_hash(["k.cu"]) == h0
    (tmp_path / "k.cu").write_text("__global__ void k(float* x) { x[0] = 2.f; }\n")
    assert b.kernel_source_hash(["k.cu"]) != h0


def test_recorded_traffic_matches_kernel_workload_and_hash(tmp_path, monkeypatch):
    b = _bench()
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    assert b.recorded_traffic("wkv4_bwd_kernel", "w", "abc") is None  # no file
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "dram_traffic.txt").write_text(
        "# kernel workload source_hash bytes_per_launch\n"
        "# wkv4_bwd_kernel w abc 1\n"
        "wkv4_bwd_kernel w abc 1772982272\n"
        "wkv4_fwd_kernel w abc 5\n")
    assert b.recorded_traffic("wkv4_bwd_kernel", "w", "abc") == 1772982272.0
    assert b.recorded_traffic("wkv4_bwd_kernel", "w", "abd") is None
    assert b.recorded_traffic("wkv4_bwd_kernel", "v", "abc") is None
    assert b.recorded_traffic("wkv4_fwd_kernel", "w", "abc") == 5.0


def test_committed_traffic_record_parses():
    """The committed record has the four fields the bench reads, for the
    bench's own workload."""
    b = _bench()
    rows = [ln.split() for ln in open(os.path.join(ROOT, "profiles", "dram_traffic.txt")) if not ln.startswith("#")]
    rows = [r for r in rows if r]
    assert rows and all(len(r) == 4 for r in rows)
    kern, workload, h, nbytes = rows[0]
    assert kern == "wkv4_bwd_kernel" and workload == b.WORKLOAD and len(h) == 16 and float(nbytes) > 0
