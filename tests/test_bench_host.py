"""Host-side logic of bench.py that decides whether a profile's DRAM traffic
still applies to the kernel being timed (CPU only)."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("kda_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_code_only_drops_comments_and_layout(bench):
    a = "int a = 1;  // one\n/* block\n comment */ float b =\n 2.0f;\n"
    b = "int a = 1;\nfloat b = 2.0f;   // two\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(a.replace("1;", "3;"))


def test_code_only_keeps_literals(bench):
    src = 'const char* s = "a // not a comment /* nor this */"; char c = \'/\'; char e = \'\\\'\';'
    out = bench._code_only(src)
    assert '"a // not a comment /* nor this */"' in out
    assert "'/'" in out and "'\\''" in out


def _profile(path, sha, traffic):
    with open(path, "w") as f:
        f.write(f"# summary\n\ntraffic_bytes_per_launch = {traffic}\nkernel_source_sha256 = {sha}\n")


def test_recorded_traffic_only_for_matching_code(bench, tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("__global__ void k() { int x = 1; }  // v1\n")
    monkeypatch.setattr(bench, "KERNEL_SOURCES", [str(src)])
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    prof = tmp_path / "profiles" / "kda_fwd_w.md"
    sha = bench.kernel_source_sha()
    _profile(prof, sha, 1234)
    assert bench.recorded_traffic("kda_fwd_w") == 1234.0
    # a comment-only edit keeps the counters valid
    src.write_text("// header\n__global__ void k() {\n  int x = 1;\n}\n")
    assert bench.kernel_source_sha() == sha
    assert bench.recorded_traffic("kda_fwd_w") == 1234.0
    # a code edit makes them stale
    src.write_text("__global__ void k() { int x = 2; }\n")
    assert bench.recorded_traffic("kda_fwd_w") is None
    # no summary for the workload: nothing to report
    assert bench.recorded_traffic("kda_fwd_other") is None


def test_recorded_traffic_hashes_only_the_named_sources(bench, tmp_path, monkeypatch):
    csrc = tmp_path / "csrc"
    csrc.mkdir()
    (csrc / "a.cuh").write_text("int a = 1;\n")
    (csrc / "b.cuh").write_text("int b = 1;\n")
    monkeypatch.setattr(bench, "CSRC", str(csrc))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    sha = bench.kernel_source_sha(["a.cuh"])
    with open(tmp_path / "profiles" / "kda_decode_w.md", "w") as f:
        f.write(f"traffic_bytes_per_launch = 99\nkernel_sources = a.cuh\nkernel_source_sha256 = {sha}\n")
    assert bench.recorded_traffic("kda_decode_w") == 99.0
    (csrc / "b.cuh").write_text("int b = 2;\n")    # another kernel's source: still valid
    assert bench.recorded_traffic("kda_decode_w") == 99.0
    (csrc / "a.cuh").write_text("int a = 2;\n")    # its own source: stale
    assert bench.recorded_traffic("kda_decode_w") is None
