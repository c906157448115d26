"""bench.py's roofline `traffic` comes from a committed ncu summary only while the kernel's
code is the code that was profiled: comment or layout edits keep it, code edits drop it."""
import os

import bench


def test_code_only_drops_comments_and_layout_but_keeps_literals():
    src = 'int a = 1;  // note\n/* block\n comment */ const char* s = "//x";\nchar q = \'"\';'
    assert bench.code_only(src) == 'int a = 1; const char* s = "//x"; char q = \'"\';'


def test_traffic_follows_the_kernel_code(tmp_path, monkeypatch):
    os.makedirs(tmp_path / "k")
    os.makedirs(tmp_path / "profiles")
    (tmp_path / "k" / "kern.cu").write_text("__global__ void k() { int x = 1; }  // v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", {"kern": ["k/kern.cu"]})
    monkeypatch.setattr(bench, "TRAFFIC_SUMMARIES", {"kern": "profiles/kern.md"})
    h = bench.sources_sha256("kern")
    (tmp_path / "profiles" / "kern.md").write_text(
        f"# summary\n\ntraffic_bytes_per_launch: 12345\nkernel_sources_sha256: {h}\n")
    assert bench.measured_traffic("kern") == 12345.0
    # a comment and layout change keeps the figure
    (tmp_path / "k" / "kern.cu").write_text("// header\n__global__ void k()\n{\n    int x = 1;\n}\n")
    assert bench.measured_traffic("kern") == 12345.0
    # a code change drops it
    (tmp_path / "k" / "kern.cu").write_text("__global__ void k() { int x = 2; }\n")
    assert bench.measured_traffic("kern") is None
    # no summary, no figure
    assert bench.measured_traffic("other") is None
