"""bench.py's roofline `traffic` comes from the committed ncu figures (a small JSON file beside
the summaries) only while the kernel's code is the code that was profiled: comment or layout
edits keep it, code edits drop it."""
import os

import bench


def test_code_only_drops_comments_and_layout_but_keeps_literals():
    src = 'int a = 1;  // note\n/* block\n comment */ const char* s = "//x";\nchar q = \'"\';'
    assert bench.code_only(src) == 'int a = 1; const char* s = "//x"; char q = \'"\';'


def test_traffic_follows_the_kernel_code(tmp_path, monkeypatch):
    import json
    os.makedirs(tmp_path / "k")
    os.makedirs(tmp_path / "profiles")
    (tmp_path / "k" / "kern.cu").write_text("__global__ void k() { int x = 1; }  // v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", {"kern": ["k/kern.cu"]})
    h = bench.sources_sha256("kern")
    (tmp_path / bench.TRAFFIC_FILE).write_text(json.dumps({"entries": [
        {"kernel": "kern", "workload": "wl", "traffic_bytes_per_call": 12345, "kernel_sources_sha256": h}]}))
    assert bench.measured_traffic("kern", "wl") == 12345.0
    # another workload has no figure
    assert bench.measured_traffic("kern", "other_wl") is None
    # a comment and layout change keeps the figure
    (tmp_path / "k" / "kern.cu").write_text("// header\n__global__ void k()\n{\n    int x = 1;\n}\n")
    assert bench.measured_traffic("kern", "wl") == 12345.0
    # a code change drops it
    (tmp_path / "k" / "kern.cu").write_text("__global__ void k() { int x = 2; }\n")
    assert bench.measured_traffic("kern", "wl") is None
    # no entry, no figure
    assert bench.measured_traffic("other", "wl") is None


def test_committed_traffic_file_is_well_formed():
    import json
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), bench.TRAFFIC_FILE)
    if not os.path.exists(path):
        return
    data = json.load(open(path))
    for e in data["entries"]:
        assert e["kernel"] in bench.KERNEL_SOURCES
        assert float(e["traffic_bytes_per_call"]) > 0
        assert len(e["kernel_sources_sha256"]) == 64 and e["workload"] and e["command"]
