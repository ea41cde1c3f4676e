"""Host-side logic of bench.py that needs no GPU."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_traffic_summary_matches_kernel_code():
    """The committed ncu summary carries the hash of the kernel code it was taken
    on; the hash ignores comments and whitespace but not code."""
    sys.path.insert(0, ROOT)
    import bench
    a = "int f(int x) { return x + 1; } // one\n/* two */"
    b = "int f(int x) {\n  return x + 1;  // another comment\n}"
    c = "int f(int x) { return x + 2; }"
    assert bench._code_only(a) == bench._code_only(b) != bench._code_only(c)


def test_traffic_figure_is_used_only_on_the_captured_code(monkeypatch):
    """roofline.traffic comes from the committed ncu summary only while the kernel
    sources hash to the value recorded beside the figure; otherwise it is null."""
    sys.path.insert(0, ROOT)
    import bench
    path = os.path.join(ROOT, bench.TRAFFIC_SUMMARY)
    fields = {}
    for line in open(path):
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    per_seq = float(fields["dram_bytes_per_sequence"])
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: fields["source_sha256"])
    assert bench.measured_traffic(4) == per_seq * 4
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.measured_traffic(4) is None
