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
    assert bench.measured_traffic(1) is not None, "profiles summary is stale for the kernel sources"
