"""The roofline's DRAM traffic comes from the committed ncu summary only while that summary
was taken on the kernel code as it is now (CPU only)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_digest_ignores_comments_and_whitespace():
    a = "int f(int x) {\n  return x + 1;  // one\n}\n/* block\n comment */\n"
    b = "int f(int x){return x+1;}\n// other comment\n"
    c = "int f(int x){return x+2;}\n"
    assert bench.code_digest_text(a) == bench.code_digest_text(b)
    assert bench.code_digest_text(a) != bench.code_digest_text(c)
    assert len(bench.code_digest(bench.GEMV_SOURCE)) == 16


def test_traffic_only_for_matching_code():
    lines = ["# summary\n", "traffic_bytes_per_launch: 1234\n", "kernel_code_digest: abcdef0123456789\n"]
    assert bench.traffic_from_summary(lines, "abcdef0123456789") == (1234, None)
    t, note = bench.traffic_from_summary(lines, "0000000000000000")
    assert t is None and "1234" in note
    assert bench.traffic_from_summary(lines[:2], "abcdef0123456789")[0] is None      # no digest line
    assert bench.traffic_from_summary(["traffic_bytes_per_launch: x\n"], "a")[0] is None


def test_committed_summary_parses():
    with open(bench.GEMV_PROFILE) as f:
        lines = f.readlines()
    t, note = bench.traffic_from_summary(lines, "?")
    assert t is None and note.startswith("the ncu counters (")
