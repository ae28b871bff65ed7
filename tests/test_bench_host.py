"""Host logic of bench.py that needs no GPU: the DRAM-traffic figure of the
roofline object is taken from the committed ncu summary only while the
kernel code it was measured on is unchanged (comments may change)."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_strip_comments_keeps_code_and_string_literals():
    src = 'int a = 1; // one\n/* block\n comment */ const char *p = "x//y/*z*/";\nint  b;'
    assert bench._strip_comments(src) == 'int a = 1; const char *p = "x//y/*z*/"; int b;'


def test_recorded_traffic_follows_the_kernel_code(tmp_path, monkeypatch):
    shutil.copytree(os.path.join(ROOT, "hash_indexed_top_b200", "csrc"), tmp_path / "hash_indexed_top_b200" / "csrc")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    summary = tmp_path / "profiles" / "c128k_step_kernels_full.txt"
    assert bench.recorded_traffic("select_fused") is None  # no summary, no figure
    summary.write_text(f"kernel sources sha256: {bench.kernel_sources_sha()}\n"
                       "traffic_per_launch select_fused_kernel 123456\n")
    assert bench.recorded_traffic("select_fused") == 123456  # taken from these kernels
    assert bench.recorded_traffic("score_hist") is None  # not measured
    src = tmp_path / "hash_indexed_top_b200" / "csrc" / "select.cuh"
    src.write_text("// a comment-only change\n" + src.read_text())
    assert bench.recorded_traffic("select_fused") == 123456  # comments do not make the counters stale
    src.write_text(src.read_text() + "\nstatic int changed_code = 1;\n")
    assert bench.recorded_traffic("select_fused") is None  # a code change does
