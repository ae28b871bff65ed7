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


def _copy_tree(tmp_path):
    for sub in ("hash_indexed_top_b200/csrc", "profiles"):
        shutil.copytree(os.path.join(ROOT, sub), tmp_path / sub)
    return tmp_path


def test_recorded_traffic_follows_the_kernel_code(tmp_path, monkeypatch):
    root = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    summary = root / "profiles" / "c128k_step_kernels_full.txt"
    recorded = [ln for ln in summary.read_text().splitlines() if ln.startswith("traffic_per_launch select_fused")]
    assert recorded, "the summary records the select kernel's traffic"
    expect = int(recorded[0].split()[2])
    assert bench.recorded_traffic("select_fused") == expect  # committed summary matches the committed code
    src = root / "hash_indexed_top_b200" / "csrc" / "select.cuh"
    src.write_text("// a comment-only change\n" + src.read_text())
    assert bench.recorded_traffic("select_fused") == expect  # comments do not make the counters stale
    src.write_text(src.read_text() + "\nstatic int changed_code = 1;\n")
    assert bench.recorded_traffic("select_fused") is None  # a code change does
