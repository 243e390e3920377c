"""Host logic that ties the bench line's ncu traffic to the kernels it was measured on:
the kernel-code hash ignores comments and blank lines but not code, and a traffic
entry is reported only while its hash matches the current kernel sources."""

import json
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_text_drops_comments_and_blank_lines():
    src = "// header\nint a = 1;  // trailing\n\n   \n  // indented comment\nint b = 2;\n"
    assert bench.code_text(src) == "int a = 1;\nint b = 2;"


def _copy_sources(tmp_path):
    for rel in bench.KERNEL_SOURCES:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(ROOT, rel), dst)


def test_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_hash()
    target = tmp_path / bench.KERNEL_SOURCES[1]
    text = target.read_text()
    target.write_text("// a comment-only edit\n\n" + text.replace("\n", "  // note\n", 1))
    assert bench.kernel_hash() == h0
    target.write_text(text + "\nstatic int extra_symbol;\n")
    assert bench.kernel_hash() != h0


def test_traffic_reported_only_for_matching_kernels(tmp_path, monkeypatch):
    _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    entry = {"dram_bytes_per_launch": 1234, "kernel_hash": bench.kernel_hash()}
    (tmp_path / "profiles" / "traffic.json").write_text(
        json.dumps({"some-workload": {"append_kernel": entry}}))
    assert bench.ncu_traffic("append_kernel", "some-workload") == 1234
    assert bench.ncu_traffic("decode_kernel", "some-workload") is None
    assert bench.ncu_traffic("append_kernel", "other-workload") is None
    target = tmp_path / bench.KERNEL_SOURCES[0]
    target.write_text(target.read_text() + "\nstatic int changed;\n")
    assert bench.ncu_traffic("append_kernel", "some-workload") is None
