"""The validity check of the committed ncu traffic counters (CPU only).

bench.py reports a kernel's DRAM traffic from profiles/ncu_traffic.json only
while the CUDA sources hash to the value stored with the capture.  The hash
ignores comments and blank lines, so that a comment edit keeps the counters,
and changes with any change to the code.
"""
import json
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

CSRC = os.path.join(ROOT, "fine_grained_fp8_token_b200", "csrc")


def _copy_tree(tmp_path):
    dst = tmp_path / "fine_grained_fp8_token_b200" / "csrc"
    shutil.copytree(CSRC, dst)
    return dst


def test_hash_of_a_copy_equals_the_tree(tmp_path):
    _copy_tree(tmp_path)
    assert bench.kernel_source_sha256(str(tmp_path)) == bench.kernel_source_sha256()


def test_comment_and_blank_line_edits_keep_the_hash(tmp_path):
    dst = _copy_tree(tmp_path)
    f = dst / "gemm.cuh"
    text = f.read_text()
    text = text.replace("namespace fgfp8 {", "// an added comment line\n\nnamespace fgfp8 {  // trailing note\n/* a block\n   comment */", 1)
    f.write_text(text)
    assert bench.kernel_source_sha256(str(tmp_path)) == bench.kernel_source_sha256()


def test_code_edits_change_the_hash(tmp_path):
    dst = _copy_tree(tmp_path)
    f = dst / "gemm.cuh"
    text = f.read_text()
    assert "constexpr int kScaleAhead = 2;" in text
    f.write_text(text.replace("constexpr int kScaleAhead = 2;", "constexpr int kScaleAhead = 3;", 1))
    assert bench.kernel_source_sha256(str(tmp_path)) != bench.kernel_source_sha256()


def test_a_new_source_file_changes_the_hash(tmp_path):
    dst = _copy_tree(tmp_path)
    (dst / "extra.cuh").write_text("#pragma once\n")
    assert bench.kernel_source_sha256(str(tmp_path)) != bench.kernel_source_sha256()


def test_stale_capture_reports_no_traffic(tmp_path, monkeypatch):
    """A capture whose stored hash differs from the sources' is not reported."""
    cap = {"captures": {"w": {"dram_read_bytes": 10, "dram_write_bytes": 5, "source_sha256": "0" * 64},
                        "v": {"dram_read_bytes": 7, "dram_write_bytes": 3,
                              "source_sha256": bench.kernel_source_sha256()}}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(cap))
    shutil.copytree(CSRC, tmp_path / "fine_grained_fp8_token_b200" / "csrc")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("w") is None
    assert bench.ncu_traffic("v") == 10
    assert bench.ncu_traffic("missing") is None
