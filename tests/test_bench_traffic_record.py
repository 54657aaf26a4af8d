"""The recorded ncu traffic in profiles/attn_fwd_wan13b.md is reported by bench.py only
while the attention kernel's sources hash to the recorded value. The hash ignores
comments and blank lines (they do not change the kernel) and nothing else."""

import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

CSRC = os.path.join(ROOT, "block_sparse_attention_ab_b200", "csrc")


def _copy(tmp_path):
    d = tmp_path / "csrc"
    d.mkdir()
    for f in ("attn_kernel.cu", "ab_device.cuh"):
        shutil.copy(os.path.join(CSRC, f), d / f)
    return d


def test_record_matches_current_sources():
    assert bench.attn_traffic_from_profile() is not None


def test_comment_edits_keep_the_hash(tmp_path):
    d = _copy(tmp_path)
    h0 = bench.kernel_source_hash(str(d))
    p = d / "attn_kernel.cu"
    src = p.read_text(encoding="utf-8")
    p.write_text("// a new comment line\n\n" + src.replace("// ", "//  ", 5)
                 + "\n/* a block\n   comment */\n", encoding="utf-8")
    assert bench.kernel_source_hash(str(d)) == h0


def test_code_edits_change_the_hash(tmp_path):
    d = _copy(tmp_path)
    h0 = bench.kernel_source_hash(str(d))
    p = d / "attn_kernel.cu"
    src = p.read_text(encoding="utf-8")
    p.write_text(src + "\nstatic int hash_probe = 1;\n", encoding="utf-8")
    assert bench.kernel_source_hash(str(d)) != h0
