"""bench.py reports a recorded ncu traffic figure for the headline attention launch only
while the attention kernel's sources hash to the value recorded beside it. The hash
ignores comments and blank lines (they do not change the kernel) and nothing else, and
covers every file that decides the kernel's memory traffic: the kernel, its device
helpers, the tensor-map construction and the launch setup."""

import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

CSRC = os.path.join(ROOT, "block_sparse_attention_ab_b200", "csrc")


def _copy(tmp_path):
    d = tmp_path / "csrc"
    d.mkdir(parents=True)
    for f in bench.KERNEL_FILES:
        shutil.copy(os.path.join(CSRC, f), d / f)
    return d


def test_hashed_files_include_the_launch_setup_and_tensor_maps():
    assert {"attn_kernel.cu", "ab_device.cuh", "tmap_host.h", "ab_api.cu"} <= set(bench.KERNEL_FILES)


def test_record_is_used_only_while_the_hash_matches(tmp_path):
    d = _copy(tmp_path)
    rec = tmp_path / "rec.md"
    rec.write_text("# test record\n\ntraffic_bytes_per_launch: 1000\nheads_captured: 2\n"
                   f"kernel_source_sha256_16: {bench.kernel_source_hash(str(d))}\n")
    # scaled from the captured heads to the full launch
    assert bench.attn_traffic_from_profile(24, path=str(rec), csrc=str(d)) == 12000.0
    (d / "tmap_host.h").write_text((d / "tmap_host.h").read_text() + "\nstatic int x = 1;\n")
    assert bench.attn_traffic_from_profile(24, path=str(rec), csrc=str(d)) is None
    assert bench.attn_traffic_from_profile(24, path=str(tmp_path / "missing.md"), csrc=str(d)) is None


def test_comment_edits_keep_the_hash(tmp_path):
    d = _copy(tmp_path)
    h0 = bench.kernel_source_hash(str(d))
    p = d / "attn_kernel.cu"
    src = p.read_text(encoding="utf-8")
    p.write_text("// a new comment line\n\n" + src.replace("// ", "//  ", 5)
                 + "\n/* a block\n   comment */\n", encoding="utf-8")
    assert bench.kernel_source_hash(str(d)) == h0


def test_code_edits_change_the_hash(tmp_path):
    for f in ("attn_kernel.cu", "tmap_host.h", "ab_api.cu"):
        d = _copy(tmp_path / f.replace(".", "_"))
        h0 = bench.kernel_source_hash(str(d))
        p = d / f
        p.write_text(p.read_text(encoding="utf-8") + "\nstatic int hash_probe = 1;\n", encoding="utf-8")
        assert bench.kernel_source_hash(str(d)) != h0
