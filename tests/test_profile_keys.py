"""The bench line's `roofline.traffic` comes from a committed ncu summary keyed by a hash of the
kernel's code: edits of comments or layout keep the key, any code change drops it (CPU only)."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

FILES = ("mk_kernel.cu", "mk_common.h", "mk_kernel.h")


def _copy_tree(dst):
    d = os.path.join(dst, "bandwidth_bound_b200", "csrc")
    os.makedirs(d)
    for f in FILES:
        shutil.copy(os.path.join(ROOT, "bandwidth_bound_b200", "csrc", f), d)
    return d


def test_hash_ignores_comments_and_layout(tmp_path):
    d = _copy_tree(str(tmp_path))
    before = bench.kernel_source_hash(str(tmp_path))
    assert before == bench.kernel_source_hash()
    p = os.path.join(d, "mk_kernel.cu")
    src = open(p).read()
    src = "// a new leading comment\n/* and a block\n   comment */\n" + src.replace("\n", "\n\n", 5)
    open(p, "w").write(src)
    assert bench.kernel_source_hash(str(tmp_path)) == before


def test_hash_follows_code_changes(tmp_path):
    d = _copy_tree(str(tmp_path))
    before = bench.kernel_source_hash(str(tmp_path))
    p = os.path.join(d, "mk_common.h")
    open(p, "a").write("\nconstexpr int kUnusedForTheTest = 1;\n")
    assert bench.kernel_source_hash(str(tmp_path)) != before


def test_committed_traffic_summary_is_plausible():
    t = bench.traffic_from_profile("llama3-8b-b8")
    if t is None:
        import pytest

        pytest.skip("the committed traffic summary was taken on other kernel code (the bench reports null)")
    # every weight and KV byte crosses HBM once: within a few percent of the workload's
    # algorithmic bytes (17.157 GB), never below them
    assert 17.157e9 <= t <= 1.05 * 17.157e9
