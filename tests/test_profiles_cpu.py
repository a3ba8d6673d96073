"""Every committed ncu summary was taken on the kernel sources as they are
now: its recorded source hash (over the files it lists) matches the files,
and it names the command that produced it."""
import glob
import os
import re
import sys

from conftest import ROOT

sys.path.insert(0, ROOT)


def _summaries():
    return sorted(glob.glob(os.path.join(ROOT, "profiles", "*_ncu.md")))


def test_profiles_exist_for_the_main_kernels():
    names = {os.path.basename(p) for p in _summaries()}
    for kernel in ("attn_fwd_kernel", "rope_apply_kernel", "temporal_kernel"):
        assert any(n.startswith(kernel) for n in names), kernel
    assert os.path.exists(os.path.join(ROOT, "profiles", "launches_c81f480.md"))


def test_profile_hashes_match_the_sources():
    import bench
    for path in _summaries():
        txt = open(path).read()
        h = re.search(r"source_hash: `(\w+)`", txt)
        files = re.search(r"source_files: `([^`]+)`", txt)
        assert h and files, path
        assert bench.kernel_source_hash(files.group(1).split(",")) == h.group(1), (
            f"{os.path.basename(path)} was captured on other sources")
        assert "--clock-control none" in txt and "```" in txt, path
