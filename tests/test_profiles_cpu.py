"""Committed ncu summaries: each names the command that produced it (with
--clock-control none) and records the hash of the kernel sources it was taken
on; bench.py reads a summary's DRAM traffic only while that hash matches the
current sources, so counters of an older kernel never reach a bench line."""
import glob
import os
import re
import sys

from conftest import ROOT

sys.path.insert(0, ROOT)


def _summaries():
    return sorted(glob.glob(os.path.join(ROOT, "profiles", "*_ncu.md")))


def _fields(path):
    txt = open(path).read()
    h = re.search(r"source_hash: `(\w+)`", txt)
    files = re.search(r"source_files: `([^`]+)`", txt)
    return txt, h, files


def test_profiles_exist_for_the_main_kernels():
    names = {os.path.basename(p) for p in _summaries()}
    for kernel in ("attn_fwd_kernel", "rope_apply_kernel", "temporal_tc_kernel"):
        assert any(n.startswith(kernel) for n in names), kernel
    assert os.path.exists(os.path.join(ROOT, "profiles", "launches_c81f480.md"))


def test_summaries_name_their_command_and_sources():
    for path in _summaries():
        txt, h, files = _fields(path)
        assert h and files, path
        assert "--clock-control none" in txt and "```" in txt, path
        for f in files.group(1).split(","):
            assert os.path.exists(os.path.join(ROOT, "full_spatiotemporal_attention_b200", "csrc", f)), f


def test_traffic_is_read_only_from_current_summaries():
    import bench
    for path in _summaries():
        _, h, files = _fields(path)
        m = re.match(r"(.+)_([a-z0-9]+)_ncu\.md$", os.path.basename(path))
        kernel, workload = m.group(1), m.group(2)
        current = bench.kernel_source_hash(files.group(1).split(",")) == h.group(1)
        traffic = bench.recorded_traffic(kernel, workload)
        if current:
            assert traffic is not None and traffic > 0, path
        else:
            assert traffic is None, path


def test_source_hash_ignores_comments(tmp_path, monkeypatch):
    import bench
    a = "int f(int x) { return x + 1; }  // one\n/* block\n comment */\n"
    b = "int f(int x)   {\n  return x + 1;\n}\n// another comment\n"
    c = "int f(int x) { return x + 2; }\n"
    assert bench.strip_comments(a) == bench.strip_comments(b)
    assert bench.strip_comments(a) != bench.strip_comments(c)
