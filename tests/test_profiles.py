"""The committed ncu summaries and how bench.py reads them (CPU only).

Every ncu command in profiles/ leaves the GPU clocks alone
(--clock-control none), runs committed files only, and the summary gives
the figures bench.py reads: a K1 summary that names its launch shape and
source hash is used for the bench line's `traffic` only while the kernel
sources are unchanged.
"""
import os
import re
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

PROFILES = os.path.join(ROOT, "profiles")


def _summaries():
    return [os.path.join(PROFILES, f) for f in sorted(os.listdir(PROFILES)) if f.endswith((".md", ".txt"))]


def test_every_ncu_command_leaves_clocks_alone_and_runs_committed_files():
    seen = 0
    for path in _summaries():
        text = open(path, encoding="utf-8").read()
        # join continuation lines of the command blocks
        text = re.sub(r"\\\n\s*", " ", text)
        for line in text.splitlines():
            if re.match(r"\s*ncu\s+-", line):
                seen += 1
                assert "--clock-control none" in line, (path, line)
                assert "_work" not in line and "/root/" not in line, (path, line)
    assert seen >= len(_summaries())


def test_summaries_are_short_text():
    for path in _summaries():
        assert os.path.getsize(path) < 16 * 1024, path


def test_traffic_lookup_follows_shape_and_source_hash(tmp_path, monkeypatch):
    h = bench.kernel_source_hash()
    (tmp_path / "a.md").write_text("shape: k_step_tma nd=16 bucket_elems=33554432 view=replicas\n"
                                   "source_sha256_16: %s\ndram_bytes_per_element: 86.5\n" % h)
    (tmp_path / "b.md").write_text("shape: k_step_tma nd=8 bucket_elems=25000000 view=replicas\n"
                                   "source_sha256_16: 0000000000000000\ndram_bytes_per_element: 53.8\n")
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    assert bench.k1_traffic_per_elem("k_step_tma", 16, 33554432, "replicas") == 86.5
    assert bench.k1_traffic_per_elem("k_step_tma", 16, 33554432, "shards") is None
    assert bench.k1_traffic_per_elem("k_step_vec8", 16, 33554432, "replicas") is None
    # a summary of other sources is not used
    assert bench.k1_traffic_per_elem("k_step_tma", 8, 25000000, "replicas") is None


def test_default_line_summary_is_parseable():
    txt = open(os.path.join(PROFILES, "k_step_tma_sweep_nd16_64mb.md"), encoding="utf-8").read()
    assert re.search(r"^shape: k_step_tma nd=16 bucket_elems=33554432 view=replicas$", txt, re.M)
    b = float(re.search(r"dram_bytes_per_element:\s*([0-9.]+)", txt).group(1))
    assert 0.9 * 88 < b <= 88      # never above the algorithmic bytes by a re-read
