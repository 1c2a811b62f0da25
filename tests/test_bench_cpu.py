"""Host logic of bench.py that needs no GPU: reading the DRAM traffic of a
kernel from its committed ncu summary, and refusing it once the kernel's
sources have changed since the capture."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def _summary(tmp_path, sha):
    prof = tmp_path / "profiles"
    prof.mkdir(exist_ok=True)
    (prof / "k_fwd_pp_some-workload.md").write_text(
        "# k_fwd_pp, some workload\n\n"
        f"- source_sha256_16: `{sha}` (SHA-256 over the kernel's files)\n"
        "- kernel: `k_fwd_pp<128, 0>`\n"
        "- dram_bytes_per_launch: 843183104\n")


def test_traffic_is_read_when_the_sources_match(tmp_path, monkeypatch):
    sha = bench.kernel_source_hash("k_fwd_pp")
    assert sha is not None and len(sha) == 16
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # the hash is over the real sources: compute it before moving ROOT
    monkeypatch.setattr(bench, "kernel_source_hash", lambda base: sha)
    _summary(tmp_path, sha)
    assert bench.committed_traffic("k_fwd_pp<128,0>", "some-workload") == 843183104


def test_traffic_is_null_for_stale_or_missing_summaries(tmp_path, monkeypatch):
    sha = bench.kernel_source_hash("k_fwd_pp")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda base: sha)
    _summary(tmp_path, "0" * 16)
    assert bench.committed_traffic("k_fwd_pp<128,0>", "some-workload") is None
    assert bench.committed_traffic("k_fwd_pp<128,0>", "other-workload") is None


def test_committed_summaries_parse():
    # every committed kernel summary carries a hash and a DRAM figure in the
    # form the bench reads
    prof = os.path.join(bench.ROOT, "profiles")
    seen = 0
    for name in sorted(os.listdir(prof)):
        base = next((k for k in bench.KERNEL_SOURCES if name.startswith(k + "_")), None)
        if base is None or not name.endswith(".md"):
            continue
        text = open(os.path.join(prof, name)).read()
        assert "- source_sha256_16: `" in text, name
        assert "- dram_bytes_per_launch: " in text, name
        seen += 1
    assert seen >= 1
