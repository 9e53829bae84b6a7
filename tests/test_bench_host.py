"""Host-side pieces of bench.py that need no GPU: the rule that attaches a committed ncu traffic
figure to a kernel only while the kernel's source is the one it was measured on, and the oracle
sample sizing of the CPU baseline."""
import hashlib
import os

import bench


def _tree(tmp_path, src_text, profile_text):
    (tmp_path / "csrc").mkdir()
    (tmp_path / "profiles").mkdir()
    (tmp_path / "csrc" / "k.cu").write_text(src_text)
    (tmp_path / "profiles" / "kern.md").write_text(profile_text)
    return hashlib.sha1(src_text.encode()).hexdigest()[:12]


def test_traffic_attached_only_for_the_measured_source(tmp_path, monkeypatch):
    sha = _tree(tmp_path, "__global__ void k() {}\n", "")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles" / "kern.md").write_text(f"x\ntraffic_bytes_per_launch: 1234 source_sha1: {sha}\n")
    assert bench.kernel_traffic("kern", ["csrc/k.cu"]) == (1234, sha)
    # one byte of the source changes: the figure no longer applies
    (tmp_path / "csrc" / "k.cu").write_text("__global__ void k() { }\n")
    traffic, new_sha = bench.kernel_traffic("kern", ["csrc/k.cu"])
    assert traffic is None and new_sha != sha


def test_traffic_absent_profile_or_line(tmp_path, monkeypatch):
    sha = _tree(tmp_path, "int x;\n", "no figure here\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("kern", ["csrc/k.cu"]) == (None, sha)
    assert bench.kernel_traffic("missing", ["csrc/k.cu"]) == (None, sha)


def test_committed_profiles_carry_a_traffic_line():
    root = os.path.dirname(bench.__file__)
    for tag in ("chunk_prefill_bf16", "decode_bf16"):
        text = open(os.path.join(root, "profiles", f"{tag}.md")).read()
        assert "traffic_bytes_per_launch:" in text and "source_sha1:" in text, tag


def test_cpu_sample_units_cover_the_batch_in_order():
    # the oracle runs the whole headline batch (about a second on 16 cores)
    assert bench.cpu_sample_units(4, 32, 16) == [(u // 32, u % 32) for u in range(128)]
    assert bench.cpu_sample_units(1, 2, 0) == [(0, 0), (0, 1)]
