"""The benchmark reports a committed ncu traffic figure only while the decode
kernel's sources are those it was captured on (CPU only)."""
from __future__ import annotations

import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_traffic_only_for_the_current_kernel_sources(tmp_path, monkeypatch):
    bench = _bench()
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "ternary_weight_linear_int8_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.KERNEL_SOURCES:
        (csrc / f).write_text(f"// {f} v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_hash()
    assert len(h) == 16
    (tmp_path / "profiles" / "p.md").write_text(
        f"kernel_sources_sha256_16: {h}\ndram_bytes_per_launch: 4513536\n")
    assert bench.profile_traffic("p.md") == 4513536.0
    # any edit of a kernel source voids the figure
    (csrc / bench.KERNEL_SOURCES[-1]).write_text("// changed\n")
    assert bench.kernel_hash() != h
    assert bench.profile_traffic("p.md") is None
    # a summary without the hash or the figure gives none
    (tmp_path / "profiles" / "q.md").write_text("dram_bytes_per_launch: 1\n")
    assert bench.profile_traffic("q.md") is None
    assert bench.profile_traffic("missing.md") is None



def test_committed_decode_profile_is_for_the_current_sources():
    """The committed summary of the headline kernel was captured on the
    sources in the tree, so the benchmark line carries its traffic figure
    (an edit of the kernel without a new capture fails here)."""
    bench = _bench()
    t = bench.profile_traffic("decode_resident_2b_m1.md")
    assert t is not None
    # the capture read the packed weights about once: algorithmic bytes of a
    # 2B layer (4,423,680 packed + 2 K + 2 N + 4) within 2 %
    assert abs(t / 4442628.0 - 1.0) < 0.02
