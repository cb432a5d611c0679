"""Host logic of bench.py that needs no GPU: the DRAM-traffic figure of the roofline is
taken from a profile summary only while the kernel sources match the captured ones."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_ratio_requires_the_captured_source(tmp_path, monkeypatch):
    csrc = tmp_path / "int8_quantized_glmq_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.DECODE_SOURCES:
        (csrc / f).write_text("// kernel source " + f)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.source_digest()
    (tmp_path / "profiles" / "k.md").write_text(
        f"# summary\nsource_digest: {digest}\ntraffic_over_algorithmic: 1.05\n")
    assert bench.profile_traffic_ratio("k") == 1.05
    (csrc / bench.DECODE_SOURCES[0]).write_text("// changed")          # the kernel changed
    assert bench.source_digest() != digest
    assert bench.profile_traffic_ratio("k") is None
    assert bench.profile_traffic_ratio("no_such_profile") is None


def test_digest_covers_every_decode_source(tmp_path, monkeypatch):
    csrc = tmp_path / "int8_quantized_glmq_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.DECODE_SOURCES:
        (csrc / f).write_text("a")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.source_digest()
    for f in bench.DECODE_SOURCES:
        (csrc / f).write_text("b")
        assert bench.source_digest() != base, f
        (csrc / f).write_text("a")
    assert bench.source_digest() == base
