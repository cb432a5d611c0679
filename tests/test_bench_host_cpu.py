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


def test_highlights_summarise_the_extras():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}
    res = {"value": 4800.0, "roofline": {"frac": 0.8},
           "extras": {"prefill_int4_m2048": {"qkv": {"tflops": 1200.0, "frac_burst": 0.8},
                                             "attn_out": {"tflops": 1050.0, "frac_burst": 0.7}},
                      "int4_m64": {"qkv": {"frac_binding_roof": 0.6}},
                      "int8": {"qkv": {"M=64": {"frac_hbm": 0.5}}},
                      "quantize_int4": {"qkv": {"frac_hbm": 0.77}},
                      "sweep_70_layers_int4": {"tokens_per_s": 95.0, "frac_hbm": 0.9, "quantize_all_ms": 70.0},
                      "decode_per_launch": {"a": {"gbs": 3000.0}, "b": {"gbs": 4500.0}}}}
    h = bench.highlights(res, peaks)
    assert h["decode_step_gbs"] == 4800.0 and h["decode_frac_hbm"] == 0.8
    assert h["prefill_frac_burst_min"] == 0.7
    assert h["int4_m64_frac_binding_roof"] == {"qkv": 0.6}
    assert h["int8_m64_frac_hbm"] == {"qkv": 0.5}
    assert h["sweep_70_layers"]["tokens_per_s"] == 95.0
    assert h["decode_min_call_frac_hbm"] == 0.5
    assert bench.highlights({"value": 1.0, "roofline": {"frac": 0.1}}, peaks) == {"decode_step_gbs": 1.0,
                                                                                 "decode_frac_hbm": 0.1}
