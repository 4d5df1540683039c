"""Host arithmetic of bench.py's roofline fields (CPU only).

The bench line reports algorithmic bytes and FLOPs per call, the fraction of
the measured peaks, and a DRAM-traffic figure scaled from a committed ncu
record that is dropped once the kernel source differs from the captured one.
These checks pin that arithmetic against closed forms.
"""
import hashlib
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from routed_expert_ffn_fp32_b200 import synth  # noqa: E402


def test_expert_bytes_closed_form():
    # 3 projections x H x I values at 4 bits plus one scale byte per 32
    assert bench.expert_bytes(synth.DECODE64) == 3 * 4096 * 1408 * 17 // 32 == 9_191_424
    assert bench.expert_bytes(synth.FINEGRAINED) == 3 * 4096 * 2048 * 17 // 32 == 13_369_344


def test_ffn_flops_closed_form():
    cfg = synth.PREFILL
    # 2 FLOPs per multiply-add, three projections, k routed pairs plus the shared expert
    assert bench.ffn_flops(cfg, 2048) == 2 * 3 * 4096 * 2048 * 2048 * (8 + 1)


def test_activated_bytes_counts_shared_expert():
    counts = [0, 3, 0, 1]
    assert bench.activated_bytes(synth.DECODE64, counts) == 2 * bench.expert_bytes(synth.DECODE64)
    assert (bench.activated_bytes(synth.FINEGRAINED, counts)
            == 3 * bench.expert_bytes(synth.FINEGRAINED))


def test_roofline_fractions():
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "source": "test"}
    r = {"ms_ffn": 0.05, "bytes_ffn": 91.0e6}
    out = bench.roofline_of(synth.DECODE64, 5, r, peaks, uses_tc=False)
    assert out["achieved"] == pytest.approx(91.0e6 / 0.05e-3 / 1e9, abs=0.1)
    assert out["frac"] == pytest.approx(out["achieved"] / 6500.0, abs=1e-4)
    assert out["traffic"] is None and "tensor" not in out
    cfg = synth.PREFILL
    r = {"ms_ffn": 1.0, "bytes_ffn": 3.4e9}
    out = bench.roofline_of(cfg, 2048, r, peaks, uses_tc=True)
    t = out["tensor"]
    flops = bench.ffn_flops(cfg, 2048)
    assert t["achieved_tflops"] == pytest.approx(flops / 1e-3 / 1e12, abs=0.1)
    assert t["fp4_peak_tflops"] == pytest.approx(4 * 1600.0)
    # the attainable fraction: the slower of the two bounds over the time taken
    t_hbm, t_tc = 3.4e9 / 6500e9, flops / 6400e12
    assert t["attainable_frac"] == pytest.approx(max(t_hbm, t_tc) / 1e-3, abs=1e-4)
    assert t["bound_by"] == ("hbm" if t_hbm >= t_tc else "tensor")


def test_measured_traffic_scales_and_checks_the_source(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = {"source": "kernel.cu",
           "source_sha256": hashlib.sha256(src.read_bytes()).hexdigest(),
           "dram_bytes_per_call": 103, "algorithmic_bytes_per_call": 100}
    (prof / "rec.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("rec.json", 1000) == 1030
    assert bench.measured_traffic("missing.json", 1000) is None
    src.write_text("// kernel, edited after the capture\n")
    assert bench.measured_traffic("rec.json", 1000) is None


@pytest.mark.parametrize("name", ["k_ffn_mma_decode64_t5.json", "k_ffn_gemm_prefill_t2048.json"])
def test_committed_traffic_records_are_consistent(name):
    """A committed record names its kernel source and holds DRAM bytes a few
    percent to some tens of percent above its algorithmic bytes (weights read
    once, plus activations, partial rows and re-reads); never below them."""
    d = json.load(open(os.path.join(ROOT, "profiles", name)))
    assert os.path.exists(os.path.join(ROOT, d["source"]))
    ratio = d["dram_bytes_per_call"] / d["algorithmic_bytes_per_call"]
    assert 1.0 <= ratio < 1.5
