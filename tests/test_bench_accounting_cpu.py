"""The bench's accounting, checked on the CPU: the FLOPs and algorithmic bytes
its roofline divides by, the peaks it divides into, and the rule that a
committed DRAM-traffic capture is reported only for the kernel source it was
taken on."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_mlp_flops_is_the_closed_form_of_the_swiglu_layer():
    # A SwiGLU MLP of hidden h and ffn f: forward 2Th(2f) + 2Tfh = 6Thf, the
    # backward twice that (dgrad + wgrad of both GEMMs): 18Thf in all.
    T, h, f = 32768, 4096, 11008
    assert bench.mlp_flops(T, h, f) == pytest.approx(18.0 * T * h * f, rel=1e-15)
    assert bench.mlp_flops(T, h, f) / 1e12 == pytest.approx(26.594, abs=5e-4)


def test_gemm_algorithmic_bytes_of_the_7b_step():
    # GB per launch as the GEMM traffic profile prints them (operands read once,
    # outputs written once, bf16): column fwd, row fwd, dgrad, dW2, dW1, dX.
    got = [b / 1e9 for b in bench.gemm_algorithmic_bytes(32768, 4096, 11008)]
    assert got == pytest.approx([2.61, 1.08, 3.24, 1.08, 1.89, 1.89], abs=0.006)
    # every launch moves at least its largest tensor
    T, h, f = 512, 256, 768
    alg = bench.gemm_algorithmic_bytes(T, h, f)
    assert all(a >= T * 2 * f * 2 for a in (alg[0], alg[2], alg[4], alg[5]))  # those touching Z / dZ
    # linear in T once the weights are subtracted
    a1 = bench.gemm_algorithmic_bytes(T, h, f)
    a2 = bench.gemm_algorithmic_bytes(2 * T, h, f)
    a3 = bench.gemm_algorithmic_bytes(3 * T, h, f)
    for x, y, z in zip(a1, a2, a3):
        assert z - y == y - x


def test_traffic_record_is_reported_only_for_its_source(monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "gemm_traffic.json")))
    assert len(rec["per_launch_bytes"]) == 6
    assert rec["bytes_per_launch"] == pytest.approx(sum(rec["per_launch_bytes"]) / 6)
    # the committed capture belongs to the committed GEMM source
    assert rec["source_sha256"] == bench.gemm_source_hash()
    got = bench.measured_traffic(rec["tokens"], rec["variant"])
    assert got is not None and got[0] == rec["bytes_per_launch"]
    assert bench.measured_traffic(rec["tokens"] // 2, rec["variant"]) is None
    assert bench.measured_traffic(rec["tokens"], "partials") is None
    monkeypatch.setattr(bench, "gemm_source_hash", lambda: "0" * 64)
    assert bench.measured_traffic(rec["tokens"], rec["variant"]) is None


def test_peaks_fall_back_and_say_so(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback"
    assert {k: p[k] for k in bench.FALLBACK_PEAKS} == bench.FALLBACK_PEAKS
    # a complete measured file is taken as it stands
    full = {"hbm_gbs": 6532.5, "bf16_tflops": 1672.3, "bf16_tflops_sustained": 1370.4}
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(full))
    p = bench.load_peaks()
    assert p["source"] == "measured" and all(p[k] == v for k, v in full.items())
    # a partial file: the missing sustained figure is scaled from the measured burst
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"bf16_tflops": 1672.3, "hbm_gbs": 0}))
    p = bench.load_peaks()
    fb = bench.FALLBACK_PEAKS
    assert p["bf16_tflops"] == 1672.3 and p["hbm_gbs"] == fb["hbm_gbs"]
    assert p["bf16_tflops_sustained"] == pytest.approx(1672.3 * fb["bf16_tflops_sustained"] / fb["bf16_tflops"])
    assert p["source"].startswith("measured (") and "hbm_gbs" in p["source"]
    # an unreadable file is the fallback
    (tmp_path / "MEASURED_PEAKS.json").write_text("{not json")
    assert bench.load_peaks()["source"] == "fallback"
