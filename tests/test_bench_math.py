"""The bench's algorithmic work and layer roofline against hand-computed
numbers (no GPU): a slip in the flop or byte count, or in which bound wins,
would misreport every fraction the bench prints."""
import os
import sys
import types

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    sys.path.insert(0, ROOT)
    import bench as b
    return b


def _shape(T):
    return types.SimpleNamespace(T=T, d=2048, E=128, k=8, f=768, group=64)


def test_algorithmic_work_of_the_8192_token_layer(bench):
    counts = np.full(128, 512)          # every expert touched
    w = bench.algorithmic(_shape(8192), counts)
    # 3 projections of 768 x 2048 int4 weights (half a byte each) plus a
    # (scale, bias) bf16 pair per row and 64-wide group
    assert w["per_expert"] == 3 * 768 * 2048 // 2 + 3 * 768 * 32 * 4 == 2_654_208
    assert w["touched"] == 128
    # gate and up: 2 x 2 T k d f; down: 2 T k d f
    assert w["flops"] == 6 * 8192 * 8 * 2048 * 768 == 618_475_290_624
    assert w["flops_gateup"] == 2 * w["flops_down"]
    # weights of the touched experts, x read and y written once (bf16)
    assert w["bytes"] == 128 * 2_654_208 + 2 * 8192 * 2048 * 2


def test_layer_roofline_picks_the_slower_bound(bench):
    peaks = {"bf16_tflops": 1637.9, "hbm_gbs": 7000.0, "source": "measured"}
    w = bench.algorithmic(_shape(8192), np.full(128, 512))
    r = bench.layer_roofline(w, 0.8404, peaks)
    assert r["bound"] == "tensor"
    assert abs(r["time_us"] - 618_475_290_624 / 1637.9e12 * 1e6) < 1e-6   # 377.6 us
    assert abs(r["time_us"] - 377.6) < 0.05
    assert abs(r["frac"] - r["time_us"] / 840.4) < 1e-9
    # one token: 8 experts' weights dominate, HBM-bound
    counts = np.zeros(128, int)
    counts[:8] = 1
    w1 = bench.algorithmic(_shape(1), counts)
    r1 = bench.layer_roofline(w1, 0.031, peaks)
    assert r1["bound"] == "hbm"
    assert abs(r1["time_us"] - (8 * 2_654_208 + 2 * 2048 * 2) / 7000e9 * 1e6) < 1e-9


def test_fallback_peaks(bench, tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["bf16_tflops"] == 1590.0 and p["hbm_gbs"] == 6650.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        '{"hbm_gbs": 7100.5, "bf16_tflops": 1637.9, "bf16_tflops_sustained": 1372.1}')
    p = bench.load_peaks()
    assert p["source"] == "measured" and p["bf16_tflops"] == 1637.9 and p["hbm_gbs"] == 7100.5
