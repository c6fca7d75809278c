"""The benchmark's roofline accounting, checked by hand on CPU.

The algorithmic bytes and flops per (token, head) are the numerators of the
reported roofline fractions; each is recomputed here from the tensors it
counts, so a changed formula shows up as a failed test rather than as a
silently different fraction.
"""
import json
import os

import pytest

import bench
import gdn_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_path_bytes_and_flops_at_d128_bf16():
    # q, k, v, z bf16 in (4 x 128 x 2), g and b fp32 (8), y bf16 out (128 x 2)
    assert bench.path_bytes_per_token_head(128, 2, 2) == 4 * 256 + 8 + 256 == 1288
    # per 64-token chunk and head: five 64x64x128 block products (x2 flops) and three 64x128x128
    # products, divided by the chunk's 64 tokens
    per_chunk = 5 * (2 * 64 * 64 * 128) + 3 * (2 * 64 * 128 * 128)
    assert bench.path_flops_per_token_head(128) == per_chunk // 64 == 180224


def test_headline_roofline_time():
    w = gdn_inputs.HEADLINE
    units = w.B * w.T * w.H
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else None
    p = bench.load_peaks()
    t_mem = 1288 * units / (p["hbm_gbs"] * 1e9)
    t_mma = 180224 * units / (p["bf16_tflops"] * 1e12)
    assert t_mem > t_mma  # the path is bound by HBM traffic
    if peaks is not None:
        assert t_mem * 1e6 == pytest.approx(78.5, abs=0.5)


@pytest.mark.parametrize("name,expected_bytes", [
    ("prep", 3 * 128 * 2 + 3 * 128 * 2),                      # q k v bf16 in, q^ k^ v^ fp16 out
    ("chunk", 3 * 256 + 8 + 4 * 256 + 192 + 12),              # q^ k^ v^, g b; W U Qt Kt, 3/4 Aqk, G beta log-alpha
    ("transfer", 3 * 256),                                    # W U Kt
    ("scan", 4 * 256 + 192 + 256 + 256),                      # W U Qt Kt, 3/4 Aqk, z; y
])
def test_kernel_bytes(name, expected_bytes):
    assert bench.kernel_work_per_token_head(name, 128, 2, 2)[0] == expected_bytes


def test_chunk_launch_bytes_at_the_headline():
    w = gdn_inputs.HEADLINE
    kb, kf = bench.kernel_work_per_token_head("chunk", w.d, 2, 2)
    assert kb * w.B * w.T * w.H == 787812480
    assert kf == 4 * 2 * 128 * 128  # K K^T, Q K^T, T V~, T K~ as 128-row tiles


def test_traffic_is_dropped_when_the_kernel_source_changed(monkeypatch):
    real = bench.kernel_source_sha("chunk")
    monkeypatch.setattr(bench, "kernel_source_sha", lambda name: "0" * 16 if name == "chunk" else real)
    assert bench.ncu_traffic("chunk", "wan21_480x832_81f") is None


def test_sample_text():
    w = gdn_inputs.HEADLINE
    assert bench.sample_text(w, w.T).startswith("the whole")
    assert "T=1000 instead of" in bench.sample_text(w, 1000)
