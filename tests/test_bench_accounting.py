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
    ("prep", 3 * 128 * 2 + 3 * 128 * 2),    # raw q, k, v bf16 in; q^, k^, v^ fp16 out
    # q^ k^ v^ fp16 + g b in; W U Qt Kt fp16 out, the 96 live Aqk columns per row, G beta log-alpha
    ("chunk", 3 * 128 * 2 + 8 + 4 * 128 * 2 + 96 * 2 + 12),
    ("transfer", 3 * 128 * 2),              # W, U, Kt fp16 in
    ("scan", 4 * 128 * 2 + 96 * 2 + 128 * 2 + 128 * 2),  # W U Qt Kt, Aqk, z in; y out
    ("combine", 0),                         # per-segment states only
    ("fused_transfer", 2 * 128 * 2 + 8),    # raw k, v bf16 in; g, b fp32 in
    ("fused_out", 4 * 128 * 2 + 8 + 128 * 2),  # raw q, k, v, z bf16 in; g, b fp32 in; y bf16 out
    ("fused_combine", 0),
])
def test_kernel_bytes(name, expected_bytes):
    assert bench.kernel_work_per_token_head(name, 128, 2, 2)[0] == expected_bytes


def test_fused_kernel_flops_per_64_token_block():
    C, d = 64, 128
    gram = 2 * 128 * C * d          # [K; Q] K^T: M = 128 stacked rows, N = C, K = d
    wu = 2 * (2 * 128 * C * C)      # W^T = K^T T_w^T and U^T = V^T T_u^T: M = d, N = K = C
    delta = 2 * 128 * C * d         # Delta^T = U^T + N W^T: M = d_v, N = C, K = d_k
    state = 2 * 128 * 128 * C       # N += E Kt: M = d_v, N = d_k, K = C
    o1, o2 = 2 * 128 * C * d, 2 * 128 * C * C
    assert bench.kernel_work_per_token_head("fused_out", d, 2, 2)[1] * C == gram + wu + delta + state + o1 + o2
    assert bench.kernel_work_per_token_head("fused_transfer", d, 2, 2)[1] * C == gram + wu + 2 * (delta + state)
    # the output pass's products are exactly the method's chunk count per token-head
    assert bench.kernel_work_per_token_head("fused_out", d, 2, 2)[1] == bench.path_flops_per_token_head(d)


def test_tensor_path_kernel_flops_per_128_token_block():
    C, d = 128, 128
    # chunk: K K^T and Q K^T (C x C x d each), W = T (beta K) and U = T (beta V) (C x C x d each)
    assert bench.kernel_work_per_token_head("chunk", d, 2, 2)[1] * C == 4 * 2 * C * C * d
    # scan: W S^T and Qt S^T (C x d x d), Kt^T Delta (d x d x C), Aqk Delta (C x C x d)
    assert bench.kernel_work_per_token_head("scan", d, 2, 2)[1] * C == 4 * 2 * C * d * d
    # transfer: W [S | P]^T (C x 2d x d) and Kt^T Delta with N = 2d
    assert bench.kernel_work_per_token_head("transfer", d, 2, 2)[1] * C == 2 * 2 * C * 2 * d * d


def test_dominant_launch_units():
    class P:
        segments = 12
    w = gdn_inputs.HEADLINE
    assert bench.launch_units("scan", w, P) == w.B * w.H * w.T
    assert bench.launch_units("fused_out", w, P) == w.B * w.H * w.T
    nb = -(-w.T // 128)
    ls = -(-nb // 12)
    assert bench.launch_units("transfer", w, P) == w.H * 11 * ls * 128
    nb = -(-w.T // 64)
    ls = -(-nb // 12)
    assert bench.launch_units("fused_transfer", w, P) == w.H * 11 * ls * 64


def test_kernel_names_per_path():
    class P:
        uses_tensor_path = True
        segments = 3
    assert bench.kernel_names(P) == ("prep", "chunk", "transfer", "combine", "scan")
    assert bench.kernel_names(P, fused=True) == ("fused_transfer", "fused_combine", "fused_out")
    P.segments = 1
    assert bench.kernel_names(P) == ("prep", "chunk", "scan")
    assert bench.kernel_names(P, fused=True) == ("fused_out",)
    P.uses_tensor_path = False
    assert bench.kernel_names(P) == ("prep", "recurrence", "output")


def test_path_roofline_fraction():
    w = gdn_inputs.HEADLINE
    p = bench.load_peaks()
    r = bench.path_roofline(w, 2, 2, 0.5, p)
    assert r["bound"] == "hbm"
    assert r["frac"] == pytest.approx(r["roofline_ms"] / 0.5)
    assert r["roofline_Mtokens_s"] == pytest.approx(w.B * w.T / (r["roofline_ms"] / 1e3) / 1e6)


def test_traffic_is_dropped_when_the_kernel_source_changed(monkeypatch, tmp_path):
    real = bench.kernel_source_sha("scan")
    monkeypatch.setattr(bench, "kernel_source_sha", lambda name: "0" * 16 if name == "scan" else real)
    assert bench.ncu_traffic("scan", "wan21_480x832_81f") is None


def test_sample_text():
    w = gdn_inputs.HEADLINE
    assert bench.sample_text(w, w.T).startswith("the whole")
    assert "T=1000 instead of" in bench.sample_text(w, 1000)


def test_block_flops_per_layer():
    # x W_in^T: M = B*T rows, N = 4*H*d + 2*H, K = D; y W_out^T: M, N = D, K = H*d
    w = gdn_inputs.HEADLINE
    f_in, f_out = bench.block_flops(w, 1536)
    M = w.B * w.T
    assert f_in == 2 * M * (4 * 1536 + 2 * 12) * 1536
    assert f_out == 2 * M * 1536 * 1536
    # the T3-Video page's Table 1 counts 7.0T QKV and 2.3T O MACs over the 30 layers of Wan2.1-1.3B at
    # 480x832x81f; one layer's q, k, v and o projections here are 3 and 1 of those D x D products
    qkv_macs_per_layer = 3 * M * 1536 * 1536
    assert 30 * qkv_macs_per_layer == pytest.approx(7.0e12, rel=0.01)
    assert 30 * M * 1536 * 1536 == pytest.approx(2.3e12, rel=0.02)


def test_recorded_traffic_covers_every_forward_kernel():
    # profiles/dram_traffic.json holds one full-size capture per kernel of the tensor path; the sum is
    # the path's DRAM bytes, reported beside the method's 1288 B per token-head
    w = gdn_inputs.HEADLINE
    names = bench.KERNELS_TENSOR_SEG
    kt = [bench.ncu_traffic(n, w.name) for n in names]
    if any(x is None for x in kt):
        pytest.skip("a kernel changed since its capture")
    assert sum(kt) > bench.path_bytes_per_token_head(128, 2, 2) * w.B * w.T * w.H
    assert kt[names.index("chunk")] <= bench.kernel_work_per_token_head("chunk", 128, 2, 2)[0] * w.B * w.T * w.H


def test_backward_launch_names_and_block_gradient_flops():
    # the tensor-core backward's launches (with and without the segment passes) and the fp32 one's
    assert len(bench.backward_kernel_names(12)) == 12 and len(bench.backward_kernel_names(8)) == 8
    assert bench.backward_kernel_names(12)[9] == "bwd_grad" and bench.backward_kernel_names(8)[5] == "bwd_grad"
    assert bench.backward_kernel_names(6) == ("prep_f32", "fwd_rows", "out_bwd", "core_bwd", "tokens_bwd", "params")
    with pytest.raises(ValueError):
        bench.backward_kernel_names(7)
    # 16 products of 128 x 128 x 128 per 128-token block: at the headline (12 heads, 256 blocks each)
    assert bench.backward_grad_flops(1, 1) == 16 * 2 * 128 ** 3
    assert bench.backward_grad_flops(12, 256) == 12 * 256 * 16 * 2 * 128 ** 3
