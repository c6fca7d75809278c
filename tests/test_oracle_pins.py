"""Pins of the fp64 oracle to facts that do not come from the oracle itself:
a hand-derived worked case, closed forms, invariants the gated delta rule
fixes, special cases, and an independent algorithm (the chunked UT form) on
small inputs.  CPU only.

The invariants follow the operator as the LinMorph page names its parts
("Why learn the initialization?": update gates, decay terms, short
convolutions, normalization) and the gated delta rule (reference [57] on the
VMonarch page).
"""
import math
import os

import numpy as np
import pytest

import gdn_inputs
import oracle
from chunk_model import chunk_core

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def silu(x):
    return x / (1.0 + np.exp(-x))


def unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# ---------------------------------------------------------------- worked case
def test_golden_hand_derived_core():
    rows, S_ref = [], None
    for line in open(os.path.join(GOLDEN, "core_d2_T3.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = line.split()
        if parts[0] == "S":
            S_ref = np.array([float(x) for x in parts[1:]]).reshape(2, 2)
        else:
            rows.append([float(x) for x in parts])
    a = np.array(rows)
    T = a.shape[0]
    k = a[:, 1:3].reshape(1, T, 1, 2)
    q = a[:, 3:5].reshape(1, T, 1, 2)
    v = a[:, 5:7].reshape(1, T, 1, 2)
    al = a[:, 7].reshape(1, T, 1)
    be = a[:, 8].reshape(1, T, 1)
    o, S = oracle.core(q, k, v, al, be, return_state=True)
    np.testing.assert_allclose(o[0, :, 0] * math.sqrt(2.0), a[:, 9:11], rtol=0, atol=1e-13)
    np.testing.assert_allclose(S[0, 0], S_ref, rtol=0, atol=1e-13)


# ------------------------------------------------------------- step 1: conv
def test_conv_tap_order_and_padding():
    # x_t = t+1 on every channel, taps (0.1, 0.2, 0.3, 0.4): tap 3 multiplies the current token
    B, T, H, d = 2, 6, 1, 3
    x = np.broadcast_to(np.arange(1, T + 1, dtype=np.float32)[None, :, None, None], (B, T, H, d)).copy()
    w = np.tile(np.array([0.1, 0.2, 0.3, 0.4], np.float32), (H * d, 1))
    u = oracle.conv_silu(x, w)
    wd = w[0].astype(np.float64)
    # t = 0, 1, 2 see zero history: only the last 1, 2, 3 taps contribute
    expect_pre = [wd[3] * 1, wd[2] * 1 + wd[3] * 2, wd[1] * 1 + wd[2] * 2 + wd[3] * 3]
    expect_pre += [wd[0] * (t - 2) + wd[1] * (t - 1) + wd[2] * t + wd[3] * (t + 1) for t in range(3, T)]
    for b in range(B):  # restarts per batch item
        np.testing.assert_allclose(u[b, :, 0, 0], silu(np.array(expect_pre)), rtol=1e-14)


def test_conv_identity_and_shift():
    B, T, H, d = 2, 9, 2, 4
    x = rng.standard_normal((B, T, H, d)).astype(np.float32)
    ident = np.tile(np.array([0, 0, 0, 1], np.float32), (H * d, 1))
    shift = np.tile(np.array([0, 0, 1, 0], np.float32), (H * d, 1))
    np.testing.assert_allclose(oracle.conv_silu(x, ident), silu(x.astype(np.float64)), rtol=1e-15)
    s = oracle.conv_silu(x, shift)
    np.testing.assert_array_equal(s[:, 0], 0.0)
    np.testing.assert_allclose(s[:, 1:], silu(x[:, :-1].astype(np.float64)), rtol=1e-15)


def test_conv_is_depthwise():
    # channel c uses only its own weights and its own input channel
    B, T, H, d = 1, 7, 2, 3
    x = np.zeros((B, T, H, d), np.float32)
    x[0, 2, 1, 2] = 1.0
    w = rng.standard_normal((H * d, 4)).astype(np.float32)
    u = oracle.conv_silu(x, w)
    c = 1 * d + 2
    for t in range(T):
        for h in range(H):
            for i in range(d):
                j = 3 - (t - 2)
                pre = float(w[c, j]) if (h == 1 and i == 2 and 0 <= j <= 3) else 0.0
                assert u[0, t, h, i] == pytest.approx(silu(pre), rel=1e-15, abs=0)


# ------------------------------------------------------------ step 2: L2 norm
def test_l2_norm_unit_and_eps():
    x = rng.standard_normal((5, 16))
    y = oracle.l2norm(x, eps=0.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(y / y[:, :1], x / x[:, :1], rtol=1e-13)
    eps = 0.5
    y2 = oracle.l2norm(x, eps=eps)
    n2 = (x ** 2).sum(-1)
    np.testing.assert_allclose((y2 ** 2).sum(-1), n2 / (n2 + eps), rtol=1e-14)
    np.testing.assert_array_equal(oracle.l2norm(np.zeros((1, 8)), eps=1e-6), 0.0)


# -------------------------------------------------------------- step 3: gates
def test_gate_closed_forms():
    # g + dt_bias = 0 -> softplus = ln 2; A_log = 0 -> alpha = 1/2; A_log = ln 2 -> alpha = 1/4
    g = np.array([[[0.25, 0.25, 30.0]]], np.float32)
    b = np.array([[[0.0, 40.0, -40.0]]], np.float32)
    A_log = np.array([0.0, math.log(2.0), 0.0], np.float32)
    dt = np.array([-0.25, -0.25, 0.0], np.float32)
    alpha, beta = oracle.gates(g, b, A_log, dt)
    assert alpha[0, 0, 0] == pytest.approx(0.5, rel=1e-15)
    assert alpha[0, 0, 1] == pytest.approx(math.exp(-math.exp(float(np.float32(math.log(2.0)))) * math.log(2.0)),
                                           rel=1e-15)
    assert alpha[0, 0, 1] == pytest.approx(0.25, rel=1e-7)
    # softplus(30) = 30 + log1p(e^-30)
    assert alpha[0, 0, 2] == pytest.approx(math.exp(-(30.0 + math.log1p(math.exp(-30.0)))), rel=1e-14)
    assert beta[0, 0, 0] == 0.5
    assert beta[0, 0, 1] == pytest.approx(1.0, abs=1e-17)
    assert beta[0, 0, 2] == pytest.approx(math.exp(-40.0), rel=1e-12)
    # decay is monotone: larger g -> smaller alpha; alpha in (0, 1)
    gs = np.linspace(-20, 20, 41, dtype=np.float32).reshape(1, 41, 1)
    al, _ = oracle.gates(gs, np.zeros_like(gs), np.array([0.7], np.float32), np.array([0.0], np.float32))
    assert np.all(np.diff(al[0, :, 0]) < 0) and np.all(al > 0) and np.all(al < 1)


# ------------------------------------------------------- step 4: recurrence
def test_t1_closed_form_full_pipeline():
    # T = 1: S_0 = beta v k^T, so o = beta v (k . q) / sqrt(d_k) before the norm
    B, T, H, d = 2, 1, 3, 16
    inp = gdn_inputs.make_inputs(B, T, H, d, "f32", 0.0, seed=7)
    y, it = oracle.forward(inp, intermediates=True)
    for b in range(B):
        for h in range(H):
            wq, wk, wv = (inp[n][h * d:(h + 1) * d, 3].astype(np.float64) for n in ("conv_q", "conv_k", "conv_v"))
            qq = silu(wq * inp["q"][b, 0, h]); kk = silu(wk * inp["k"][b, 0, h]); vv = silu(wv * inp["v"][b, 0, h])
            qq = qq / math.sqrt((qq ** 2).sum() + 1e-6); kk = kk / math.sqrt((kk ** 2).sum() + 1e-6)
            x = float(inp["g"][b, 0, h]) + float(inp["dt_bias"][h])
            beta = 1.0 / (1.0 + math.exp(-float(inp["b"][b, 0, h])))
            o = beta * vv * float(kk @ qq) / math.sqrt(d)
            np.testing.assert_allclose(it["o"][b, 0, h], o, rtol=1e-12, atol=1e-300)
            yy = o / math.sqrt((o ** 2).mean() + 1e-6) * inp["norm_w"] * silu(inp["z"][b, 0, h].astype(np.float64))
            np.testing.assert_allclose(y[b, 0, h], yy, rtol=1e-12)
            assert it["alpha"][b, 0, h] == pytest.approx(
                math.exp(-math.exp(float(inp["A_log"][h])) * (max(x, 0) + math.log1p(math.exp(-abs(x))))), rel=1e-14)


def test_beta_zero_gives_zero_state_and_output():
    B, T, H, d = 1, 40, 2, 8
    q = unit(rng.standard_normal((B, T, H, d)))
    k = unit(rng.standard_normal((B, T, H, d)))
    v = rng.standard_normal((B, T, H, d))
    al = rng.uniform(0.1, 1.0, (B, T, H))
    o, S = oracle.core(q, k, v, al, np.zeros((B, T, H)), return_state=True)
    assert np.all(o == 0.0) and np.all(S == 0.0)
    # and through the full pipeline: b -> -inf makes beta exactly 0, so y = 0
    inp = gdn_inputs.make_inputs(B, T, H, d, "f32", 0.0, seed=3)
    inp["b"][:] = -1e4
    y = oracle.forward(inp)
    assert np.all(y == 0.0)


def test_orthonormal_keys_are_retrieved_exactly():
    # alpha = beta = 1 and orthonormal keys: S k_i = v_i for every key written
    d, n = 16, 12
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Qm[:, :n].T
    vals = rng.standard_normal((n, d))
    T = n
    k = keys.reshape(1, T, 1, d)
    v = vals.reshape(1, T, 1, d)
    # query at token t a random key written at or before t
    idx = [int(rng.integers(0, t + 1)) for t in range(T)]
    q = keys[idx].reshape(1, T, 1, d)
    o, S = oracle.core(q, k, v, np.ones((1, T, 1)), np.ones((1, T, 1)), return_state=True)
    np.testing.assert_allclose(o[0, :, 0] * math.sqrt(d), vals[idx], atol=1e-12)
    np.testing.assert_allclose(S[0, 0] @ keys.T, vals.T, atol=1e-12)


def test_repeated_key_returns_latest_value():
    # one key written repeatedly with beta = 1: S_t k = v_t whatever alpha is
    d, T = 8, 30
    kk = unit(rng.standard_normal(d))
    k = np.broadcast_to(kk, (1, T, 1, d)).copy()
    v = rng.standard_normal((1, T, 1, d))
    al = rng.uniform(0.05, 1.0, (1, T, 1))
    o = oracle.core(k, k, v, al, np.ones((1, T, 1)))
    np.testing.assert_allclose(o[0, :, 0] * math.sqrt(d), v[0, :, 0], atol=1e-12)


def test_pure_decay_after_single_write():
    # beta_0 = 1, beta_t = 0 afterwards: o_t = (prod_{s=1..t} alpha_s) v_0 (k_0 . q_t) / sqrt(d)
    d, T = 8, 25
    k = unit(rng.standard_normal((1, T, 1, d)))
    q = unit(rng.standard_normal((1, T, 1, d)))
    v = rng.standard_normal((1, T, 1, d))
    al = rng.uniform(0.5, 1.0, (1, T, 1))
    be = np.zeros((1, T, 1)); be[0, 0, 0] = 1.0
    o = oracle.core(q, k, v, al, be)
    for t in range(T):
        dec = np.prod(al[0, 1:t + 1, 0])
        np.testing.assert_allclose(o[0, t, 0], dec * v[0, 0, 0] * (k[0, 0, 0] @ q[0, t, 0]) / math.sqrt(d),
                                   rtol=1e-12, atol=1e-15)


def test_constant_key_geometric_sum():
    # constant unit key = query, constant alpha, beta, v:
    # x_t = S_t k = a x_{t-1} + beta v with a = alpha (1 - beta)  =>  x_t = beta v (1 - a^{t+1}) / (1 - a)
    d, T = 8, 60
    kk = unit(rng.standard_normal(d))
    vv = rng.standard_normal(d)
    alpha, beta = 0.93, 0.3
    k = np.broadcast_to(kk, (1, T, 1, d)).copy()
    v = np.broadcast_to(vv, (1, T, 1, d)).copy()
    o = oracle.core(k, k, v, np.full((1, T, 1), alpha), np.full((1, T, 1), beta))
    a = alpha * (1 - beta)
    for t in range(T):
        np.testing.assert_allclose(o[0, t, 0] * math.sqrt(d), beta * vv * (1 - a ** (t + 1)) / (1 - a), rtol=1e-12)


def test_initial_state_and_final_state_compose():
    # running [0, T) equals running [0, t0) then [t0, T) from the returned state
    B, T, H, d = 1, 50, 2, 8
    q = unit(rng.standard_normal((B, T, H, d))); k = unit(rng.standard_normal((B, T, H, d)))
    v = rng.standard_normal((B, T, H, d)); al = rng.uniform(0.3, 1, (B, T, H)); be = rng.uniform(0, 1, (B, T, H))
    o, S = oracle.core(q, k, v, al, be, return_state=True)
    t0 = 23
    o1, S1 = oracle.core(q[:, :t0], k[:, :t0], v[:, :t0], al[:, :t0], be[:, :t0], return_state=True)
    o2, S2 = oracle.core(q[:, t0:], k[:, t0:], v[:, t0:], al[:, t0:], be[:, t0:], s0=S1, return_state=True)
    np.testing.assert_allclose(np.concatenate([o1, o2], 1), o, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(S2, S, rtol=1e-12, atol=1e-15)


# ------------------------------------------------------- step 5: output norm
def test_output_norm_closed_form():
    dv = 16
    c = 0.37
    o = np.full((3, dv), c)
    z = rng.standard_normal((3, dv)).astype(np.float32)
    w = rng.uniform(0.5, 2, dv).astype(np.float32)
    eps = 1e-3
    y = oracle.output(o, z, w, eps)
    np.testing.assert_allclose(y, c / math.sqrt(c * c + eps) * w.astype(np.float64) * silu(z.astype(np.float64)),
                               rtol=1e-14)
    # scale invariance when eps = 0
    o2 = rng.standard_normal((4, dv))
    np.testing.assert_allclose(oracle.output(5.0 * o2, z[:1].repeat(4, 0), w, 0.0),
                               oracle.output(o2, z[:1].repeat(4, 0), w, 0.0), rtol=1e-13)


# ----------------------------------------------------- whole-method properties
def test_head_permutation_equivariance_and_batch_independence():
    B, T, H, d = 2, 70, 3, 16
    inp = gdn_inputs.make_inputs(B, T, H, d, "f32", 0.0, seed=11)
    y = oracle.forward(inp)
    perm = np.array([2, 0, 1])
    p = dict(inp)
    for n in ("q", "k", "v", "z"):
        p[n] = inp[n][:, :, perm]
    for n in ("g", "b"):
        p[n] = inp[n][:, :, perm]
    for n in ("conv_q", "conv_k", "conv_v"):
        p[n] = inp[n].reshape(H, d, 4)[perm].reshape(H * d, 4)
    for n in ("A_log", "dt_bias"):
        p[n] = inp[n][perm]
    np.testing.assert_array_equal(oracle.forward(p), y[:, :, perm])
    one = {n: (a[1:2] if isinstance(a, np.ndarray) and a.ndim >= 3 else a) for n, a in inp.items()}
    np.testing.assert_array_equal(oracle.forward(one), y[1:2])


def test_causality_prefix_unchanged():
    B, T, H, d = 1, 90, 2, 16
    inp = gdn_inputs.make_inputs(B, T, H, d, "f32", 0.0, seed=5)
    y = oracle.forward(inp)
    t0 = 41
    p = {n: (a.copy() if isinstance(a, np.ndarray) else a) for n, a in inp.items()}
    for n in ("q", "k", "v", "z"):
        p[n][:, t0] += 1.0
    p["g"][:, t0] -= 2.0
    p["b"][:, t0] += 2.0
    y2 = oracle.forward(p)
    np.testing.assert_array_equal(y2[:, :t0], y[:, :t0])
    assert np.abs(y2[:, t0:] - y[:, t0:]).max() > 1e-3


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 128, 129, 200])
@pytest.mark.parametrize("C", [64, 128])
def test_chunked_ut_form_equals_sequential_oracle(T, C):
    # an independent algorithm (block UT transform + inter-block state) agrees with
    # the token-by-token recurrence to fp64 rounding
    B, H, d = 1, 2, 32
    inp = gdn_inputs.make_inputs(B, T, H, d, "f32", -2.0, seed=T)
    _, it = oracle.forward(inp, intermediates=True)
    o = chunk_core(it["qh"], it["kh"], it["vh"], np.log(it["alpha"]), it["beta"], C=C)
    np.testing.assert_allclose(o, it["o"], rtol=0, atol=1e-12 * np.abs(it["o"]).max())


def test_workload_shapes_match_video_geometry():
    # T = latent frames x (H/16) x (W/16); 480x832 -> 30x52 latent plane
    names = [w.name for w in gdn_inputs.WORKLOADS]
    assert len(set(names)) == 5
    assert gdn_inputs.WORKLOADS[2].T == 32760 and gdn_inputs.WORKLOADS[2].H == 12
    assert gdn_inputs.WORKLOADS[1].T == 7800 and gdn_inputs.WORKLOADS[4].T == 126360
    assert gdn_inputs.WORKLOADS[3].T == 27280 and gdn_inputs.WORKLOADS[3].B == 2
    # the T3-Video page's Table 1 attention MACs for Wan2.1-1.3B at 480x832 (98.9T)
    # equal 2 * T^2 * d_model * layers at T = 32760, d_model = 1536, 30 layers
    assert abs(2 * 32760 ** 2 * 1536 * 30 / 1e12 - 98.9) < 0.05


@pytest.mark.parametrize("Ls", [1, 2, 3])
def test_segment_parallel_states_equal_sequential_states(Ls):
    # the segment form (per-segment transfer matrices combined afterwards) gives
    # the same state at every segment start as the token-by-token recurrence
    from chunk_model import segment_start_states
    T, d, C = 700, 16, 64
    inp = gdn_inputs.make_inputs(1, T, 1, d, "f32", -3.0, seed=Ls)
    _, it = oracle.forward(inp, intermediates=True)
    starts = segment_start_states(it["kh"][0, :, 0], it["vh"][0, :, 0], np.log(it["alpha"][0, :, 0]),
                                  it["beta"][0, :, 0], C=C, Ls=Ls)
    assert len(starts) == -(-(-(-T // C)) // Ls)
    for j, St in enumerate(starts[1:], start=1):
        t_end = j * Ls * C
        _, S = oracle.core(it["qh"][:, :t_end], it["kh"][:, :t_end], it["vh"][:, :t_end], it["alpha"][:, :t_end],
                           it["beta"][:, :t_end], return_state=True)
        np.testing.assert_allclose(St, S[0, 0].T, rtol=0, atol=1e-12 * max(1.0, np.abs(S).max()))


# ------------------------------------------------ carried state (streaming)
def test_forward_with_zero_initial_state_is_the_plain_forward():
    inp = gdn_inputs.make_inputs(1, 130, 2, 16, "f32", -1.0, seed=61)
    y, s = oracle.forward_with_state(inp)
    np.testing.assert_allclose(y, oracle.forward(inp), rtol=1e-12, atol=1e-14)
    assert s.shape == (1, 2, 16, 16)


def test_streaming_in_two_pieces_equals_one_pass():
    # g ~ N(-6, 1): alpha ~ 0.95-0.99, so the carried state dominates the second piece
    from state_util import split_stream
    inp = gdn_inputs.make_inputs(1, 300, 2, 32, "f32", -6.0, seed=62)
    y, s = oracle.forward_with_state(inp)
    p1, p2 = split_stream(inp, 170)
    y1, s1 = oracle.forward_with_state(p1)
    y2, s2 = oracle.forward_with_state(p2, s0=s1)
    np.testing.assert_allclose(y1, y[:, :170], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(y2[:, 3:], y[:, 170:], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(s2, s, rtol=1e-9, atol=1e-12)
    # without the carried state the second piece differs
    y2z, _ = oracle.forward_with_state(p2)
    assert np.abs(y2z[:, 3:] - y[:, 170:]).max() > 1e-3


# ------------------------------------------------ reverse-direction scan
def test_reverse_scan_is_anti_causal():
    # outputs at t > t0 never see token t0; the output at t0 does
    inp = gdn_inputs.make_inputs(1, 90, 2, 16, "f32", -1.0, seed=71)
    y, _ = oracle.reverse(inp)
    t0 = 40
    p = {n: (a.copy() if isinstance(a, np.ndarray) else a) for n, a in inp.items()}
    p["k"][:, t0] += 0.5
    p["g"][:, t0] -= 2.0
    y2, _ = oracle.reverse(p)
    np.testing.assert_array_equal(y2[:, t0 + 1:], y[:, t0 + 1:])
    assert np.abs(y2[:, t0] - y[:, t0]).max() > 1e-6


def test_reverse_scan_last_token_is_a_one_token_forward():
    # the last token is the first of the reversed sequence: zero conv history and zero state,
    # so its output is the forward of that token alone
    from state_util import slice_tokens
    inp = gdn_inputs.make_inputs(1, 50, 3, 16, "f32", 0.0, seed=72)
    y, _ = oracle.reverse(inp)
    one = oracle.forward(slice_tokens(inp, 49, 50))
    np.testing.assert_allclose(y[:, 49], one[:, 0], rtol=1e-13, atol=1e-15)
    # and the first token's output differs from the causal forward's (the direction matters)
    assert np.abs(y[:, 0] - oracle.forward(inp)[:, 0]).max() > 1e-3


def test_reverse_scan_conv_looks_ahead():
    # with the decay at full strength for every token after the first (alpha ~ 0: the state keeps
    # only the current token), token t's output depends on tokens t..t+3 only, through the conv
    inp = gdn_inputs.make_inputs(1, 40, 1, 16, "f32", 0.0, seed=73)
    inp["g"][:] = 60.0
    inp["A_log"][:] = np.log(16.0)
    y, _ = oracle.reverse(inp)
    from state_util import slice_tokens
    for t in (5, 20, 36):
        window = oracle.reverse(slice_tokens(inp, t, min(t + 4, 40)))[0]
        np.testing.assert_allclose(y[:, t], window[:, 0], rtol=1e-9, atol=1e-12)
