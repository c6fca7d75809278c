"""Pins of the oracle's backward (oracle/backward.py).

Its numpy forward is pinned to the C oracle's forward; its gradient is pinned
by central finite differences of that forward in fp64, along a random
direction for every input and parameter at once (a dropped term, a wrong sign
or a transposed operand anywhere in the backward shows up in one of them);
and planted mistakes in copies of its source must each fail a check.
"""
import numpy as np
import pytest

import gdn_inputs
import oracle
from oracle import backward as ob

NAMES = ("q", "k", "v", "z", "g", "b", "conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "norm_w")


def _case(seed, T=20, H=2, d=8, g_mean=-1.0, B=1):
    inp = gdn_inputs.make_inputs(B, T, H, d, "f32", g_mean, seed=seed)
    inp = {n: (np.asarray(a, np.float64) if isinstance(a, np.ndarray) else a) for n, a in inp.items()}
    rng = np.random.default_rng(seed)
    inp["norm_w"] = 1.0 + 0.3 * rng.standard_normal(d)  # a non-trivial norm weight
    dy = rng.standard_normal((B, T, H, d))
    return inp, dy


def _fd_check(mod, inp, dy, h=1e-6, rtol=1e-6):
    grads = mod.vjp(inp, dy)
    rng = np.random.default_rng(1)
    bad = []
    for n in NAMES:
        e = rng.standard_normal(np.shape(inp[n]))
        p = dict(inp)
        p[n] = inp[n] + h * e
        lp = float((mod.forward(p) * dy).sum())
        p[n] = inp[n] - h * e
        lm = float((mod.forward(p) * dy).sum())
        fd = (lp - lm) / (2 * h)
        an = float((grads[n] * e).sum())
        if not abs(fd - an) <= rtol * max(abs(fd), abs(an), 1e-8):
            bad.append((n, fd, an))
    return bad


def test_numpy_forward_equals_the_c_oracle():
    for seed, gm in ((81, -1.0), (82, 1.0)):
        inp, _ = _case(seed, T=70, H=3, d=16, g_mean=gm, B=2)
        c_in = dict(inp)
        for n in NAMES:  # the C oracle takes fp32 arrays: give it values exact in fp32
            c_in[n] = np.asarray(inp[n], np.float32)
            inp[n] = c_in[n].astype(np.float64)
        np.testing.assert_allclose(ob.forward(inp), oracle.forward(c_in), rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("seed,g_mean,T", [(83, -1.0, 20), (84, 1.0, 7), (85, -4.0, 33), (86, 0.0, 2)])
def test_gradient_matches_central_differences(seed, g_mean, T):
    inp, dy = _case(seed, T=T, g_mean=g_mean)
    assert _fd_check(ob, inp, dy) == []


MUTANTS = {
    "drop_state_term_of_dalpha": ("dalpha[b, t, h] = (D * Sp).sum() - be", "dalpha[b, t, h] = 0.0 - be"),
    "no_decay_of_the_carried_gradient": ("D = a_ * D + np.outer(du, kh[b, t, h])", "D = D + np.outer(du, kh[b, t, h])"),
    "drop_key_term_through_u": ("dkh[b, t, h] += Sp.T @ du ", "dkh[b, t, h] += 0.0 * du.sum() "),
    "transposed_dq": ("dqh[b, t, h] = St.T @ dot", "dqh[b, t, h] = St @ dot"),
    "l2norm_without_projection": ("ds = (dh - xhat * (xhat * dh).sum(-1, keepdims=True)) / nrm", "ds = dh / nrm"),
    "rmsnorm_without_mean_term": ("do = rn * gz - o * rn ** 3", "do = rn * gz - 0.0 * o * rn ** 3"),
    "conv_transpose_wrong_direction": ("dx[:, :-sh] += wr[None, None, :, :, k] * da[:, sh:]",
                                       "dx[:, sh:] += wr[None, None, :, :, k] * da[:, :-sh]"),
    "softplus_slope_sign": ("grads[\"g\"] = dla * (-eA * sp_grad)", "grads[\"g\"] = dla * (eA * sp_grad)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_check(name):
    import inspect
    import types
    src = inspect.getsource(ob)
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    mod = types.ModuleType("mutant_" + name)
    exec(compile(src.replace(old, new), mod.__name__, "exec"), mod.__dict__)
    inp, dy = _case(87, T=20, g_mean=-1.0)
    assert _fd_check(mod, inp, dy) != []


@pytest.mark.parametrize("T,C", [(1, 64), (63, 64), (64, 64), (65, 64), (200, 64), (50, 16)])
def test_blocked_backward_algebra_equals_the_oracle_backward(T, C):
    # the design of a blocked (UT-form) backward, checked against the sequential backward in fp64
    from chunk_model import chunk_core_backward
    inp, dy = _case(90 + T, T=T, H=2, d=16, g_mean=-1.0)
    _, tp = ob._tape(inp, ob.DEFAULT_L2_EPS, ob.DEFAULT_NORM_EPS)
    ref = ob.vjp(inp, dy)
    got = chunk_core_backward(tp["h_q"], tp["h_k"], tp["s_v"], tp["la"], tp["beta"], ref["do"], C=C)
    for n, m in (("dq", "dqh"), ("dk", "dkh"), ("dv", "dvh"), ("dbeta", "dbeta")):
        np.testing.assert_allclose(got[n], ref[m], rtol=1e-9, atol=1e-11, err_msg=n)
    np.testing.assert_allclose(got["dla"], ref["dalpha"] * tp["alpha"], rtol=1e-9, atol=1e-11, err_msg="dla")


@pytest.mark.parametrize("T,C", [(1, 128), (127, 128), (128, 128), (300, 128), (130, 64)])
def test_kernel_form_backward_equals_the_oracle_backward(T, C):
    # the block backward as the tensor-core kernels take it (reverse recurrence of dS at block ends,
    # then each block's gradients from its tiles, S0 and dS alone), against the sequential backward
    from chunk_model import ut_backward
    inp, dy = _case(120 + T, T=T, H=2, d=16, g_mean=-0.5)
    _, tp = ob._tape(inp, ob.DEFAULT_L2_EPS, ob.DEFAULT_NORM_EPS)
    ref = ob.vjp(inp, dy)
    got = ut_backward(tp["h_q"], tp["h_k"], tp["s_v"], tp["la"], tp["beta"], ref["do"], C=C)
    for n, m in (("dq", "dqh"), ("dk", "dkh"), ("dv", "dvh"), ("dbeta", "dbeta")):
        np.testing.assert_allclose(got[n], ref[m], rtol=1e-9, atol=1e-11, err_msg=n)
    np.testing.assert_allclose(got["dla"], ref["dalpha"] * tp["alpha"], rtol=1e-9, atol=1e-11, err_msg="dla")


def test_sum_magnitudes_bound_the_parameter_gradients():
    # the scale used for the parity bound of the sums over tokens: at least the sum's own magnitude
    # (triangle inequality); and equal to it when every term has one sign, as norm_w's terms do in
    # the second case (every input and dy positive, z > 1)
    inp, dy = _case(140, T=30, H=2, d=8)
    ref = ob.vjp(inp, dy)
    mags = ob.sum_magnitudes(inp, dy)
    for k in ("A_log", "dt_bias", "norm_w"):
        assert np.all(mags[k] >= np.abs(ref[k]) * (1 - 1e-12)), k
    one_sign = {n: np.abs(v) if isinstance(v, np.ndarray) else v for n, v in inp.items()}
    dy_pos = np.abs(dy)
    one_sign["z"] = np.abs(inp["z"]) + 1.0
    ref1 = ob.vjp(one_sign, dy_pos)
    mags1 = ob.sum_magnitudes(one_sign, dy_pos)
    np.testing.assert_allclose(mags1["norm_w"], np.abs(ref1["norm_w"]), rtol=1e-9)
