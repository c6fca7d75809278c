"""Pins of the block oracle (oracle/block.py): the layer with its projections.

With permutation matrices for both weights the projections select input
features exactly, so the block oracle must equal the core oracle (pinned on
its own in test_oracle_pins.py) run on those selected features, with the output
permuted.  A wrong split order of q | k | v | z | g | b, a head-minor reshape,
or a transposed weight changes the result and fails here.
"""
import numpy as np
import pytest

import gdn_inputs
import oracle
import oracle.block as ob


@pytest.mark.parametrize("B,T,H,d", [(1, 37, 2, 8), (2, 20, 4, 4)])
def test_block_oracle_with_permutation_weights_is_the_core_oracle(B, T, H, d):
    rng = np.random.default_rng(7)
    Hd = H * d
    N = 4 * Hd + 2 * H
    D = N
    core = gdn_inputs.make_inputs(B, T, H, d, "f32", 0.0, seed=11)
    pi = rng.permutation(N)                 # projection row n reads feature pi[n]
    x = np.zeros((B, T, D), np.float32)
    feats = np.concatenate([core["q"].reshape(B, T, Hd), core["k"].reshape(B, T, Hd), core["v"].reshape(B, T, Hd),
                            core["z"].reshape(B, T, Hd), core["g"], core["b"]], axis=-1)
    x[..., pi] = feats                      # feature pi[n] holds the n-th projection
    w_in = np.zeros((N, D), np.float32)
    w_in[np.arange(N), pi] = 1.0
    sigma = rng.permutation(Hd)             # output column j reads y column sigma[j]
    w_out = np.zeros((Hd, Hd), np.float32)
    w_out[np.arange(Hd), sigma] = 1.0
    inp = dict(x=x, w_in=w_in, w_out=w_out)
    for n in ("conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "norm_w"):
        inp[n] = core[n]
    out = ob.forward(inp)
    y = oracle.forward(core).reshape(B, T, Hd)
    np.testing.assert_allclose(out, y[..., sigma], rtol=1e-12, atol=1e-15)
    # the projections themselves are the selected features
    parts = ob.project_in(x, w_in, H, d)
    for n in ("q", "k", "v", "z", "g", "b"):
        np.testing.assert_array_equal(parts[n], core[n])


def test_block_oracle_output_is_linear_in_w_out():
    inp = gdn_inputs.make_block_inputs(1, 50, 2, 8, 64, seed=3)
    out1, it = ob.forward(inp, intermediates=True)
    y = it["y"].reshape(1, 50, 16)
    # out = y W_out^T: column j of out is y . W_out[j]
    j = 5
    np.testing.assert_allclose(out1[..., j], y @ inp["w_out"][j].astype(np.float64), rtol=1e-12)


@pytest.mark.parametrize("mutant", ["swap_qk", "head_minor", "g_b_swapped", "w_out_transposed"])
def test_planted_mistakes_in_the_block_oracle_fail_the_pin(mutant, monkeypatch):
    real_project = ob.project_in

    def project(x, w_in, H, d):
        parts = real_project(x, w_in, H, d)
        B, T = parts["q"].shape[:2]
        if mutant == "swap_qk":
            parts["q"], parts["k"] = parts["k"], parts["q"]
        elif mutant == "head_minor":
            for n in ("q", "k", "v", "z"):
                parts[n] = parts[n].reshape(B, T, d, H).swapaxes(2, 3)
        elif mutant == "g_b_swapped":
            parts["g"], parts["b"] = parts["b"], parts["g"]
        return parts

    monkeypatch.setattr(ob, "project_in", project)
    if mutant == "w_out_transposed":
        real_forward = ob.forward

        def fwd(inp, **kw):
            return real_forward(dict(inp, w_out=np.ascontiguousarray(np.asarray(inp["w_out"]).T)), **kw)
        monkeypatch.setattr(ob, "forward", fwd)
    with pytest.raises(AssertionError):
        test_block_oracle_with_permutation_weights_is_the_core_oracle(1, 37, 2, 8)
