"""The GDN layer with its projections, as a plain composition: an fp64 matrix
product for the input projection, the core oracle (gdn_oracle.c) for the GDN
forward, and an fp64 matrix product for the output projection.

TEST INFRASTRUCTURE ONLY, like the rest of this package: the tests, the smoke
check and the benchmark's CPU baseline may use it; the CUDA library never does.

For every token row m = b*T + t (the layer the LinMorph page builds its GDN
module into, "Why learn the initialization?"; the projections are those the
T3-Video page counts in Table 1):
    [q | k | v | z | g | b]_m = x_m W_in^T     W_in [4*H*d + 2*H][D], rows in that order
    y = GDN forward (q, k, v, z, g, b)         the core oracle, causal scan
    out_m = y_m W_out^T                        W_out [D][H*d]
q, k, v, z are head-major within their H*d columns.  The core oracle takes its
activations in fp32, so the fp64 projections are rounded to fp32 on the way in
(a relative change of at most 2^-24, far below any tolerance used with it).
"""
from __future__ import annotations

import numpy as np

from . import DEFAULT_L2_EPS, DEFAULT_NORM_EPS
from . import forward as core_forward


def project_in(x, w_in, H: int, d: int) -> dict:
    """x [B,T,D] times w_in^T, split into q, k, v, z [B,T,H,d] and g, b [B,T,H] (fp64)."""
    P = np.asarray(x, np.float64) @ np.asarray(w_in, np.float64).T
    B, T, _ = P.shape
    Hd = H * d
    parts = {n: P[..., i * Hd:(i + 1) * Hd].reshape(B, T, H, d) for i, n in enumerate(("q", "k", "v", "z"))}
    parts["g"] = P[..., 4 * Hd:4 * Hd + H]
    parts["b"] = P[..., 4 * Hd + H:4 * Hd + 2 * H]
    return parts


def forward(inp: dict, l2_eps=DEFAULT_L2_EPS, norm_eps=DEFAULT_NORM_EPS, nthreads=None, intermediates=False):
    """The layer on an input dict from gdn_inputs.make_block_inputs: returns out [B,T,D] fp64
    (and, with intermediates, the projections and y)."""
    H = int(np.asarray(inp["A_log"]).shape[0])
    d = int(np.asarray(inp["norm_w"]).shape[0])
    x = np.asarray(inp["x"])
    B, T, _ = x.shape
    parts = project_in(x, inp["w_in"], H, d)
    core_inp = dict(parts)
    for n in ("conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "norm_w"):
        core_inp[n] = inp[n]
    core_inp["meta"] = dict(B=B, T=T, H=H, d_k=d, d_v=d, dtype="f32")
    y = core_forward(core_inp, l2_eps, norm_eps, nthreads)
    out = y.reshape(B, T, H * d) @ np.asarray(inp["w_out"], np.float64).T
    if intermediates:
        return out, dict(parts, y=y)
    return out
