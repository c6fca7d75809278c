"""Seeded synthetic inputs for the GDN forward, shared by the tests, the smoke
check and the benchmark.

This module only draws random numbers and converts storage formats; it holds
none of the method's arithmetic.  Neither the oracle nor the CUDA library is
imported here.

Workloads.  The token geometry follows the video DiTs on the pages: latent
frames x (H/16) x (W/16) with frame-major flattening.  480x832 gives a 30x52
latent plane (VMonarch page, section 4.3 quotes the (28,52)-class spatial
size for 448x832; the T3-Video page, Table 1, gives attention MACs for
Wan2.1-1.3B at 480x832 that fix T = 21*30*52 = 32,760 tokens at 81 frames,
d_model = 12*128).  Frame counts 17/81/321 are the LinMorph page's clip
lengths ("Fit on short clips", "Acceleration grows with video length");
704x1280x121f is the Wan2.2-5B geometry (31x22x40 latent, CFG pair B=2,
24 heads).

Value distributions: q, k, v, z ~ N(0, 1); conv weights ~ N(0, 0.1) (std);
g ~ N(mu_g, 1) and b ~ N(0, 1) per (b, t, h); A_log ~ U(0, ln 16) per head;
dt_bias ~ N(0, 0.1) per head; RMSNorm weight = 1.  Values are drawn in fp32
with numpy's PCG64 seeded by the workload's seed, in a fixed order, and q, k,
v, z are rounded to bf16 (round to nearest even) for the bf16 workloads.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d: int
    dtype: str  # "f32" or "bf16": storage of q, k, v, z (and of y by default)
    g_mean: float
    seed: int
    note: str = ""

    @property
    def tokens(self) -> int:
        return self.B * self.T


# The five seeded workloads.  index = seed.
WORKLOADS = [
    Workload("tiny_fp32_T256", 1, 2, 256, 64, "f32", 0.0, 0,
             "tiny fp32 case, B1 H2 T256 d64"),
    Workload("wan21_480x832_17f", 1, 12, 5 * 30 * 52, 128, "bf16", 0.0, 1,
             "Wan2.1-1.3B-shaped block, 480x832, 17 frames (5 latent)"),
    Workload("wan21_480x832_81f", 1, 12, 21 * 30 * 52, 128, "bf16", 0.0, 2,
             "Wan2.1-1.3B-shaped block, 480x832, 81 frames (21 latent)"),
    Workload("wan22_704x1280_121f_cfg", 2, 24, 31 * 22 * 40, 128, "bf16", -1.0, 3,
             "Wan2.2-5B-shaped block, 704x1280, 121 frames, CFG pair"),
    Workload("long_480x832_321f", 1, 12, 81 * 30 * 52, 128, "bf16", 1.0, 4,
             "long video, 480x832, 321 frames (81 latent)"),
]
HEADLINE = WORKLOADS[2]


def by_name(name: str) -> Workload:
    for w in WORKLOADS:
        if w.name == name:
            return w
    raise KeyError(name)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 exactly."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def make_inputs(B: int, T: int, H: int, d: int, dtype: str = "bf16", g_mean: float = 0.0,
                seed: int = 0, d_v: int | None = None) -> dict:
    """Draw one seeded input set.

    Returns a dict of numpy arrays.  Activations are [B, T, H, d]; gates are
    [B, T, H]; conv weights are [H*d, 4]; A_log, dt_bias are [H]; norm_w is
    [d_v].  For dtype "bf16", q/k/v/z hold the exact fp32 widening of their bf16
    values and q_bits/k_bits/v_bits/z_bits hold the bf16 patterns (uint16).
    """
    dv = d if d_v is None else d_v
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    for name, dd in (("q", d), ("k", d), ("v", dv), ("z", dv)):
        x = rng.standard_normal((B, T, H, dd), dtype=np.float32)
        if dtype == "bf16":
            bits = f32_to_bf16_bits(x)
            out[name + "_bits"] = bits
            out[name] = bf16_bits_to_f32(bits)
        elif dtype == "f32":
            out[name] = x
        else:
            raise ValueError(dtype)
    out["g"] = (rng.standard_normal((B, T, H), dtype=np.float32) + np.float32(g_mean)).astype(np.float32)
    out["b"] = rng.standard_normal((B, T, H), dtype=np.float32)
    out["conv_q"] = (np.float32(0.1) * rng.standard_normal((H * d, 4), dtype=np.float32))
    out["conv_k"] = (np.float32(0.1) * rng.standard_normal((H * d, 4), dtype=np.float32))
    out["conv_v"] = (np.float32(0.1) * rng.standard_normal((H * dv, 4), dtype=np.float32))
    out["A_log"] = rng.uniform(0.0, math.log(16.0), H).astype(np.float32)
    out["dt_bias"] = (np.float32(0.1) * rng.standard_normal(H, dtype=np.float32))
    out["norm_w"] = np.ones(dv, dtype=np.float32)
    out["meta"] = dict(B=B, T=T, H=H, d_k=d, d_v=dv, dtype=dtype, g_mean=g_mean, seed=seed)
    return out


def workload_inputs(w: Workload, T: int | None = None, B: int | None = None,
                    H: int | None = None) -> dict:
    """Inputs for a named workload; T/B/H may be overridden for reduced cases
    (same seed and distributions, smaller shape)."""
    return make_inputs(B if B is not None else w.B, T if T is not None else w.T,
                       H if H is not None else w.H, w.d, w.dtype, w.g_mean, w.seed)


def make_block_inputs(B: int, T: int, H: int, d: int, D: int, seed: int = 0) -> dict:
    """Draw one seeded input set for the GDN layer with its projections.

    x [B, T, D] ~ N(0, 1) and the weights W_in [4*H*d + 2*H, D] ~ N(0, 1/D) and
    W_out [D, H*d] ~ N(0, 1/(H*d)) are rounded to bf16 (bits in x_bits,
    w_in_bits, w_out_bits; the exact fp32 widenings in x, w_in, w_out), so that
    the projections of q, k, v, z, g, b come out near N(0, 1) like the core's
    inputs.  The conv weights, A_log, dt_bias and norm_w follow make_inputs.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    N = 4 * H * d + 2 * H
    for name, shape, std in (("x", (B, T, D), 1.0), ("w_in", (N, D), 1.0 / math.sqrt(D)),
                             ("w_out", (D, H * d), 1.0 / math.sqrt(H * d))):
        x = rng.standard_normal(shape, dtype=np.float32) * np.float32(std)
        bits = f32_to_bf16_bits(x)
        out[name + "_bits"] = bits
        out[name] = bf16_bits_to_f32(bits)
    out["conv_q"] = (np.float32(0.1) * rng.standard_normal((H * d, 4), dtype=np.float32))
    out["conv_k"] = (np.float32(0.1) * rng.standard_normal((H * d, 4), dtype=np.float32))
    out["conv_v"] = (np.float32(0.1) * rng.standard_normal((H * d, 4), dtype=np.float32))
    out["A_log"] = rng.uniform(0.0, math.log(16.0), H).astype(np.float32)
    out["dt_bias"] = (np.float32(0.1) * rng.standard_normal(H, dtype=np.float32))
    out["norm_w"] = np.ones(d, dtype=np.float32)
    out["meta"] = dict(B=B, T=T, H=H, d=d, D=D, seed=seed)
    return out
