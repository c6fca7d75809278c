"""Helpers for the GPU tests: move a seeded input set to the device, run the
CUDA forward through the C ABI, and compare with the oracle under the
tolerances of the method's parity bar.

Tolerances (fixed here, used by every parity test):
  * fp32 inputs:              rel-L2 <= 1e-5
  * bf16 inputs, fp32 output: rel-L2 <= 2e-3 and max |y - y_ref| <= 2e-2
  * bf16 inputs, bf16 output: rel-L2 <= 2e-3 + rel-L2(bf16(y_ref), y_ref) and
    |y - y_ref| <= 2e-2 + 1 bf16 ulp(|y_ref|) elementwise.  The 2e-3 bar is on
    the computed value; rounding the output to bf16 adds an error that does
    not depend on the implementation.  By the triangle inequality a value
    within the bar, rounded to bf16, is within the bar plus the rounding error
    of the exact result (about 1.7e-3 on large outputs, up to 3e-3 on a few
    hundred elements).  Half an ulp also exceeds 2e-2 for |y| >= 8, hence the
    elementwise ulp.
rel-L2 = ||y - y_ref||_2 / ||y_ref||_2 over the whole tensor.
"""
from __future__ import annotations

import numpy as np

REL_L2_F32 = 1e-5
REL_L2_BF16 = 2e-3
MAX_ABS_BF16 = 2e-2


def torch_inputs(inp: dict, device="cuda"):
    import torch
    out = {}
    meta = inp["meta"]
    for n in ("q", "k", "v", "z"):
        if meta["dtype"] == "bf16":
            out[n] = torch.from_numpy(inp[n + "_bits"].view(np.int16)).view(torch.bfloat16).to(device)
        else:
            out[n] = torch.from_numpy(inp[n]).to(device)
    for n in ("g", "b", "conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "norm_w"):
        out[n] = torch.from_numpy(np.ascontiguousarray(inp[n], dtype=np.float32)).to(device)
    return out


def run_gdn(inp: dict, out_dtype=None, flags=0, device="cuda", return_plan=False):
    import torch

    import gated_deltanet_06_b200 as gdn
    t = torch_inputs(inp, device)
    B, T, H, d = t["q"].shape
    odt = out_dtype or t["q"].dtype
    plan = gdn.Plan(B, T, H, d, gdn._torch_dtype_code(t["q"].dtype), gdn._torch_dtype_code(odt), flags=flags)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=device)
    y = gdn.forward(**t, plan=plan, workspace=ws, out_dtype=odt)
    st = plan.device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == gdn.OK, gdn.status_string(st)
    yn = y.float().cpu().numpy().astype(np.float64)
    return (yn, plan, ws) if return_plan else yn


def rel_l2(y, ref):
    return float(np.linalg.norm((y - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))


def bf16_ulp(x):
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 7), 2.0 ** -133)


def check_parity(y, ref, in_dtype: str, out_dtype: str, what=""):
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    r = rel_l2(y, ref)
    err = np.abs(y - ref)
    if in_dtype == "f32":
        assert r <= REL_L2_F32, f"{what}: rel-L2 {r:.3e} > {REL_L2_F32}"
        return r, float(err.max())
    bar = REL_L2_BF16
    if out_dtype == "bf16":
        import gdn_inputs
        rounded = gdn_inputs.bf16_bits_to_f32(gdn_inputs.f32_to_bf16_bits(ref.astype(np.float32)))
        bar += rel_l2(rounded.astype(np.float64), ref)
    assert r <= bar, f"{what}: rel-L2 {r:.3e} > {bar:.3e}"
    if out_dtype == "bf16":
        bound = MAX_ABS_BF16 + bf16_ulp(ref)
        bad = err > bound
        assert not bad.any(), f"{what}: {int(bad.sum())} elements over 2e-2 + 1 ulp (max err {err.max():.3e})"
    else:
        assert err.max() <= MAX_ABS_BF16, f"{what}: max-abs {err.max():.3e} > {MAX_ABS_BF16}"
    return r, float(err.max())


def head_slice(inp: dict, b: int, h: int) -> dict:
    """The inputs of one (b, h) as a B = H = 1 problem (heads are independent)."""
    d = inp["meta"]["d_k"]
    out = {}
    for n in ("q", "k", "v", "z"):
        out[n] = np.ascontiguousarray(inp[n][b:b + 1, :, h:h + 1])
    for n in ("g", "b"):
        out[n] = np.ascontiguousarray(inp[n][b:b + 1, :, h:h + 1])
    for n in ("conv_q", "conv_k", "conv_v"):
        out[n] = np.ascontiguousarray(inp[n][h * d:(h + 1) * d])
    for n in ("A_log", "dt_bias"):
        out[n] = np.ascontiguousarray(inp[n][h:h + 1])
    out["norm_w"] = inp["norm_w"]
    out["meta"] = dict(inp["meta"], B=1, H=1)
    return out
