"""The strict parity bar at full size.

Every bf16 workload runs in the benchmark's launch configuration with fp32
output, so that no output rounding enters the comparison, and sampled heads are
recomputed by the oracle over their whole sequence: rel-L2 <= 2e-3 and
max |y - y_ref| <= 2e-2, element by element (the tolerances of the tensor
path's parity bar).  The default tensor path and the fused one (FLAG_FUSED) run
on the same inputs against the same oracle heads.  The carried-state and
reverse variants run on the 81-frame 480x832 workload (T = 32760, H = 12).

Large activations: q, k, v, z scaled by 32 and by 128 (powers of two, so the
bf16 values scale exactly) check that the fp16 tensor-core operands stay in
range; the output grows with z (SiLU(s z) -> s z), so the max-abs bound scales
with s while the relative bar stays.  Past the fp16 range (v scaled by 2^20)
the tensor path must report the overflow through the debug check, and the
fp32 CUDA-core path must still meet the bar.
"""
import numpy as np
import pytest

import gdn_inputs
import oracle
from gpu_util import MAX_ABS_BF16, REL_L2_BF16, check_parity, head_slice, rel_l2, torch_inputs
from state_util import random_state

pytestmark = pytest.mark.gpu


def _forward_heads(inp, picks, flags=0, s0=None, reverse=False):
    """The whole forward on the GPU (fp32 y), returned only at the picked (b, h) heads."""
    import torch
    import gated_deltanet_06_b200 as gdn
    t = torch_inputs(inp)
    B, T, H, d = t["q"].shape
    if reverse:
        flags |= gdn.FLAG_REVERSE
    plan = gdn.Plan(B, T, H, d, gdn._torch_dtype_code(t["q"].dtype), gdn.DTYPE_F32, flags=flags)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    y = torch.empty((B, T, H, d), dtype=torch.float32, device="cuda")
    s_end = None
    stream = torch.cuda.current_stream().cuda_stream
    if s0 is None:
        plan.forward_raw(gdn.tensor_ptrs(t), y.data_ptr(), ws.data_ptr(), stream)
    else:
        s0_t = torch.from_numpy(s0).cuda()
        s_end = torch.empty_like(s0_t)
        plan.forward_state_raw(gdn.tensor_ptrs(t), s0_t.data_ptr(), y.data_ptr(), s_end.data_ptr(), ws.data_ptr(),
                               stream)
    assert plan.device_status(ws.data_ptr(), stream) == gdn.OK
    out = {bh: y[bh[0], :, bh[1]].double().cpu().numpy() for bh in picks}
    st = None if s_end is None else {bh: s_end[bh[0], bh[1]].double().cpu().numpy() for bh in picks}
    return out, st


def _picks(w, seed):
    rng = np.random.default_rng(seed)
    return sorted({(w.B - 1, w.H - 1), (int(rng.integers(0, w.B)), int(rng.integers(0, w.H)))})


@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_full_size_fp32_output_sampled_heads(idx):
    import gated_deltanet_06_b200 as gdn
    w = gdn_inputs.WORKLOADS[idx]
    inp = gdn_inputs.workload_inputs(w)
    picks = _picks(w, 100 + idx)
    runs = {name: _forward_heads(inp, picks, flags)[0] for name, flags in (("tensor", 0), ("fused", gdn.FLAG_FUSED))}
    for b, h in picks:
        ref = oracle.forward(head_slice(inp, b, h))[0, :, 0]
        for name, y in runs.items():
            check_parity(y[(b, h)], ref, "bf16", "f32", f"{name} {w.name} b={b} h={h}")


@pytest.mark.parametrize("fused", [False, True])
def test_full_size_fp32_output_with_state(fused):
    import gated_deltanet_06_b200 as gdn
    w = gdn_inputs.HEADLINE
    inp = gdn_inputs.workload_inputs(w)
    s0 = random_state(w.B, w.H, w.d, seed=510)
    picks = [(0, 3), (w.B - 1, w.H - 1)]
    y, s = _forward_heads(inp, picks, gdn.FLAG_FUSED if fused else 0, s0=s0)
    for b, h in picks:
        y_ref, s_ref = oracle.forward_with_state(head_slice(inp, b, h), s0=s0[b:b + 1, h:h + 1].astype(np.float64))
        check_parity(y[(b, h)], y_ref[0, :, 0], "bf16", "f32", f"state {w.name} b={b} h={h}")
        r = rel_l2(s[(b, h)], s_ref[0, 0])
        assert r <= REL_L2_BF16, f"final state b={b} h={h}: rel-L2 {r:.3e}"


@pytest.mark.parametrize("fused", [False, True])
def test_full_size_fp32_output_reverse(fused):
    import gated_deltanet_06_b200 as gdn
    w = gdn_inputs.HEADLINE
    inp = gdn_inputs.workload_inputs(w)
    picks = [(0, 7), (w.B - 1, w.H - 1)]
    y, _ = _forward_heads(inp, picks, gdn.FLAG_FUSED if fused else 0, reverse=True)
    for b, h in picks:
        ref, _ = oracle.reverse(head_slice(inp, b, h))
        check_parity(y[(b, h)], ref[0, :, 0], "bf16", "f32", f"reverse {w.name} b={b} h={h}")


def _scaled(inp, scale, names=("q", "k", "v", "z")):
    out = dict(inp)
    for n in names:
        x = inp[n] * np.float32(scale)  # a power of two: exact in bf16
        out[n + "_bits"] = gdn_inputs.f32_to_bf16_bits(x)
        out[n] = gdn_inputs.bf16_bits_to_f32(out[n + "_bits"])
        assert np.array_equal(out[n], x)
    return out


@pytest.mark.parametrize("scale", [32.0, 128.0])
@pytest.mark.parametrize("fused", [False, True])
def test_large_activations_stay_in_fp16_range(scale, fused):
    import gated_deltanet_06_b200 as gdn
    base = gdn_inputs.make_inputs(1, 1500, 2, 128, "bf16", -1.0, seed=520)
    inp = _scaled(base, scale)
    picks = [(0, 0), (0, 1)]
    y, _ = _forward_heads(inp, picks, gdn.FLAG_FUSED if fused else 0)
    ref = oracle.forward(inp)
    for b, h in picks:
        got, want = y[(b, h)], ref[b, :, h]
        assert np.all(np.isfinite(got))
        r = rel_l2(got, want)
        assert r <= REL_L2_BF16, f"x{scale:g} head {h}: rel-L2 {r:.3e}"
        err = np.abs(got - want).max()
        assert err <= MAX_ABS_BF16 * scale, f"x{scale:g} head {h}: max-abs {err:.3e} > {MAX_ABS_BF16 * scale:.3e}"


def test_overflow_past_fp16_range_is_reported():
    import torch
    import gated_deltanet_06_b200 as gdn
    base = gdn_inputs.make_inputs(1, 300, 2, 128, "bf16", -1.0, seed=530)
    inp = _scaled(base, 2.0 ** 20, names=("v",))  # conv4(v) reaches ~1e5: past fp16's 65504
    t = torch_inputs(inp)
    s = torch.cuda.current_stream().cuda_stream
    for flags in (0, gdn.FLAG_FUSED):
        plan = gdn.Plan(1, 300, 2, 128, gdn.DTYPE_BF16, gdn.DTYPE_F32, flags=flags | gdn.FLAG_DEBUG_CHECKS)
        assert plan.uses_tensor_path
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
        gdn.forward(**t, plan=plan, workspace=ws, out_dtype=torch.float32)
        assert plan.device_status(ws.data_ptr(), s) == gdn.ERR_DEVICE_CHECK, flags
    # the fp32 CUDA-core path holds the same inputs
    plan = gdn.Plan(1, 300, 2, 128, gdn.DTYPE_BF16, gdn.DTYPE_F32, flags=gdn.FLAG_FORCE_SIMT)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    y = gdn.forward(**t, plan=plan, workspace=ws, out_dtype=torch.float32)
    assert plan.device_status(ws.data_ptr(), s) == gdn.OK
    check_parity(y.double().cpu().numpy(), oracle.forward(inp), "bf16", "f32", "x2^20 v, CUDA-core path")
