"""The recurrent state carried in and out (gdn_forward_state), on a B200,
against the oracle's forward with the same initial state.

The state bar: the end state is what every later output is computed from, so
it takes the outputs' relative budget: rel-L2 <= 2e-3 with bf16 inputs (the
tensor path's 16-bit operands), 1e-5 with fp32 inputs (CUDA-core path).
Outputs keep the parity bar of the other tests.
"""
import numpy as np
import pytest

import gdn_inputs
import oracle
from gpu_util import REL_L2_BF16, REL_L2_F32, check_parity, head_slice, rel_l2, torch_inputs
from state_util import random_state, split_stream

pytestmark = pytest.mark.gpu


def _run(inp, s0=None, out_dtype=None, flags=0, want_state=True):
    import torch
    import gated_deltanet_06_b200 as gdn
    t = torch_inputs(inp)
    B, T, H, d = t["q"].shape
    odt = out_dtype or torch.float32
    plan = gdn.Plan(B, T, H, d, gdn._torch_dtype_code(t["q"].dtype), gdn._torch_dtype_code(odt), flags=flags)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    s0_t = None if s0 is None else torch.from_numpy(s0).cuda()
    res = gdn.forward(**t, plan=plan, workspace=ws, out_dtype=odt, s0=s0_t, return_state=want_state)
    st = plan.device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == gdn.OK, gdn.status_string(st)
    y, s = res if want_state else (res, None)
    return y.double().cpu().numpy(), (None if s is None else s.double().cpu().numpy()), plan


def _check_state(s, ref, in_dtype, what):
    assert np.all(np.isfinite(s)), f"{what}: non-finite state"
    r = rel_l2(s, ref)
    bar = REL_L2_F32 if in_dtype == "f32" else REL_L2_BF16
    assert r <= bar, f"{what}: state rel-L2 {r:.3e} > {bar}"
    return r


@pytest.mark.parametrize("B,T,H,g_mean", [(1, 100, 2, -1.0),    # one block, one segment
                                          (1, 1500, 3, -6.0),   # 12 segments, long memory, ragged
                                          (2, 1000, 24, 0.0)])  # 48 heads, 3 segments
def test_tensor_path_state_in_and_out(B, T, H, g_mean):
    inp = gdn_inputs.make_inputs(B, T, H, 128, "bf16", g_mean, seed=300 + T)
    s0 = random_state(B, H, 128, seed=T)
    y, s, plan = _run(inp, s0)
    assert plan.uses_tensor_path
    y_ref, s_ref = oracle.forward_with_state(inp, s0=s0.astype(np.float64))
    check_parity(y, y_ref, "bf16", "f32", f"T={T} y")
    _check_state(s, s_ref, "bf16", f"T={T}")
    # the initial state matters for this case
    y0, _ = oracle.forward_with_state(inp)
    assert rel_l2(y0, y_ref) > 10 * REL_L2_BF16


@pytest.mark.parametrize("d", [64, 128])
def test_cuda_core_path_state_in_and_out(d):
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_inputs(2, 333, 2, d, "f32", -3.0, seed=310 + d)
    s0 = random_state(2, 2, d, seed=d)
    y, s, plan = _run(inp, s0, flags=gdn.FLAG_FORCE_SIMT)
    assert not plan.uses_tensor_path
    y_ref, s_ref = oracle.forward_with_state(inp, s0=s0.astype(np.float64))
    check_parity(y, y_ref, "f32", "f32", f"simt d={d} y")
    _check_state(s, s_ref, "f32", f"simt d={d}")


def test_zero_or_absent_initial_state_is_the_plain_forward_bitwise():
    import torch
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_inputs(1, 1500, 3, 128, "bf16", -1.0, seed=320)
    t = torch_inputs(inp)
    y_plain = gdn.forward(**t)
    y_none, s_none = gdn.forward(**t, return_state=True)
    y_zero, s_zero = gdn.forward(**t, s0=torch.zeros((1, 3, 128, 128), device="cuda"), return_state=True)
    y_only = gdn.forward(**t, s0=torch.zeros((1, 3, 128, 128), device="cuda"))
    assert torch.equal(y_plain, y_none) and torch.equal(y_plain, y_zero) and torch.equal(y_plain, y_only)
    assert torch.equal(s_none, s_zero)
    _check_state(s_none.double().cpu().numpy(), oracle.forward_with_state(inp)[1], "bf16", "zero s0")


@pytest.mark.parametrize("t1", [700, 1280])  # a cut inside a block, and on a block boundary
def test_streaming_in_two_pieces_matches_one_pass(t1):
    import torch
    inp = gdn_inputs.make_inputs(1, 2000, 2, 128, "bf16", -6.0, seed=330)
    p1, p2 = split_stream(inp, t1)
    y1, s1, _ = _run(p1)
    y2, s2, _ = _run(p2, s0=s1.astype(np.float32))
    y_ref, s_ref = oracle.forward_with_state(inp)
    check_parity(np.concatenate([y1, y2[:, 3:]], axis=1), y_ref, "bf16", "f32", f"two pieces cut at {t1}")
    _check_state(s2, s_ref, "bf16", f"two pieces cut at {t1}")
    # and against the GPU's own one-pass run
    y_one, s_one, _ = _run(inp)
    assert rel_l2(np.concatenate([y1, y2[:, 3:]], axis=1), y_one) <= REL_L2_BF16
    assert rel_l2(s2, s_one) <= REL_L2_BF16


def test_headline_workload_with_state_sampled_heads():
    # 12 heads of the 81-frame 480x832 workload (32760 tokens) in the benchmark's launch
    # configuration, bf16 output, with an initial state; two heads recomputed by the oracle
    import torch
    w = gdn_inputs.HEADLINE
    inp = gdn_inputs.workload_inputs(w)
    s0 = random_state(w.B, w.H, w.d, seed=340)
    y, s, _ = _run(inp, s0, out_dtype=torch.bfloat16)
    for b, h in ((0, 0), (w.B - 1, w.H - 1)):
        one = head_slice(inp, b, h)
        y_ref, s_ref = oracle.forward_with_state(one, s0=s0[b:b + 1, h:h + 1].astype(np.float64))
        check_parity(y[b, :, h], y_ref[0, :, 0], "bf16", "bf16", f"{w.name} b={b} h={h}")
        _check_state(s[b:b + 1, h:h + 1], s_ref, "bf16", f"{w.name} b={b} h={h}")


def test_state_argument_errors():
    import torch
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_inputs(1, 300, 2, 128, "bf16", 0.0, seed=350)
    t = torch_inputs(inp)
    plan = gdn.Plan(1, 300, 2, 128, gdn.DTYPE_BF16)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    y = torch.empty_like(t["q"])
    st = torch.zeros((2 * 2 * 128 * 128 + 16,), device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    ptrs = gdn.tensor_ptrs(t)
    base = st.data_ptr()
    for s0, se in ((base, base),             # the same buffer
                   (base, base + 4096),      # overlapping
                   (base + 4, 0),            # misaligned s0
                   (0, base + 8)):           # misaligned s_end
        with pytest.raises(gdn.GDNError) as e:
            plan.forward_state_raw(ptrs, s0, y.data_ptr(), se, ws.data_ptr(), s)
        assert e.value.status == gdn.ERR_INVALID_ARG
    with pytest.raises(ValueError):
        gdn.forward(**t, s0=torch.zeros((1, 2, 128, 64), device="cuda"))
