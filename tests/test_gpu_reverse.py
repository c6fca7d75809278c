"""The reverse (anti-causal) scan, GDN_FLAG_REVERSE, on a B200: parity with
the oracle's reverse scan, bitwise equality with the forward scan of the
time-reversed input (both run the same arithmetic in the same internal
order), bitwise anti-causality, and the carried state in the reverse
direction.  Tolerances are the parity bar of the forward tests."""
import numpy as np
import pytest

import gdn_inputs
import oracle
from gpu_util import check_parity, head_slice, rel_l2, REL_L2_BF16, REL_L2_F32, torch_inputs
from state_util import random_state

pytestmark = pytest.mark.gpu


def _flip(inp):
    out = dict(inp)
    for n in ("q", "k", "v", "z", "q_bits", "k_bits", "v_bits", "z_bits", "g", "b"):
        if n in inp:
            out[n] = np.ascontiguousarray(inp[n][:, ::-1])
    return out


def _run(inp, reverse, out_dtype=None, flags=0, s0=None, want_state=False):
    import torch
    import gated_deltanet_06_b200 as gdn
    t = torch_inputs(inp)
    B, T, H, d = t["q"].shape
    odt = out_dtype or t["q"].dtype
    fl = flags | (gdn.FLAG_REVERSE if reverse else 0)
    plan = gdn.Plan(B, T, H, d, gdn._torch_dtype_code(t["q"].dtype), gdn._torch_dtype_code(odt), flags=fl)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    s0_t = None if s0 is None else torch.from_numpy(s0).cuda()
    res = gdn.forward(**t, plan=plan, workspace=ws, out_dtype=odt, s0=s0_t, return_state=want_state,
                      reverse=reverse)
    st = plan.device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == gdn.OK, gdn.status_string(st)
    if want_state:
        return res[0].double().cpu().numpy(), res[1].double().cpu().numpy()
    return res.double().cpu().numpy()


@pytest.mark.parametrize("T", [1, 3, 63, 64, 65, 129, 300, 1500])
def test_reverse_tensor_path_ragged_T(T):
    import torch
    inp = gdn_inputs.make_inputs(1, T, 3, 128, "bf16", -2.0, seed=400 + T)
    ref, _ = oracle.reverse(inp)
    check_parity(_run(inp, True, out_dtype=torch.float32), ref, "bf16", "f32", f"reverse T={T} f32-out")
    check_parity(_run(inp, True), ref, "bf16", "bf16", f"reverse T={T} bf16-out")


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("f32", 128), ("bf16", 64)])
def test_reverse_cuda_core_path(dtype, d):
    import torch
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_inputs(2, 333, 2, d, dtype, -1.0, seed=410 + d)
    y = _run(inp, True, out_dtype=torch.float32, flags=gdn.FLAG_FORCE_SIMT)
    check_parity(y, oracle.reverse(inp)[0], "f32" if dtype == "f32" else "bf16", "f32", f"reverse simt {dtype} d={d}")


@pytest.mark.parametrize("simt", [False, True])
def test_reverse_equals_forward_of_the_reversed_input_bitwise(simt):
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_inputs(2, 1000, 24, 128, "bf16", -1.0, seed=420)  # 48 heads: several segments
    fl = gdn.FLAG_FORCE_SIMT if simt else 0
    y_rev = _run(inp, True, flags=fl)
    y_fwd_flipped = _run(_flip(inp), False, flags=fl)[:, ::-1]
    np.testing.assert_array_equal(y_rev, y_fwd_flipped)


def test_reverse_anti_causality_bitwise():
    inp = gdn_inputs.make_inputs(1, 700, 2, 128, "bf16", 0.0, seed=430)
    y = _run(inp, True)
    t0 = 333
    p = {n: (a.copy() if isinstance(a, np.ndarray) else a) for n, a in inp.items()}
    for n in ("q", "k", "v", "z"):
        bits = p[n + "_bits"]
        bits[:, t0] ^= np.uint16(0x0040)
        p[n] = gdn_inputs.bf16_bits_to_f32(bits)
    p["g"][:, t0] -= 3.0
    y2 = _run(p, True)
    np.testing.assert_array_equal(y2[:, t0 + 1:], y[:, t0 + 1:])
    assert np.abs(y2[:, :t0 + 1] - y[:, :t0 + 1]).max() > 0


@pytest.mark.parametrize("simt", [False, True])
def test_reverse_with_carried_state(simt):
    import torch
    import gated_deltanet_06_b200 as gdn
    dtype = "f32" if simt else "bf16"
    inp = gdn_inputs.make_inputs(1, 1500, 3, 128, dtype, -6.0, seed=440)
    s0 = random_state(1, 3, 128, seed=441)
    y, s = _run(inp, True, out_dtype=torch.float32, flags=gdn.FLAG_FORCE_SIMT if simt else 0, s0=s0,
                want_state=True)
    y_ref, s_ref = oracle.reverse(inp, s0=s0.astype(np.float64))
    check_parity(y, y_ref, dtype, "f32", "reverse with state")
    assert rel_l2(s, s_ref) <= (REL_L2_F32 if simt else REL_L2_BF16)


def test_reverse_headline_workload_sampled_heads():
    w = gdn_inputs.HEADLINE
    inp = gdn_inputs.workload_inputs(w)
    y = _run(inp, True)
    for b, h in ((0, 5), (w.B - 1, w.H - 1)):
        ref, _ = oracle.reverse(head_slice(inp, b, h))
        check_parity(y[b, :, h], ref[0, :, 0], "bf16", "bf16", f"reverse {w.name} b={b} h={h}")


def test_plan_direction_must_match():
    import torch
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_inputs(1, 130, 2, 128, "bf16", 0.0, seed=450)
    t = torch_inputs(inp)
    plan = gdn.Plan(1, 130, 2, 128, gdn.DTYPE_BF16)
    with pytest.raises(ValueError):
        gdn.forward(**t, plan=plan, reverse=True)
