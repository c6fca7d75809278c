"""gdn_forward_noalloc: the forward for callers that cannot allocate device
memory (code where cudaMalloc is not allowed, or whose device memory is all
held by a framework that passes in only inputs and outputs).  It takes its
workspace from a fixed array in the library's device image instead.

Each test compares it, through the C ABI, with gdn_forward run on a
caller-allocated workspace, on two calls in a row, under the same tolerances
as the parity tests.  The file is named so that pytest collects it last; it
depends on no state left by other tests.
"""
import numpy as np
import pytest

import gdn_inputs
from gpu_util import REL_L2_BF16, REL_L2_F32, MAX_ABS_BF16, rel_l2, torch_inputs

pytestmark = pytest.mark.gpu


def _plan_for(t, out_dtype):
    import gated_deltanet_06_b200 as gdn
    B, T, H, d = t["q"].shape
    return gdn.Plan(B, T, H, d, gdn._torch_dtype_code(t["q"].dtype), gdn._torch_dtype_code(out_dtype))


def _close(y, ref, in_dtype):
    y = y.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    assert np.all(np.isfinite(y))
    r = rel_l2(y, ref)
    if in_dtype == "f32":
        assert r <= REL_L2_F32, r
    else:
        assert r <= REL_L2_BF16, r
        assert np.abs(y - ref).max() <= MAX_ABS_BF16


@pytest.mark.parametrize("shape,dtype", [((1, 700, 2, 128), "bf16"), ((2, 300, 3, 128), "bf16"),
                                         ((1, 256, 2, 64), "f32")])
def test_noalloc_matches_forward_on_two_calls_in_a_row(shape, dtype):
    import torch
    import gated_deltanet_06_b200 as gdn
    B, T, H, d = shape
    stream = torch.cuda.current_stream().cuda_stream
    for call, seed in enumerate((11, 12)):  # two calls, different inputs: nothing stale may leak through
        inp = gdn_inputs.make_inputs(B, T, H, d, dtype, -1.0, seed=seed)
        t = torch_inputs(inp)
        plan = _plan_for(t, torch.float32)
        assert plan.workspace_bytes <= gdn.NOALLOC_SCRATCH_BYTES
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
        ref = gdn.forward(**t, plan=plan, workspace=ws, out_dtype=torch.float32)
        y = torch.full_like(ref, float("nan"))
        plan.forward_noalloc_raw(gdn.tensor_ptrs(t), y.data_ptr(), stream)
        torch.cuda.synchronize()
        _close(y, ref, dtype)


def test_noalloc_rejects_a_plan_larger_than_its_array():
    import torch
    import gated_deltanet_06_b200 as gdn
    plan = gdn.Plan(1, 32760, 12, 128, gdn.DTYPE_BF16)
    assert plan.workspace_bytes > gdn.NOALLOC_SCRATCH_BYTES
    inp = gdn_inputs.make_inputs(1, 128, 12, 128, "bf16", 0.0, seed=1)  # pointers only; nothing may run
    t = torch_inputs(inp)
    y = torch.zeros(4, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gdn.GDNError) as e:
        plan.forward_noalloc_raw(gdn.tensor_ptrs(t), y.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert e.value.status == gdn.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0
