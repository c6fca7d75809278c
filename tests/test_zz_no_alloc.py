"""gdn_forward_noalloc: the forward for callers that cannot allocate device
memory (code where cudaMalloc is not allowed, or whose device memory is all
held by a framework that passes in only inputs and outputs).  It takes its
workspace from a fixed array in the library's device image instead.

Each test compares it, through the C ABI, with gdn_forward run on a
caller-allocated, zero-filled workspace: the same plan on the same inputs runs
the same kernels, so the two outputs must agree bit for bit, whatever an
earlier call left in the array.  The file is named so that pytest collects it
last; it depends on no state left by other tests.
"""
import os
import subprocess
import sys

import pytest

import gdn_inputs
from gpu_util import torch_inputs

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def _plan_for(t, out_dtype, flags=0):
    import gated_deltanet_06_b200 as gdn
    B, T, H, d = t["q"].shape
    return gdn.Plan(B, T, H, d, gdn._torch_dtype_code(t["q"].dtype), gdn._torch_dtype_code(out_dtype), flags=flags)


def _both(t, plan, out_dtype):
    """(gdn_forward on a fresh zeroed workspace, gdn_forward_noalloc) on the same inputs."""
    import torch
    import gated_deltanet_06_b200 as gdn
    stream = torch.cuda.current_stream().cuda_stream
    assert plan.workspace_bytes <= gdn.NOALLOC_SCRATCH_BYTES
    ws = torch.zeros(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    ref = gdn.forward(**t, plan=plan, workspace=ws, out_dtype=out_dtype)
    assert plan.device_status(ws.data_ptr(), stream) == gdn.OK
    y = torch.full_like(ref, float("nan"))
    plan.forward_noalloc_raw(gdn.tensor_ptrs(t), y.data_ptr(), stream)
    torch.cuda.synchronize()
    return ref, y


@pytest.mark.parametrize("shape,dtype,fused", [((1, 700, 2, 128), "bf16", False), ((2, 300, 3, 128), "bf16", False),
                                               ((1, 700, 2, 128), "bf16", True), ((1, 256, 2, 64), "f32", False)])
def test_noalloc_is_bitwise_the_forward_on_two_calls_in_a_row(shape, dtype, fused):
    import torch
    import gated_deltanet_06_b200 as gdn
    B, T, H, d = shape
    for seed in (11, 12):  # two calls, different inputs: nothing stale may leak through
        t = torch_inputs(gdn_inputs.make_inputs(B, T, H, d, dtype, -1.0, seed=seed))
        plan = _plan_for(t, torch.float32, gdn.FLAG_FUSED if fused else 0)
        ref, y = _both(t, plan, torch.float32)
        assert torch.isfinite(ref).all()
        assert torch.equal(y, ref)


def test_noalloc_after_a_larger_call():
    """A long sequence fills far more of the array than the short one that follows it reads; the
    short call's result must not see any of the long call's intermediates."""
    import torch
    for (B, T, H), seed in (((1, 3000, 4), 21), ((1, 300, 2), 22), ((2, 129, 1), 23)):
        t = torch_inputs(gdn_inputs.make_inputs(B, T, H, 128, "bf16", -1.0, seed=seed))
        ref, y = _both(t, _plan_for(t, torch.bfloat16), torch.bfloat16)
        assert torch.equal(y, ref), (B, T, H)


def test_noalloc_rejects_a_plan_larger_than_its_array():
    import torch
    import gated_deltanet_06_b200 as gdn
    plan = gdn.Plan(1, 32760, 12, 128, gdn.DTYPE_BF16)
    assert plan.workspace_bytes > gdn.NOALLOC_SCRATCH_BYTES
    t = torch_inputs(gdn_inputs.make_inputs(1, 128, 12, 128, "bf16", 0.0, seed=1))  # pointers only; nothing may run
    y = torch.zeros(4, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gdn.GDNError) as e:
        plan.forward_noalloc_raw(gdn.tensor_ptrs(t), y.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert e.value.status == gdn.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0


def test_noalloc_after_device_reset():
    """cudaDeviceReset ends the context the array's address was looked up in; the next call must
    look it up again in the new context.  Run in a child process that uses the CUDA runtime
    directly (no torch, whose own state would not survive the reset)."""
    r = subprocess.run([sys.executable, os.path.join(HERE, "noalloc_reset_child.py")], capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "noalloc after reset: bitwise equal" in r.stdout
