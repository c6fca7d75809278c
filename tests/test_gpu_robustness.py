"""Robustness of the forward on a B200: random shapes against the oracle, CUDA-graph capture and
replay, and concurrent forwards on two streams.

Random shapes (seeded) cover B, H and ragged T together on the tensor path, the fused path and the
CUDA-core path at the parity bars of gpu_util.  A forward captured in a CUDA graph and replayed must
give the eager forward's output bit for bit (the library's launches, tensor maps and status reset are
all capturable).  Two forwards with their own workspaces on two unordered streams must each give the
output of running alone: nothing is shared between calls but the plan.
"""
import numpy as np
import pytest

import gdn_inputs
import oracle
from gpu_util import check_parity, torch_inputs

pytestmark = pytest.mark.gpu


def _shapes(seed, n):
    rng = np.random.default_rng(seed)
    return [(int(rng.integers(1, 4)), int(rng.integers(1, 1800)), int(rng.integers(1, 7))) for _ in range(n)]


@pytest.mark.parametrize("path", ["tensor", "fused", "simt"])
@pytest.mark.parametrize("B,T,H", _shapes(2026, 6))
def test_random_shapes_against_oracle(path, B, T, H):
    import torch
    import gated_deltanet_06_b200 as gdn
    d, dt = (64, "f32") if path == "simt" else (128, "bf16")
    flags = {"tensor": 0, "fused": gdn.FLAG_FUSED, "simt": 0}[path]
    inp = gdn_inputs.make_inputs(B, T, H, d, dt, float(np.random.default_rng(T).uniform(-3, 1)), seed=B * 1000 + T)
    t = torch_inputs(inp)
    plan = gdn.Plan(B, T, H, d, gdn._torch_dtype_code(t["q"].dtype), gdn.DTYPE_F32, flags=flags)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    y = gdn.forward(**t, plan=plan, workspace=ws, out_dtype=torch.float32)
    assert plan.device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == gdn.OK
    check_parity(y.double().cpu().numpy(), oracle.forward(inp), dt, "f32", f"{path} B={B} T={T} H={H}")


@pytest.mark.parametrize("flags_name", ["tensor", "fused"])
def test_cuda_graph_replay_is_bitwise_the_eager_forward(flags_name):
    import torch
    import gated_deltanet_06_b200 as gdn
    flags = gdn.FLAG_FUSED if flags_name == "fused" else 0
    inp = gdn_inputs.make_inputs(1, 3000, 4, 128, "bf16", -1.0, seed=61)
    t = torch_inputs(inp)
    plan = gdn.Plan(1, 3000, 4, 128, gdn.DTYPE_BF16, flags=flags)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    ptrs = gdn.tensor_ptrs(t)
    eager = torch.empty((1, 3000, 4, 128), dtype=torch.bfloat16, device="cuda")
    plan.forward_raw(ptrs, eager.data_ptr(), ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    y = torch.zeros_like(eager)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        plan.forward_raw(ptrs, y.data_ptr(), ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    for _ in range(3):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, eager)
    assert plan.device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == gdn.OK


def test_two_streams_with_their_own_workspaces():
    import torch
    import gated_deltanet_06_b200 as gdn
    inps = [gdn_inputs.make_inputs(1, 2500, 6, 128, "bf16", 0.0, seed=71 + i) for i in range(2)]
    ts = [torch_inputs(x) for x in inps]
    plan = gdn.Plan(1, 2500, 6, 128, gdn.DTYPE_BF16)
    alone = []
    for t in ts:
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
        alone.append(gdn.forward(**t, plan=plan, workspace=ws))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    wss = [torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
    ys = [torch.empty_like(alone[0]) for _ in range(2)]
    for _ in range(5):
        for i in range(2):
            plan.forward_raw(gdn.tensor_ptrs(ts[i]), ys[i].data_ptr(), wss[i].data_ptr(), streams[i].cuda_stream)
    torch.cuda.synchronize()
    for i in range(2):
        assert plan.device_status(wss[i].data_ptr(), streams[i].cuda_stream) == gdn.OK
        assert torch.equal(ys[i], alone[i])
