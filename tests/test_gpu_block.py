"""The GDN layer with its projections (gdn_block_forward) on a B200 against
the block oracle (oracle/block.py).

Tolerances: the layer's output with fp32 storage is held to the parity bar of
the tensor path (rel-L2 <= 2e-3, max |out - ref| <= 2e-2); with bf16 output the
bf16 rounding of the exact result is added as for the core (gpu_util's bf16
bar).  The cases cover ragged M tiles (the input projection's tiles advance by
125 rows), batch boundaries inside a tile (the conv must not reach across batch
items), H = 2 .. 12, D from 128 to the Wan2.1-1.3B width 1536, and the full
81-frame 480x832 layer.
"""
import numpy as np
import pytest

import gdn_inputs
import oracle.block as ob
from gpu_util import check_parity

pytestmark = pytest.mark.gpu


def _device(inp):
    import torch
    t = {}
    for n in ("x", "w_in", "w_out"):
        t[n] = torch.from_numpy(inp[n + "_bits"].view(np.int16)).view(torch.bfloat16).cuda()
    for n in ("conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "norm_w"):
        t[n] = torch.from_numpy(np.ascontiguousarray(inp[n], dtype=np.float32)).cuda()
    return t


def _run(inp, out_dtype, flags=0):
    import torch
    import gated_deltanet_06_b200 as gdn
    m = inp["meta"]
    t = _device(inp)
    plan = gdn.BlockPlan(m["B"], m["T"], m["H"], m["d"], m["D"], gdn._torch_dtype_code(out_dtype), flags=flags)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    out = gdn.block_forward(**t, out_dtype=out_dtype, plan=plan, workspace=ws)
    st = plan.device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == gdn.OK, gdn.status_string(st)
    return out


@pytest.mark.parametrize("B,T,H,D", [(1, 300, 2, 256), (1, 129, 2, 128), (2, 1001, 4, 512), (3, 250, 2, 192),
                                     (1, 4000, 12, 1536), (1, 1, 2, 128), (2, 3, 2, 128), (1, 125, 2, 64),
                                     (3, 126, 4, 320)])
def test_block_matches_oracle_fp32_out(B, T, H, D):
    import torch
    inp = gdn_inputs.make_block_inputs(B, T, H, 128, D, seed=T + D)
    out = _run(inp, torch.float32).double().cpu().numpy()
    check_parity(out, ob.forward(inp), "bf16", "f32", f"block B={B} T={T} H={H} D={D}")


def test_block_bf16_out_and_bitwise_repeat():
    import torch
    inp = gdn_inputs.make_block_inputs(2, 700, 4, 128, 512, seed=5)
    a = _run(inp, torch.bfloat16)
    b = _run(inp, torch.bfloat16)
    assert torch.equal(a, b)
    check_parity(a.float().double().cpu().numpy(), ob.forward(inp), "bf16", "bf16", "block bf16 out")


def test_block_debug_checks_pass_bit_for_bit():
    import torch
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_block_inputs(2, 1001, 4, 128, 512, seed=9)
    assert torch.equal(_run(inp, torch.float32), _run(inp, torch.float32, flags=gdn.FLAG_DEBUG_CHECKS))


def test_block_full_81_frame_layer():
    # the 81-frame 480x832 Wan2.1-1.3B-shaped layer: T = 32760, H = 12, D = 1536, every output
    import torch
    inp = gdn_inputs.make_block_inputs(1, 32760, 12, 128, 1536, seed=2)
    out = _run(inp, torch.float32).double().cpu().numpy()
    check_parity(out, ob.forward(inp), "bf16", "f32", "block 81f")


def test_block_plan_rejections():
    import gated_deltanet_06_b200 as gdn
    for kw in (dict(H=3), dict(d=64), dict(D=100), dict(out_dtype=gdn.DTYPE_F16), dict(flags=gdn.FLAG_REVERSE)):
        args = dict(B=1, T=100, H=2, d=128, D=256, out_dtype=gdn.DTYPE_BF16, flags=0)
        args.update(kw)
        with pytest.raises(gdn.GDNError) as e:
            gdn.BlockPlan(args["B"], args["T"], args["H"], args["d"], args["D"], args["out_dtype"], flags=args["flags"])
        assert e.value.status == gdn.ERR_UNSUPPORTED, kw
