"""gdn_backward's tensor-core path (16-bit inputs, d = 128) on a B200 against
the oracle's backward (fp64, written out per step and pinned by finite
differences).

The bar, per gradient tensor: rel-L2 <= 2e-3 and max |g - g_ref| <= 2e-2 *
max |g_ref|, the bf16 parity bar of the forward applied to each gradient (its
elementwise bound scaled by the tensor's largest entry, since the gradients'
magnitudes differ from tensor to tensor).  The path rounds every tensor-core
operand to fp16, as the forward does; the CPU model of that rounding (the
block algebra with every operand rounded to fp16) gives about 7e-4 on the
per-token gradients, so the bar leaves a factor of about 3.

dA_log, ddt_bias and dnorm_w are sums over every token of terms of both
signs.  A sum whose terms are each within a relative e is within e times the
sum of the terms' magnitudes, so their bound is 2e-3 * ||sum |terms| ||_2
(oracle.backward.sum_magnitudes) in place of 2e-3 * ||g_ref||_2, and their
elementwise bound scales the same way.  With cancellation, ||g_ref|| can be
much smaller than the magnitudes.

The workspace stage test compares the kernels' intermediates (the state S at
every block start, the state gradient dS at every block end, dq^, dk^, dv^,
d log alpha, dbeta) with the block model in tests/chunk_model.py, itself
pinned to the oracle's backward on the CPU.
"""
import numpy as np
import pytest

import gdn_inputs
from gpu_util import rel_l2, torch_inputs
from oracle import backward as ob

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
MAX_REL = 2e-2
KEY = {"dq": "q", "dk": "k", "dv": "v", "dz": "z", "dg": "g", "db": "b", "dconv_q": "conv_q",
       "dconv_k": "conv_k", "dconv_v": "conv_v", "dA_log": "A_log", "ddt_bias": "dt_bias", "dnorm_w": "norm_w"}


def _dy(shape, seed):
    rng = np.random.default_rng(seed)
    return gdn_inputs.bf16_bits_to_f32(gdn_inputs.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32)))


def _run(inp, dy, out_f32=False, flags=0, keep=False):
    import torch
    import gated_deltanet_06_b200 as gdn
    t = torch_inputs(inp)
    B, T, H, d = t["q"].shape
    odt = torch.float32 if out_f32 else torch.bfloat16
    plan = gdn.Plan(B, T, H, d, gdn.DTYPE_BF16, gdn._torch_dtype_code(odt), flags=flags)
    if not flags & gdn.FLAG_FORCE_SIMT:
        assert plan.uses_tensor_path and plan.backward_launches in (8, 12)
    ws = torch.empty(plan.backward_workspace_bytes, dtype=torch.uint8, device="cuda")
    out = gdn.backward(**t, dy=torch.from_numpy(dy).to("cuda", odt), plan=plan, workspace=ws)
    torch.cuda.synchronize()
    assert plan.device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == gdn.OK
    got = {n: v.double().cpu().numpy() for n, v in out.items()}
    if keep:
        return got, plan, ws
    return got


def _check_all(got, ref, what, mags=None):
    # mags: oracle.backward.sum_magnitudes of the case (the scale of the sums over tokens)
    errs = {}
    for n, rn in KEY.items():
        scale = ref[rn]
        if mags is not None and rn in mags:
            scale = mags[rn]
        e = float(np.linalg.norm((got[n] - ref[rn]).ravel()) / max(np.linalg.norm(np.ravel(scale)), 1e-300))
        m = float(np.abs(got[n] - ref[rn]).max() / max(np.abs(scale).max(), 1e-300))
        errs[n] = (e, m)
    bad = {n: v for n, v in errs.items() if not (v[0] <= REL_L2 and v[1] <= MAX_REL)}
    assert not bad, f"{what}: {bad} (all: {errs})"
    return errs


@pytest.mark.parametrize("B,T,H,g_mean,out_f32", [(1, 300, 2, 0.0, False),    # segments of one block
                                                  (2, 200, 3, -1.0, True),     # two sequences, ragged
                                                  (1, 100, 2, 1.0, False),     # one block: one segment
                                                  (1, 128, 2, 0.0, True),      # exactly one block
                                                  (1, 129, 2, 0.0, False),     # one token in the last block
                                                  (1, 1, 2, 0.0, False)])      # a single token
def test_tensor_core_backward_matches_the_oracle(B, T, H, g_mean, out_f32):
    inp = gdn_inputs.make_inputs(B, T, H, 128, "bf16", g_mean, seed=700 + T)
    rng = np.random.default_rng(T)
    inp["norm_w"] = (1.0 + 0.3 * rng.standard_normal(128)).astype(np.float32)
    dy = _dy((B, T, H, 128), 800 + T)
    _check_all(_run(inp, dy, out_f32=out_f32), ob.vjp(inp, dy), f"B={B} T={T} H={H}", ob.sum_magnitudes(inp, dy))


def test_tensor_core_backward_with_segments_of_several_blocks():
    # 12 heads (the video configurations' count): about 12 segments per head, so 14 blocks make
    # segments of two blocks and the combine chains seven of them; the last block is ragged
    import gated_deltanet_06_b200 as gdn
    B, T, H = 1, 1700, 12
    inp = gdn_inputs.make_inputs(B, T, H, 128, "bf16", 0.0, seed=731)
    plan = gdn.Plan(B, T, H, 128, gdn.DTYPE_BF16, gdn.DTYPE_BF16)
    dy = _dy((B, T, H, 128), 832)
    got = _run(inp, dy)
    if plan.segments * 2 > -(-T // 128):
        pytest.skip(f"{plan.segments} segments on this GPU: segments hold one block each")
    _check_all(got, ob.vjp(inp, dy), "T=1700 H=12", ob.sum_magnitudes(inp, dy))


def test_stages_match_the_block_model():
    import torch
    import gated_deltanet_06_b200 as gdn
    from chunk_model import ut_backward
    B, T, H = 1, 333, 2
    inp = gdn_inputs.make_inputs(B, T, H, 128, "bf16", -0.5, seed=741)
    dy = _dy((B, T, H, 128), 842)
    _, plan, ws = _run(inp, dy, keep=True)
    _, tp = ob._tape(inp, ob.DEFAULT_L2_EPS, ob.DEFAULT_NORM_EPS)
    ref = ob.vjp(inp, dy)
    model = ut_backward(tp["h_q"], tp["h_k"], tp["s_v"], tp["la"], tp["beta"], ref["do"])
    off = plan.backward_workspace_offsets()
    Tp = -(-T // 128) * 128
    nc = Tp // 128

    def view(name, dtype, shape):
        n = int(np.prod(shape))
        esz = np.dtype(dtype).itemsize
        raw = ws[off[name]:off[name] + n * esz].cpu().numpy()
        return raw.view(dtype).reshape(shape).astype(np.float64)

    s0 = view("S0", np.float16, (B, H, nc, 128, 128))
    np.testing.assert_array_less(rel_l2(s0, model["S0T"]), 2e-3)
    dst = view("dSb", np.float16, (B, H, nc, 128, 128))
    assert rel_l2(dst, model["dST"]) <= 3e-3, rel_l2(dst, model["dST"])
    for name, mk in (("dqh", "dq"), ("dkh", "dk"), ("dvh", "dv")):
        g = view(name, np.float32, (B, H, Tp, 128))[:, :, :T].transpose(0, 2, 1, 3)
        if name == "dqh":  # the workspace holds dL/dQ for Q = q^ / sqrt(d_k)
            g = g / np.sqrt(128.0)
        assert rel_l2(g, model[mk]) <= REL_L2, (name, rel_l2(g, model[mk]))
    for name, mk in (("dla", "dla"), ("dbeta", "dbeta")):
        g = view(name, np.float32, (B, H, Tp))[:, :, :T].transpose(0, 2, 1)
        assert rel_l2(g, model[mk]) <= REL_L2, (name, rel_l2(g, model[mk]))
    torch.cuda.synchronize()


def test_tensor_core_backward_at_the_headline_size():
    # 12 heads x 32760 tokens, beyond the oracle's tape: bitwise repeatability, finiteness, linearity
    # in dy within the bar (fp16 operand rounding makes it approximate), and agreement with the fp32
    # CUDA-core backward of the same inputs within the bar
    import gated_deltanet_06_b200 as gdn
    w = gdn_inputs.HEADLINE
    inp = gdn_inputs.workload_inputs(w)
    dy1 = _dy((w.B, w.T, w.H, w.d), 850)
    dy2 = _dy((w.B, w.T, w.H, w.d), 851)
    g1 = _run(inp, dy1, out_f32=True)
    g1b = _run(inp, dy1, out_f32=True)
    for n in KEY:
        assert np.array_equal(g1[n], g1b[n]), n
        assert np.all(np.isfinite(g1[n])), n
    g2 = _run(inp, dy2, out_f32=True)
    gs = _run(inp, dy1 + dy2, out_f32=True)
    for n in KEY:
        assert rel_l2(gs[n], g1[n] + g2[n]) <= REL_L2, (n, rel_l2(gs[n], g1[n] + g2[n]))
    del g1b, g2, gs
    simt = _run(inp, dy1, out_f32=True, flags=gdn.FLAG_FORCE_SIMT)
    for n in KEY:
        assert rel_l2(g1[n], simt[n]) <= REL_L2, (n, rel_l2(g1[n], simt[n]))


def test_tensor_core_backward_with_f16_inputs_and_output():
    # fp16 activations and an fp16 dy (the draws rounded to fp16, and the oracle given the same
    # values): the same path with the 16-bit loads of the other type
    import torch
    import gated_deltanet_06_b200 as gdn
    B, T, H = 1, 200, 2
    inp = gdn_inputs.make_inputs(B, T, H, 128, "bf16", -0.5, seed=761)
    t = torch_inputs(inp)
    for n in ("q", "k", "v", "z"):
        inp[n] = inp[n].astype(np.float16).astype(np.float32)
        t[n] = torch.from_numpy(inp[n]).to("cuda", torch.float16)
    dy = _dy((B, T, H, 128), 862).astype(np.float16).astype(np.float32)
    plan = gdn.Plan(B, T, H, 128, gdn.DTYPE_F16, gdn.DTYPE_F16)
    assert plan.uses_tensor_path and plan.backward_launches in (8, 12)
    ws = torch.empty(plan.backward_workspace_bytes, dtype=torch.uint8, device="cuda")
    out = gdn.backward(**t, dy=torch.from_numpy(dy).to("cuda", torch.float16), plan=plan, workspace=ws)
    torch.cuda.synchronize()
    assert plan.device_status(ws.data_ptr(), torch.cuda.current_stream().cuda_stream) == gdn.OK
    got = {n: v.double().cpu().numpy() for n, v in out.items()}
    _check_all(got, ob.vjp(inp, dy), "f16 T=200", ob.sum_magnitudes(inp, dy))
