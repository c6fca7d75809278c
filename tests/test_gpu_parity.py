"""Parity of the CUDA forward (through the C ABI) with the fp64 oracle, on a
B200.  Element-by-element on small and ragged cases, on sampled heads of the
five full-size workloads (run in the same launch configuration the benchmark
times), plus the invariants and error paths of the ABI.
"""
import numpy as np
import pytest

import gdn_inputs
import oracle
from gpu_util import check_parity, head_slice, run_gdn, torch_inputs

pytestmark = pytest.mark.gpu


def _oracle(inp):
    return oracle.forward(inp)


# --------------------------------------------------------------- small cases
def test_tiny_fp32_workload_full():
    w = gdn_inputs.WORKLOADS[0]
    inp = gdn_inputs.workload_inputs(w)
    y = run_gdn(inp)
    check_parity(y, _oracle(inp), "f32", "f32", w.name)


@pytest.mark.parametrize("T", [1, 2, 3, 63, 64, 65, 127, 128, 129, 255, 256, 300, 1000])
def test_bf16_tensor_path_ragged_T(T):
    import torch
    inp = gdn_inputs.make_inputs(1, T, 2, 128, "bf16", 0.0, seed=100 + T)
    ref = _oracle(inp)
    check_parity(run_gdn(inp, out_dtype=torch.float32), ref, "bf16", "f32", f"T={T} f32-out")
    check_parity(run_gdn(inp), ref, "bf16", "bf16", f"T={T} bf16-out")


@pytest.mark.parametrize("g_mean", [-6.0, -1.0, 1.0])
def test_decay_regimes_including_long_memory(g_mean):
    # g ~ N(-6, 1) gives alpha ~ 0.95-0.99: the inter-block state dominates
    import torch
    inp = gdn_inputs.make_inputs(1, 1500, 3, 128, "bf16", g_mean, seed=7)
    check_parity(run_gdn(inp, out_dtype=torch.float32), _oracle(inp), "bf16", "f32", f"g_mean={g_mean}")


def test_fp16_inputs_tensor_path():
    import torch
    inp = gdn_inputs.make_inputs(2, 700, 2, 128, "f32", -2.0, seed=9)
    t = torch_inputs(inp)
    import gated_deltanet_06_b200 as gdn
    args = {n: (t[n].half() if n in ("q", "k", "v", "z") else t[n]) for n in t}
    y = gdn.forward(**args, out_dtype=torch.float32)
    ref_inp = dict(inp)
    for n in ("q", "k", "v", "z"):
        ref_inp[n] = args[n].float().cpu().numpy()
    check_parity(y.double().cpu().numpy(), _oracle(ref_inp), "bf16", "f32", "fp16 inputs")


@pytest.mark.parametrize("dtype,d", [("bf16", 64), ("f32", 128), ("bf16", 128)])
def test_cuda_core_path(dtype, d):
    import torch
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_inputs(2, 333, 2, d, dtype, -0.5, seed=d)
    flags = gdn.FLAG_FORCE_SIMT
    y = run_gdn(inp, out_dtype=torch.float32, flags=flags)
    check_parity(y, _oracle(inp), "f32" if dtype == "f32" else "bf16", "f32", f"simt {dtype} d={d}")


# ----------------------------------------------------- full-size workloads
@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_workload_reduced_length_all_heads(idx):
    w = gdn_inputs.WORKLOADS[idx]
    inp = gdn_inputs.workload_inputs(w, T=1100)
    check_parity(run_gdn(inp), _oracle(inp), "bf16", "bf16", w.name + " T=1100")


@pytest.mark.parametrize("idx", [1, 2, 3, 4])
def test_workload_full_size_sampled_heads(idx):
    # the full workload on the GPU (bench launch configuration, bf16 in/out);
    # two (b, h) heads recomputed by the oracle over their whole sequence
    w = gdn_inputs.WORKLOADS[idx]
    inp = gdn_inputs.workload_inputs(w)
    y = run_gdn(inp)
    rng = np.random.default_rng(idx)
    picks = {(w.B - 1, w.H - 1), (int(rng.integers(0, w.B)), int(rng.integers(0, w.H)))}
    for b, h in sorted(picks):
        ref = _oracle(head_slice(inp, b, h))[0, :, 0]
        check_parity(y[b, :, h], ref, "bf16", "bf16", f"{w.name} b={b} h={h}")


# ---------------------------------------------------------------- invariants
def test_causality_bitwise_prefix():
    inp = gdn_inputs.make_inputs(1, 700, 2, 128, "bf16", 0.0, seed=21)
    y = run_gdn(inp)
    t0 = 333
    p = {n: (a.copy() if isinstance(a, np.ndarray) else a) for n, a in inp.items()}
    for n in ("q", "k", "v", "z"):
        bits = p[n + "_bits"]
        bits[:, t0] ^= np.uint16(0x0040)
        p[n] = gdn_inputs.bf16_bits_to_f32(bits)
    p["g"][:, t0] -= 3.0
    y2 = run_gdn(p)
    np.testing.assert_array_equal(y2[:, :t0], y[:, :t0])
    assert np.abs(y2[:, t0:] - y[:, t0:]).max() > 0


def test_batch_items_independent_bitwise():
    inp = gdn_inputs.make_inputs(2, 500, 3, 128, "bf16", 0.0, seed=22)
    y = run_gdn(inp)
    for b in range(2):
        one = {n: (a[b:b + 1] if isinstance(a, np.ndarray) and a.ndim >= 3 else a) for n, a in inp.items()}
        one["meta"] = dict(inp["meta"], B=1)
        np.testing.assert_array_equal(run_gdn(one), y[b:b + 1])


def test_beta_zero_gives_zero_output():
    inp = gdn_inputs.make_inputs(1, 300, 2, 128, "bf16", 0.0, seed=23)
    inp["b"][:] = -1e4
    assert np.all(run_gdn(inp) == 0.0)


def test_strided_token_layout():
    # q, k, v, z as views into a wider packed projection output (token stride > H*d)
    import torch
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_inputs(1, 400, 2, 128, "bf16", 0.0, seed=24)
    t = torch_inputs(inp)
    B, T, H, d = t["q"].shape
    packed = torch.zeros((B, T, 4 * H * d + 64), dtype=torch.bfloat16, device="cuda")
    views = {}
    for i, n in enumerate(("q", "k", "v", "z")):
        packed[:, :, i * H * d:(i + 1) * H * d] = t[n].reshape(B, T, H * d)
        views[n] = packed[:, :, i * H * d:(i + 1) * H * d].view(B, T, H, d)
    args = dict(t, **views)
    y = gdn.forward(**args)
    y_dense = gdn.forward(**t)
    assert torch.equal(y, y_dense)


def test_forward_host_matches_device_forward():
    import torch
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_inputs(1, 500, 2, 128, "bf16", 0.0, seed=25)
    t = torch_inputs(inp)
    y_dev = gdn.forward(**t)
    plan = gdn.Plan(1, 500, 2, 128, gdn.DTYPE_BF16)
    host = {n: t[n].cpu().pin_memory() for n in t}
    y_host = torch.empty_like(y_dev, device="cpu").pin_memory()
    staging = torch.empty(plan.staging_bytes, dtype=torch.uint8, device="cuda")
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    plan.forward_host_raw(gdn.tensor_ptrs(host), y_host.data_ptr(), staging.data_ptr(), ws.data_ptr(), s)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_dev.cpu())


def test_forward_timed_records_every_launch_and_matches_forward():
    import torch
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_inputs(1, 400, 2, 128, "bf16", 0.0, seed=28)
    t = torch_inputs(inp)
    plan = gdn.Plan(1, 400, 2, 128, gdn.DTYPE_BF16)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    y1 = gdn.forward(**t, plan=plan, workspace=ws)
    y2 = torch.empty_like(y1)
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(plan.launches + 1)]
    for e in ev:
        e.record(stream)
    plan.forward_timed_raw(gdn.tensor_ptrs(t), y2.data_ptr(), ws.data_ptr(), stream.cuda_stream,
                           [e.cuda_event for e in ev])
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    times = [ev[i].elapsed_time(ev[i + 1]) for i in range(plan.launches)]
    assert all(x >= 0 for x in times) and sum(times) > 0
    with pytest.raises(gdn.GDNError):
        plan.forward_timed_raw(gdn.tensor_ptrs(t), y2.data_ptr(), ws.data_ptr(), stream.cuda_stream,
                               [e.cuda_event for e in ev[:-1]])


# ---------------------------------------------------------------- error paths
def test_invalid_arguments_are_rejected_before_launch():
    import torch
    import gated_deltanet_06_b200 as gdn
    inp = gdn_inputs.make_inputs(1, 130, 2, 128, "bf16", 0.0, seed=26)
    t = torch_inputs(inp)
    plan = gdn.Plan(1, 130, 2, 128, gdn.DTYPE_BF16)
    ws = torch.empty(plan.workspace_bytes + 512, dtype=torch.uint8, device="cuda")
    y = torch.empty_like(t["q"])
    s = torch.cuda.current_stream().cuda_stream
    ptrs = gdn.tensor_ptrs(t)
    for bad in (dict(ptrs, q=0), dict(ptrs, v=ptrs["v"] + 2), dict(ptrs, norm_w=0)):
        with pytest.raises(gdn.GDNError) as e:
            plan.forward_raw(bad, y.data_ptr(), ws.data_ptr(), s)
        assert e.value.status == gdn.ERR_INVALID_ARG
    with pytest.raises(gdn.GDNError) as e:
        plan.forward_raw(ptrs, y.data_ptr(), ws.data_ptr() + 16, s)  # workspace not 256-aligned
    assert e.value.status == gdn.ERR_INVALID_ARG
    for kw in (dict(d=96), dict(d=128, T=0), dict(d=128, tok_stride=100)):
        args = dict(B=1, T=130, H=2, d=128)
        args.update(kw)
        with pytest.raises(gdn.GDNError):
            gdn.Plan(args["B"], args["T"], args["H"], args["d"], gdn.DTYPE_BF16, tok_stride=kw.get("tok_stride", 0))


@pytest.mark.parametrize("fused", [False, True])
def test_bounded_wait_timeout_mid_pipeline(fused):
    # the last kernel's producer, mid-pipeline with TMA loads and tensor-core work in flight, waits
    # on a barrier nothing arrives on; the wait gives up after ~50 ms, every thread leaves its loop,
    # the work in flight is drained, the status word reports the timeout, and the next forward on
    # the same context is exact.  Each drain waits only for the last phase started on its barrier:
    # a drain that picked the wrong phase would sit out its whole 2 s limit, so the forward must
    # come back well inside that.  B = 2, H = 12, T = 1000 gives segments of 2 blocks on the tensor
    # path, so the next block's loads are in flight when the wait starts.
    import torch
    import gated_deltanet_06_b200 as gdn
    B, T, H = 2, 1000, 12
    inp = gdn_inputs.make_inputs(B, T, H, 128, "bf16", 0.0, seed=27)
    t = torch_inputs(inp)
    base = gdn.FLAG_FUSED if fused else 0
    plan = gdn.Plan(B, T, H, 128, gdn.DTYPE_BF16, flags=base | gdn.FLAG_TEST_WAIT_TIMEOUT)
    if not fused:
        assert plan.segments > 1 and -(-T // 128) >= 2 * (plan.segments - 1)
    ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
    gdn.forward(**t, plan=plan, workspace=ws)  # warm-up: module load, attribute set-up
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    gdn.forward(**t, plan=plan, workspace=ws)
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    assert 45.0 <= ms < 1000.0, ms
    assert plan.device_status(ws.data_ptr(), s.cuda_stream) == gdn.ERR_TIMEOUT
    assert plan.device_status(ws.data_ptr(), s.cuda_stream) == gdn.OK  # reading clears it
    check_parity(run_gdn(inp, flags=base), _oracle(inp), "bf16", "bf16", "after timeout")


@pytest.mark.parametrize("simt", [False, True])
def test_debug_checks_report_non_finite_outputs(simt):
    # GDN_FLAG_DEBUG_CHECKS: a NaN in z reaches one output value, which the device check reports
    # through the status word; without the flag the status stays OK; a clean input passes the
    # checks with the same output bit for bit
    import torch
    import gated_deltanet_06_b200 as gdn
    dt = "f32" if simt else "bf16"
    inp = gdn_inputs.make_inputs(1, 300, 2, 128, dt, 0.0, seed=27)
    clean = torch_inputs(inp)
    bad = dict(clean, z=clean["z"].clone())
    bad["z"][0, 100, 1, 5] = float("nan")
    code = gdn._torch_dtype_code(clean["q"].dtype)
    s = torch.cuda.current_stream().cuda_stream
    base = gdn.FLAG_FORCE_SIMT if simt else 0
    outs = {}
    for name, t in (("bad", bad), ("clean", clean)):
        for flags in (gdn.FLAG_DEBUG_CHECKS, 0):
            plan = gdn.Plan(1, 300, 2, 128, code, flags=base | flags)
            ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
            outs[(name, flags)] = gdn.forward(**t, plan=plan, workspace=ws)
            st = plan.device_status(ws.data_ptr(), s)
            expect = gdn.ERR_DEVICE_CHECK if (name == "bad" and flags) else gdn.OK
            assert st == expect, (name, flags, gdn.status_string(st))
    assert torch.isnan(outs[("bad", 0)].float()).sum().item() == 1
    assert torch.equal(outs[("clean", gdn.FLAG_DEBUG_CHECKS)], outs[("clean", 0)])


@pytest.mark.parametrize("B,T,H,flags", [(1, 1, 2, 0), (2, 129, 3, 0), (1, 3000, 12, 0), (2, 1000, 12, "rev"),
                                         (1, 2000, 4, "state"), (2, 1000, 12, "fused"), (1, 777, 2, "simt")])
def test_debug_bounds_checks_pass_clean_runs_bit_for_bit(B, T, H, flags):
    # GDN_FLAG_DEBUG_CHECKS adds index-bounds checks on every kernel's global accesses (a failed one
    # skips the access and reports GDN_ERR_DEVICE_CHECK); on valid inputs none may fire, and the
    # checked run must give the unchecked run's output bit for bit, over ragged, multi-segment,
    # reverse, carried-state, fused and CUDA-core plans
    import torch
    import gated_deltanet_06_b200 as gdn
    from state_util import random_state
    inp = gdn_inputs.make_inputs(B, T, H, 128, "bf16", -1.0, seed=T)
    t = torch_inputs(inp)
    base = {0: 0, "rev": gdn.FLAG_REVERSE, "state": 0, "fused": gdn.FLAG_FUSED, "simt": gdn.FLAG_FORCE_SIMT}[flags]
    s = torch.cuda.current_stream().cuda_stream
    s0 = torch.from_numpy(random_state(B, H, 128, seed=T)).cuda() if flags == "state" else None
    outs = []
    for dbg in (0, gdn.FLAG_DEBUG_CHECKS):
        plan = gdn.Plan(B, T, H, 128, gdn.DTYPE_BF16, gdn.DTYPE_F32, flags=base | dbg)
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device="cuda")
        y = gdn.forward(**t, plan=plan, workspace=ws, out_dtype=torch.float32, s0=s0,
                        reverse=bool(base & gdn.FLAG_REVERSE))
        assert plan.device_status(ws.data_ptr(), s) == gdn.OK, (flags, dbg)
        outs.append(y)
    assert torch.equal(outs[0], outs[1])
