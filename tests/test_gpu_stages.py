"""Per-stage checks of the tensor path on a B200: each kernel's output, read
back from the workspace, against an fp64 reference of that stage computed
from the oracle's intermediates.  These localise a failure to one kernel
(prep, UT transform, scan, output)."""
import math

import numpy as np
import pytest

import gdn_inputs
import oracle
from gpu_util import check_parity, run_gdn

pytestmark = pytest.mark.gpu
BLK = 128


def _ws_array(ws, off, count, dtype):
    import torch
    nbytes = count * (2 if dtype == torch.float16 else 4)
    return ws[off:off + nbytes].view(dtype).double().cpu().numpy()


def _stage_refs(inp):
    y, it = oracle.forward(inp, intermediates=True)
    B, T, H, d = inp["q"].shape
    NB = -(-T // BLK)
    Tp = NB * BLK

    def headmajor(x):  # [B,T,H,...] -> [B,H,Tp,...] zero-padded
        x = np.moveaxis(x, 2, 1)
        pad = [(0, 0)] * x.ndim
        pad[2] = (0, Tp - T)
        return np.pad(x, pad)

    ref = dict(qh=headmajor(it["qh"]) / math.sqrt(d), kh=headmajor(it["kh"]), vh=headmajor(it["vh"]),
               beta=headmajor(it["beta"]), la=headmajor(np.log(it["alpha"])), o=it["o"], y=y)
    G = ref["la"].reshape(B, H, NB, BLK).cumsum(-1).reshape(B, H, Tp)
    ref["G"] = G
    W = np.zeros((B, H, Tp, d)); U = np.zeros_like(W); Qt = np.zeros_like(W); Kt = np.zeros_like(W)
    Aqk = np.zeros((B, H, Tp, BLK))
    for b in range(B):
        for h in range(H):
            for c in range(NB):
                sl = slice(c * BLK, (c + 1) * BLK)
                K, V, Q = ref["kh"][b, h, sl], ref["vh"][b, h, sl], ref["qh"][b, h, sl]
                g, be = G[b, h, sl], ref["beta"][b, h, sl]
                D = np.minimum(g[:, None] - g[None, :], 0.0)
                L = np.tril(np.ones((BLK, BLK)), -1) * be[:, None] * np.exp(D) * (K @ K.T)
                Tm = np.linalg.inv(np.eye(BLK) + L)
                W[b, h, sl] = Tm @ ((be * np.exp(g))[:, None] * K)
                U[b, h, sl] = Tm @ (be[:, None] * V)
                Qt[b, h, sl] = np.exp(g)[:, None] * Q
                Kt[b, h, sl] = np.exp(g[-1] - g)[:, None] * K
                Aqk[b, h, sl] = np.tril(np.ones((BLK, BLK))) * np.exp(D) * (Q @ K.T)
    ref.update(W=W, U=U, Qt=Qt, Kt=Kt, Aqk=Aqk)
    return ref


def _rel(a, b):
    return np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300)


@pytest.mark.parametrize("T,g_mean", [(300, -1.0), (129, -6.0), (1100, -6.0)])
def test_stage_outputs_of_tensor_path(T, g_mean):
    import torch
    inp = gdn_inputs.make_inputs(1, T, 2, 128, "bf16", g_mean, seed=31)
    y, plan, ws = run_gdn(inp, out_dtype=torch.float32, return_plan=True)
    assert plan.uses_tensor_path
    off = plan.workspace_offsets()
    ref = _stage_refs(inp)
    B, H, d = 1, 2, 128
    Tp = -(-T // BLK) * BLK
    n_act = B * H * Tp * d
    # K1: prep
    for name in ("qh", "kh", "vh"):
        got = _ws_array(ws, off[name], n_act, torch.float16).reshape(B, H, Tp, d)
        err = np.abs(got - ref[name])
        assert np.all(err <= 6e-4 * np.abs(ref[name]) + 1e-7), f"{name}: max err {err.max():.3e}"
    for name, key in (("G", "G"), ("beta", "beta"), ("log_alpha", "la")):
        got = _ws_array(ws, off[name], B * H * Tp, torch.float32).reshape(B, H, Tp)
        np.testing.assert_allclose(got, ref[key], rtol=1e-5, atol=2e-5 * (1 + np.abs(ref[key]).max()),
                                   err_msg=name)
    # K2: UT transform and decayed operands
    for name in ("Kt", "Qt", "Aqk", "W", "U"):
        got = _ws_array(ws, off[name], n_act, torch.float16).reshape(ref[name].shape)
        want = ref[name]
        if name == "Aqk":  # block lower triangular: the zero upper-right 64x64 quadrant is not stored
            keep = np.ones((BLK, BLK), bool)
            keep[:64, 64:] = False
            keep = np.tile(keep, (Tp // BLK, 1))
            got, want = got[..., keep], want[..., keep]
        r = _rel(got, want)
        assert r < 5e-3, f"{name}: rel-L2 {r:.3e}"
    # segment transfer + combine: S^T at every segment start vs the oracle's state there
    NB = Tp // BLK
    ns = plan.segments
    if ns > 1:
        ls = -(-NB // ns)
        St = _ws_array(ws, off["Sstart"], B * H * ns * d * d, torch.float32).reshape(B, H, ns, d, d)
        _, it = oracle.forward(inp, intermediates=True)
        for j in range(1, ns):
            t_end = min(j * ls * BLK, T)
            _, S = oracle.core(it["qh"][:, :t_end], it["kh"][:, :t_end], it["vh"][:, :t_end],
                               it["alpha"][:, :t_end], it["beta"][:, :t_end], return_state=True)
            for h in range(H):
                r = _rel(St[0, h, j], S[0, h].T)
                assert r < 3e-3, f"segment {j} head {h} start state: rel {r:.3e}"
    # scan with the fused output step
    check_parity(y, ref["y"], "bf16", "f32", "y")
