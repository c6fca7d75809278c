"""Chunked (UT / WY) form of the gated delta rule in numpy: a design aid for
the CUDA kernels, not the oracle.

It restates the algebra the kernels implement, block by block, so that the
tests can check that algebra against the sequential oracle (they agree to
rounding in fp64), and so that the effect of storing intermediates in a
narrower type can be measured on the CPU.

Algebra (per (b, h), block of C tokens r = 0..C-1, incoming state S0, d_v x d_k):
  G_r    = sum_{s<=r} log alpha_s                       (in-block cumulative log decay)
  L_rj   = beta_r exp(G_r - G_j) (k_r . k_j)   for j < r, else 0
  T      = (I + L)^-1                                   (unit lower triangular)
  W      = T diag(beta exp(G)) K,   U = T diag(beta) V
  Delta  = U - W S0^T                                   (rows delta_r of the delta rule)
  O      = diag(exp(G)) Q S0^T + (M o exp(G_r - G_i) o Q K^T) Delta,  M_ri = [i <= r]
  S_C    = exp(G_C) S0 + Delta^T diag(exp(G_C - G)) K
Only exponentials of non-positive differences are ever taken.

Derivation: with delta_t = beta_t (v_t - alpha_t S_{t-1} k_t) the recurrence
reads S_t = alpha_t S_{t-1} + delta_t k_t^T; unrolling inside the block gives
(I + L) Delta = diag(beta) V - diag(beta exp(G)) K S0^T, and the state and
output follow by substitution.
"""
from __future__ import annotations

import numpy as np


def _round(x, mode):
    if mode is None or mode == "f64":
        return x
    if mode == "f32":
        return x.astype(np.float32).astype(np.float64)
    if mode == "f16":
        return x.astype(np.float16).astype(np.float64)
    if mode == "bf16":
        u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
        r = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
        return (((u + r) >> np.uint32(16)) << np.uint32(16)).view(np.float32).astype(np.float64)
    raise ValueError(mode)


def chunk_core(qh, kh, vh, log_alpha, beta, C=64, operand=None, store=None):
    """o [B,T,H,d_v] from prepared q^ (unscaled), k^, v^ and log alpha, beta,
    by the block algebra above.

    operand: rounding applied to every tensor-core operand (None = exact).
    store:   rounding applied to intermediates the kernels keep in memory.
    """
    B, T, H, dk = qh.shape
    dv = vh.shape[-1]
    nc = -(-T // C)
    Tp = nc * C
    scale = 1.0 / np.sqrt(dk)
    o = np.zeros((B, T, H, dv))
    tril_strict = np.tril(np.ones((C, C)), -1)
    tril_incl = np.tril(np.ones((C, C)))
    for b in range(B):
        for h in range(H):
            def pad(x):
                out = np.zeros((Tp,) + x.shape[1:])
                out[:T] = x
                return out
            Q = _round(pad(qh[b, :, h] * scale), store)
            K = _round(pad(kh[b, :, h]), store)
            V = _round(pad(vh[b, :, h]), store)
            la = pad(log_alpha[b, :, h])
            be = pad(beta[b, :, h])
            S = np.zeros((dv, dk))
            for c in range(nc):
                sl = slice(c * C, (c + 1) * C)
                Kc, Vc, Qc = K[sl], V[sl], Q[sl]
                G = np.cumsum(la[sl])
                bc = be[sl]
                Akk = _round(Kc, operand) @ _round(Kc, operand).T
                D = G[:, None] - G[None, :]
                L = tril_strict * bc[:, None] * np.exp(np.minimum(D, 0.0)) * Akk
                Tm = np.linalg.inv(np.eye(C) + L)
                W = _round(Tm * (bc * np.exp(G))[None, :], operand) @ _round(Kc, operand)
                U = _round(Tm * bc[None, :], operand) @ _round(Vc, operand)
                W, U = _round(W, store), _round(U, store)
                St = _round(S, operand)
                Delta = U - W @ St.T
                Dl = _round(Delta, operand)
                Aqk = _round(tril_incl * np.exp(np.minimum(D, 0.0)) * (_round(Qc, operand) @ _round(Kc, operand).T), operand)
                Qt = _round(np.exp(G)[:, None] * Qc, operand)
                O = Qt @ St.T + Aqk @ Dl
                Kt = _round(np.exp(G[-1] - G)[:, None] * Kc, operand)
                S = np.exp(G[-1]) * S + Dl.T @ Kt
                rows = min(C, T - c * C)
                o[b, c * C:c * C + rows, h] = O[:rows]
    return o


def segment_start_states(kh, vh, log_alpha, beta, C=128, Ls=2):
    """Segment-parallel form of the inter-block state (one (b, h), inputs
    [T, d]): each segment of Ls blocks runs the combined state [S^T | P^T]
    from [0 | I] block by block (P is the segment's transfer matrix, S_loc its
    end state from zero), then S_start(j+1)^T = P_j^T S_start(j)^T + S_loc(j)^T.
    Returns the list of S^T at every segment start (d_k x d_v)."""
    T, d = kh.shape
    nb = -(-T // C)
    Tp = nb * C

    def pad(x):
        out = np.zeros((Tp,) + x.shape[1:])
        out[:T] = x
        return out
    K, V, la, be = pad(kh), pad(vh), pad(log_alpha), pad(beta)
    ns = -(-nb // Ls)
    zloc = []
    for j in range(ns - 1):
        Zt = np.zeros((d, 2 * d))
        Zt[:, d:] = np.eye(d)
        for c in range(j * Ls, min((j + 1) * Ls, nb)):
            sl = slice(c * C, (c + 1) * C)
            Kc, Vc, G, bc = K[sl], V[sl], np.cumsum(la[sl]), be[sl]
            D = np.minimum(G[:, None] - G[None, :], 0.0)
            L = np.tril(np.ones((C, C)), -1) * bc[:, None] * np.exp(D) * (Kc @ Kc.T)
            Tm = np.linalg.inv(np.eye(C) + L)
            W = Tm @ ((bc * np.exp(G))[:, None] * Kc)
            U = Tm @ (bc[:, None] * Vc)
            Kt = np.exp(G[-1] - G)[:, None] * Kc
            Delta = np.concatenate([U, np.zeros((C, d))], 1) - W @ Zt
            Zt = np.exp(G[-1]) * Zt + Kt.T @ Delta
        zloc.append(Zt)
    St = np.zeros((d, d))
    starts = [St]
    for j in range(ns - 1):
        St = zloc[j][:, d:] @ St + zloc[j][:, :d]
        starts.append(St)
    return starts


def chunk_core_backward(qh, kh, vh, log_alpha, beta, do, C=64):
    """Gradients of the recurrence (step 4) by the block algebra above, for
    L with dL/do = do: returns dq^ (unscaled q^), dk^, dv^, d log alpha and
    dbeta, all [B,T,H,...] fp64.  The design of a blocked backward: per
    block, last block first, carrying dS = dL/dS at the block's end:

      O   = diag(e^G) Q S0^T + P Delta,  P = (M o e^(G_r-G_i) o Q K^T)
      S_C = e^(G_C) S0 + Delta^T Kd,     Kd = diag(e^(G_C-G)) K
      Delta = U - W S0^T,  W = T diag(beta e^G) K,  U = T diag(beta) V,
      T = (I + L)^-1,      L = tril_strict(beta_r e^(G_r-G_j) K K^T)

    taken back in reverse order (dT to dL through dL = -T^T dT T^T), with
    every e^G factor's gradient collected into dG and d log alpha the
    reverse cumulative sum of dG."""
    B, T, H, dk = qh.shape
    dv = vh.shape[-1]
    nc = -(-T // C)
    Tp = nc * C
    scale = 1.0 / np.sqrt(dk)
    out = {n: np.zeros(s) for n, s in (("dq", qh.shape), ("dk", kh.shape), ("dv", vh.shape),
                                       ("dla", log_alpha.shape), ("dbeta", beta.shape))}
    strict = np.tril(np.ones((C, C)), -1)
    incl = np.tril(np.ones((C, C)))
    I = np.eye(C)
    for b in range(B):
        for h in range(H):
            def pad(x):
                o_ = np.zeros((Tp,) + x.shape[1:])
                o_[:T] = x
                return o_
            Q = pad(qh[b, :, h]) * scale
            K, V = pad(kh[b, :, h]), pad(vh[b, :, h])
            la, be, dO = pad(log_alpha[b, :, h]), pad(beta[b, :, h]), pad(do[b, :, h])

            def block(c, S0):
                sl = slice(c * C, (c + 1) * C)
                G = np.cumsum(la[sl])
                Dm = np.minimum(G[:, None] - G[None, :], 0.0)
                f = dict(sl=sl, G=G, E=np.exp(G), bc=be[sl], Kc=K[sl], Vc=V[sl], Qc=Q[sl], dOc=dO[sl])
                f["Gam"], f["Gs"] = incl * np.exp(Dm), strict * np.exp(Dm)
                f["A"] = f["Kc"] @ f["Kc"].T
                f["L"] = f["Gs"] * f["bc"][:, None] * f["A"]
                f["Tm"] = np.linalg.inv(I + f["L"])
                f["Kb"] = (f["bc"] * f["E"])[:, None] * f["Kc"]
                f["Vb"] = f["bc"][:, None] * f["Vc"]
                f["W"], f["U"] = f["Tm"] @ f["Kb"], f["Tm"] @ f["Vb"]
                f["Delta"] = f["U"] - f["W"] @ S0.T
                f["P"] = f["Gam"] * (f["Qc"] @ f["Kc"].T)
                f["Kd"] = np.exp(G[-1] - G)[:, None] * f["Kc"]
                return f

            S = np.zeros((dv, dk))
            starts = []
            for c in range(nc):
                starts.append(S)
                f = block(c, S)
                S = np.exp(f["G"][-1]) * S + f["Delta"].T @ f["Kd"]
            dS = np.zeros((dv, dk))
            for c in range(nc - 1, -1, -1):
                S0 = starts[c]
                f = block(c, S0)
                G, E, bc, Kc, Vc, Qc, dOc = f["G"], f["E"], f["bc"], f["Kc"], f["Vc"], f["Qc"], f["dOc"]
                Tm, W, Delta, P, Kd, L, A, Gs, Gam = (f[n] for n in ("Tm", "W", "Delta", "P", "Kd", "L", "A", "Gs", "Gam"))
                gC = G[-1]
                dG, dE, dgC = np.zeros(C), np.zeros(C), 0.0
                dbeta = np.zeros(C)
                # O = diag(E) Q S0^T + P Delta
                dS0 = dOc.T @ (E[:, None] * Qc)
                dQ = E[:, None] * (dOc @ S0)
                dE += (dOc * (Qc @ S0.T)).sum(1)
                dP = (dOc @ Delta.T) * incl
                dDelta = P.T @ dOc
                dQK = dP * Gam
                dQ += dQK @ Kc
                dK = dQK.T @ Qc
                dPP = dP * P
                dG += dPP.sum(1) - dPP.sum(0)
                # S_C = e^gC S0 + Delta^T Kd
                dS0 += np.exp(gC) * dS
                dgC += np.exp(gC) * float((dS * S0).sum())
                dDelta += Kd @ dS.T
                dKd = Delta @ dS
                dK += np.exp(gC - G)[:, None] * dKd
                t = (dKd * Kd).sum(1)
                dgC += float(t.sum())
                dG -= t
                # Delta = U - W S0^T
                dU, dW = dDelta, -dDelta @ S0
                dS0 -= dDelta.T @ W
                # W = T Kb, U = T Vb
                dT = dW @ f["Kb"].T + dU @ f["Vb"].T
                dKb, dVb = Tm.T @ dW, Tm.T @ dU
                dK += (bc * E)[:, None] * dKb
                tk = (dKb * Kc).sum(1)
                dbeta += E * tk
                dE += bc * tk
                dV = bc[:, None] * dVb
                dbeta += (dVb * Vc).sum(1)
                # T = (I + L)^-1;  L = Gs beta_r A
                dL = -(Tm.T @ dT @ Tm.T) * strict
                dA = dL * Gs * bc[:, None]
                dK += (dA + dA.T) @ Kc
                dbeta += (dL * Gs * A).sum(1)
                dLL = dL * L
                dG += dLL.sum(1) - dLL.sum(0)
                # E = e^G, gC = G_{C-1}, G = cumsum(log alpha)
                dG += E * dE
                dG[-1] += dgC
                dla = np.cumsum(dG[::-1])[::-1]
                rows = min(C, T - c * C)
                r0 = c * C
                out["dq"][b, r0:r0 + rows, h] = dQ[:rows] * scale
                out["dk"][b, r0:r0 + rows, h] = dK[:rows]
                out["dv"][b, r0:r0 + rows, h] = dV[:rows]
                out["dla"][b, r0:r0 + rows, h] = dla[:rows]
                out["dbeta"][b, r0:r0 + rows, h] = dbeta[:rows]
                dS = dS0
    return out


def ut_backward(qh, kh, vh, log_alpha, beta, do, C=128):
    """The block backward as the tensor-core kernels take it (fp64, no rounding):
    the forward's block tiles (T, W, U, P = Aqk, Qt, Kt) and S0 at every block
    start, the state gradient dS at every block end by the reverse recurrence
      dDelta = P^T dO + Kt dS^T,  dS_start = e^(G_last) dS + dO^T Qt - dDelta^T W,
    then every block's local gradients from its tiles, S0 and dS alone:
      dQ  = diag(E) dO S0 + dQK K,  dQK = (dO Delta^T) o Gam
      dK  = dQK^T Q + diag(e^(G_last - G)) Delta dS + diag(beta E) T^T dW + (dA + dA^T) K
      dV  = diag(beta) T^T dDelta,  dW = -dDelta S0
      dL  = -(dKb W^T + dVb U^T) o strict,  dA = diag(beta) dL o Gam
    with dG collected from every e^G factor (row sums minus column sums of the
    decay-masked products) and d log alpha its reverse cumulative sum over the
    block, plus e^(G_last) <dS, S0> + sum(dKd o Kt) on every token.
    Returns the gradients (as chunk_core_backward) and the per-(b, h) lists of
    S0^T and dS^T per block (d_k x d_v)."""
    B, T, H, dk = qh.shape
    dv = vh.shape[-1]
    nc = -(-T // C)
    Tp = nc * C
    scale = 1.0 / np.sqrt(dk)
    out = {n: np.zeros(s) for n, s in (("dq", qh.shape), ("dk", kh.shape), ("dv", vh.shape),
                                       ("dla", log_alpha.shape), ("dbeta", beta.shape))}
    out["S0T"] = np.zeros((B, H, nc, dk, dv))
    out["dST"] = np.zeros((B, H, nc, dk, dv))
    strict = np.tril(np.ones((C, C)), -1)
    incl = np.tril(np.ones((C, C)))
    for b in range(B):
        for h in range(H):
            def pad(x):
                o_ = np.zeros((Tp,) + x.shape[1:])
                o_[:T] = x
                return o_
            Q = pad(qh[b, :, h]) * scale
            K, V = pad(kh[b, :, h]), pad(vh[b, :, h])
            la, be, dO = pad(log_alpha[b, :, h]), pad(beta[b, :, h]), pad(do[b, :, h])
            blocks = []
            S = np.zeros((dv, dk))
            for c in range(nc):
                sl = slice(c * C, (c + 1) * C)
                G = np.cumsum(la[sl])
                E, bc = np.exp(G), be[sl]
                Dm = np.minimum(G[:, None] - G[None, :], 0.0)
                Gs, Gam = strict * np.exp(Dm), incl * np.exp(Dm)
                Kc, Vc, Qc = K[sl], V[sl], Q[sl]
                A = Kc @ Kc.T
                Tm = np.linalg.inv(np.eye(C) + Gs * bc[:, None] * A)
                W, U = Tm @ ((bc * E)[:, None] * Kc), Tm @ (bc[:, None] * Vc)
                P = Gam * (Qc @ Kc.T)
                Qt, Kt = E[:, None] * Qc, np.exp(G[-1] - G)[:, None] * Kc
                blocks.append(dict(G=G, E=E, bc=bc, Kc=Kc, Vc=Vc, Qc=Qc, Tm=Tm, W=W, U=U, P=P, Qt=Qt, Kt=Kt,
                                   S0=S.copy(), Gs=Gs, Gam=Gam, A=A, dO=dO[sl]))
                out["S0T"][b, h, c] = S.T
                S = np.exp(G[-1]) * S + (U - W @ S.T).T @ Kt
            dS = np.zeros((dv, dk))
            dS_end = [None] * nc
            for c in range(nc - 1, -1, -1):
                f = blocks[c]
                dS_end[c] = dS
                out["dST"][b, h, c] = dS.T
                dDelta = f["P"].T @ f["dO"] + f["Kt"] @ dS.T
                dS = np.exp(f["G"][-1]) * dS + f["dO"].T @ f["Qt"] - dDelta.T @ f["W"]
            for c in range(nc):
                f = blocks[c]
                G, E, bc, Kc, Vc, Qc = f["G"], f["E"], f["bc"], f["Kc"], f["Vc"], f["Qc"]
                Tm, W, U, P, Kt, S0, Gs, Gam, A, dOc = (f[n] for n in ("Tm", "W", "U", "P", "Kt", "S0", "Gs", "Gam",
                                                                        "A", "dO"))
                dSc, gL = dS_end[c], G[-1]
                Delta = U - W @ S0.T
                dDelta = P.T @ dOc + Kt @ dSc.T
                dOS = dOc @ S0
                dE = (dOS * Qc).sum(1)
                dPr = dOc @ Delta.T
                dQK = dPr * Gam
                dPP = dPr * P
                dG = dPP.sum(1) - dPP.sum(0)
                dQ = E[:, None] * dOS + dQK @ Kc
                dKd = Delta @ dSc
                t = (dKd * Kt).sum(1)
                dG -= t
                dgC = np.exp(gL) * float((dSc * S0).sum()) + float(t.sum())
                dK = dQK.T @ Qc + np.exp(gL - G)[:, None] * dKd
                dW = -dDelta @ S0
                dKb, dVb = Tm.T @ dW, Tm.T @ dDelta
                tk = (dKb * Kc).sum(1)
                dK += (bc * E)[:, None] * dKb
                dbeta = E * tk + (dVb * Vc).sum(1)
                dE += bc * tk
                dL = -(dKb @ W.T + dVb @ U.T) * strict
                dLGA = dL * Gs * A
                dbeta += dLGA.sum(1)
                dLL = bc[:, None] * dLGA
                dG += dLL.sum(1) - dLL.sum(0)
                dA = bc[:, None] * dL * Gs
                dK += (dA + dA.T) @ Kc
                dG += E * dE
                dla = np.cumsum(dG[::-1])[::-1] + dgC
                rows = min(C, T - c * C)
                r0 = c * C
                out["dq"][b, r0:r0 + rows, h] = dQ[:rows] * scale
                out["dk"][b, r0:r0 + rows, h] = dK[:rows]
                out["dv"][b, r0:r0 + rows, h] = bc[:rows, None] * dVb[:rows]
                out["dla"][b, r0:r0 + rows, h] = dla[:rows]
                out["dbeta"][b, r0:r0 + rows, h] = dbeta[:rows]
    return out
