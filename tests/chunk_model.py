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
