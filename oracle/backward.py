"""The oracle's backward: the gradient of the Gated DeltaNet forward (steps
1-5 of the oracle's forward) with respect to every input and parameter, by
reverse-mode differentiation written out step by step in plain fp64 numpy.

TEST INFRASTRUCTURE ONLY, like the rest of the oracle package.

The method's pages train the GDN modules (the LinMorph page: distillation and
joint recovery after the weight mapping), which needs this gradient; they do
not write it out.  It is the derivative of the forward the oracle already
defines, taken one step at a time in reverse order:

  5  y = o * rn * w * SiLU(z),  rn = 1/sqrt(mean(o^2) + eps)
  4  S_t = alpha_t S_{t-1} + delta_t k^_t^T,  delta_t = beta_t (v^_t - alpha_t u_t),
     u_t = S_{t-1} k^_t,  o_t = S_t q^_t / sqrt(d_k)   (the gated delta rule of
     reference [57] on the VMonarch page, rearranged)
  3  log alpha = -exp(A_log) softplus(g + dt_bias),  beta = sigmoid(b)
  2  q^ = q'/sqrt(|q'|^2 + eps), k^ likewise
  1  q' = SiLU(a), a = conv4(q) (tap 3 on the current token); likewise k', v^

forward() here recomputes the forward in numpy (pinned against the C oracle),
and vjp() returns dL/dx for L = sum(y * dy).  Pinned by central finite
differences of forward() in fp64.  Small cases only: the tape keeps every
state S_t.
"""
from __future__ import annotations

import numpy as np

DEFAULT_L2_EPS = 1e-6
DEFAULT_NORM_EPS = 1e-6


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _softplus(x):
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def _conv4(x, w):
    """a[t] = sum_k w[:, k] * x[t-3+k], zero before t = 0.  x [B,T,H,d], w [H*d, 4]."""
    B, T, H, d = x.shape
    wr = w.reshape(H, d, 4)
    a = np.zeros_like(x)
    for k in range(4):
        sh = 3 - k  # x[t - sh]
        if sh == 0:
            a += wr[None, None, :, :, k] * x
        elif sh < T:
            a[:, sh:] += wr[None, None, :, :, k] * x[:, :-sh]
    return a


def _tape(inp, l2_eps, norm_eps):
    f = {n: np.asarray(inp[n], dtype=np.float64) for n in
         ("q", "k", "v", "z", "g", "b", "conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "norm_w")}
    B, T, H, dk = f["q"].shape
    dv = f["v"].shape[-1]
    tp = {"f": f}
    for n in ("q", "k", "v"):
        a = _conv4(f[n], f["conv_" + n])
        tp["a_" + n] = a
        tp["s_" + n] = a * _sigmoid(a)  # SiLU
    for n in ("q", "k"):
        x = tp["s_" + n]
        nrm = np.sqrt((x * x).sum(-1, keepdims=True) + l2_eps)
        tp["n_" + n] = nrm
        tp["h_" + n] = x / nrm
    qh, kh, vh = tp["h_q"], tp["h_k"], tp["s_v"]
    xg = f["g"] + f["dt_bias"][None, None, :]
    la = -np.exp(f["A_log"])[None, None, :] * _softplus(xg)
    alpha, beta = np.exp(la), _sigmoid(f["b"])
    tp.update(xg=xg, la=la, alpha=alpha, beta=beta)
    scale = 1.0 / np.sqrt(dk)
    S = np.zeros((B, H, T + 1, dv, dk))  # S[:, :, t + 1] = state after token t
    u = np.zeros((B, T, H, dv))
    dl = np.zeros((B, T, H, dv))
    o = np.zeros((B, T, H, dv))
    for b in range(B):
        for h in range(H):
            St = np.zeros((dv, dk))
            for t in range(T):
                a_, be = alpha[b, t, h], beta[b, t, h]
                ut = St @ kh[b, t, h]
                dlt = be * (vh[b, t, h] - a_ * ut)
                St = a_ * St + np.outer(dlt, kh[b, t, h])
                S[b, h, t + 1] = St
                u[b, t, h], dl[b, t, h] = ut, dlt
                o[b, t, h] = St @ qh[b, t, h] * scale
    tp.update(S=S, u=u, dl=dl, o=o, scale=scale)
    rn = 1.0 / np.sqrt((o * o).mean(-1, keepdims=True) + norm_eps)
    sz = f["z"] * _sigmoid(f["z"])
    tp.update(rn=rn, sz=sz)
    y = o * rn * f["norm_w"] * sz
    return y, tp


def forward(inp: dict, l2_eps=DEFAULT_L2_EPS, norm_eps=DEFAULT_NORM_EPS):
    """y [B,T,H,d_v] fp64, recomputed in numpy (the same definition as the C oracle)."""
    return _tape(inp, l2_eps, norm_eps)[0]


def vjp(inp: dict, dy, l2_eps=DEFAULT_L2_EPS, norm_eps=DEFAULT_NORM_EPS) -> dict:
    """Gradients of L = sum(y * dy) with respect to q, k, v, z [B,T,H,d], g, b
    [B,T,H], conv_q, conv_k, conv_v [H*d,4], A_log, dt_bias [H] and norm_w
    [d_v], all fp64, plus the intermediate gradients do (w.r.t. o), dqh, dkh,
    dvh (w.r.t. q^ k^ v^), dalpha and dbeta [B,T,H]."""
    y, tp = _tape(inp, l2_eps, norm_eps)
    f = tp["f"]
    dy = np.asarray(dy, dtype=np.float64)
    B, T, H, dk = f["q"].shape
    dv = f["v"].shape[-1]
    grads = {}

    # 5: output norm and gate
    o, rn, sz, w, z = tp["o"], tp["rn"], tp["sz"], f["norm_w"], f["z"]
    grads["norm_w"] = (dy * o * rn * sz).sum(axis=(0, 1, 2))
    sig = _sigmoid(z)
    grads["z"] = dy * o * rn * w * sig * (1.0 + z * (1.0 - sig))
    gz = dy * w * sz  # dL/d(o * rn)
    do = rn * gz - o * rn ** 3 * (o * gz).sum(-1, keepdims=True) / dv
    grads["do"] = do

    # 4: the recurrence, backwards in time
    qh, kh, vh = tp["h_q"], tp["h_k"], tp["s_v"]
    alpha, beta, S, u, dl, scale = tp["alpha"], tp["beta"], tp["S"], tp["u"], tp["dl"], tp["scale"]
    dqh = np.zeros_like(qh)
    dkh = np.zeros_like(kh)
    dvh = np.zeros_like(vh)
    dalpha = np.zeros((B, T, H))
    dbeta = np.zeros((B, T, H))
    for b in range(B):
        for h in range(H):
            D = np.zeros((dv, dk))  # dL/dS_t
            for t in range(T - 1, -1, -1):
                a_, be = alpha[b, t, h], beta[b, t, h]
                St, Sp = S[b, h, t + 1], S[b, h, t]
                dot = do[b, t, h] * scale
                D = D + np.outer(dot, qh[b, t, h])
                dqh[b, t, h] = St.T @ dot
                ddl = D @ kh[b, t, h]                      # dL/d delta_t
                dkh[b, t, h] = D.T @ dl[b, t, h]           # through delta_t k^_t^T
                dvh[b, t, h] = be * ddl
                dbeta[b, t, h] = ddl @ (vh[b, t, h] - a_ * u[b, t, h])
                du = -a_ * be * ddl                        # dL/du_t
                dalpha[b, t, h] = (D * Sp).sum() - be * (ddl @ u[b, t, h])
                dkh[b, t, h] += Sp.T @ du                  # through u_t = S_{t-1} k^_t
                D = a_ * D + np.outer(du, kh[b, t, h])     # dL/dS_{t-1}
    grads.update(dqh=dqh, dkh=dkh, dvh=dvh, dalpha=dalpha, dbeta=dbeta)

    # 3: gates
    dla = dalpha * alpha                                   # d log alpha
    sp_grad = _sigmoid(tp["xg"])                           # softplus'
    eA = np.exp(f["A_log"])[None, None, :]
    grads["g"] = dla * (-eA * sp_grad)
    grads["dt_bias"] = grads["g"].sum(axis=(0, 1))
    grads["A_log"] = (dla * tp["la"]).sum(axis=(0, 1))     # d log alpha / dA_log = log alpha
    grads["b"] = dbeta * beta * (1.0 - beta)

    # 2: L2 norms;  1: SiLU and the short convolutions
    for n, dh in (("q", dqh), ("k", dkh), ("v", dvh)):
        if n != "v":
            x, nrm = tp["s_" + n], tp["n_" + n]
            xhat = x / nrm
            ds = (dh - xhat * (xhat * dh).sum(-1, keepdims=True)) / nrm
        else:
            ds = dh
        a = tp["a_" + n]
        sa = _sigmoid(a)
        da = ds * sa * (1.0 + a * (1.0 - sa))
        x = f[n]
        wr = f["conv_" + n].reshape(H, dv if n == "v" else dk, 4)
        dx = np.zeros_like(x)
        dw = np.zeros_like(wr)
        for k in range(4):
            sh = 3 - k  # a[t] uses x[t - sh] with weight w[:, k]
            if sh == 0:
                dx += wr[None, None, :, :, k] * da
                dw[:, :, k] = (da * x).sum(axis=(0, 1))
            elif sh < T:
                dx[:, :-sh] += wr[None, None, :, :, k] * da[:, sh:]
                dw[:, :, k] = (da[:, sh:] * x[:, :-sh]).sum(axis=(0, 1))
        grads[n] = dx
        grads["conv_" + n] = dw.reshape(-1, 4)
    return grads


def sum_magnitudes(inp: dict, dy, l2_eps=DEFAULT_L2_EPS, norm_eps=DEFAULT_NORM_EPS) -> dict:
    """For the parameter gradients that are sums over tokens, the sum of their terms' magnitudes:
    A_log and dt_bias [H] (terms d log alpha * log alpha and dL/dg, summed over b, t), norm_w [d_v]
    (terms dy * o * rn * SiLU(z), summed over b, t, h).  A sum whose terms carry a relative error e
    is off by at most e times this, so it sets the scale of a parity bound on such a gradient."""
    g = vjp(inp, dy, l2_eps, norm_eps)
    _, tp = _tape(inp, l2_eps, norm_eps)
    dy = np.asarray(dy, dtype=np.float64)
    dla = g["dalpha"] * tp["alpha"]
    return {"A_log": np.abs(dla * tp["la"]).sum(axis=(0, 1)),
            "dt_bias": np.abs(g["g"]).sum(axis=(0, 1)),
            "norm_w": np.abs(dy * tp["o"] * tp["rn"] * tp["sz"]).sum(axis=(0, 1, 2))}
