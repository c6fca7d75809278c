"""The oracle: a plain sequential fp64 CPU statement of the Gated DeltaNet
forward (gdn_oracle.c), with a thin ctypes wrapper.

TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's CPU
baseline leg may use it; the CUDA library and its Python binding never import
it, and it imports nothing from them.  See gdn_oracle.c for the definition
and the readings it takes where the method's pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_SO = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None

DEFAULT_L2_EPS = 1e-6
DEFAULT_NORM_EPS = 1e-6


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c with gcc -O2 (no fast-math) into oracle/_build."""
    os.makedirs(os.path.dirname(_SO), exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-o", _SO, _SRC, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_SO)
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def default_threads(units: int) -> int:
    return max(1, min(units, os.cpu_count() or 1))


def conv_silu(x, w):
    """Step 1: causal kernel-4 depthwise conv + SiLU.  x [B,T,H,d], w [H*d,4]."""
    lib = _load()
    x = _f32(x)
    B, T, H, d = x.shape
    out = np.empty(x.shape, np.float64)
    lib.oracle_conv_silu(ctypes.c_int(B), ctypes.c_int(T), ctypes.c_int(H), ctypes.c_int(d),
                         _p(x), _p(_f32(w)), _p(out))
    return out


def l2norm(x, eps=DEFAULT_L2_EPS):
    """Step 2: x / sqrt(|x|^2 + eps) over the last axis (returns a copy)."""
    lib = _load()
    y = _f64(x).copy()
    d = y.shape[-1]
    lib.oracle_l2norm(ctypes.c_longlong(y.size // d), ctypes.c_int(d), ctypes.c_double(eps), _p(y))
    return y


def gates(g, b, A_log, dt_bias):
    """Step 3: alpha, beta per (b, t, h).  g, b [B,T,H]."""
    lib = _load()
    g = _f32(g)
    B, T, H = g.shape
    alpha = np.empty(g.shape, np.float64)
    beta = np.empty(g.shape, np.float64)
    lib.oracle_gates(ctypes.c_int(B), ctypes.c_int(T), ctypes.c_int(H), _p(g), _p(_f32(b)),
                     _p(_f32(A_log)), _p(_f32(dt_bias)), _p(alpha), _p(beta))
    return alpha, beta


def core(qh, kh, vh, alpha, beta, s0=None, return_state=False, nthreads=None):
    """Step 4: the gated delta-rule recurrence on given (already prepared)
    q^, k^ [B,T,H,d_k], v^ [B,T,H,d_v], alpha, beta [B,T,H].  Returns o
    [B,T,H,d_v] = S_t q^_t / sqrt(d_k); with return_state, also the final
    states [B,H,d_v,d_k].  s0 is an optional initial state [B,H,d_v,d_k]."""
    lib = _load()
    qh, kh, vh = _f64(qh), _f64(kh), _f64(vh)
    alpha, beta = _f64(alpha), _f64(beta)
    B, T, H, dk = qh.shape
    dv = vh.shape[-1]
    o = np.empty((B, T, H, dv), np.float64)
    s0a = _f64(s0) if s0 is not None else None
    s_end = np.empty((B, H, dv, dk), np.float64) if return_state else None
    n = nthreads or default_threads(B * H)
    lib.oracle_core(ctypes.c_int(B), ctypes.c_int(T), ctypes.c_int(H), ctypes.c_int(dk),
                    ctypes.c_int(dv), _p(qh), _p(kh), _p(vh), _p(alpha), _p(beta), _p(o),
                    _p(s0a), _p(s_end), ctypes.c_int(n))
    return (o, s_end) if return_state else o


def output(o, z, norm_w, eps=DEFAULT_NORM_EPS):
    """Step 5: RMSNorm over d_v times norm_w times SiLU(z)."""
    lib = _load()
    o = _f64(o)
    z = _f32(z)
    dv = o.shape[-1]
    y = np.empty(o.shape, np.float64)
    lib.oracle_output(ctypes.c_longlong(o.size // dv), ctypes.c_int(dv), _p(o), _p(z),
                      _p(_f32(norm_w)), ctypes.c_double(eps), _p(y))
    return y


def forward(inp: dict, l2_eps=DEFAULT_L2_EPS, norm_eps=DEFAULT_NORM_EPS, nthreads=None,
            intermediates=False):
    """Steps 1-5 on an input dict from gdn_inputs.make_inputs.  Returns y
    [B,T,H,d_v] fp64 (and, with intermediates, a dict of q^, k^, v^, alpha,
    beta, o)."""
    lib = _load()
    q, k, v, z = (_f32(inp[n]) for n in ("q", "k", "v", "z"))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    y = np.empty((B, T, H, dv), np.float64)
    inter = None
    ptrs = [None] * 6
    if intermediates:
        inter = dict(qh=np.empty(q.shape), kh=np.empty(k.shape), vh=np.empty(v.shape),
                     alpha=np.empty((B, T, H)), beta=np.empty((B, T, H)), o=np.empty(v.shape))
        ptrs = [inter[n] for n in ("qh", "kh", "vh", "alpha", "beta", "o")]
    n = nthreads or default_threads(B * H)
    rc = lib.oracle_forward(
        ctypes.c_int(B), ctypes.c_int(T), ctypes.c_int(H), ctypes.c_int(dk), ctypes.c_int(dv),
        _p(q), _p(k), _p(v), _p(z), _p(_f32(inp["g"])), _p(_f32(inp["b"])),
        _p(_f32(inp["conv_q"])), _p(_f32(inp["conv_k"])), _p(_f32(inp["conv_v"])),
        _p(_f32(inp["A_log"])), _p(_f32(inp["dt_bias"])), _p(_f32(inp["norm_w"])),
        ctypes.c_double(l2_eps), ctypes.c_double(norm_eps), ctypes.c_int(n), _p(y),
        *[_p(a) for a in ptrs])
    if rc != 0:
        raise MemoryError("oracle_forward: out of host memory")
    return (y, inter) if intermediates else y


def forward_with_state(inp: dict, s0=None, l2_eps=DEFAULT_L2_EPS, norm_eps=DEFAULT_NORM_EPS, nthreads=None):
    """Steps 1-5 with the recurrent state carried in and out: s0
    [B,H,d_v,d_k] (None = zero) is the state S before token 0; returns y and
    the state after token T-1.  Composed of the step functions above; the
    short convolutions still see zero history before token 0."""
    qh = l2norm(conv_silu(inp["q"], inp["conv_q"]), l2_eps)
    kh = l2norm(conv_silu(inp["k"], inp["conv_k"]), l2_eps)
    vh = conv_silu(inp["v"], inp["conv_v"])
    alpha, beta = gates(inp["g"], inp["b"], inp["A_log"], inp["dt_bias"])
    o, s_end = core(qh, kh, vh, alpha, beta, s0=s0, return_state=True, nthreads=nthreads)
    return output(o, inp["z"], inp["norm_w"], norm_eps), s_end


_T_AXIS = ("q", "k", "v", "z", "g", "b")


def _flip_time(inp: dict) -> dict:
    out = dict(inp)
    for n in _T_AXIS:
        out[n] = np.ascontiguousarray(inp[n][:, ::-1])
    return out


def reverse(inp: dict, s0=None, l2_eps=DEFAULT_L2_EPS, norm_eps=DEFAULT_NORM_EPS, nthreads=None):
    """The anti-causal (reverse-direction) scan: steps 1-5 over the token order
    T-1, ..., 0, i.e. the forward of the time-reversed sequence, with its
    outputs put back in the original order.  Its short convolutions see the
    current and the three FOLLOWING tokens (zero past T-1), and the state runs
    from token T-1 down to token 0.  The pages leave the scan direction open
    (the LinGen page's linear branch is a bidirectional Mamba2 block); this is
    the one direction-reversal reading: the same operator on the reversed
    sequence.  Returns (y, state after token 0); s0 is the state before token
    T-1."""
    y, s_end = forward_with_state(_flip_time(inp), s0=s0, l2_eps=l2_eps, norm_eps=norm_eps, nthreads=nthreads)
    return np.ascontiguousarray(y[:, ::-1]), s_end


class _swapped_library:
    """Context manager used by the oracle's own mutation tests: temporarily
    route every call above to another build of gdn_oracle.c (a copy with a
    planted mistake, compiled on the CPU)."""

    def __init__(self, so_path):
        self.so_path = so_path

    def __enter__(self):
        global _lib
        self.saved = _load()
        _lib = ctypes.CDLL(self.so_path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def compile_variant(src_text: str, out_path: str) -> str:
    """Compile a (modified) copy of the oracle source to out_path; test use only."""
    c_path = out_path[:-3] + ".c"
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-o", out_path, c_path, "-lm"])
    return out_path


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()
