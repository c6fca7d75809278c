"""Input helpers for the carried-state tests (no arithmetic of the method)."""
import numpy as np

_T_AXIS = ("q", "k", "v", "z", "q_bits", "k_bits", "v_bits", "z_bits", "g", "b")


def slice_tokens(inp: dict, t0: int, t1: int) -> dict:
    """Tokens [t0, t1) of every (b, h) as an input of its own."""
    out = {}
    for n, a in inp.items():
        if n in _T_AXIS:
            out[n] = np.ascontiguousarray(a[:, t0:t1])
        elif n == "meta":
            out[n] = dict(a, T=t1 - t0)
        else:
            out[n] = a
    return out


def split_stream(inp: dict, t1: int, hist: int = 3):
    """One input as two pieces for streaming: tokens [0, t1), and [t1 - hist, T) whose first hist
    tokens only carry the short convolutions' history: their gates are made neutral (g = b = -200:
    alpha = 1 and beta = 0 to working precision), so the state passes through them unchanged and
    their outputs are dropped."""
    first = slice_tokens(inp, 0, t1)
    second = slice_tokens(inp, t1 - hist, inp["q"].shape[1])
    for n in ("g", "b"):
        second[n] = second[n].copy()
        second[n][:, :hist] = -200.0
    return first, second


def random_state(B: int, H: int, d: int, seed: int, scale: float = 0.5) -> np.ndarray:
    """A seeded [B, H, d, d] fp32 state S (S[i][j]: i over d_v, j over d_k)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return (np.float32(scale) * rng.standard_normal((B, H, d, d), dtype=np.float32)).astype(np.float32)
