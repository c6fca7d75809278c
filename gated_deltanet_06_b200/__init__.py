"""Python binding of libgdn_b200.so, the sm_100a Gated DeltaNet forward.

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  The binding fails loudly (ImportError) when the library has
not been built; there is no fallback.  PyTorch is used for device memory and
streams only.

    import gated_deltanet_06_b200 as gdn
    y = gdn.forward(q, k, v, z, g, b, conv_q, conv_k, conv_v, A_log, dt_bias, norm_w)
"""
from __future__ import annotations

import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "gdn.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python gated_deltanet_06_b200/build.py` "
                      "(the GDN forward has no CPU fallback)")
_lib = ctypes.CDLL(LIB_PATH)

# gdn_status
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE_CHECK, ERR_NO_DEVICE = range(7)
# gdn_dtype
DTYPE_BF16, DTYPE_F32, DTYPE_F16 = 0, 1, 2
FLAG_DEBUG_CHECKS = 0x1
FLAG_FORCE_SIMT = 0x2
FLAG_REVERSE = 0x4
FLAG_FUSED = 0x8
FLAG_TEST_WAIT_TIMEOUT = 0x100


class Config(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("d_k", ctypes.c_int),
                ("d_v", ctypes.c_int), ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
                ("conv_size", ctypes.c_int), ("chunk", ctypes.c_int), ("l2_eps", ctypes.c_float),
                ("norm_eps", ctypes.c_float), ("tok_stride", ctypes.c_longlong), ("flags", ctypes.c_uint)]


class Inputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("q", "k", "v", "z", "g", "b", "conv_q", "conv_k", "conv_v",
                                                 "A_log", "dt_bias", "norm_w")]


GRAD_NAMES = ("dq", "dk", "dv", "dz", "dg", "db", "dconv_q", "dconv_k", "dconv_v", "dA_log", "ddt_bias", "dnorm_w")


class Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in GRAD_NAMES]


_vp = ctypes.c_void_p
_lib.gdn_plan.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(_vp), ctypes.POINTER(ctypes.c_size_t)]
_lib.gdn_plan.restype = ctypes.c_int
_lib.gdn_forward.argtypes = [_vp, ctypes.POINTER(Inputs), _vp, _vp, _vp]
_lib.gdn_forward.restype = ctypes.c_int
_lib.gdn_forward_state.argtypes = [_vp, ctypes.POINTER(Inputs), _vp, _vp, _vp, _vp, _vp]
_lib.gdn_forward_state.restype = ctypes.c_int
_lib.gdn_backward.argtypes = [_vp, ctypes.POINTER(Inputs), _vp, ctypes.POINTER(Grads), _vp, _vp]
_lib.gdn_backward.restype = ctypes.c_int
_lib.gdn_backward_timed.argtypes = [_vp, ctypes.POINTER(Inputs), _vp, ctypes.POINTER(Grads), _vp, _vp,
                                    ctypes.POINTER(_vp), ctypes.c_int]
_lib.gdn_backward_timed.restype = ctypes.c_int
_lib.gdn_backward_workspace_bytes.argtypes = [_vp]
_lib.gdn_backward_workspace_bytes.restype = ctypes.c_size_t
_lib.gdn_backward_workspace_offsets.argtypes = [_vp, ctypes.POINTER(ctypes.c_size_t), ctypes.c_int]
_lib.gdn_backward_workspace_offsets.restype = ctypes.c_int
_lib.gdn_backward_launches.argtypes = [_vp]
_lib.gdn_backward_launches.restype = ctypes.c_int
_lib.gdn_forward_timed.argtypes = [_vp, ctypes.POINTER(Inputs), _vp, _vp, _vp, ctypes.POINTER(_vp), ctypes.c_int]
_lib.gdn_forward_timed.restype = ctypes.c_int
_lib.gdn_forward_host.argtypes = [_vp, ctypes.POINTER(Inputs), _vp, _vp, _vp, _vp]
_lib.gdn_forward_host.restype = ctypes.c_int
_lib.gdn_forward_noalloc.argtypes = [_vp, ctypes.POINTER(Inputs), _vp, _vp]
_lib.gdn_forward_noalloc.restype = ctypes.c_int
NOALLOC_SCRATCH_BYTES = 64 << 20
_lib.gdn_staging_bytes.argtypes = [_vp]
_lib.gdn_staging_bytes.restype = ctypes.c_size_t
_lib.gdn_get_device_status.argtypes = [_vp, _vp, _vp]
_lib.gdn_get_device_status.restype = ctypes.c_int
_lib.gdn_launches_per_forward.argtypes = [_vp]
_lib.gdn_launches_per_forward.restype = ctypes.c_int
_lib.gdn_plan_uses_tensor_path.argtypes = [_vp]
_lib.gdn_plan_uses_tensor_path.restype = ctypes.c_int
_lib.gdn_plan_segments.argtypes = [_vp]
_lib.gdn_plan_segments.restype = ctypes.c_int
_lib.gdn_workspace_offsets.argtypes = [_vp, ctypes.POINTER(ctypes.c_size_t), ctypes.c_int]
_lib.gdn_workspace_offsets.restype = ctypes.c_int
_lib.gdn_destroy.argtypes = [_vp]
_lib.gdn_destroy.restype = ctypes.c_int
_lib.gdn_status_string.argtypes = [ctypes.c_int]
_lib.gdn_status_string.restype = ctypes.c_char_p


class BlockConfig(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("D", ctypes.c_int), ("out_dtype", ctypes.c_int), ("l2_eps", ctypes.c_float),
                ("norm_eps", ctypes.c_float), ("flags", ctypes.c_uint)]


BLOCK_NAMES = ("x", "w_in", "w_out", "conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "norm_w")


class BlockInputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in BLOCK_NAMES]


_lib.gdn_block_plan.argtypes = [ctypes.POINTER(BlockConfig), ctypes.POINTER(_vp), ctypes.POINTER(ctypes.c_size_t)]
_lib.gdn_block_plan.restype = ctypes.c_int
_lib.gdn_block_forward.argtypes = [_vp, ctypes.POINTER(BlockInputs), _vp, _vp, _vp]
_lib.gdn_block_forward.restype = ctypes.c_int
_lib.gdn_block_forward_timed.argtypes = [_vp, ctypes.POINTER(BlockInputs), _vp, _vp, _vp, ctypes.POINTER(_vp),
                                         ctypes.c_int]
_lib.gdn_block_forward_timed.restype = ctypes.c_int
_lib.gdn_block_launches.argtypes = [_vp]
_lib.gdn_block_launches.restype = ctypes.c_int
_lib.gdn_block_device_status.argtypes = [_vp, _vp, _vp]
_lib.gdn_block_device_status.restype = ctypes.c_int
_lib.gdn_block_destroy.argtypes = [_vp]
_lib.gdn_block_destroy.restype = ctypes.c_int


class GDNError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


def status_string(s: int) -> str:
    return _lib.gdn_status_string(int(s)).decode()


def declared_symbols() -> list[str]:
    """Function names include/gdn.h declares."""
    text = open(HEADER_PATH).read()
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(gdn_\w+)\s*\(", text, flags=re.M)))


def library():
    return _lib


def _check(rc: int, where: str):
    if rc != OK:
        raise GDNError(rc, where)


class Plan:
    """A gdn_plan_t: validated shapes and the workspace layout (host state only)."""

    def __init__(self, B, T, H, d, in_dtype=DTYPE_BF16, out_dtype=None, l2_eps=1e-6, norm_eps=1e-6,
                 tok_stride=0, flags=0):
        self.cfg = Config(B, T, H, d, d, in_dtype, in_dtype if out_dtype is None else out_dtype, 4, 64,
                          l2_eps, norm_eps, tok_stride, flags)
        self._h = _vp()
        ws = ctypes.c_size_t()
        _check(_lib.gdn_plan(ctypes.byref(self.cfg), ctypes.byref(self._h), ctypes.byref(ws)), "gdn_plan")
        self.workspace_bytes = ws.value

    @property
    def handle(self):
        return self._h

    @property
    def staging_bytes(self) -> int:
        return _lib.gdn_staging_bytes(self._h)

    @property
    def launches(self) -> int:
        return _lib.gdn_launches_per_forward(self._h)

    @property
    def uses_tensor_path(self) -> bool:
        return bool(_lib.gdn_plan_uses_tensor_path(self._h))

    @property
    def segments(self) -> int:
        return _lib.gdn_plan_segments(self._h)

    def forward_raw(self, ptrs: dict, y: int, workspace: int, stream: int) -> None:
        """gdn_forward with raw device addresses (ints)."""
        ins = Inputs(*[ptrs[n] for n, _ in Inputs._fields_])
        _check(_lib.gdn_forward(self._h, ctypes.byref(ins), y, workspace, stream), "gdn_forward")

    def forward_state_raw(self, ptrs: dict, s0: int, y: int, s_end: int, workspace: int, stream: int) -> None:
        """gdn_forward_state: s0 / s_end are device addresses of [B][H][d][d] fp32 states (0 = none)."""
        ins = Inputs(*[ptrs[n] for n, _ in Inputs._fields_])
        _check(_lib.gdn_forward_state(self._h, ctypes.byref(ins), s0 or None, y, s_end or None, workspace, stream),
               "gdn_forward_state")

    @property
    def backward_workspace_bytes(self) -> int:
        return _lib.gdn_backward_workspace_bytes(self._h)

    @property
    def backward_launches(self) -> int:
        return _lib.gdn_backward_launches(self._h)

    def backward_raw(self, ptrs: dict, dy: int, grads: dict, workspace: int, stream: int) -> None:
        """gdn_backward with raw device addresses: grads maps GRAD_NAMES to fp32 buffers."""
        ins = Inputs(*[ptrs[n] for n, _ in Inputs._fields_])
        gr = Grads(*[grads[n] for n in GRAD_NAMES])
        _check(_lib.gdn_backward(self._h, ctypes.byref(ins), dy, ctypes.byref(gr), workspace, stream), "gdn_backward")

    def backward_timed_raw(self, ptrs: dict, dy: int, grads: dict, workspace: int, stream: int, events: list) -> None:
        """gdn_backward_timed: `events` are cudaEvent_t handles (ints), backward_launches + 1 of them."""
        ins = Inputs(*[ptrs[n] for n, _ in Inputs._fields_])
        gr = Grads(*[grads[n] for n in GRAD_NAMES])
        arr = (_vp * len(events))(*events)
        _check(_lib.gdn_backward_timed(self._h, ctypes.byref(ins), dy, ctypes.byref(gr), workspace, stream, arr,
                                       len(events)), "gdn_backward_timed")

    def forward_timed_raw(self, ptrs: dict, y: int, workspace: int, stream: int, events: list) -> None:
        """gdn_forward_timed: `events` are cudaEvent_t handles (ints), launches + 1 of them."""
        ins = Inputs(*[ptrs[n] for n, _ in Inputs._fields_])
        arr = (_vp * len(events))(*events)
        _check(_lib.gdn_forward_timed(self._h, ctypes.byref(ins), y, workspace, stream, arr, len(events)),
               "gdn_forward_timed")

    def forward_noalloc_raw(self, ptrs: dict, y: int, stream: int) -> None:
        """gdn_forward_noalloc: the workspace comes from the library's fixed
        device array instead of the caller (for callers that cannot allocate)."""
        ins = Inputs(*[ptrs[n] for n, _ in Inputs._fields_])
        _check(_lib.gdn_forward_noalloc(self._h, ctypes.byref(ins), y, stream), "gdn_forward_noalloc")

    def forward_host_raw(self, ptrs: dict, y_host: int, staging: int, workspace: int, stream: int) -> None:
        """gdn_forward_host with raw host input addresses and device staging/workspace."""
        ins = Inputs(*[ptrs[n] for n, _ in Inputs._fields_])
        _check(_lib.gdn_forward_host(self._h, ctypes.byref(ins), y_host, staging, workspace, stream),
               "gdn_forward_host")

    WS_FIELDS = ("status", "qh", "kh", "vh", "G", "beta", "log_alpha", "W", "U", "Qt", "Kt", "Aqk", "o", "Zloc",
                 "Sstart", "seg_states", "seg_start")

    def workspace_offsets(self) -> dict:
        arr = (ctypes.c_size_t * len(self.WS_FIELDS))()
        n = _lib.gdn_workspace_offsets(self._h, arr, len(self.WS_FIELDS))
        return {self.WS_FIELDS[i]: arr[i] for i in range(n)}

    BWD_WS_FIELDS = ("T", "S0", "o", "dO", "dSloc", "dSend", "dSb", "dqh", "dkh", "dvh", "dla", "dbeta",
                     "dnw_part", "dconv_part", "dA_part")

    def backward_workspace_offsets(self) -> dict:
        """Offsets of the tensor-core backward's buffers in the gdn_backward workspace (empty for
        plans without that backward)."""
        arr = (ctypes.c_size_t * len(self.BWD_WS_FIELDS))()
        n = _lib.gdn_backward_workspace_offsets(self._h, arr, len(self.BWD_WS_FIELDS))
        return {self.BWD_WS_FIELDS[i]: arr[i] for i in range(n)}

    def device_status(self, workspace: int, stream: int) -> int:
        return _lib.gdn_get_device_status(self._h, workspace, stream)

    def close(self):
        if self._h:
            _lib.gdn_destroy(self._h)
            self._h = _vp()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------- torch helpers
def _torch_dtype_code(t):
    import torch
    return {torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16, torch.float32: DTYPE_F32}[t]


_NAMES = ("q", "k", "v", "z", "g", "b", "conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "norm_w")


def tensor_ptrs(tensors: dict) -> dict:
    return {n: tensors[n].data_ptr() for n in _NAMES}


def forward(q, k, v, z, g, b, conv_q, conv_k, conv_v, A_log, dt_bias, norm_w, out_dtype=None,
            l2_eps=1e-6, norm_eps=1e-6, plan: Plan | None = None, workspace=None, y=None, stream=None,
            s0=None, return_state=False, reverse=False):
    """GDN forward on CUDA tensors (q, k, v, z [B,T,H,d]; g, b [B,T,H] fp32; conv_* [H*d,4];
    A_log, dt_bias [H]; norm_w [d]).  Returns y [B,T,H,d].  With s0 (a [B,H,d,d] fp32 state S[i][j],
    i over d_v, j over d_k) the recurrence starts from it; with return_state=True the call returns
    (y, s_end), s_end the [B,H,d,d] fp32 state after the last token.  reverse=True runs the
    anti-causal scan (token T-1 first; s0 / s_end are then the states before token T-1 and after
    token 0); a given plan must carry FLAG_REVERSE exactly when reverse=True."""
    import torch
    B, T, H, d = q.shape
    in_code = _torch_dtype_code(q.dtype)
    odt = q.dtype if out_dtype is None else out_dtype
    if plan is None:
        plan = Plan(B, T, H, d, in_code, _torch_dtype_code(odt), l2_eps, norm_eps, q.stride(1),
                    flags=FLAG_REVERSE if reverse else 0)
    elif bool(plan.cfg.flags & FLAG_REVERSE) != bool(reverse):
        raise ValueError("the plan's scan direction differs from reverse=")
    if workspace is None:
        workspace = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=q.device)
    if y is None:
        y = torch.empty((B, T, H, d), dtype=odt, device=q.device)
    s = torch.cuda.current_stream(q.device).cuda_stream if stream is None else stream
    t = dict(q=q, k=k, v=v, z=z, g=g, b=b, conv_q=conv_q, conv_k=conv_k, conv_v=conv_v, A_log=A_log,
             dt_bias=dt_bias, norm_w=norm_w)
    if s0 is None and not return_state:
        plan.forward_raw(tensor_ptrs(t), y.data_ptr(), workspace.data_ptr(), s)
        return y
    if s0 is not None and (s0.dtype != torch.float32 or tuple(s0.shape) != (B, H, d, d) or not s0.is_contiguous()):
        raise ValueError("s0 must be a contiguous [B, H, d, d] float32 tensor")
    s_end = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device) if return_state else None
    plan.forward_state_raw(tensor_ptrs(t), 0 if s0 is None else s0.data_ptr(), y.data_ptr(),
                           0 if s_end is None else s_end.data_ptr(), workspace.data_ptr(), s)
    return (y, s_end) if return_state else y


def backward(q, k, v, z, g, b, conv_q, conv_k, conv_v, A_log, dt_bias, norm_w, dy, l2_eps=1e-6, norm_eps=1e-6,
             plan: Plan | None = None, workspace=None, stream=None) -> dict:
    """Gradients of sum(y * dy) for the forward of the same arguments (dy [B,T,H,d], the output's
    dtype).  Returns a dict of fp32 CUDA tensors keyed by GRAD_NAMES (dq .. dnorm_w)."""
    import torch
    B, T, H, d = q.shape
    if plan is None:
        plan = Plan(B, T, H, d, _torch_dtype_code(q.dtype), _torch_dtype_code(dy.dtype), l2_eps, norm_eps,
                    q.stride(1))
    if workspace is None:
        workspace = torch.empty(plan.backward_workspace_bytes, dtype=torch.uint8, device=q.device)
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    out = {n: torch.empty((B, T, H, d), **f32) for n in ("dq", "dk", "dv", "dz")}
    out.update(dg=torch.empty((B, T, H), **f32), db=torch.empty((B, T, H), **f32),
               dA_log=torch.empty(H, **f32), ddt_bias=torch.empty(H, **f32), dnorm_w=torch.empty(d, **f32))
    for n in ("dconv_q", "dconv_k", "dconv_v"):
        out[n] = torch.empty((H * d, 4), **f32)
    s = torch.cuda.current_stream(dev).cuda_stream if stream is None else stream
    t = dict(q=q, k=k, v=v, z=z, g=g, b=b, conv_q=conv_q, conv_k=conv_k, conv_v=conv_v, A_log=A_log,
             dt_bias=dt_bias, norm_w=norm_w)
    plan.backward_raw(tensor_ptrs(t), dy.contiguous().data_ptr(), {n: out[n].data_ptr() for n in GRAD_NAMES},
                      workspace.data_ptr(), s)
    return out


# ------------------------------------------------------------------ the layer
class BlockPlan:
    """A gdn_block_plan_t: the GDN layer with its input and output projections (host state only)."""

    def __init__(self, B, T, H, d, D, out_dtype=DTYPE_BF16, l2_eps=1e-6, norm_eps=1e-6, flags=0):
        self.cfg = BlockConfig(B, T, H, d, D, out_dtype, l2_eps, norm_eps, flags)
        self._h = _vp()
        ws = ctypes.c_size_t()
        _check(_lib.gdn_block_plan(ctypes.byref(self.cfg), ctypes.byref(self._h), ctypes.byref(ws)),
               "gdn_block_plan")
        self.workspace_bytes = ws.value

    @property
    def launches(self) -> int:
        return _lib.gdn_block_launches(self._h)

    def forward_raw(self, ptrs: dict, out: int, workspace: int, stream: int) -> None:
        ins = BlockInputs(*[ptrs[n] for n in BLOCK_NAMES])
        _check(_lib.gdn_block_forward(self._h, ctypes.byref(ins), out, workspace, stream), "gdn_block_forward")

    def forward_timed_raw(self, ptrs: dict, out: int, workspace: int, stream: int, events: list) -> None:
        ins = BlockInputs(*[ptrs[n] for n in BLOCK_NAMES])
        arr = (_vp * len(events))(*events)
        _check(_lib.gdn_block_forward_timed(self._h, ctypes.byref(ins), out, workspace, stream, arr, len(events)),
               "gdn_block_forward_timed")

    BWD_WS_FIELDS = ("T", "S0", "o", "dO", "dSloc", "dSend", "dSb", "dqh", "dkh", "dvh", "dla", "dbeta",
                     "dnw_part", "dconv_part", "dA_part")

    def backward_workspace_offsets(self) -> dict:
        """Offsets of the tensor-core backward's buffers in the gdn_backward workspace (empty for
        plans without that backward)."""
        arr = (ctypes.c_size_t * len(self.BWD_WS_FIELDS))()
        n = _lib.gdn_backward_workspace_offsets(self._h, arr, len(self.BWD_WS_FIELDS))
        return {self.BWD_WS_FIELDS[i]: arr[i] for i in range(n)}

    def device_status(self, workspace: int, stream: int) -> int:
        return _lib.gdn_block_device_status(self._h, workspace, stream)

    def close(self):
        if self._h:
            _lib.gdn_block_destroy(self._h)
            self._h = _vp()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def block_forward(x, w_in, w_out, conv_q, conv_k, conv_v, A_log, dt_bias, norm_w, out_dtype=None, l2_eps=1e-6,
                  norm_eps=1e-6, plan: BlockPlan | None = None, workspace=None, out=None, stream=None):
    """The GDN layer on CUDA tensors: x [B,T,D] bf16, w_in [4*H*d + 2*H, D] bf16 (rows q, k, v, z, g, b),
    w_out [D, H*d] bf16, conv_* [H*d, 4], A_log, dt_bias [H], norm_w [d] fp32.  Returns out [B,T,D]
    (bf16, or out_dtype=torch.float32): (x W_in^T -> GDN forward -> y W_out^T)."""
    import torch
    B, T, D = x.shape
    H = A_log.shape[0]
    d = norm_w.shape[0]
    odt = torch.bfloat16 if out_dtype is None else out_dtype
    if plan is None:
        plan = BlockPlan(B, T, H, d, D, _torch_dtype_code(odt), l2_eps, norm_eps)
    if workspace is None:
        workspace = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((B, T, D), dtype=odt, device=x.device)
    s = torch.cuda.current_stream(x.device).cuda_stream if stream is None else stream
    t = dict(x=x, w_in=w_in, w_out=w_out, conv_q=conv_q, conv_k=conv_k, conv_v=conv_v, A_log=A_log,
             dt_bias=dt_bias, norm_w=norm_w)
    for n, v in t.items():
        if not v.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    plan.forward_raw({n: v.data_ptr() for n, v in t.items()}, out.data_ptr(), workspace.data_ptr(), s)
    return out
