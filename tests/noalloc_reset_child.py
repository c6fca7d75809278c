"""Child process of the noalloc reset test (run by test_zz_no_alloc.py; not a
test module).  Runs gdn_forward and gdn_forward_noalloc on the same inputs,
resets the device with cudaDeviceReset, and runs both again: every output must
be bitwise equal.  Device memory comes straight from the CUDA runtime that the
library loaded, through ctypes."""
import ctypes
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))

import gdn_inputs  # noqa: E402
import gated_deltanet_06_b200 as gdn  # noqa: E402


def _runtime():
    # the process's one CUDA runtime: the shared library the GDN library itself was linked against
    with open("/proc/self/maps") as f:
        for line in f:
            if "libcudart.so" in line:
                rt = ctypes.CDLL(line.split()[-1])
                rt.cudaMalloc.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_size_t]
                rt.cudaMemcpy.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int]
                rt.cudaMemset.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t]
                return rt
    raise SystemExit("the CUDA runtime is not loaded")


RT = _runtime()
H2D, D2H = 1, 2


def _ok(rc, what):
    if rc != 0:
        raise SystemExit(f"{what}: CUDA error {rc}")


def _alloc(nbytes):
    p = ctypes.c_void_p()
    _ok(RT.cudaMalloc(ctypes.byref(p), nbytes), "cudaMalloc")
    return p.value


def _upload(a):
    a = np.ascontiguousarray(a)
    p = _alloc(a.nbytes)
    _ok(RT.cudaMemcpy(p, a.ctypes.data, a.nbytes, H2D), "cudaMemcpy H2D")
    return p


def _download(p, nbytes):
    out = np.empty(nbytes, dtype=np.uint8)
    _ok(RT.cudaMemcpy(out.ctypes.data, p, nbytes, D2H), "cudaMemcpy D2H")
    return out


def run_both(plan, inp):
    ptrs = {n: _upload(inp[n + "_bits"]) for n in ("q", "k", "v", "z")}
    for n in ("g", "b", "conv_q", "conv_k", "conv_v", "A_log", "dt_bias", "norm_w"):
        ptrs[n] = _upload(np.asarray(inp[n], dtype=np.float32))
    B, T, H, d = inp["q"].shape
    ybytes = B * T * H * d * 4
    y_ref, y, ws = _alloc(ybytes), _alloc(ybytes), _alloc(plan.workspace_bytes)
    _ok(RT.cudaMemset(ws, 0, plan.workspace_bytes), "cudaMemset")
    _ok(RT.cudaMemset(y, 0xFF, ybytes), "cudaMemset")
    plan.forward_raw(ptrs, y_ref, ws, 0)
    plan.forward_noalloc_raw(ptrs, y, 0)
    _ok(RT.cudaDeviceSynchronize(), "cudaDeviceSynchronize")
    if plan.device_status(ws, 0) != gdn.OK:
        raise SystemExit("device status of the forward")
    return _download(y_ref, ybytes), _download(y, ybytes)


def main():
    _ok(RT.cudaSetDevice(0), "cudaSetDevice")
    inp = gdn_inputs.make_inputs(1, 700, 2, 128, "bf16", -1.0, seed=41)
    plan = gdn.Plan(1, 700, 2, 128, gdn.DTYPE_BF16, gdn.DTYPE_F32)
    ref1, y1 = run_both(plan, inp)
    if not np.isfinite(ref1.view(np.float32)).all():
        raise SystemExit("non-finite forward output")
    if not np.array_equal(ref1, y1):
        raise SystemExit("noalloc differs from the forward before the reset")
    _ok(RT.cudaDeviceReset(), "cudaDeviceReset")
    ref2, y2 = run_both(plan, inp)
    if not (np.array_equal(ref2, ref1) and np.array_equal(y2, ref1)):
        raise SystemExit("noalloc differs from the forward after the reset")
    print("noalloc after reset: bitwise equal")


if __name__ == "__main__":
    main()
