"""The C-ABI library loads and exports every function include/gdn.h declares,
and host-side validation behaves as documented -- no GPU and no compute
calls needed."""
import ctypes

import pytest


def _gdn():
    import gated_deltanet_06_b200 as gdn
    return gdn


def test_library_loads_and_exports_every_declared_symbol():
    gdn = _gdn()
    lib = gdn.library()
    declared = gdn.declared_symbols()
    assert len(declared) >= 9
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/gdn.h but not exported"


def test_status_strings():
    gdn = _gdn()
    for s in range(7):
        assert gdn.status_string(s) and gdn.status_string(s) != "unknown status"
    assert gdn.status_string(99) == "unknown status"


def _plan_rc(**kw):
    gdn = _gdn()
    cfg = dict(B=1, T=256, H=2, d_k=128, d_v=128, in_dtype=gdn.DTYPE_BF16, out_dtype=gdn.DTYPE_BF16, conv_size=4,
               chunk=64, l2_eps=1e-6, norm_eps=1e-6, tok_stride=0, flags=0)
    cfg.update(kw)
    c = gdn.Config(**cfg)
    h = ctypes.c_void_p()
    ws = ctypes.c_size_t()
    return gdn.library().gdn_plan(ctypes.byref(c), ctypes.byref(h), ctypes.byref(ws))


@pytest.mark.parametrize("kw,expect", [
    (dict(T=0), "INVALID_ARG"), (dict(B=0), "INVALID_ARG"), (dict(H=-1), "INVALID_ARG"),
    (dict(l2_eps=-1.0), "INVALID_ARG"), (dict(norm_eps=float("nan")), "INVALID_ARG"),
    (dict(tok_stride=100), "INVALID_ARG"), (dict(tok_stride=2 * 128 + 4), "INVALID_ARG"),
    (dict(d_k=96, d_v=96), "UNSUPPORTED"), (dict(d_k=128, d_v=64), "UNSUPPORTED"),
    (dict(conv_size=3), "UNSUPPORTED"), (dict(chunk=32), "UNSUPPORTED"), (dict(in_dtype=7), "UNSUPPORTED"),
])
def test_plan_validation_without_device(kw, expect):
    gdn = _gdn()
    assert _plan_rc(**kw) == getattr(gdn, "ERR_" + expect)


def test_plan_null_arguments():
    gdn = _gdn()
    assert gdn.library().gdn_plan(None, None, None) == gdn.ERR_INVALID_ARG
    assert gdn.library().gdn_destroy(None) == gdn.OK
    assert gdn.library().gdn_forward(None, None, None, None, None) == gdn.ERR_INVALID_ARG
    assert gdn.library().gdn_staging_bytes(None) == 0


def test_valid_plan_needs_an_sm100_device():
    gdn = _gdn()
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present; covered by the GPU tests")
    assert _plan_rc() == gdn.ERR_NO_DEVICE
