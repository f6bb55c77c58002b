"""The allocation-free forward scan, esa_scan_fwd_noalloc, through the C ABI.

Some callers cannot allocate device memory where they run the scan (a
serving loop with a device-memory budget fixed at start-up, a latency-critical
path where cudaMalloc may synchronise the device, a foreign-language caller
that is only handed tensor pointers).  For them the library keeps its scratch
in a built-in static device array.  These tests check that entry point
against the ordinary esa_scan_fwd (which takes a caller-allocated workspace)
on two calls in a row -- the array is shared and keeps the previous call's
contents -- and that shapes needing more scratch than the array holds are
refused before anything runs.
"""
import ctypes

import pytest
import torch

from gated_linear_recurrence_b200 import esa, inputs
from tests._parity import DT, TOL, assert_close, host64

pytestmark = pytest.mark.gpu

ESA_ERR_NOALLOC_LIMIT = -8
NOALLOC_BYTES = 64 * 1024 * 1024
_CODE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}


def _lib():
    lib = esa.load_library()
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.esa_scan_fwd_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I, P]
    lib.esa_scan_fwd_noalloc.restype = I
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_fwd(lib, a, v, q, mode, E_init):
    B, T, H, D = a.shape
    y = torch.empty_like(a)
    E_final = torch.empty(B, H, D, dtype=torch.float32, device=a.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream(a.device).cuda_stream)
    rc = lib.esa_scan_fwd_noalloc(_ptr(a), _ptr(v), _ptr(q), _ptr(y), _ptr(E_final), B, T, H, D, mode,
                                  _ptr(E_init), _CODE[a.dtype], stream)
    return rc, y, E_final


def test_noalloc_forward_matches_workspace_forward_on_two_calls(cuda_device):
    lib = _lib()
    cases = [  # B, T, H, D, dtype, mode, seed: two different problems back to back
        (4, 1000, 4, 32, "f16", esa.CONTROLLED, 21),
        (3, 333, 2, 64, "bf16", esa.DIRECT, 22),
    ]
    for B, T, H, D, dt, mode, seed in cases:
        assert esa.esa_workspace_size(B, T, H, D, DT[dt]) <= NOALLOC_BYTES
        x = inputs.make_scan_inputs(B, T, H, D, dt, a_mean=2.0, seed=seed, with_dy=False)
        a, v, q = (x[k].to(cuda_device) for k in ("a", "v", "q"))
        E0 = inputs.make_state(B, H, D, seed=seed + 100, scale=0.5).to(cuda_device)
        y_ref, Ef_ref, _ = esa.esa_scan_fwd(a, v, q, mode=mode, E_init=E0)
        rc, y, Ef = _noalloc_fwd(lib, a, v, q, mode, E0)
        assert rc == 0, esa.esa_strerror(rc)
        torch.cuda.synchronize()
        tol = TOL[DT[dt]]
        assert_close(y, host64(y_ref), tol, f"noalloc y ({dt})")
        assert_close(Ef, host64(Ef_ref), tol, f"noalloc E_final ({dt})")


def test_noalloc_refuses_shapes_beyond_its_scratch(cuda_device):
    lib = _lib()
    B, T, H, D = 64, 16384, 4, 32
    assert esa.esa_workspace_size(B, T, H, D, torch.float16) > NOALLOC_BYTES
    a = torch.zeros(B, T, H, D, dtype=torch.float16, device=cuda_device)
    rc, _, _ = _noalloc_fwd(lib, a, a, a, esa.CONTROLLED, None)
    assert rc == ESA_ERR_NOALLOC_LIMIT
    assert "64 MiB" in esa.esa_strerror(rc)
