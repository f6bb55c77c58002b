"""The allocation-free forward scan, esa_scan_fwd_noalloc, through the C ABI.

Some callers cannot allocate device memory where they run the scan (a
serving loop with a device-memory budget fixed at start-up, a latency-critical
path where cudaMalloc may synchronise the device, a foreign-language caller
that is only handed tensor pointers).  For them the library keeps its scratch
in a built-in static device array.  These tests check that entry point:

* against the fp64 oracle on the same inputs, for every input dtype (fp8
  e4m3 inputs give fp16 outputs), and against the ordinary esa_scan_fwd,
  on calls in a row with different shapes: the array is shared and keeps
  the previous call's contents;
* its status call, esa_check_noalloc: a bounded wait that gives up (planted
  on the host by advancing the array's ticket counter, so the first chunk of
  every chain is never scanned) is reported as ESA_ERR_TIMEOUT, and the
  next calls are correct again;
* the restart of its call counter: with the array's epoch set just below
  and at the point where the guard starts the array afresh, the next calls
  still match the oracle;
* shapes needing more scratch than the array holds are refused before
  anything runs.

The file is named so that pytest collects it last.
"""
import ctypes
import time

import pytest
import torch

import oracle
from gated_linear_recurrence_b200 import esa, inputs
from tests._parity import DT, TOL, assert_close, host64

pytestmark = pytest.mark.gpu

ESA_ERR_NOALLOC_LIMIT = -8
NOALLOC_BYTES = 64 * 1024 * 1024
EPOCH_RESTART = 0xFFFFFF00
F8 = torch.float8_e4m3fn
_CODE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2, F8: 3}
TICKET_FWD, EPOCH_WORD = 4, 2   # int32 indices of ticket[0] and of the epoch in the array's header


def _lib():
    lib = esa.load_library()
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.esa_scan_fwd_noalloc.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I, P]
    lib.esa_scan_fwd_noalloc.restype = I
    lib.esa_check_noalloc.argtypes = [P]
    lib.esa_check_noalloc.restype = I
    lib.esa_noalloc_scratch.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_size_t)]
    lib.esa_noalloc_scratch.restype = I
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _noalloc_fwd(lib, a, v, q, mode, E_init):
    B, T, H, D = a.shape
    y = torch.empty(a.shape, dtype=esa.out_dtype(a.dtype), device=a.device)
    E_final = torch.empty(B, H, D, dtype=torch.float32, device=a.device)
    rc = lib.esa_scan_fwd_noalloc(_ptr(a), _ptr(v), _ptr(q), _ptr(y), _ptr(E_final), B, T, H, D, mode,
                                  _ptr(E_init), _CODE[a.dtype], _stream(a.device))
    return rc, y, E_final


class _DeviceWords:
    """int32 words of library-owned device memory, for torch.as_tensor (no copy, no allocation)."""

    def __init__(self, addr, n):
        self.__cuda_array_interface__ = {"shape": (n,), "typestr": "<i4", "data": (addr, False), "version": 3}


def _header(lib):
    """The array's 256-byte header as an int32 tensor aliasing it (device memory owned by the library)."""
    p, n = ctypes.c_void_p(), ctypes.c_size_t()
    assert lib.esa_noalloc_scratch(ctypes.byref(p), ctypes.byref(n)) == 0
    assert n.value == NOALLOC_BYTES and p.value % 256 == 0
    return torch.as_tensor(_DeviceWords(p.value, 64), device="cuda")


def _write_word(hdr, index, value):
    torch.cuda.synchronize()
    hdr[index] = value - 2**32 if value >= 2**31 else value
    torch.cuda.synchronize()


def _read_word(hdr, index):
    torch.cuda.synchronize()
    return int(hdr[index].item()) & 0xFFFFFFFF


def _check(lib, dev):
    return lib.esa_check_noalloc(_stream(dev))


def _case_inputs(B, T, H, D, dt, seed, dev):
    if dt == "e4m3":
        x = inputs.make_scan_inputs(B, T, H, D, "f32", 2.0, seed, with_dy=False)
        return tuple(x[k].to(F8).to(dev) for k in ("a", "v", "q"))
    x = inputs.make_scan_inputs(B, T, H, D, dt, a_mean=2.0, seed=seed, with_dy=False)
    return tuple(x[k].to(dev) for k in ("a", "v", "q"))


def _f64(t):
    return t.to(torch.float32).to("cpu", torch.float64).numpy()


def _against_oracle(lib, dev, B, T, H, D, dt, mode, seed, label):
    a, v, q = _case_inputs(B, T, H, D, dt, seed, dev)
    E0 = inputs.make_state(B, H, D, seed=seed + 100, scale=0.5).to(dev)
    rc, y, Ef = _noalloc_fwd(lib, a, v, q, mode, E0)
    assert rc == 0, esa.esa_strerror(rc)
    assert _check(lib, dev) == 0
    y_r, Ef_r = oracle.scan_fwd(_f64(a), _f64(v), _f64(q), mode, E_init=host64(E0))
    tol = TOL[torch.float16] if dt == "e4m3" else TOL[DT[dt]]
    assert_close(y, y_r, tol, f"{label} y ({dt})")
    assert_close(Ef, Ef_r, tol, f"{label} E_final ({dt})")
    return a, v, q, E0, y, Ef


CASES = [  # B, T, H, D, dtype, mode, seed: different problems back to back
    (4, 1000, 4, 32, "f16", esa.CONTROLLED, 21),
    (3, 333, 2, 64, "bf16", esa.DIRECT, 22),
    (2, 200, 3, 32, "f32", esa.CONTROLLED, 23),
    (2, 300, 4, 32, "e4m3", esa.DIRECT, 24),
    (1, 129, 1, 128, "f16", esa.CONTROLLED, 25),
]


def test_noalloc_forward_matches_oracle_on_calls_in_a_row(cuda_device):
    lib = _lib()
    for B, T, H, D, dt, mode, seed in CASES:
        assert esa.esa_workspace_size(B, T, H, D, F8 if dt == "e4m3" else DT[dt]) <= NOALLOC_BYTES
        a, v, q, E0, y, Ef = _against_oracle(lib, cuda_device, B, T, H, D, dt, mode, seed, "call")
        # the ordinary entry point (caller-allocated workspace) on the same inputs: the same arithmetic
        y_w, Ef_w, _ = esa.esa_scan_fwd(a, v, q, mode=mode, E_init=E0)
        torch.cuda.synchronize()
        assert torch.equal(y, y_w) and torch.equal(Ef, Ef_w)


def test_noalloc_reports_a_wait_that_gave_up_and_recovers(cuda_device):
    lib = _lib()
    B, T, H, D, dt, mode = 2, 1024, 4, 32, "f16", esa.CONTROLLED   # 8 tiles of 128 rows per chain
    _against_oracle(lib, cuda_device, B, T, H, D, dt, mode, 31, "before")   # the array is initialised
    hdr = _header(lib)
    nchains = B * (H * D // 64)
    _write_word(hdr, TICKET_FWD, nchains)   # the scan starts at its second chunk
    a, v, q = _case_inputs(B, T, H, D, dt, 32, cuda_device)
    t0 = time.time()
    rc, _, _ = _noalloc_fwd(lib, a, v, q, mode, None)
    assert rc == 0
    assert _check(lib, cuda_device) == esa.ESA_ERR_TIMEOUT
    assert time.time() - t0 < 60
    assert _read_word(hdr, TICKET_FWD) == 0          # the kernel reset its ticket counter
    assert _check(lib, cuda_device) == 0              # the status was cleared by the first check
    for k in range(2):
        _against_oracle(lib, cuda_device, B, T, H, D, dt, mode, 33 + k, f"after{k}")


@pytest.mark.parametrize("start", [EPOCH_RESTART - 1, 0xFFFFFFFE])
def test_noalloc_call_counter_restarts_before_it_runs_out(cuda_device, start):
    lib = _lib()
    B, T, H, D, dt, mode = 3, 700, 4, 32, "f16", esa.CONTROLLED
    _against_oracle(lib, cuda_device, B, T, H, D, dt, mode, 41, "before")
    hdr = _header(lib)
    _write_word(hdr, EPOCH_WORD, start)
    for k in range(2):   # different inputs each call: a stale carry would show
        _against_oracle(lib, cuda_device, B, T, H, D, dt, mode, 42 + k, f"call{k}")
        ep = _read_word(hdr, EPOCH_WORD)
        assert 1 <= ep <= EPOCH_RESTART, hex(ep)
    assert _read_word(hdr, EPOCH_WORD) < start


def test_noalloc_refuses_shapes_beyond_its_scratch(cuda_device):
    lib = _lib()
    B, T, H, D = 64, 16384, 4, 32
    assert esa.esa_workspace_size(B, T, H, D, torch.float16) > NOALLOC_BYTES
    a = torch.zeros(B, T, H, D, dtype=torch.float16, device=cuda_device)
    rc, _, _ = _noalloc_fwd(lib, a, a, a, esa.CONTROLLED, None)
    assert rc == ESA_ERR_NOALLOC_LIMIT
    assert "64 MiB" in esa.esa_strerror(rc)
    bad = torch.zeros(2, 64, 4, 32, dtype=torch.float16, device=cuda_device)
    rc = lib.esa_scan_fwd_noalloc(ctypes.c_void_p(bad.data_ptr() + 2), _ptr(bad), _ptr(bad), _ptr(bad), None,
                                  2, 63, 4, 32, 1, None, 1, _stream(cuda_device))
    assert rc == esa.ESA_ERR_ALIGN
    assert _check(lib, cuda_device) == 0
