"""ctypes binding of the ESA scan C ABI (``include/esa.h``).

Argument marshalling only: every step of the scan runs in the CUDA library
``lib/libesa_b200.so``.  PyTorch supplies device memory and the current CUDA
stream.  There is no CPU path: CPU tensors, a missing library or a non-B200
device raise an error.

The functions carry the C names:

* :func:`esa_scan_fwd`  -- forward scan (+ E_final, + checkpoints in the workspace)
* :func:`esa_scan_bwd`  -- backward scan (da, dv, dq, dE_init)
* :func:`esa_step`      -- one-token decode update (in place on E); :class:`PreparedStep`
  is the same call on fixed buffers with its arguments resolved once (decode loops)
* :func:`esa_scan_map`, :func:`esa_scan_bwd_map` -- forward / backward segment
  maps ``(P, S)`` of a time slice (context parallelism)
* :func:`esa_compose`   -- apply a sequence of segment maps to a state
* :func:`esa_fused_fwd` -- forward scan with the a / v / q projections fused in
* :func:`esa_fused_layer_fwd` -- the same with the output projection z = y W_O^T (C = 64)
* :func:`esa_check`     -- synchronise and read the device status of a workspace
* :func:`esa_workspace_init` -- zero a new workspace and write its header
* :func:`esa_workspace_size`, :func:`esa_strerror`, :func:`esa_version`

The two scans also take row-strided a, v, q (and da, dv, dq): column blocks
of one ``[B, T, 3 H D]`` buffer, passed to ``esa_scan_fwd_ld`` /
``esa_scan_bwd_ld`` with their row stride.

Input dtypes: float32, float16, bfloat16, and float8_e4m3fn (outputs then
float16) for every call except the fused forward, which takes 16-bit inputs.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libesa_b200.so")

DIRECT = 0
CONTROLLED = 1
_DTYPE_CODE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2, torch.float8_e4m3fn: 3}


def out_dtype(dtype):
    """The dtype of a scan's outputs for inputs of `dtype`: the same, except
    that fp8 (e4m3) inputs give fp16 outputs."""
    return torch.float16 if dtype == torch.float8_e4m3fn else dtype

ESA_OK = 0
ESA_ERR_ARG = -1
ESA_ERR_ALIGN = -2
ESA_ERR_UNSUPPORTED = -3
ESA_ERR_WORKSPACE = -4
ESA_ERR_LAUNCH = -5
ESA_ERR_TIMEOUT = -6
ESA_ERR_DEVICE = -7

_lock = threading.Lock()
_lib = None


class EsaError(RuntimeError):
    """A non-zero status returned by the C ABI."""

    def __init__(self, func, code):
        self.code = code
        super().__init__(f"{func} failed: {esa_strerror(code)} (status {code})")


def load_library():
    """Load ``libesa_b200.so`` (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"ESA CUDA library not found at {LIB_PATH}; build it with "
                "`python -m gated_linear_recurrence_b200.build` (there is no CPU fallback)")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.esa_workspace_size.argtypes = [I, I, I, I, I]
        lib.esa_workspace_size.restype = S
        lib.esa_scan_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, P, I, P, S, P]
        lib.esa_scan_fwd.restype = I
        lib.esa_scan_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, P, I, P, S, P]
        lib.esa_scan_bwd.restype = I
        L = ctypes.c_longlong
        lib.esa_scan_fwd_ld.argtypes = [P, P, P, L, P, P, I, I, I, I, I, P, I, P, S, P]
        lib.esa_scan_fwd_ld.restype = I
        lib.esa_scan_bwd_ld.argtypes = [P, P, P, L, P, P, P, P, P, L, P, I, I, I, I, I, P, I, P, S, P]
        lib.esa_scan_bwd_ld.restype = I
        lib.esa_scan_map.argtypes = [P, P, P, P, I, I, I, I, I, I, P, S, P]
        lib.esa_scan_map.restype = I
        lib.esa_scan_bwd_map.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P, I, P, S, P]
        lib.esa_scan_bwd_map.restype = I
        lib.esa_compose.argtypes = [P, P, I, ctypes.c_longlong, I, P, P, P]
        lib.esa_compose.restype = I
        lib.esa_fused_fwd.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P, I, P, S, P]
        lib.esa_fused_fwd.restype = I
        lib.esa_fused_layer_fwd.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, P, I, P, S, P]
        lib.esa_fused_layer_fwd.restype = I
        lib.esa_step.argtypes = [P, P, P, P, P, I, I, I, I, I, P]
        lib.esa_step.restype = I
        lib.esa_check.argtypes = [P, P]
        lib.esa_check.restype = I
        lib.esa_workspace_init.argtypes = [P, S, P]
        lib.esa_workspace_init.restype = I
        lib.esa_strerror.argtypes = [I]
        lib.esa_strerror.restype = ctypes.c_char_p
        lib.esa_version.argtypes = []
        lib.esa_version.restype = I
        _lib = lib
        return lib


def esa_strerror(code: int) -> str:
    return load_library().esa_strerror(int(code)).decode()


def esa_version() -> int:
    return int(load_library().esa_version())


def esa_workspace_size(B: int, T: int, H: int, D: int, dtype) -> int:
    code = _DTYPE_CODE[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    return int(load_library().esa_workspace_size(B, T, H, D, code))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device, stream):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


class _NoDeviceSwitch:
    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


_SAME_DEVICE = _NoDeviceSwitch()


def _on(device):
    """Make `device` current for a library call; a no-op when it already is
    (the common case, and the one on decode's latency-bound path)."""
    if device.index is None or device.index == torch.cuda.current_device():
        return _SAME_DEVICE
    return torch.cuda.device(device)


def _check_seq(name, t, ref):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (the ESA library has no CPU path)")
    if t.shape != ref.shape or t.dtype != ref.dtype or t.device != ref.device:
        raise ValueError(f"{name} must match a: shape {tuple(ref.shape)}, dtype {ref.dtype}, {ref.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous [B, T, H, D]")


def row_stride(t):
    """Elements between consecutive tokens' rows of a ``[B, T, H, D]`` tensor
    whose H * D channels per token are contiguous (e.g. a column block of a
    ``[B, T, 3 H D]`` projection output); None for any other layout."""
    B, T, H, D = (int(x) for x in t.shape)
    st = t.stride()
    if (D > 1 and st[3] != 1) or (H > 1 and st[2] != D):
        return None
    if T > 1:
        ld = st[1]
        if B > 1 and st[0] != T * ld:
            return None
    elif B > 1:
        ld = st[0]
    else:
        ld = H * D
    return ld if ld >= H * D else None


def _strided_seq(names, ts, ref):
    """Common row stride of same-shaped sequence tensors (checked)."""
    lds = set()
    for name, t in zip(names, ts):
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise TypeError(f"{name} must be a CUDA tensor (the ESA library has no CPU path)")
        if t.shape != ref.shape or t.device != ref.device:
            raise ValueError(f"{name} must have shape {tuple(ref.shape)} on {ref.device}")
        ld = row_stride(t)
        if ld is None:
            raise ValueError(f"{name} must be [B, T, H, D] with each token's H*D channels contiguous")
        lds.add(ld)
    if len(lds) != 1:
        raise ValueError(f"{', '.join(names)} must share one row stride (got {sorted(lds)})")
    return lds.pop()


def _check_state(name, t, B, H, D, device):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.device != device:
        raise TypeError(f"{name} must be a CUDA tensor on {device}")
    if tuple(t.shape) != (B, H, D) or t.dtype != torch.float32 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous float32 tensor of shape {(B, H, D)}")


def _dims(a, strided=False):
    if not isinstance(a, torch.Tensor) or not a.is_cuda:
        raise TypeError("a must be a CUDA tensor (the ESA library has no CPU path)")
    if a.dim() != 4:
        raise ValueError("sequence tensors must be [B, T, H, D]")
    if a.dtype not in _DTYPE_CODE:
        raise TypeError(f"unsupported dtype {a.dtype}")
    if not strided and not a.is_contiguous():
        raise ValueError("a must be contiguous [B, T, H, D]")
    return tuple(int(s) for s in a.shape)


def esa_workspace_init(workspace, stream=None):
    """Zero a workspace and write its header (once, after allocation)."""
    lib = load_library()
    with _on(workspace.device):
        rc = lib.esa_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(workspace.device, stream))
    if rc != 0:
        raise EsaError("esa_workspace_init", rc)
    return workspace


def new_workspace(B, T, H, D, dtype, device, stream=None):
    """Allocate and initialise a workspace of the size the C ABI asks for
    (torch memory, caller-owned)."""
    n = esa_workspace_size(B, T, H, D, dtype)
    if n == 0:
        raise ValueError("unsupported shape for the ESA scan")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    return esa_workspace_init(ws, stream)


def esa_scan_fwd(a, v, q, y=None, E_final=None, mode=CONTROLLED, E_init=None, workspace=None,
                 stream=None, want_E_final=True):
    """Forward scan.  Returns ``(y, E_final, workspace)``.

    ``workspace`` (uint8 CUDA tensor) is allocated when not given; keep it for
    :func:`esa_scan_bwd`.  ``E_final`` is allocated when not given unless
    ``want_E_final`` is False.  a, v, q may be row-strided views (each
    token's channels contiguous, one row stride for the three, e.g. column
    blocks of one projection output): they then go through
    ``esa_scan_fwd_ld``.
    """
    B, T, H, D = _dims(a, strided=True)
    ld = _strided_seq(("a", "v", "q"), (a, v, q), a)
    for name, t in (("v", v), ("q", q)):
        if t.dtype != a.dtype:
            raise ValueError(f"{name} must match a: dtype {a.dtype}")
    ydt = out_dtype(a.dtype)
    if y is None:
        y = torch.empty(a.shape, dtype=ydt, device=a.device)
    if not isinstance(y, torch.Tensor) or tuple(y.shape) != tuple(a.shape) or y.dtype != ydt \
            or y.device != a.device or not y.is_contiguous():
        raise ValueError(f"y must be a contiguous {ydt} tensor of shape {tuple(a.shape)} on {a.device}")
    if E_final is None and want_E_final:
        E_final = torch.empty((B, H, D), dtype=torch.float32, device=a.device)
    _check_state("E_final", E_final, B, H, D, a.device)
    _check_state("E_init", E_init, B, H, D, a.device)
    if workspace is None:
        workspace = new_workspace(B, T, H, D, a.dtype, a.device)
    lib = load_library()
    with _on(a.device):
        if ld == H * D:
            rc = lib.esa_scan_fwd(_ptr(a), _ptr(v), _ptr(q), _ptr(y), _ptr(E_final), B, T, H, D, int(mode),
                                  _ptr(E_init), _DTYPE_CODE[a.dtype], _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(a.device, stream))
        else:
            rc = lib.esa_scan_fwd_ld(_ptr(a), _ptr(v), _ptr(q), ld, _ptr(y), _ptr(E_final), B, T, H, D,
                                     int(mode), _ptr(E_init), _DTYPE_CODE[a.dtype], _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(a.device, stream))
    if rc != 0:
        raise EsaError("esa_scan_fwd" if ld == H * D else "esa_scan_fwd_ld", rc)
    return y, E_final, workspace


def esa_scan_bwd(a, v, q, dy, workspace, mode=CONTROLLED, E_init=None, dE_final=None, da=None, dv=None,
                 dq=None, dE_init=None, stream=None, want_dE_init=True):
    """Backward scan.  ``workspace`` must be the one the matching forward wrote.

    Returns ``(da, dv, dq, dE_init)``.  a, v, q (one row stride) and the
    given da, dv, dq (another) may be row-strided views, e.g. column blocks
    of one ``[B, T, 3 H D]`` buffer; dy is contiguous.  Strided rows go
    through ``esa_scan_bwd_ld``.
    """
    B, T, H, D = _dims(a, strided=True)
    ld_in = _strided_seq(("a", "v", "q"), (a, v, q), a)
    for name, t in (("v", v), ("q", q)):
        if t.dtype != a.dtype:
            raise ValueError(f"{name} must match a: dtype {a.dtype}")
    _check_seq("dy", dy, a)
    odt = out_dtype(a.dtype)
    da = torch.empty(a.shape, dtype=odt, device=a.device) if da is None else da
    dv = torch.empty(a.shape, dtype=odt, device=a.device) if dv is None else dv
    dq = torch.empty(a.shape, dtype=odt, device=a.device) if dq is None else dq
    for name, t in (("da", da), ("dv", dv), ("dq", dq)):
        if not isinstance(t, torch.Tensor) or tuple(t.shape) != tuple(a.shape) or t.dtype != odt \
                or t.device != a.device:
            raise ValueError(f"{name} must be a {odt} tensor of shape {tuple(a.shape)} on {a.device}")
    ld_g = _strided_seq(("da", "dv", "dq"), (da, dv, dq), a)
    if dE_init is None and want_dE_init:
        dE_init = torch.empty((B, H, D), dtype=torch.float32, device=a.device)
    _check_state("dE_init", dE_init, B, H, D, a.device)
    _check_state("dE_final", dE_final, B, H, D, a.device)
    _check_state("E_init", E_init, B, H, D, a.device)
    if workspace is None or not workspace.is_cuda:
        raise ValueError("esa_scan_bwd needs the CUDA workspace written by the matching esa_scan_fwd")
    lib = load_library()
    plain = ld_in == H * D and ld_g == H * D
    with _on(a.device):
        if plain:
            rc = lib.esa_scan_bwd(_ptr(a), _ptr(v), _ptr(q), _ptr(dy), _ptr(dE_final), _ptr(da), _ptr(dv),
                                  _ptr(dq), _ptr(dE_init), B, T, H, D, int(mode), _ptr(E_init),
                                  _DTYPE_CODE[a.dtype], _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(a.device, stream))
        else:
            rc = lib.esa_scan_bwd_ld(_ptr(a), _ptr(v), _ptr(q), ld_in, _ptr(dy), _ptr(dE_final), _ptr(da),
                                     _ptr(dv), _ptr(dq), ld_g, _ptr(dE_init), B, T, H, D, int(mode),
                                     _ptr(E_init), _DTYPE_CODE[a.dtype], _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(a.device, stream))
    if rc != 0:
        raise EsaError("esa_scan_bwd" if plain else "esa_scan_bwd_ld", rc)
    return da, dv, dq, dE_init


def esa_scan_map(a, v, mode=CONTROLLED, workspace=None, P=None, S=None, stream=None):
    """Forward segment map of a time slice: ``E_T = P * E_0 + S`` per channel.

    Returns ``(P, S, workspace)`` (float32 ``[B, H, D]``).  Only the
    workspace's chunk-map words are written.
    """
    B, T, H, D = _dims(a)
    _check_seq("v", v, a)
    P = torch.empty((B, H, D), dtype=torch.float32, device=a.device) if P is None else P
    S = torch.empty((B, H, D), dtype=torch.float32, device=a.device) if S is None else S
    _check_state("P", P, B, H, D, a.device)
    _check_state("S", S, B, H, D, a.device)
    if workspace is None:
        workspace = new_workspace(B, T, H, D, a.dtype, a.device)
    lib = load_library()
    with _on(a.device):
        rc = lib.esa_scan_map(_ptr(a), _ptr(v), _ptr(P), _ptr(S), B, T, H, D, int(mode), _DTYPE_CODE[a.dtype],
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(a.device, stream))
    if rc != 0:
        raise EsaError("esa_scan_map", rc)
    return P, S, workspace


def esa_scan_bwd_map(a, v, q, dy, workspace, mode=CONTROLLED, E_init=None, P=None, S=None, stream=None):
    """Backward segment map of a time slice: ``dE_init = P * dE_final + S``.

    ``workspace`` must hold the chunk states of the matching forward (same
    inputs and ``E_init``); they are kept.  Returns ``(P, S)``.
    """
    B, T, H, D = _dims(a)
    for name, t in (("v", v), ("q", q), ("dy", dy)):
        _check_seq(name, t, a)
    P = torch.empty((B, H, D), dtype=torch.float32, device=a.device) if P is None else P
    S = torch.empty((B, H, D), dtype=torch.float32, device=a.device) if S is None else S
    _check_state("P", P, B, H, D, a.device)
    _check_state("S", S, B, H, D, a.device)
    _check_state("E_init", E_init, B, H, D, a.device)
    if workspace is None or not workspace.is_cuda:
        raise ValueError("esa_scan_bwd_map needs the CUDA workspace written by the matching esa_scan_fwd")
    lib = load_library()
    with _on(a.device):
        rc = lib.esa_scan_bwd_map(_ptr(a), _ptr(v), _ptr(q), _ptr(dy), _ptr(P), _ptr(S), B, T, H, D, int(mode),
                                  _ptr(E_init), _DTYPE_CODE[a.dtype], _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(a.device, stream))
    if rc != 0:
        raise EsaError("esa_scan_bwd_map", rc)
    return P, S


def esa_compose(P, S, x0=None, reverse=False, out=None, stream=None):
    """Apply the maps ``x -> P[j] * x + S[j]`` for j in order (``reverse``:
    from the last index down) to ``x0`` (zeros when None).

    ``P``, ``S``: float32 CUDA tensors ``[n, *shape]``; ``x0`` and the result
    have ``shape``.
    """
    if not isinstance(P, torch.Tensor) or not P.is_cuda or P.dtype != torch.float32 or P.dim() < 1:
        raise TypeError("P must be a float32 CUDA tensor [n, ...]")
    if S.shape != P.shape or S.dtype != P.dtype or S.device != P.device:
        raise ValueError("S must match P")
    if not (P.is_contiguous() and S.is_contiguous()):
        raise ValueError("P and S must be contiguous")
    n, shape = int(P.shape[0]), tuple(P.shape[1:])
    count = 1
    for d in shape:
        count *= int(d)
    for name, t in (("x0", x0), ("out", out)):
        if t is not None and (tuple(t.shape) != shape or t.dtype != torch.float32 or t.device != P.device
                              or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous float32 tensor of shape {shape} on {P.device}")
    out = torch.empty(shape, dtype=torch.float32, device=P.device) if out is None else out
    lib = load_library()
    with _on(P.device):
        rc = lib.esa_compose(_ptr(P), _ptr(S), n, count, int(bool(reverse)), _ptr(x0), _ptr(out),
                             _stream(P.device, stream))
    if rc != 0:
        raise EsaError("esa_compose", rc)
    return out


def esa_fused_fwd(x, W, H, mode=CONTROLLED, E_init=None, y=None, E_final=None, workspace=None, stream=None,
                  want_E_final=True, want_avq=False, avq=None):
    """Forward scan of the projections of ``x``: a, v, q = x W[:C]^T,
    x W[C:2C]^T, x W[2C:]^T (rounded to x's dtype), computed on the tensor
    cores inside the scan.  ``x``: [B, T, C_in] float16 / bfloat16; ``W``:
    [3C, C_in] of the same dtype; ``H`` heads of D = C / H channels.

    Returns ``(y, E_final, workspace)`` with ``y`` [B, T, H, D], or with
    ``want_avq`` (or ``avq``, three preallocated [B, T, H, D] tensors of x's
    dtype) ``(y, E_final, workspace, (a, v, q))``: the projections the scan
    consumed, for :func:`esa_scan_bwd`.
    """
    if not isinstance(x, torch.Tensor) or not x.is_cuda or x.dim() != 3:
        raise TypeError("x must be a CUDA tensor [B, T, C_in] (the ESA library has no CPU path)")
    if not isinstance(W, torch.Tensor) or not W.is_cuda or W.dim() != 2 or W.dtype != x.dtype or W.device != x.device:
        raise TypeError("W must be a CUDA tensor [3C, C_in] of x's dtype and device")
    if x.dtype not in _DTYPE_CODE or not x.is_contiguous() or not W.is_contiguous():
        raise ValueError("x and W must be contiguous float16 / bfloat16 tensors")
    B, T, C_in = (int(s) for s in x.shape)
    if W.shape[1] != C_in or W.shape[0] % 3 != 0 or (W.shape[0] // 3) % H != 0:
        raise ValueError("W must be [3C, C_in] with C divisible by H")
    C = W.shape[0] // 3
    D = C // H
    if y is None:
        y = torch.empty((B, T, H, D), dtype=x.dtype, device=x.device)
    if tuple(y.shape) != (B, T, H, D) or y.dtype != x.dtype or not y.is_contiguous():
        raise ValueError(f"y must be a contiguous {x.dtype} tensor of shape {(B, T, H, D)}")
    if E_final is None and want_E_final:
        E_final = torch.empty((B, H, D), dtype=torch.float32, device=x.device)
    _check_state("E_final", E_final, B, H, D, x.device)
    _check_state("E_init", E_init, B, H, D, x.device)
    if workspace is None:
        workspace = new_workspace(B, T, H, D, x.dtype, x.device)
    if avq is not None:
        want_avq = True
        avq = tuple(avq)
        if len(avq) != 3:
            raise ValueError("avq must be three tensors (a, v, q)")
        for name, t in zip(("a", "v", "q"), avq):
            if (not isinstance(t, torch.Tensor) or tuple(t.shape) != (B, T, H, D) or t.dtype != x.dtype
                    or t.device != x.device or not t.is_contiguous()):
                raise ValueError(f"{name} must be a contiguous {x.dtype} tensor of shape {(B, T, H, D)} on {x.device}")
    elif want_avq:
        avq = tuple(torch.empty((B, T, H, D), dtype=x.dtype, device=x.device) for _ in range(3))
    else:
        avq = (None, None, None)
    lib = load_library()
    with _on(x.device):
        rc = lib.esa_fused_fwd(_ptr(x), _ptr(W), _ptr(y), _ptr(E_final), *(_ptr(t) for t in avq), B, T, H, D, C_in,
                               int(mode), _ptr(E_init),
                               _DTYPE_CODE[x.dtype], _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(x.device, stream))
    if rc != 0:
        raise EsaError("esa_fused_fwd", rc)
    return (y, E_final, workspace, avq) if want_avq else (y, E_final, workspace)


def esa_fused_layer_fwd(x, W, W_O, H, mode=CONTROLLED, E_init=None, z=None, y=None, want_y=False, E_final=None,
                        workspace=None, stream=None, want_E_final=True):
    """The layer's forward from its input, output projection included:
    :func:`esa_fused_fwd` followed by z = y W_O^T in the same kernel, for a
    layer of C = 64 channels.  ``x`` [B, T, C_in] float16 / bfloat16 (C_in of
    64 or 128); ``W`` [192, C_in] and ``W_O`` [64, 64] ([out, in]) of x's
    dtype.  Returns ``(z, y, E_final, workspace)``: z [B, T, 64]; y
    [B, T, H, D] when ``want_y`` (or ``y`` given), else None."""
    if not isinstance(x, torch.Tensor) or not x.is_cuda or x.dim() != 3:
        raise TypeError("x must be a CUDA tensor [B, T, C_in] (the ESA library has no CPU path)")
    for name, t in (("W", W), ("W_O", W_O)):
        if (not isinstance(t, torch.Tensor) or not t.is_cuda or t.dim() != 2 or t.dtype != x.dtype
                or t.device != x.device or not t.is_contiguous()):
            raise TypeError(f"{name} must be a contiguous CUDA tensor of x's dtype and device")
    if x.dtype not in _DTYPE_CODE or not x.is_contiguous():
        raise ValueError("x must be a contiguous float16 / bfloat16 tensor")
    B, T, C_in = (int(s) for s in x.shape)
    if W.shape[1] != C_in or W.shape[0] % 3 != 0 or (W.shape[0] // 3) % H != 0:
        raise ValueError("W must be [3C, C_in] with C divisible by H")
    C = W.shape[0] // 3
    D = C // H
    if tuple(W_O.shape) != (C, C):
        raise ValueError(f"W_O must be [{C}, {C}]")
    if z is None:
        z = torch.empty((B, T, C), dtype=x.dtype, device=x.device)
    if tuple(z.shape) != (B, T, C) or z.dtype != x.dtype or not z.is_contiguous():
        raise ValueError(f"z must be a contiguous {x.dtype} tensor of shape {(B, T, C)}")
    if y is None and want_y:
        y = torch.empty((B, T, H, D), dtype=x.dtype, device=x.device)
    if y is not None and (tuple(y.shape) != (B, T, H, D) or y.dtype != x.dtype or not y.is_contiguous()):
        raise ValueError(f"y must be a contiguous {x.dtype} tensor of shape {(B, T, H, D)}")
    if E_final is None and want_E_final:
        E_final = torch.empty((B, H, D), dtype=torch.float32, device=x.device)
    _check_state("E_final", E_final, B, H, D, x.device)
    _check_state("E_init", E_init, B, H, D, x.device)
    if workspace is None:
        workspace = new_workspace(B, T, H, D, x.dtype, x.device)
    lib = load_library()
    with _on(x.device):
        rc = lib.esa_fused_layer_fwd(_ptr(x), _ptr(W), _ptr(W_O), _ptr(z), _ptr(y), _ptr(E_final), B, T, H, D, C_in,
                                     int(mode), _ptr(E_init), _DTYPE_CODE[x.dtype], _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream(x.device, stream))
    if rc != 0:
        raise EsaError("esa_fused_layer_fwd", rc)
    return z, y, E_final, workspace


def esa_step(a_t, v_t, q_t, E, y_t=None, mode=CONTROLLED, stream=None):
    """One-token update: E (float32 [B, H, D]) is updated in place.  Returns ``y_t``."""
    if not isinstance(a_t, torch.Tensor) or not a_t.is_cuda or a_t.dim() != 3:
        raise TypeError("a_t must be a CUDA tensor [B, H, D] (the ESA library has no CPU path)")
    if a_t.dtype not in _DTYPE_CODE or not a_t.is_contiguous():
        raise ValueError("a_t must be contiguous with dtype float32, float16 or bfloat16")
    B, H, D = (int(s) for s in a_t.shape)
    for name, t in (("v_t", v_t), ("q_t", q_t)):
        if t.shape != a_t.shape or t.dtype != a_t.dtype or t.device != a_t.device or not t.is_contiguous():
            raise ValueError(f"{name} must match a_t")
    _check_state("E", E, B, H, D, a_t.device)
    if E is None:
        raise ValueError("E (the recurrent state) is required")
    if y_t is None:
        y_t = torch.empty(a_t.shape, dtype=out_dtype(a_t.dtype), device=a_t.device)
    if tuple(y_t.shape) != tuple(a_t.shape) or y_t.dtype != out_dtype(a_t.dtype) or y_t.device != a_t.device \
            or not y_t.is_contiguous():
        raise ValueError(f"y_t must be a contiguous {out_dtype(a_t.dtype)} tensor of shape {tuple(a_t.shape)}")
    lib = load_library()
    with _on(a_t.device):
        rc = lib.esa_step(_ptr(a_t), _ptr(v_t), _ptr(q_t), _ptr(E), _ptr(y_t), B, H, D, int(mode),
                          _DTYPE_CODE[a_t.dtype], _stream(a_t.device, stream))
    if rc != 0:
        raise EsaError("esa_step", rc)
    return y_t


class PreparedStep:
    """``esa_step`` on fixed buffers, with the argument checks, the device
    pointers and the stream resolved once, at construction.

    A decode loop usually writes each new token's a_t, v_t, q_t into the same
    buffers (the projections' outputs) and keeps one state E; for it each
    call of this object is a single C call with prebuilt arguments, which
    removes most of the host cost of :func:`esa_step` (the kernel itself
    moves a few hundred KB at most and is launch-bound).  Work is enqueued on
    the stream given here, or on the stream that was current at construction;
    the buffers must outlive the object.  Calling it returns ``y_t``.
    """

    def __init__(self, a_t, v_t, q_t, E, y_t=None, mode=CONTROLLED, stream=None):
        if not isinstance(a_t, torch.Tensor) or not a_t.is_cuda or a_t.dim() != 3:
            raise TypeError("a_t must be a CUDA tensor [B, H, D] (the ESA library has no CPU path)")
        if a_t.dtype not in _DTYPE_CODE or not a_t.is_contiguous():
            raise ValueError("a_t must be contiguous with dtype float32, float16, bfloat16 or float8_e4m3fn")
        B, H, D = (int(s) for s in a_t.shape)
        for name, t in (("v_t", v_t), ("q_t", q_t)):
            if t.shape != a_t.shape or t.dtype != a_t.dtype or t.device != a_t.device or not t.is_contiguous():
                raise ValueError(f"{name} must match a_t")
        if E is None:
            raise ValueError("E (the recurrent state) is required")
        _check_state("E", E, B, H, D, a_t.device)
        if y_t is None:
            y_t = torch.empty(a_t.shape, dtype=out_dtype(a_t.dtype), device=a_t.device)
        if tuple(y_t.shape) != tuple(a_t.shape) or y_t.dtype != out_dtype(a_t.dtype) or \
                y_t.device != a_t.device or not y_t.is_contiguous():
            raise ValueError(f"y_t must be a contiguous {out_dtype(a_t.dtype)} tensor of shape {tuple(a_t.shape)}")
        self.device = a_t.device
        self.y_t = y_t
        self._keep = (a_t, v_t, q_t, E, y_t)   # the buffers stay alive as long as this object
        self._fn = load_library().esa_step
        self._args = (_ptr(a_t), _ptr(v_t), _ptr(q_t), _ptr(E), _ptr(y_t), B, H, D, int(mode),
                      _DTYPE_CODE[a_t.dtype], _stream(a_t.device, stream))
        if self.device.index is not None and self.device.index != torch.cuda.current_device():
            raise ValueError("make the tensors' device current before preparing and calling the step")

    def __call__(self):
        rc = self._fn(*self._args)
        if rc != 0:
            raise EsaError("esa_step", rc)
        return self.y_t


def esa_check(workspace, stream=None):
    """Synchronise the stream and raise :class:`EsaError` if a device-side wait gave up."""
    lib = load_library()
    with _on(workspace.device):
        rc = lib.esa_check(_ptr(workspace), _stream(workspace.device, stream))
    if rc != 0:
        raise EsaError("esa_check", rc)
