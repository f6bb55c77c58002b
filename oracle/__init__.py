"""Double-precision CPU oracle for the ESA gated linear recurrence.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The GPU
library does not import it, link it or call it, and the two share no code.

The arithmetic lives in ``esa_oracle.c`` (plain C, double precision,
sequential per head and per time step).  This module compiles it with gcc
when needed and exposes three numpy-level functions with the semantics of the
three GPU entry points:

* :func:`scan_fwd` -- the forward scan with the per-head RMS readout,
* :func:`scan_bwd` -- the backward (reverse) scan,
* :func:`step`     -- the one-token recurrent update,

and, for splitting one sequence along time (context parallelism), the maps
that summarise a time slice and their composition:

* :func:`scan_map`     -- forward map (P, S) of a slice: E_T = P E_0 + S,
* :func:`scan_bwd_map` -- backward map: dE_init = P dE_final + S,
* :func:`compose`      -- a sequence of such maps applied to a state,

and the forward of the layer from its input:

* :func:`project`      -- a, v, q as projections of x, rounded to the I/O type,
* :func:`fused_fwd`    -- those projections followed by :func:`scan_fwd`,
* :func:`output_projection` -- the layer's output z = W_O y of the readout.

Sources for each formula are given in the C file's header: the recurrence and
its two modes ("entangled-state-attention 0.1.0", section "Core idea"), the
readout (same section), the state shape (mlbricks-web.pages.dev/esa,
"Generation / memory"), and the chain-rule derivation of the backward pass.

Parity pins: every function here is checked against closed forms, invariants,
special cases, a high-precision brute-force evaluation and finite differences
in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "esa_oracle.c")
_LIB = os.path.join(_HERE, "libesa_oracle.so")

DIRECT = 0
CONTROLLED = 1
EPS = 1e-6

_lock = threading.Lock()
_lib = None

# Mutation testing only: load a deliberately altered build of the oracle from
# this path instead of the real one (see tests/test_oracle_mutations.py).
_LIB_OVERRIDE_ENV = "ESA_ORACLE_LIB_OVERRIDE"


def build(force: bool = False) -> str:
    """Compile ``esa_oracle.c`` into ``libesa_oracle.so`` with gcc (-O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            override = os.environ.get(_LIB_OVERRIDE_ENV)
            if override:
                lib = ctypes.CDLL(override)
            else:
                build()
                lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            L = ctypes.c_long
            I = ctypes.c_int
            lib.esa_oracle_scan_fwd.argtypes = [P, P, P, P, P, L, L, L, L, I, P, P]
            lib.esa_oracle_scan_fwd.restype = I
            lib.esa_oracle_scan_bwd.argtypes = [P, P, P, P, P, P, P, P, P, L, L, L, L, I, P]
            lib.esa_oracle_scan_bwd.restype = I
            lib.esa_oracle_step.argtypes = [P, P, P, P, P, L, L, L, I]
            lib.esa_oracle_step.restype = I
            _lib = lib
    return _lib


def _f64(x, shape=None):
    arr = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if shape is not None and arr.shape != tuple(shape):
        raise ValueError(f"expected shape {tuple(shape)}, got {arr.shape}")
    return arr


def _ptr(arr):
    return None if arr is None else arr.ctypes.data_as(ctypes.c_void_p)


def scan_fwd(a, v, q, mode, E_init=None, return_states=False):
    """Forward scan of [B, T, H, D] inputs.

    Returns ``(y, E_final)`` or, with ``return_states``, ``(y, E_final, E_all)``
    where ``E_all[b, t]`` is the state after token t.
    """
    a = _f64(a)
    if a.ndim != 4:
        raise ValueError("a must be [B, T, H, D]")
    B, T, H, D = a.shape
    v = _f64(v, a.shape)
    q = _f64(q, a.shape)
    E0 = None if E_init is None else _f64(E_init, (B, H, D))
    y = np.empty_like(a)
    E_final = np.empty((B, H, D), dtype=np.float64)
    E_all = np.empty_like(a) if return_states else None
    rc = _load().esa_oracle_scan_fwd(_ptr(a), _ptr(v), _ptr(q), _ptr(y), _ptr(E_final),
                                     B, T, H, D, int(mode), _ptr(E0), _ptr(E_all))
    if rc != 0:
        raise ValueError(f"esa_oracle_scan_fwd failed with {rc}")
    return (y, E_final, E_all) if return_states else (y, E_final)


def scan_bwd(a, v, q, dy, mode, E_init=None, dE_final=None):
    """Backward scan.  Returns ``(da, dv, dq, dE_init)``."""
    a = _f64(a)
    if a.ndim != 4:
        raise ValueError("a must be [B, T, H, D]")
    B, T, H, D = a.shape
    v = _f64(v, a.shape)
    q = _f64(q, a.shape)
    dy = _f64(dy, a.shape)
    E0 = None if E_init is None else _f64(E_init, (B, H, D))
    dEf = None if dE_final is None else _f64(dE_final, (B, H, D))
    da = np.empty_like(a)
    dv = np.empty_like(a)
    dq = np.empty_like(a)
    dE_init = np.empty((B, H, D), dtype=np.float64)
    rc = _load().esa_oracle_scan_bwd(_ptr(a), _ptr(v), _ptr(q), _ptr(dy), _ptr(dEf),
                                     _ptr(da), _ptr(dv), _ptr(dq), _ptr(dE_init),
                                     B, T, H, D, int(mode), _ptr(E0))
    if rc != 0:
        raise ValueError(f"esa_oracle_scan_bwd failed with {rc}")
    return da, dv, dq, dE_init


def step(a_t, v_t, q_t, E, mode):
    """One-token update of [B, H, D] inputs.  Returns ``(y_t, E_new)``; E is not modified."""
    a_t = _f64(a_t)
    if a_t.ndim != 3:
        raise ValueError("a_t must be [B, H, D]")
    B, H, D = a_t.shape
    v_t = _f64(v_t, a_t.shape)
    q_t = _f64(q_t, a_t.shape)
    E_new = np.array(_f64(E, a_t.shape), copy=True)
    y_t = np.empty_like(a_t)
    rc = _load().esa_oracle_step(_ptr(a_t), _ptr(v_t), _ptr(q_t), _ptr(E_new), _ptr(y_t),
                                 B, H, D, int(mode))
    if rc != 0:
        raise ValueError(f"esa_oracle_step failed with {rc}")
    return y_t, E_new


def _gates(a):
    """A_t = sigmoid(a_t) in double precision."""
    return 1.0 / (1.0 + np.exp(-_f64(a)))


def scan_map(a, v, mode):
    """Forward map of a time slice ([B, T, H, D] inputs): ``(P, S)``, float64
    ``[B, H, D]``, such that the slice's final state is ``P * E_0 + S`` for
    every initial state E_0.

    The recurrence E_t = A_t E_{t-1} + B_t ("entangled-state-attention
    0.1.0", section "Core idea"; B_t = v_t or (1 - A_t) v_t) is affine in
    E_{t-1} with B_t independent of E, so by induction E_T = (prod_t A_t) E_0
    + E_T|_{E_0 = 0}: P is the product of the gates, S the scan from a zero
    state.  The readout does not enter, so q is zero here.
    """
    a = _f64(a)
    P = np.prod(_gates(a), axis=1)
    _, S = scan_fwd(a, v, np.zeros_like(a), mode)
    return P, S


def scan_bwd_map(a, v, q, dy, mode, E_init=None):
    """Backward map of a time slice: ``(P, S)`` with ``dE_init = P * dE_final
    + S`` for every dE_final.

    The reverse recurrence G_t = ghat_t + A_{t+1} G_{t+1}, G_T = ghat_T +
    dE_final, dE_init = A_1 G_1, is affine in dE_final, and ghat depends only
    on the forward states (fixed by E_init), not on dE_final: dE_init =
    (prod_t A_t) dE_final + dE_init|_{dE_final = 0}.
    """
    a = _f64(a)
    P = np.prod(_gates(a), axis=1)
    S = scan_bwd(a, v, q, dy, mode, E_init=E_init, dE_final=None)[3]
    return P, S


def compose(P, S, x0=None, reverse=False):
    """Apply the maps x -> P[j] x + S[j] one after another to ``x0`` (zeros
    when None): j = 0, 1, ..., n-1, or n-1, ..., 0 with ``reverse``.
    ``P``, ``S``: ``[n, ...]``."""
    P = _f64(P)
    S = _f64(S, P.shape)
    x = np.zeros(P.shape[1:]) if x0 is None else np.array(_f64(x0, P.shape[1:]), copy=True)
    order = range(P.shape[0] - 1, -1, -1) if reverse else range(P.shape[0])
    for j in order:
        x = P[j] * x + S[j]
    return x


def round_io(x, io_dtype):
    """Round float64 values to the I/O type and widen them back: "f16" (IEEE
    half, round to nearest even, by numpy), "bf16" (the upper 16 bits of the
    float32 value, round to nearest even, after rounding to float32 first)
    or "f32"."""
    x = np.asarray(x, dtype=np.float64)
    if io_dtype == "f16":
        return x.astype(np.float16).astype(np.float64)
    if io_dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if io_dtype == "bf16":
        u = np.ascontiguousarray(x.astype(np.float32)).view(np.uint32).astype(np.uint64)
        u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16 << 16
        return u.astype(np.uint32).view(np.float32).astype(np.float64)
    raise ValueError(f"unknown I/O type {io_dtype}")


def project(x, W, io_dtype):
    """The layer's projections ("entangled-state-attention 0.1.0", section
    "Core idea": a = x W_A, v = x W_V, q = x W_Q): ``x`` [B, T, C_in], ``W``
    [3C, C_in] (W_A, W_V, W_Q stacked, each [out, in]); float64 products,
    rounded to the I/O type.  Returns a, v, q as [B, T, C] float64."""
    x = _f64(x)
    W = _f64(W)
    C = W.shape[0] // 3
    out = []
    for p in range(3):
        out.append(round_io(x @ W[p * C:(p + 1) * C].T, io_dtype))
    return tuple(out)


def output_projection(y, W_O, io_dtype):
    """The layer's output ("entangled-state-attention 0.1.0", section "Core
    idea": y_t = W_O (q_t (.) Norm(E_t))): ``y`` [B, T, H, D] -- the readout as
    the scan writes it, in the I/O type -- flattened to [B, T, C], times
    ``W_O`` [C_out, C] ([out, in], as ``W``): z = y W_O^T in float64, rounded
    to the I/O type.  Returns z as [B, T, C_out] float64."""
    y = round_io(_f64(y), io_dtype)
    B, T = y.shape[0], y.shape[1]
    return round_io(y.reshape(B, T, -1) @ _f64(W_O).T, io_dtype)


def fused_fwd(x, W, H, mode, io_dtype, E_init=None):
    """Forward of the layer from its input: :func:`project`, then
    :func:`scan_fwd` over H heads.  Returns ``(y, E_final)``, y [B, T, H, D]."""
    a, v, q = project(x, W, io_dtype)
    B, T, C = a.shape
    D = C // H
    shape = (B, T, H, D)
    return scan_fwd(a.reshape(shape), v.reshape(shape), q.reshape(shape), mode, E_init=E_init)
