"""A plain float32 evaluation of the scan's definition, one time step after
another, for sizing what float32 arithmetic itself can resolve.

It is neither an oracle nor a model of the CUDA kernels: it follows the same
definition as the fp64 oracle ("entangled-state-attention 0.1.0", "Core
idea": A = sigma(a), direct B = v, controlled B = (1 - A) v,
E_t = A_t E_{t-1} + B_t, y = q E / sqrt(mean_d E^2 + 1e-6); the backward by
the chain rule) with every operation rounded to float32, in time order.  Where
an output is a cancellation of terms much larger than itself (an eps-dominated
readout scales every gradient term by r ~ 1e3; a saturated gate sums them over
the whole sequence), this evaluation misses the fp64 result by far more than
1e-5 (1 + |ref|), and so must any float32-state implementation; the edge-regime
parity tests use its error to size their envelope there.
"""
import numpy as np

EPS = np.float32(1e-6)


def _sig(x):
    """Logistic sigmoid and its complement in float32, without cancellation:
    sigma(x) = 1 / (1 + e^-x) for x >= 0, e^x / (1 + e^x) for x < 0; 1 - sigma(x) = sigma(-x)."""
    x = x.astype(np.float32)
    with np.errstate(over="ignore"):
        ep = np.exp(-np.abs(x)).astype(np.float32)
    big = (np.float32(1) / (np.float32(1) + ep)).astype(np.float32)
    small = (ep / (np.float32(1) + ep)).astype(np.float32)
    A = np.where(x >= 0, big, small).astype(np.float32)
    Ac = np.where(x >= 0, small, big).astype(np.float32)
    return A, Ac


def fwd_bwd(a, v, q, dy, mode, E_init=None, dE_final=None):
    """float32 sequential forward and backward over [B, T, H, D] inputs.
    Returns a dict of y, E_final, da, dv, dq, dE_init (float64 arrays holding float32 values)."""
    f = np.float32
    a, v, q, dy = (np.asarray(t, dtype=np.float32) for t in (a, v, q, dy))
    B, T, H, D = a.shape
    E = np.zeros((B, H, D), np.float32) if E_init is None else np.asarray(E_init, np.float32).copy()
    E0 = E.copy()
    A, Ac = _sig(a)
    Bt = v if mode == 0 else (Ac * v).astype(np.float32)
    Es = np.empty((T, B, H, D), np.float32)
    rs = np.empty((T, B, H, 1), np.float32)
    y = np.empty_like(v)
    for t in range(T):
        E = (A[:, t] * E + Bt[:, t]).astype(np.float32)
        m = (np.sum(E * E, axis=-1, keepdims=True, dtype=np.float32) / f(D)).astype(np.float32)
        r = (f(1) / np.sqrt(m + EPS)).astype(np.float32)
        Es[t], rs[t] = E, r
        y[:, t] = q[:, t] * (E * r)
    out = {"y": y, "E_final": E.copy()}
    G = np.zeros((B, H, D), np.float32) if dE_final is None else np.asarray(dE_final, np.float32).copy()
    da = np.empty_like(v)
    dv = np.empty_like(v)
    dq = np.empty_like(v)
    carry = G   # gradient flowing into E_t from later steps (dE_final at t = T)
    for t in range(T - 1, -1, -1):
        E, r = Es[t], rs[t]
        n = (E * r).astype(np.float32)
        dq[:, t] = dy[:, t] * n
        dn = (dy[:, t] * q[:, t]).astype(np.float32)
        dot = (np.sum(dn * n, axis=-1, keepdims=True, dtype=np.float32) / f(D)).astype(np.float32)
        ghat = (r * (dn - n * dot)).astype(np.float32)
        G = (ghat + carry).astype(np.float32)
        Eprev = Es[t - 1] if t > 0 else E0
        s = (A[:, t] * Ac[:, t]).astype(np.float32)
        if mode == 0:
            dv[:, t] = G
            da[:, t] = G * Eprev * s
        else:
            dv[:, t] = G * Ac[:, t]
            da[:, t] = G * (Eprev - v[:, t]) * s
        carry = (A[:, t] * G).astype(np.float32)
    out.update(da=da, dv=dv, dq=dq, dE_init=carry)
    return {k: x.astype(np.float64) for k, x in out.items()}
