"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on
the same (I/O-dtype-rounded) inputs and compare element by element.

Tolerance (per element): |gpu - ref| <= tol * (1 + |ref|), with tol = 1e-5
for float32 I/O and 2e-3 for float16 / bfloat16 I/O (float32 state in both).
bfloat16 outputs alone get half a unit in the last place of their format on
top: an output rounded to bfloat16 (8 significant bits) carries up to
2^-8 |ref| of rounding error by construction, which exceeds 2e-3 (1 + |ref|)
once |ref| > 1.05, so no implementation that returns bfloat16 can meet the
bare bound.  float16 and float32 outputs are held to the bare bound.

Every comparison records its worst ratio |err| / bound (1.0 = at the bound);
``worst_ratios()`` returns them, and the test session prints the largest ones.
"""
import numpy as np
import torch

import oracle
from gated_linear_recurrence_b200 import esa

TOL = {torch.float32: 1e-5, torch.float16: 2e-3, torch.bfloat16: 2e-3}
DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def host64(t):
    return t.detach().to("cpu", torch.float64).numpy()


# significand bits after the leading one, and the smallest normal exponent
_FORMAT = {torch.float32: (23, -126), torch.float16: (10, -14), torch.bfloat16: (7, -126)}


def half_ulp(ref, dtype):
    """Half the spacing of `dtype` values at |ref| (normal and subnormal range)."""
    mant, emin = _FORMAT.get(dtype, (52, -1022))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.abs(ref)))
    e = np.maximum(np.where(np.isfinite(e), e, emin), emin)
    return 0.5 * np.exp2(e - mant)


_WORST = {}   # (test id, output name) -> (worst ratio, output dtype)


def worst_ratios():
    """{(test id, output name): (worst |err| / bound, output dtype name)} of this session."""
    return dict(_WORST)


def _test_id():
    import os
    return os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]


def bound(ref, tol, out_dtype):
    """The per-element error bound: tol (1 + |ref|), plus half an ulp for bfloat16 outputs."""
    b = tol * (1.0 + np.abs(ref))
    if out_dtype == torch.bfloat16:
        b = b + half_ulp(ref, out_dtype)
    return b


def assert_close(gpu, ref, tol, name, allowance=0.0):
    """|gpu - ref| <= bound(ref, tol, dtype) + allowance, element by element."""
    out_dtype = gpu.dtype if isinstance(gpu, torch.Tensor) else torch.float64
    g = host64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert g.shape == ref.shape, (name, g.shape, ref.shape)
    if g.size == 0:
        return
    assert np.all(np.isfinite(g)), f"{name}: non-finite GPU output"
    ratio = np.abs(g - ref) / (bound(ref, tol, out_dtype) + allowance)
    worst = np.unravel_index(np.argmax(ratio), ratio.shape)
    key = (_test_id(), name)
    prev = _WORST.get(key, (0.0, ""))[0]
    _WORST[key] = (max(prev, float(ratio[worst])), str(out_dtype).replace("torch.", ""))
    extra = ("+ulp/2" if out_dtype == torch.bfloat16 else "") + (f"+{allowance:.3g}" if allowance else "")
    assert ratio[worst] <= 1.0, (f"{name}: |err| {abs(g[worst] - ref[worst]):.3e} at {worst} exceeds "
                                 f"{tol:g}*(1+|ref|){extra} (gpu {g[worst]:.6g}, ref {ref[worst]:.6g}, "
                                 f"ratio {ratio[worst]:.3f})")


def gpu_fwd_bwd(x, mode, E_init=None, dE_final=None, with_bwd=True):
    """x: dict of CUDA tensors a, v, q (dy).  Returns dict of CUDA outputs."""
    y, Ef, ws = esa.esa_scan_fwd(x["a"], x["v"], x["q"], mode=mode, E_init=E_init)
    out = {"y": y, "E_final": Ef, "ws": ws}
    if with_bwd:
        da, dv, dq, dE0 = esa.esa_scan_bwd(x["a"], x["v"], x["q"], x["dy"], ws, mode=mode, E_init=E_init,
                                           dE_final=dE_final)
        out.update(da=da, dv=dv, dq=dq, dE_init=dE0)
    esa.esa_check(ws)
    return out


def oracle_fwd_bwd(x, mode, E_init=None, dE_final=None, with_bwd=True, rows=None):
    """Oracle on the same rounded inputs (optionally only batch rows `rows`)."""
    sel = slice(None) if rows is None else rows
    a, v, q = (host64(x[k][sel]) for k in ("a", "v", "q"))
    E0 = None if E_init is None else host64(E_init[sel])
    dEf = None if dE_final is None else host64(dE_final[sel])
    y, Ef = oracle.scan_fwd(a, v, q, mode, E_init=E0)
    out = {"y": y, "E_final": Ef}
    if with_bwd:
        da, dv, dq, dE0 = oracle.scan_bwd(a, v, q, host64(x["dy"][sel]), mode, E_init=E0, dE_final=dEf)
        out.update(da=da, dv=dv, dq=dq, dE_init=dE0)
    return out


def compare(gpu, ref, tol, keys, rows=None, prefix="", allowance=None):
    """assert_close over `keys`; `allowance` maps a key to an absolute allowance on top of the bound."""
    for k in keys:
        g = gpu[k] if rows is None else gpu[k][rows]
        assert_close(g, ref[k], tol, prefix + k, allowance=(allowance or {}).get(k, 0.0))
