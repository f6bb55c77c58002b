"""CPU checks of the plain float32 evaluation (``tests/_f32_sequential.py``)
that sizes the envelope of the GPU edge-regime parity tests.

1. It is a faithful float32 evaluation of the same definition as the fp64
   oracle: on well-conditioned inputs of both modes it agrees with the oracle
   within the bare fp32 bound 1e-5 (1 + |ref|) on every output.
2. The claim the envelope rests on: in the ill-conditioned regimes (an
   eps-dominated readout; saturated controlled gates from a zero state) even
   this straightforward float32 evaluation misses the fp64 result by many
   times that bound, so the bound is out of reach of any float32-state
   implementation there.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_recurrence_b200 import inputs
from tests import _f32_sequential

B, T, H, D = 2, 300, 4, 32
KEYS = ("y", "E_final", "da", "dv", "dq", "dE_init")


def _draw(seed, a_mean, a_std, v_scale, dt):
    x = inputs.make_scan_inputs(B, T, H, D, "f32", 0.0, seed)
    out = {"a": x["a"] * a_std + a_mean, "v": x["v"] * v_scale, "q": x["q"], "dy": x["dy"]}
    dtype = {"f32": torch.float32, "f16": torch.float16}[dt]
    return {k: t.to(dtype).to(torch.float64).numpy() for k, t in out.items()}


def _ratios(x, mode, tol, states, seed):
    E0 = inputs.make_state(B, H, D, seed=seed + 1, scale=0.5).double().numpy() if states else None
    dEf = inputs.make_state(B, H, D, seed=seed + 2).double().numpy() if states else None
    y, Ef = oracle.scan_fwd(x["a"], x["v"], x["q"], mode, E_init=E0)
    da, dv, dq, dE0 = oracle.scan_bwd(x["a"], x["v"], x["q"], x["dy"], mode, E_init=E0, dE_final=dEf)
    ref = {"y": y, "E_final": Ef, "da": da, "dv": dv, "dq": dq, "dE_init": dE0}
    got = _f32_sequential.fwd_bwd(x["a"], x["v"], x["q"], x["dy"], mode, E0, dEf)
    return {k: float(np.max(np.abs(got[k] - ref[k]) / (tol * (1.0 + np.abs(ref[k]))))) for k in KEYS}


@pytest.mark.parametrize("mode,a_mean", [(0, 0.0), (1, 1.5), (1, 4.0)])
def test_float32_evaluation_agrees_with_the_oracle_when_well_conditioned(mode, a_mean):
    r = _ratios(_draw(5, a_mean, 1.0, 1.0, "f32"), mode, 1e-5, True, 5)
    assert max(r.values()) <= 1.0, r
    assert max(r.values()) > 1e-4, r   # float32 rounding is visible: this is not the fp64 oracle again


def test_float32_evaluation_misses_the_bare_bound_when_ill_conditioned():
    # eps-dominated readout: controlled, zero state, v ~ 1e-3 N(0, 1), so mean_d E^2 ~ 3e-7 < eps
    r = _ratios(_draw(34, 0.0, 1.0, 1e-3, "f32"), 1, 1e-5, False, 34)
    assert r["dv"] > 3.0, r
    # saturated controlled gates (a ~ N(20, 1)) from a zero state: the gradient is summed over all T steps
    r = _ratios(_draw(31, 20.0, 1.0, 1.0, "f32"), 1, 1e-5, False, 31)
    assert r["dE_init"] > 10.0, r
