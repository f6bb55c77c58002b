"""GPU parity in the numerical edge regimes of the method.

The gate is a logistic sigmoid and the readout divides by a root mean square
with eps = 1e-6 inside the square root ("entangled-state-attention 0.1.0",
"Core idea": A = sigma(a), controlled write term (1 - A) v, y = q Norm(E)).
A fast implementation departs from that definition exactly where these tests
look:

* saturated gates (|a| around 20): A rounds to 1 (or 0) in float32, so
  1 - A must come from exp(-a) A, not from a subtraction;
* gate logits far below the kernel's clamp at -80 (and far above +80):
  exp(-a) must stay finite and A, 1 - A keep the right limits;
* an eps-dominated readout: a state so small (controlled mode, zero initial
  state, values ~1e-4 or 1e-3) that mean_d E^2 is well below eps, where the
  square root's argument is decided by eps;
* large values in float16 (|v| up to about 6e4, near the format's largest
  finite value), where E^2 is large and the readout's scale is tiny.

Each case runs the forward and the backward through the C ABI and compares
every output with the fp64 oracle on the same rounded inputs, at the bound
the tests use everywhere (float16 and float32 at tol (1 + |ref|),
bfloat16 with half an ulp of its format on top) plus an envelope sized by
float32 arithmetic itself: 4 times the worst error, on that output, of a
plain float32 evaluation of the definition in time order
(``tests/_f32_sequential.py``).  Where an output is a cancellation of terms
far larger than itself -- gradients of an eps-dominated readout are scaled by
r ~ 1e3, and with saturated gates they are summed over the whole sequence --
that evaluation misses the fp64 result by up to ~50 times 1e-5 (1 + |ref|)
(``tests/test_f32_conditioning.py`` pins this), so no float32-state
implementation can meet the bare fp32 bound there; a fast-math departure from
the definition (a gate or a norm computed wrongly) would still exceed the
envelope by orders of magnitude.  The envelope is close to zero for
well-conditioned outputs.
"""
import numpy as np
import pytest
import torch

from gated_linear_recurrence_b200 import inputs
from tests import _f32_sequential
from tests._parity import DT, TOL, compare, gpu_fwd_bwd, host64, oracle_fwd_bwd

ENVELOPE = 4.0   # times the plain float32 evaluation's worst error on the same output

pytestmark = pytest.mark.gpu

ALL = ("y", "E_final", "da", "dv", "dq", "dE_init")
B, T, H, D = 2, 300, 4, 32   # three 128-row tiles per chain with a ragged tail; two channel tiles


def _draw(seed, a_mean, a_std, v_scale, dt, dev, v_clip=None):
    """a ~ N(a_mean, a_std^2), v ~ v_scale N(0, 1) (optionally clipped), q, dy ~ N(0, 1),
    drawn in float32 from one seeded stream, then rounded to the I/O dtype."""
    x = inputs.make_scan_inputs(B, T, H, D, "f32", 0.0, seed)
    a = x["a"] * a_std + a_mean
    v = x["v"] * v_scale
    if v_clip is not None:
        v = v.clamp(-v_clip, v_clip)
    out = {"a": a, "v": v, "q": x["q"], "dy": x["dy"]}
    return {k: t.to(DT[dt]).to(dev) for k, t in out.items()}


def _run(x, mode, dt, states, dev, seed):
    E0 = inputs.make_state(B, H, D, seed=seed + 1, scale=0.5).to(dev) if states else None
    dEf = inputs.make_state(B, H, D, seed=seed + 2).to(dev) if states else None
    ref = oracle_fwd_bwd(x, mode, E0, dEf)
    f32 = _f32_sequential.fwd_bwd(*(host64(x[k]) for k in ("a", "v", "q", "dy")), mode,
                                  None if E0 is None else host64(E0), None if dEf is None else host64(dEf))
    env = {k: ENVELOPE * float(np.max(np.abs(f32[k] - ref[k]))) for k in ALL}
    compare(gpu_fwd_bwd(x, mode, E0, dEf), ref, TOL[DT[dt]], ALL, allowance=env)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("a_mean", [20.0, -20.0])
def test_saturated_gates(cuda_device, dt, mode, a_mean):
    x = _draw(31, a_mean, 1.0, 1.0, dt, cuda_device)
    _run(x, mode, dt, True, cuda_device, 31)
    if mode == 1 and a_mean > 0:   # the state barely moves from zero: eps decides the readout too
        _run(x, mode, dt, False, cuda_device, 31)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("mode", [0, 1])
def test_logits_beyond_the_clamp(cuda_device, dt, mode):
    # a ~ N(-90, 20^2): most logits below -80, some above; fp16 and bf16 hold them all.
    x = _draw(32, -90.0, 20.0, 1.0, dt, cuda_device)
    _run(x, mode, dt, True, cuda_device, 32)


@pytest.mark.parametrize("mode", [0, 1])
def test_logits_over_the_whole_float32_range(cuda_device, mode):
    # a ~ N(0, 60^2) in float32: saturated on both sides, clamped below -80, exp(-a) underflowing above +88.
    x = _draw(33, 0.0, 60.0, 1.0, "f32", cuda_device)
    _run(x, mode, "f32", True, cuda_device, 33)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("v_scale", [1e-4, 1e-3])
def test_eps_dominated_readout(cuda_device, dt, v_scale):
    # Controlled mode from a zero state: E ~ v_scale / sqrt(3) per channel, so
    # mean_d E^2 is about 3e-9 (1e-4) or 3e-7 (1e-3) against eps = 1e-6.
    x = _draw(34, 0.0, 1.0, v_scale, dt, cuda_device)
    _run(x, 1, dt, False, cuda_device, 34)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("a_mean", [2.0, 6.0])
def test_large_values_f16(cuda_device, mode, a_mean):
    # |v| up to 6e4 (fp16's largest finite value is 65504); direct mode with
    # long-memory gates lets the state grow well past the input range.
    x = _draw(35, a_mean, 1.0, 1e4, "f16", cuda_device, v_clip=6.0e4)
    _run(x, mode, "f16", True, cuda_device, 35)
