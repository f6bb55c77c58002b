"""Pins for the double-precision CPU oracle (no GPU).

The pages print no numeric worked example for the scan, so every pin here is
fixed by mathematics rather than by a printed value:

* a brute-force evaluation of the closed form
  E_t = (prod_{r<=t} A_r) E_0 + sum_{s<=t} (prod_{s<r<=t} A_r) B_s
  in 50-digit decimal arithmetic (independent of numpy and of the C code);
* special cases that reduce to library routines (numpy.cumsum for A = 1,
  scipy.signal.lfilter for a constant controlled gate);
* the controlled-mode convex-hull invariant ("entangled-state-attention
  0.1.0", Core idea: the keep gate trades retention against writing);
* readout invariants of the per-head RMS norm;
* split/resume, scan == step-by-step decode, causality;
* central finite differences and a directional-derivative (adjoint) check for
  the backward pass, plus the exact transposition of the linear state map.
"""
import decimal
import math

import numpy as np
import pytest
import scipy.signal

import oracle

D_, C_ = oracle.DIRECT, oracle.CONTROLLED


def rng_inputs(seed, B, T, H, D, a_mean=0.0, a_scale=1.0):
    r = np.random.default_rng(seed)
    a = r.normal(a_mean, a_scale, (B, T, H, D))
    v = r.normal(0, 1, (B, T, H, D))
    q = r.normal(0, 1, (B, T, H, D))
    dy = r.normal(0, 1, (B, T, H, D))
    E0 = r.normal(0, 1, (B, H, D))
    dEf = r.normal(0, 1, (B, H, D))
    return a, v, q, dy, E0, dEf


# ---------------------------------------------------------------------------
# Closed form, evaluated by brute force in 50-digit decimal arithmetic.
# ---------------------------------------------------------------------------

def _dec_sigmoid(x):
    x = decimal.Decimal(x)
    return decimal.Decimal(1) / (decimal.Decimal(1) + (-x).exp())


def _brute_closed_form(a, v, q, E0, mode):
    """y and E_final from the closed form, O(T^2) per channel, 50 digits."""
    ctx = decimal.getcontext()
    ctx.prec = 50
    Dec = decimal.Decimal
    B, T, H, D = a.shape
    y = np.zeros(a.shape)
    Ef = np.zeros((B, H, D))
    eps = Dec("1e-6")
    for b in range(B):
        for h in range(H):
            A = [[_dec_sigmoid(float(a[b, t, h, d])) for d in range(D)] for t in range(T)]
            Bt = [[Dec(float(v[b, t, h, d])) if mode == D_ else (1 - A[t][d]) * Dec(float(v[b, t, h, d]))
                   for d in range(D)] for t in range(T)]
            for t in range(T):
                E = []
                for d in range(D):
                    prod_all = Dec(1)
                    for r in range(t + 1):
                        prod_all *= A[r][d]
                    acc = prod_all * Dec(float(E0[b, h, d]))
                    for s in range(t + 1):
                        p = Dec(1)
                        for r in range(s + 1, t + 1):
                            p *= A[r][d]
                        acc += p * Bt[s][d]
                    E.append(acc)
                m = sum(e * e for e in E) / Dec(D)
                rr = Dec(1) / (m + eps).sqrt()
                for d in range(D):
                    y[b, t, h, d] = float(Dec(float(q[b, t, h, d])) * E[d] * rr)
                if t == T - 1:
                    Ef[b, h, :] = [float(e) for e in E]
    return y, Ef


@pytest.mark.parametrize("mode", [D_, C_])
def test_closed_form_brute_force(mode):
    a, v, q, _, E0, _ = rng_inputs(11 + mode, 1, 7, 2, 3)
    y, Ef = oracle.scan_fwd(a, v, q, mode, E_init=E0)
    y_ref, Ef_ref = _brute_closed_form(a, v, q, E0, mode)
    np.testing.assert_allclose(y, y_ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Ef, Ef_ref, rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------------------
# Special cases that reduce to library routines.
# ---------------------------------------------------------------------------

def test_direct_gate_one_is_cumsum():
    # sigma(1000) == 1 exactly in double, so E = E_0 + cumsum(v).
    _, v, q, _, E0, _ = rng_inputs(3, 2, 9, 2, 4)
    a = np.full(v.shape, 1000.0)
    _, Ef, Eall = oracle.scan_fwd(a, v, q, D_, E_init=E0, return_states=True)
    ref = E0[:, None] + np.cumsum(v, axis=1)
    np.testing.assert_allclose(Eall, ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(Ef, ref[:, -1], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("mode", [D_, C_])
def test_gate_zero_forgets(mode):
    # sigma(-1000) == 0 in double: the state is just the write term B_t = v_t.
    _, v, q, _, E0, _ = rng_inputs(4, 2, 6, 2, 4)
    a = np.full(v.shape, -1000.0)
    _, _, Eall = oracle.scan_fwd(a, v, q, mode, E_init=E0, return_states=True)
    np.testing.assert_array_equal(Eall, v)


def test_controlled_gate_one_freezes_state():
    _, v, q, _, E0, _ = rng_inputs(5, 2, 6, 2, 4)
    a = np.full(v.shape, 1000.0)
    _, Ef, Eall = oracle.scan_fwd(a, v, q, C_, E_init=E0, return_states=True)
    np.testing.assert_array_equal(Eall, np.broadcast_to(E0[:, None], v.shape))


@pytest.mark.parametrize("logit", [-1.3, 0.4, 2.5])
def test_controlled_constant_gate_is_ema_filter(logit):
    # g constant: E_t = g E_{t-1} + (1-g) v_t, a first-order IIR filter.
    _, v, q, _, E0, _ = rng_inputs(6, 1, 40, 1, 3)
    a = np.full(v.shape, logit)
    g = 1.0 / (1.0 + math.exp(-logit))
    _, _, Eall = oracle.scan_fwd(a, v, q, C_, E_init=E0, return_states=True)
    for d in range(3):
        ref, _ = scipy.signal.lfilter([1.0 - g], [1.0, -g], v[0, :, 0, d], zi=[g * E0[0, 0, d]])
        np.testing.assert_allclose(Eall[0, :, 0, d], ref, rtol=1e-12, atol=1e-12)


def test_controlled_constant_value():
    # v constant: E_t = v + (prod g)(E_0 - v).
    a, _, q, _, E0, _ = rng_inputs(7, 1, 12, 2, 3)
    vc = np.random.default_rng(8).normal(size=(1, 1, 2, 3))
    v = np.broadcast_to(vc, a.shape).copy()
    _, _, Eall = oracle.scan_fwd(a, v, q, C_, E_init=E0, return_states=True)
    g = 1.0 / (1.0 + np.exp(-a))
    P = np.cumprod(g, axis=1)
    ref = vc + P * (E0[:, None] - vc)
    np.testing.assert_allclose(Eall, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# Invariants.
# ---------------------------------------------------------------------------

def test_controlled_state_stays_in_convex_hull():
    a, v, q, _, E0, _ = rng_inputs(9, 3, 50, 2, 4, a_scale=3.0)
    _, _, Eall = oracle.scan_fwd(a, v, q, C_, E_init=E0, return_states=True)
    lo = np.minimum(E0[:, None], np.minimum.accumulate(v, axis=1))
    hi = np.maximum(E0[:, None], np.maximum.accumulate(v, axis=1))
    assert np.all(Eall >= lo - 1e-12)
    assert np.all(Eall <= hi + 1e-12)


@pytest.mark.parametrize("mode", [D_, C_])
def test_readout_rms_invariants(mode):
    a, v, _, _, E0, _ = rng_inputs(10, 2, 20, 3, 8)
    v = v * np.logspace(-4, 0, 20)[None, :, None, None]    # small states make eps visible
    E0 = E0 * 1e-4
    q = np.ones_like(a)
    y, _, Eall = oracle.scan_fwd(a, v, q, mode, E_init=E0, return_states=True)
    m = np.mean(Eall ** 2, axis=-1)
    # With q = 1, y is the normalised state n: mean_d n^2 = m / (m + eps).
    np.testing.assert_allclose(np.mean(y ** 2, axis=-1), m / (m + oracle.EPS), rtol=1e-12)
    # n has the sign of E.
    assert np.all(np.sign(y) == np.sign(Eall))
    # |y_i| <= |q_i| sqrt(D) for any q.
    q2 = np.random.default_rng(1).normal(size=a.shape)
    y2, _ = oracle.scan_fwd(a, v, q2, mode, E_init=E0)
    assert np.all(np.abs(y2) <= np.abs(q2) * math.sqrt(8) + 1e-12)


def test_readout_scale_invariance_direct():
    # Direct mode is linear in (E_0, v): scaling both scales E, and y is
    # unchanged up to the eps term when mean E^2 >> eps.
    a, v, q, _, E0, _ = rng_inputs(12, 1, 30, 2, 8)
    y1, _ = oracle.scan_fwd(a, v, q, D_, E_init=E0)
    y2, _ = oracle.scan_fwd(a, 1e3 * v, q, D_, E_init=1e3 * E0)
    np.testing.assert_allclose(y1, y2, rtol=1e-5, atol=1e-6)


def test_readout_single_channel():
    # D = 1: y = q E / sqrt(E^2 + eps).
    a, v, q, _, E0, _ = rng_inputs(13, 2, 10, 3, 1)
    y, _, Eall = oracle.scan_fwd(a, v, q, C_, E_init=E0, return_states=True)
    np.testing.assert_allclose(y, q * Eall / np.sqrt(Eall ** 2 + 1e-6), rtol=1e-13)


# ---------------------------------------------------------------------------
# Split / resume, scan == decode, causality.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [D_, C_])
def test_split_resume(mode):
    a, v, q, _, E0, _ = rng_inputs(14, 2, 33, 2, 4)
    y, Ef = oracle.scan_fwd(a, v, q, mode, E_init=E0)
    y1, E1 = oracle.scan_fwd(a[:, :13], v[:, :13], q[:, :13], mode, E_init=E0)
    y2, E2 = oracle.scan_fwd(a[:, 13:], v[:, 13:], q[:, 13:], mode, E_init=E1)
    np.testing.assert_array_equal(np.concatenate([y1, y2], axis=1), y)
    np.testing.assert_array_equal(E2, Ef)


@pytest.mark.parametrize("mode", [D_, C_])
def test_scan_equals_stepwise_decode(mode):
    a, v, q, _, E0, _ = rng_inputs(15, 2, 17, 2, 4)
    y, Ef = oracle.scan_fwd(a, v, q, mode, E_init=E0)
    E = E0.copy()
    for t in range(a.shape[1]):
        yt, E = oracle.step(a[:, t], v[:, t], q[:, t], E, mode)
        np.testing.assert_array_equal(yt, y[:, t])
    np.testing.assert_array_equal(E, Ef)


@pytest.mark.parametrize("mode", [D_, C_])
def test_causality(mode):
    a, v, q, _, E0, _ = rng_inputs(16, 1, 20, 2, 4)
    y, _ = oracle.scan_fwd(a, v, q, mode, E_init=E0)
    t0 = 11
    a2, v2, q2 = a.copy(), v.copy(), q.copy()
    a2[:, t0] += 0.7
    v2[:, t0:] -= 1.3
    q2[:, t0] *= -2.0
    y2, _ = oracle.scan_fwd(a2, v2, q2, mode, E_init=E0)
    np.testing.assert_array_equal(y2[:, :t0], y[:, :t0])
    assert np.all(np.abs(y2[:, t0] - y[:, t0]) > 0)


def test_empty_sequence():
    a = np.zeros((2, 0, 2, 4))
    E0 = np.random.default_rng(0).normal(size=(2, 2, 4))
    y, Ef = oracle.scan_fwd(a, a, a, C_, E_init=E0)
    assert y.shape == (2, 0, 2, 4)
    np.testing.assert_array_equal(Ef, E0)
    da, dv, dq, dE0 = oracle.scan_bwd(a, a, a, a, C_, E_init=E0, dE_final=E0)
    np.testing.assert_array_equal(dE0, E0)


# ---------------------------------------------------------------------------
# Backward pass.
# ---------------------------------------------------------------------------

def _loss(a, v, q, E0, dy, dEf, mode):
    y, Ef = oracle.scan_fwd(a, v, q, mode, E_init=E0)
    return float(np.sum(dy * y) + np.sum(dEf * Ef))


@pytest.mark.parametrize("mode", [D_, C_])
def test_backward_finite_differences(mode):
    a, v, q, dy, E0, dEf = rng_inputs(17 + mode, 1, 6, 2, 4)
    da, dv, dq, dE0 = oracle.scan_bwd(a, v, q, dy, mode, E_init=E0, dE_final=dEf)
    h = 1e-6
    for name, x, g in (("a", a, da), ("v", v, dv), ("q", q, dq), ("E0", E0, dE0)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            args = {"a": a, "v": v, "q": q, "E0": E0}
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args[name] = xp
            fp = _loss(args["a"], args["v"], args["q"], args["E0"], dy, dEf, mode)
            args[name] = xm
            fm = _loss(args["a"], args["v"], args["q"], args["E0"], dy, dEf, mode)
            num[idx] = (fp - fm) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=2e-6, atol=2e-7, err_msg=name)


@pytest.mark.parametrize("mode", [D_, C_])
def test_backward_directional_derivative(mode):
    # <grad, delta> == d/dh L(x + h delta) at h = 0, on a longer sequence.
    a, v, q, dy, E0, dEf = rng_inputs(19 + mode, 2, 48, 2, 8, a_mean=1.0)
    da, dv, dq, dE0 = oracle.scan_bwd(a, v, q, dy, mode, E_init=E0, dE_final=dEf)
    r = np.random.default_rng(21)
    dl = [r.normal(size=x.shape) for x in (a, v, q, E0)]
    h = 1e-5
    fp = _loss(a + h * dl[0], v + h * dl[1], q + h * dl[2], E0 + h * dl[3], dy, dEf, mode)
    fm = _loss(a - h * dl[0], v - h * dl[1], q - h * dl[2], E0 - h * dl[3], dy, dEf, mode)
    num = (fp - fm) / (2 * h)
    ana = sum(float(np.sum(g * d)) for g, d in zip((da, dv, dq, dE0), dl))
    assert abs(num - ana) <= 1e-6 * (1 + abs(ana))


def test_backward_transpose_of_linear_state_map():
    # With dy = 0 only E_final carries gradient.  The state map is linear in
    # (E_0, v) for fixed gates, so its transpose is explicit:
    #   dE_init = (prod_t A_t) dE_final,  dv_t = (prod_{r>t} A_r) dE_final (direct)
    #   dv_t = (1 - A_t) (prod_{r>t} A_r) dE_final                      (controlled)
    a, v, q, _, E0, dEf = rng_inputs(22, 2, 15, 2, 3)
    dy = np.zeros_like(a)
    A = 1.0 / (1.0 + np.exp(-a))
    suffix = np.flip(np.cumprod(np.flip(A, axis=1), axis=1), axis=1)   # prod_{r>=t}
    after = np.concatenate([suffix[:, 1:], np.ones_like(suffix[:, :1])], axis=1)  # prod_{r>t}
    for mode in (D_, C_):
        da, dv, dq, dE0 = oracle.scan_bwd(a, v, q, dy, mode, E_init=E0, dE_final=dEf)
        np.testing.assert_allclose(dE0, suffix[:, 0] * dEf, rtol=1e-12)
        ref_dv = after * dEf[:, None] * (1.0 if mode == D_ else (1.0 - A))
        np.testing.assert_allclose(dv, ref_dv, rtol=1e-12, atol=1e-15)
        np.testing.assert_array_equal(dq, np.zeros_like(dq))


# ---------------------------------------------------------------------------
# Segment maps (a sequence split along time).
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [D_, C_])
def test_scan_map_is_the_affine_map_of_the_slice(mode):
    # For every initial state the slice ends at P E_0 + S; two unrelated
    # initial states (and zero) pin both P and S.
    a, v, q, _, E0, dEf = rng_inputs(30, 2, 23, 2, 4, a_mean=1.0)
    P, S = oracle.scan_map(a, v, mode)
    for x in (E0, dEf, np.zeros_like(E0)):
        _, Ef = oracle.scan_fwd(a, v, q, mode, E_init=x)
        np.testing.assert_allclose(Ef, P * x + S, rtol=1e-12, atol=1e-13)


def test_scan_map_brute_force_product():
    # P is the product of the gates: 50-digit decimal evaluation, one channel.
    a, v, _, _, _, _ = rng_inputs(31, 1, 9, 1, 2)
    P, _ = oracle.scan_map(a, v, C_)
    ctx = decimal.Context(prec=50)
    for d in range(2):
        prod = decimal.Decimal(1)
        for t in range(9):
            x = decimal.Decimal(float(a[0, t, 0, d]))
            prod = ctx.multiply(prod, ctx.divide(1, ctx.add(1, ctx.exp(-x))))
        assert abs(float(prod) - P[0, 0, d]) <= 1e-14 * abs(float(prod))


@pytest.mark.parametrize("mode", [D_, C_])
def test_scan_bwd_map_is_the_affine_map_of_the_slice(mode):
    a, v, q, dy, E0, dEf = rng_inputs(32, 2, 19, 2, 4)
    P, S = oracle.scan_bwd_map(a, v, q, dy, mode, E_init=E0)
    for g in (dEf, 3.0 * E0, np.zeros_like(dEf)):
        dE0 = oracle.scan_bwd(a, v, q, dy, mode, E_init=E0, dE_final=g)[3]
        np.testing.assert_allclose(dE0, P * g + S, rtol=1e-11, atol=1e-12)


def test_compose_order_small_example():
    # maps x -> 2x + 1 then x -> 3x + 1 from x = 1: 3 then 10; reversed: 4 then 9.
    P = np.array([[2.0], [3.0]])
    S = np.array([[1.0], [1.0]])
    assert oracle.compose(P, S, np.array([1.0]))[0] == 10.0
    assert oracle.compose(P, S, np.array([1.0]), reverse=True)[0] == 9.0
    assert oracle.compose(P, S)[0] == 4.0
    assert oracle.compose(P[:0], S[:0], np.array([5.0]))[0] == 5.0


@pytest.mark.parametrize("mode", [D_, C_])
def test_slices_composed_equal_the_whole_sequence(mode):
    # Three slices of unequal length: the forward maps of the earlier slices
    # give each slice its initial state, the reverse maps of the later slices
    # give each its final-state gradient, and the per-slice scans then equal
    # the scan of the whole sequence.
    a, v, q, dy, E0, dEf = rng_inputs(33, 2, 40, 2, 4, a_mean=0.5)
    cuts = [0, 11, 12, 40]
    sl = [slice(cuts[i], cuts[i + 1]) for i in range(3)]
    y, Ef = oracle.scan_fwd(a, v, q, mode, E_init=E0)
    da, dv, dq, dE0 = oracle.scan_bwd(a, v, q, dy, mode, E_init=E0, dE_final=dEf)
    fmaps = [oracle.scan_map(a[:, s], v[:, s], mode) for s in sl]
    Pf = np.stack([m[0] for m in fmaps])
    Sf = np.stack([m[1] for m in fmaps])
    E_in = [oracle.compose(Pf[:r], Sf[:r], E0) for r in range(3)]
    np.testing.assert_allclose(oracle.compose(Pf, Sf, E0), Ef, rtol=1e-12, atol=1e-13)
    bmaps = [oracle.scan_bwd_map(a[:, s], v[:, s], q[:, s], dy[:, s], mode, E_init=E_in[r])
             for r, s in enumerate(sl)]
    Pb = np.stack([m[0] for m in bmaps])
    Sb = np.stack([m[1] for m in bmaps])
    np.testing.assert_allclose(oracle.compose(Pb, Sb, dEf, reverse=True), dE0, rtol=1e-11, atol=1e-12)
    parts = {k: [] for k in ("y", "da", "dv", "dq")}
    for r, s in enumerate(sl):
        yr, _ = oracle.scan_fwd(a[:, s], v[:, s], q[:, s], mode, E_init=E_in[r])
        dE_out = oracle.compose(Pb[r + 1:], Sb[r + 1:], dEf, reverse=True)
        dar, dvr, dqr, _ = oracle.scan_bwd(a[:, s], v[:, s], q[:, s], dy[:, s], mode, E_init=E_in[r],
                                           dE_final=dE_out)
        for k, val in zip(("y", "da", "dv", "dq"), (yr, dar, dvr, dqr)):
            parts[k].append(val)
    for k, ref in (("y", y), ("da", da), ("dv", dv), ("dq", dq)):
        np.testing.assert_allclose(np.concatenate(parts[k], axis=1), ref, rtol=1e-10, atol=1e-12, err_msg=k)


# ---------------------------------------------------------------------------
# The layer's projections (input of the fused forward).
# ---------------------------------------------------------------------------

def test_project_hand_example():
    # C = 1, C_in = 2: W_A = [1, 0], W_V = [0, 1], W_Q = [1, -1]; x = (3, 5)
    x = np.array([[[3.0, 5.0]]])
    W = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, -1.0]])
    a, v, q = oracle.project(x, W, "f32")
    assert (a.item(), v.item(), q.item()) == (3.0, 5.0, -2.0)
    # not symmetric: x W^T differs from x W
    W2 = np.array([[0.0, 2.0], [1.0, 0.0], [0.5, 0.5]])
    a, v, q = oracle.project(x, W2, "f32")
    assert (a.item(), v.item(), q.item()) == (10.0, 3.0, 4.0)


def test_round_io_matches_torch_conversions():
    import torch
    r = np.random.default_rng(40)
    x = np.concatenate([r.normal(0, 1, 2000) * 10.0 ** r.integers(-6, 5, 2000), [0.0, -0.0, 65504.0, 1e-8]])
    f16 = torch.from_numpy(x).to(torch.float16).double().numpy()
    np.testing.assert_array_equal(oracle.round_io(x, "f16"), f16)
    bf = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(oracle.round_io(x, "bf16"), bf)


def test_fused_forward_is_projection_then_scan():
    r = np.random.default_rng(41)
    x = r.normal(0, 1, (2, 9, 16))
    W = r.normal(0, 0.25, (3 * 8, 16))
    y, Ef = oracle.fused_fwd(x, W, 2, C_, "f16")
    a = oracle.round_io(x @ W[:8].T, "f16").reshape(2, 9, 2, 4)
    v = oracle.round_io(x @ W[8:16].T, "f16").reshape(2, 9, 2, 4)
    q = oracle.round_io(x @ W[16:].T, "f16").reshape(2, 9, 2, 4)
    y2, Ef2 = oracle.scan_fwd(a, v, q, C_)
    np.testing.assert_array_equal(y, y2)
    np.testing.assert_array_equal(Ef, Ef2)


def test_output_projection_hand_example_and_special_cases():
    # C = 2, C_out = 2: z_o = sum_c W_O[o, c] y_c, so y = (1, 0) picks W_O's first column
    y = np.array([[[[1.0, 0.0]]]])                  # [B=1, T=1, H=1, D=2]
    W_O = np.array([[1.0, 2.0], [3.0, 4.0]])
    np.testing.assert_array_equal(oracle.output_projection(y, W_O, "f32").ravel(), [1.0, 3.0])
    y = np.array([[[[0.0, 1.0]]]])
    np.testing.assert_array_equal(oracle.output_projection(y, W_O, "f32").ravel(), [2.0, 4.0])
    r = np.random.default_rng(43)
    yr = r.normal(0, 1, (2, 5, 2, 4))
    flat = oracle.round_io(yr, "f16").reshape(2, 5, 8)
    # identity: the rounded readout itself; a permutation: its channels permuted
    np.testing.assert_array_equal(oracle.output_projection(yr, np.eye(8), "f16"), flat)
    perm = r.permutation(8)
    np.testing.assert_array_equal(oracle.output_projection(yr, np.eye(8)[perm], "f16"), flat[..., perm])
    # C_out may differ from C, and heads are flattened head-major (channel h D + d)
    W2 = np.zeros((3, 8))
    W2[0, 5] = 1.0                                  # head 1, channel 1
    z = oracle.output_projection(yr, W2, "f16")
    assert z.shape == (2, 5, 3)
    np.testing.assert_array_equal(z[..., 0], oracle.round_io(yr[:, :, 1, 1], "f16"))
    np.testing.assert_array_equal(z[..., 1:], 0.0)


def test_output_projection_rounds_its_input_and_its_output():
    # the readout is consumed as written, in the I/O type: 1 + 0.4 ulp rounds to 1 first
    y = np.array([[[[1.0 + 0.4 * 2.0 ** -10]]]])
    assert oracle.output_projection(y, np.array([[1000.0]]), "f16").item() == 1000.0   # not 1000.5
    # and the product is rounded to the I/O type: 1.0001 is not an fp16 value
    z = oracle.output_projection(np.array([[[[1.0]]]]), np.array([[1.0001]]), "f16").item()
    assert z == float(np.float16(1.0001)) == 1.0


# ---------------------------------------------------------------------------
# The only printed worked examples are shapes.
# ---------------------------------------------------------------------------

def test_printed_shapes(golden_shapes):
    for case in golden_shapes:
        Bx, Tx, Cx = case["input"]
        H = case["heads"]
        a = np.zeros((Bx, Tx, H, Cx // H))
        y, Ef = oracle.scan_fwd(a, a, a, C_)
        assert list(y.reshape(Bx, Tx, Cx).shape) == case["output"], case["cite"]
        assert list(Ef.shape) == [Bx, H, Cx // H]


@pytest.fixture
def golden_shapes():
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "printed_shapes.json")
    with open(path) as f:
        return json.load(f)["cases"]
