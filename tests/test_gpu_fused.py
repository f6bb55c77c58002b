"""GPU parity of the fused projection + scan forward (esa_fused_fwd).

The kernel computes a, v, q = x W_A^T, x W_V^T, x W_Q^T on the tensor cores
(tcgen05), rounds them to the I/O type and scans them without writing them
out.  It is compared with

* the oracle, in two parts: every projection the kernel produced (it can
  write them out) against the float64 product, within half a unit in the
  last place plus the float32 accumulation bound -- the rounding of a value
  that lies within the accumulation error of a rounding midpoint can go
  either way, so the projections are not compared with a rounded oracle
  value; then the kernel's scan against the oracle's scan of exactly those
  projections; on ragged lengths, partial channel tiles, both input widths,
  both modes and dtypes, and a given initial state;
* the library's own forward scan on the same projections: bitwise equal;
* the library's backward on the fused forward's outputs and workspace.

Inputs: x ~ N(0, 1), weights ~ N(0, 1 / C_in), so a, v, q ~ N(0, 1).
"""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_recurrence_b200 import esa, inputs
from tests._parity import DT, TOL, assert_close, half_ulp, host64

pytestmark = pytest.mark.gpu

CASES = [
    # B, T, H, D, C_in, mode, dtype
    (2, 300, 4, 32, 128, 1, "f16"),
    (3, 1000, 2, 64, 64, 0, "bf16"),
    (1, 97, 8, 8, 128, 1, "f16"),        # C = 64: one channel tile
    (2, 257, 5, 16, 128, 0, "bf16"),     # C = 80: a partial second channel tile
    (2, 4100, 4, 32, 128, 1, "bf16"),
    (1, 129, 6, 64, 64, 1, "f16"),       # six channel tiles
    (2, 700, 8, 32, 256, 1, "f16"),      # C_in = 256: one tile group per CTA, four channel tiles
    (1, 300, 4, 64, 256, 0, "bf16"),     # C_in = 256, D = 64
]


def _inputs(B, T, C_in, C, dt, seed, device):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, T, C_in, generator=g).to(DT[dt]).to(device)
    W = (torch.randn(3 * C, C_in, generator=g) / C_in ** 0.5).to(DT[dt]).to(device)
    return x, W


def _check_projections(x, W, avq, C, dtype):
    """Each projection the kernel produced is the float64 product rounded to
    the I/O type, up to the float32 accumulation inside the tensor core: it
    lies within half a unit in the last place (of the I/O type) plus the
    accumulation error bound 2^-15 sum_k |x_k W_k| of the exact product."""
    x64, W64 = host64(x), host64(W)
    B, T, _ = x.shape
    for p, t in enumerate(avq):
        Wp = W64[p * C:(p + 1) * C]
        exact = x64 @ Wp.T
        g = host64(t).reshape(B, T, C)
        allowed = np.maximum(half_ulp(exact, dtype), half_ulp(g, dtype)) + 2.0 ** -15 * (np.abs(x64) @ np.abs(Wp).T)
        err = np.abs(g - exact)
        worst = np.unravel_index(np.argmax(err / allowed), err.shape)
        assert err[worst] <= allowed[worst], (f"projection {'avq'[p]}: |err| {err[worst]:.3e} at {worst} "
                                              f"(allowed {allowed[worst]:.3e})")


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}T{c[1]}H{c[2]}D{c[3]}Cin{c[4]}m{c[5]}{c[6]}" for c in CASES])
def test_fused_forward_matches_oracle(cuda_device, case):
    """Projections against their float64 values; the scan of the projections
    the kernel consumed against the oracle's scan of the same values."""
    B, T, H, D, C_in, mode, dt = case
    C = H * D
    x, W = _inputs(B, T, C_in, C, dt, 90 + T, cuda_device)
    E0 = inputs.make_state(B, H, D, seed=91, scale=0.5).to(cuda_device)
    y, Ef, ws, avq = esa.esa_fused_fwd(x, W, H, mode=mode, E_init=E0, want_avq=True)
    esa.esa_check(ws)
    _check_projections(x, W, avq, C, DT[dt])
    y_r, Ef_r = oracle.scan_fwd(*(host64(t) for t in avq), mode, E_init=host64(E0))
    tol = TOL[DT[dt]]
    assert_close(y, y_r, tol, "y")
    assert_close(Ef, Ef_r, tol, "E_final")


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}T{c[1]}H{c[2]}D{c[3]}Cin{c[4]}m{c[5]}{c[6]}" for c in CASES])
def test_fused_scan_is_bitwise_the_library_scan(cuda_device, case):
    """Given the same a, v, q the fused kernel's scan is the forward scan
    kernel's arithmetic, operation for operation: y and E_final are bitwise
    equal; with the projections requested or not, y is the same."""
    B, T, H, D, C_in, mode, dt = case
    C = H * D
    x, W = _inputs(B, T, C_in, C, dt, 95 + T, cuda_device)
    y, Ef, ws, avq = esa.esa_fused_fwd(x, W, H, mode=mode, want_avq=True)
    y_only, Ef_only, _ = esa.esa_fused_fwd(x, W, H, mode=mode, workspace=ws)
    y2, Ef2, _ = esa.esa_scan_fwd(*avq, mode=mode, workspace=ws)
    esa.esa_check(ws)
    assert torch.equal(y, y2) and torch.equal(Ef, Ef2)
    assert torch.equal(y, y_only) and torch.equal(Ef, Ef_only)
    # and the projections agree with cuBLAS's up to the accumulation order
    proj = [(x @ W[p * C:(p + 1) * C].T) for p in range(3)]
    for p in range(3):
        d = (avq[p].reshape(B, T, C).float() - proj[p].float()).abs()
        assert bool((d <= 2.0 ** -7 * proj[p].float().abs() + 1e-6).all()), f"projection {p} vs cuBLAS"


def test_fused_forward_then_library_backward(cuda_device):
    """With the projections written, the fused call is a training forward:
    esa_scan_bwd on its outputs and workspace gives the oracle's gradients."""
    B, T, H, D, C_in, mode, dt = 2, 600, 4, 32, 128, 1, "f16"
    C = H * D
    x, W = _inputs(B, T, C_in, C, dt, 97, cuda_device)
    dy = torch.randn(B, T, H, D, generator=torch.Generator().manual_seed(98)).to(DT[dt]).to(cuda_device)
    y, Ef, ws, (a, v, q) = esa.esa_fused_fwd(x, W, H, mode=mode, want_avq=True)
    da, dv, dq, dE0 = esa.esa_scan_bwd(a, v, q, dy, ws, mode=mode)
    esa.esa_check(ws)
    ref = oracle.scan_bwd(host64(a), host64(v), host64(q), host64(dy), mode)
    tol = TOL[DT[dt]]
    for name, g, r in zip(("da", "dv", "dq", "dE_init"), (da, dv, dq, dE0), ref):
        assert_close(g, r, tol, name)


def test_fused_forward_empty_and_reuse(cuda_device):
    H, D, C_in = 4, 32, 128
    x, W = _inputs(2, 0, C_in, H * D, "f16", 5, cuda_device)
    E0 = inputs.make_state(2, H, D, seed=6).to(cuda_device)
    y, Ef, ws = esa.esa_fused_fwd(x, W, H, E_init=E0)
    assert y.shape == (2, 0, H, D)
    assert torch.equal(Ef, E0)
    # one workspace, three calls of different lengths
    ws = esa.new_workspace(2, 700, H, D, torch.float16, cuda_device)
    for k, T in enumerate((700, 129, 511)):
        x, W = _inputs(2, T, C_in, H * D, "f16", 7 + k, cuda_device)
        y, Ef, _, avq = esa.esa_fused_fwd(x, W, H, mode=1, workspace=ws, want_avq=True)
        esa.esa_check(ws)
        y_r, Ef_r = oracle.scan_fwd(*(host64(t) for t in avq), 1)
        assert_close(y, y_r, TOL[torch.float16], f"call{k}.y")
        assert_close(Ef, Ef_r, TOL[torch.float16], f"call{k}.E_final")


def test_fused_forward_rejects_unsupported_shapes(cuda_device):
    x, W = _inputs(1, 16, 96, 128, "f16", 1, cuda_device)
    with pytest.raises(esa.EsaError):
        esa.esa_fused_fwd(x, W, 4)                      # C_in = 96
    x, W = _inputs(1, 16, 128, 256, "f16", 1, cuda_device)
    with pytest.raises(esa.EsaError):
        esa.esa_fused_fwd(x, W, 2)                      # D = 128
    x32 = torch.zeros(1, 16, 128, device=cuda_device)
    W32 = torch.zeros(384, 128, device=cuda_device)
    with pytest.raises(esa.EsaError):
        esa.esa_fused_fwd(x32, W32, 4)                  # float32 I/O


def _random_fused_cases(n, seed=20261203):
    import numpy as np
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < n:
        D = int(rng.choice([8, 16, 32, 64]))
        H = int(rng.integers(1, 9))
        C_in = int(rng.choice([64, 128, 256]))
        B = int(rng.integers(1, 4))
        T = int(rng.choice([1, 127, 128, 129, 255, 256, 700])) if rng.random() < 0.5 else int(rng.integers(1, 2000))
        if B * T * H * D > 800_000:
            continue
        cases.append((B, T, H, D, C_in, int(rng.integers(0, 2)), str(rng.choice(["f16", "bf16"])), len(cases)))
    return cases


RANDOM = _random_fused_cases(12)


@pytest.mark.parametrize("case", RANDOM, ids=[f"{c[7]}-B{c[0]}T{c[1]}H{c[2]}D{c[3]}Cin{c[4]}m{c[5]}{c[6]}" for c in RANDOM])
def test_fused_random_shapes(cuda_device, case):
    B, T, H, D, C_in, mode, dt, k = case
    C = H * D
    x, W = _inputs(B, T, C_in, C, dt, 300 + k, cuda_device)
    E0 = inputs.make_state(B, H, D, seed=301 + k, scale=0.5).to(cuda_device) if k % 2 else None
    y, Ef, ws, avq = esa.esa_fused_fwd(x, W, H, mode=mode, E_init=E0, want_avq=True)
    esa.esa_check(ws)
    _check_projections(x, W, avq, C, DT[dt])
    y_r, Ef_r = oracle.scan_fwd(*(host64(t) for t in avq), mode, E_init=None if E0 is None else host64(E0))
    tol = TOL[DT[dt]]
    assert_close(y, y_r, tol, "y")
    assert_close(Ef, Ef_r, tol, "E_final")


# ---------------------------------------------------------------------------
# The layer's whole forward: fused projections, scan and output projection
# z = y W_O^T (esa_fused_layer_fwd, C = 64).
# ---------------------------------------------------------------------------

LAYER_CASES = [
    # B, T, H, D, C_in, mode, dtype
    (2, 700, 2, 32, 64, 1, "f16"),
    (1, 300, 1, 64, 128, 0, "bf16"),
    (3, 257, 4, 16, 64, 0, "f16"),       # ragged last tile
    (1, 1030, 8, 8, 128, 1, "bf16"),
]


@pytest.mark.parametrize("case", LAYER_CASES, ids=[f"B{c[0]}T{c[1]}H{c[2]}D{c[3]}Cin{c[4]}m{c[5]}{c[6]}"
                                                   for c in LAYER_CASES])
def test_fused_layer_forward_matches_oracle(cuda_device, case):
    """z against the float64 output projection of the kernel's own y (half a
    unit in the last place plus the float32 accumulation bound), and against
    the oracle's whole layer (projections, scan, output projection) at the
    I/O tolerance; y bitwise equal to esa_fused_fwd's."""
    B, T, H, D, C_in, mode, dt = case
    C = H * D
    x, W = _inputs(B, T, C_in, C, dt, 120 + T, cuda_device)
    g = torch.Generator().manual_seed(121 + T)
    W_O = (torch.randn(C, C, generator=g) / C ** 0.5).to(DT[dt]).to(cuda_device)
    E0 = inputs.make_state(B, H, D, seed=122, scale=0.5).to(cuda_device)
    z, y, Ef, ws = esa.esa_fused_layer_fwd(x, W, W_O, H, mode=mode, E_init=E0, want_y=True)
    esa.esa_check(ws)
    y_f, Ef_f, _ = esa.esa_fused_fwd(x, W, H, mode=mode, E_init=E0)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_f.view(torch.int16))
    assert torch.equal(Ef, Ef_f)
    # z from the kernel's own y: one rounding of a float32-accumulated product
    y64 = host64(y).reshape(B, T, C)
    Wo64 = host64(W_O)
    exact = y64 @ Wo64.T
    zg = host64(z)
    allowed = np.maximum(half_ulp(exact, DT[dt]), half_ulp(zg, DT[dt])) + 2.0 ** -15 * (np.abs(y64) @ np.abs(Wo64).T)
    err = np.abs(zg - exact)
    worst = np.unravel_index(np.argmax(err / allowed), err.shape)
    assert err[worst] <= allowed[worst], f"z: |err| {err[worst]:.3e} at {worst} (allowed {allowed[worst]:.3e})"
    # the whole layer against the oracle
    y_r, Ef_r = oracle.fused_fwd(host64(x), host64(W), H, mode, dt, E_init=host64(E0))
    z_r = oracle.output_projection(y_r, host64(W_O), dt)
    tol = TOL[DT[dt]]
    assert_close(z, z_r, tol, f"z ({dt})")
    assert_close(Ef, Ef_r, tol, f"E_final ({dt})")


def test_fused_layer_forward_without_y_and_refusals(cuda_device):
    B, T, H, D, C_in = 2, 500, 2, 32, 64
    x, W = _inputs(B, T, C_in, H * D, "f16", 130, cuda_device)
    W_O = (torch.randn(64, 64, generator=torch.Generator().manual_seed(131)) / 8.0).half().to(cuda_device)
    z, y, _, ws = esa.esa_fused_layer_fwd(x, W, W_O, H, mode=esa.CONTROLLED)
    esa.esa_check(ws)
    assert y is None
    z2, _, _, _ = esa.esa_fused_layer_fwd(x, W, W_O, H, mode=esa.CONTROLLED, want_y=True)
    torch.cuda.synchronize()
    assert torch.equal(z.view(torch.int16), z2.view(torch.int16))
    # C = 128 (two channel tiles) and C_in = 256 are refused
    x2, W2 = _inputs(1, 64, 64, 128, "f16", 132, cuda_device)
    W_O2 = torch.zeros(128, 128, dtype=torch.float16, device=cuda_device)
    with pytest.raises(esa.EsaError):
        esa.esa_fused_layer_fwd(x2, W2, W_O2, 4)
    x3, W3 = _inputs(1, 64, 256, 64, "f16", 133, cuda_device)
    with pytest.raises(esa.EsaError):
        esa.esa_fused_layer_fwd(x3, W3, W_O, 2)
