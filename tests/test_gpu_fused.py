"""GPU parity of the fused projection + scan forward (esa_fused_fwd).

The kernel computes a, v, q = x W_A^T, x W_V^T, x W_Q^T on the tensor cores
(tcgen05), rounds them to the I/O type and scans them without writing them
out.  It is compared with

* the oracle: float64 projections rounded to the I/O type, then the fp64
  scan (``oracle.fused_fwd``), on ragged lengths, partial channel tiles,
  both input widths, both modes and dtypes, and a given initial state;
* the unfused library path: the projections by torch (cuBLAS) in the I/O
  type, then ``esa_scan_fwd``.

Inputs: x ~ N(0, 1), weights ~ N(0, 1 / C_in), so a, v, q ~ N(0, 1).
"""
import pytest
import torch

import oracle
from gated_linear_recurrence_b200 import esa, inputs
from tests._parity import DT, TOL, assert_close, host64

pytestmark = pytest.mark.gpu

CASES = [
    # B, T, H, D, C_in, mode, dtype
    (2, 300, 4, 32, 128, 1, "f16"),
    (3, 1000, 2, 64, 64, 0, "bf16"),
    (1, 97, 8, 8, 128, 1, "f16"),        # C = 64: one channel tile
    (2, 257, 5, 16, 128, 0, "bf16"),     # C = 80: a partial second channel tile
    (2, 4100, 4, 32, 128, 1, "bf16"),
    (1, 129, 6, 64, 64, 1, "f16"),       # six channel tiles
]


def _inputs(B, T, C_in, C, dt, seed, device):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, T, C_in, generator=g).to(DT[dt]).to(device)
    W = (torch.randn(3 * C, C_in, generator=g) / C_in ** 0.5).to(DT[dt]).to(device)
    return x, W


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}T{c[1]}H{c[2]}D{c[3]}Cin{c[4]}m{c[5]}{c[6]}" for c in CASES])
def test_fused_forward_matches_oracle(cuda_device, case):
    B, T, H, D, C_in, mode, dt = case
    C = H * D
    x, W = _inputs(B, T, C_in, C, dt, 90 + T, cuda_device)
    E0 = inputs.make_state(B, H, D, seed=91, scale=0.5).to(cuda_device)
    y, Ef, ws = esa.esa_fused_fwd(x, W, H, mode=mode, E_init=E0)
    esa.esa_check(ws)
    y_r, Ef_r = oracle.fused_fwd(host64(x), host64(W), H, mode, dt, E_init=host64(E0))
    tol = TOL[DT[dt]]
    assert_close(y, y_r, tol, "y")
    assert_close(Ef, Ef_r, tol, "E_final")


@pytest.mark.parametrize("case", CASES[:3], ids=[f"B{c[0]}T{c[1]}H{c[2]}D{c[3]}" for c in CASES[:3]])
def test_fused_forward_matches_unfused_library_path(cuda_device, case):
    B, T, H, D, C_in, mode, dt = case
    C = H * D
    x, W = _inputs(B, T, C_in, C, dt, 95 + T, cuda_device)
    y, Ef, ws = esa.esa_fused_fwd(x, W, H, mode=mode)
    proj = [(x @ W[p * C:(p + 1) * C].T).reshape(B, T, H, D).contiguous() for p in range(3)]
    y2, Ef2, _ = esa.esa_scan_fwd(*proj, mode=mode, workspace=ws)
    esa.esa_check(ws)
    tol = TOL[DT[dt]]
    assert_close(y, host64(y2), tol, "y")
    assert_close(Ef, host64(Ef2), tol, "E_final")


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
        y, Ef, _ = esa.esa_fused_fwd(x, W, H, mode=1, workspace=ws)
        esa.esa_check(ws)
        y_r, Ef_r = oracle.fused_fwd(host64(x), host64(W), H, 1, "f16")
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
