"""Host logic of the ESA layer's autograd functions, on the CPU.

The layer's projection paths are plumbing around the library calls: one
projection GEMM whose column blocks are the scan's a, v, q (row stride 3C),
the backward's da, dv, dq written into the column blocks of one gradient
buffer, and dx = G W, dW = G^T x, db = column sums of G.  Here the two scan
calls are replaced by the oracle (a test double that honours the same
strided views), so the plumbing is checked without a GPU against a float64
per-token reference of the whole layer: output, final state and the
gradients of the input, the initial state, the four weights and the biases.
The library calls themselves are covered by the GPU parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_recurrence_b200 import ESA, esa, layer as layer_mod


def _oracle_scan_fwd(a, v, q, mode=1, E_init=None, workspace=None, **_):
    f64 = lambda t: t.detach().double().numpy()   # noqa: E731
    y, Ef = oracle.scan_fwd(f64(a), f64(v), f64(q), mode, E_init=None if E_init is None else f64(E_init))
    return torch.from_numpy(y).to(a.dtype), torch.from_numpy(Ef).float(), {"E_init": E_init}


def _oracle_scan_bwd(a, v, q, dy, workspace, mode=1, E_init=None, dE_final=None, da=None, dv=None, dq=None,
                     want_dE_init=True, **_):
    f64 = lambda t: None if t is None else t.detach().double().numpy()   # noqa: E731
    g = oracle.scan_bwd(f64(a), f64(v), f64(q), f64(dy), mode, E_init=f64(E_init), dE_final=f64(dE_final))
    outs = []
    for dst, val in zip((da, dv, dq), g[:3]):
        src = torch.from_numpy(val).to(a.dtype)
        if dst is None:
            dst = src
        else:
            assert dst.shape == src.shape
            dst.copy_(src)   # into the caller's (possibly strided) view
        outs.append(dst)
    dE0 = torch.from_numpy(g[3]).float() if want_dE_init else None
    return outs[0], outs[1], outs[2], dE0


def _oracle_fused_fwd(x, W, H, mode=1, E_init=None, want_avq=False, **_):
    B, T, _ = x.shape
    C = W.shape[0] // 3
    P = (x @ W.t()).reshape(B, T, 3, H, C // H)
    a, v, q = (P[:, :, i].contiguous() for i in range(3))
    y, Ef, ws = _oracle_scan_fwd(a, v, q, mode, E_init)
    return (y, Ef, ws, (a, v, q)) if want_avq else (y, Ef, ws)


@pytest.fixture
def oracle_scans(monkeypatch):
    monkeypatch.setattr(esa, "esa_scan_fwd", _oracle_scan_fwd)
    monkeypatch.setattr(esa, "esa_scan_bwd", _oracle_scan_bwd)
    monkeypatch.setattr(esa, "esa_fused_fwd", _oracle_fused_fwd)


def _reference(x, E0, Ws, bs, H, mode, eps=1e-6):
    """Float64 per-token loop of the layer (projections with biases, the
    recurrence per head, the per-head RMS readout, the output projection)."""
    B, T, C = x.shape
    D = C // H
    a, v, q = ((x @ Ws[i].T + (0 if bs[i] is None else bs[i])).reshape(B, T, H, D) for i in range(3))
    E = E0
    ys = []
    for t in range(T):
        A = torch.sigmoid(a[:, t])
        E = A * E + (v[:, t] if mode == "direct" else (1.0 - A) * v[:, t])
        r = torch.rsqrt(E.pow(2).mean(dim=-1, keepdim=True) + eps)
        ys.append(q[:, t] * E * r)
    y = torch.stack(ys, dim=1).reshape(B, T, C)
    return y @ Ws[3].T + (0 if bs[3] is None else bs[3]), E


@pytest.mark.parametrize("mode,bias", [("controlled", True), ("direct", False)])
def test_one_gemm_projection_path_gradients(oracle_scans, mode, bias):
    torch.manual_seed(3)
    B, T, C, H = 2, 9, 16, 2
    lay = ESA(C, H, mode=mode, bias=bias, dtype=torch.float64, fused=False)
    x = torch.randn(B, T, C, dtype=torch.float64, requires_grad=True)
    E0 = (torch.randn(B, H, C // H, dtype=torch.float64) * 0.3).requires_grad_(True)
    g = torch.randn(B, T, C, dtype=torch.float64)
    u = torch.randn(B, H, C // H, dtype=torch.float64)

    out, E = lay(x, state=E0.float(), return_state=True)
    ((out * g).sum() + (E.double() * u).sum()).backward()

    lins = [lay.W_A, lay.W_V, lay.W_Q, lay.W_O]
    Ws = [m.weight.detach().clone().requires_grad_(True) for m in lins]
    bs = [None if m.bias is None else m.bias.detach().clone().requires_grad_(True) for m in lins]
    x2 = x.detach().clone().requires_grad_(True)
    E02 = E0.detach().float().double().requires_grad_(True)
    ref, E_ref = _reference(x2, E02, Ws, bs, H, mode)
    ((ref * g).sum() + (E_ref * u).sum()).backward()

    tol = dict(rtol=1e-5, atol=1e-6)   # the state passes through float32 at the boundary
    torch.testing.assert_close(out, ref, **tol)
    torch.testing.assert_close(E.double(), E_ref, **tol)
    torch.testing.assert_close(x.grad, x2.grad, **tol)
    for m, W in zip(lins, Ws):
        torch.testing.assert_close(m.weight.grad, W.grad, **tol)
    if bias:
        for m, b in zip(lins, bs):
            torch.testing.assert_close(m.bias.grad, b.grad, **tol)


def test_fused_path_backward_gradients(oracle_scans):
    """The fused function's backward (G buffer, dx = G W, dW = G^T x)."""
    torch.manual_seed(4)
    B, T, C, H = 2, 7, 16, 2
    x = torch.randn(B, T, C, dtype=torch.float64, requires_grad=True)
    W = (torch.randn(3 * C, C, dtype=torch.float64) / C ** 0.5).requires_grad_(True)
    E0 = (torch.randn(B, H, C // H) * 0.3).requires_grad_(True)
    g = torch.randn(B, T, H, C // H, dtype=torch.float64)
    y, E = layer_mod._FusedProjScanFn.apply(x, W, E0, 1, H)
    ((y * g).sum() + E.sum()).backward()

    x2 = x.detach().clone().requires_grad_(True)
    W2 = W.detach().clone().requires_grad_(True)
    E02 = E0.detach().double().requires_grad_(True)
    WO = torch.eye(C, dtype=torch.float64)
    y_ref, E_ref = _reference(x2, E02, [W2[:C], W2[C:2 * C], W2[2 * C:], WO], [None] * 4, H, "controlled")
    ((y_ref.reshape(B, T, H, C // H) * g).sum() + E_ref.sum()).backward()
    tol = dict(rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(y.double(), y_ref.reshape(B, T, H, C // H), **tol)
    torch.testing.assert_close(x.grad, x2.grad, **tol)
    torch.testing.assert_close(W.grad, W2.grad, **tol)
    torch.testing.assert_close(E0.grad.double(), E02.grad, **tol)
    assert np.isfinite(x.grad.numpy()).all()
