"""The autograd scan and the ESA layer over the C ABI.

* ``esa_scan`` forward values and every gradient (a, v, q, E_init) against the
  fp64 oracle, for a loss that uses both y and E_final.
* The ``ESA`` layer (projections + scan + readout + output projection) against
  a float64 PyTorch reference written out as the plain per-token loop of the
  "entangled-state-attention 0.1.0" page ("Core idea"), output and gradients
  of the input and of all four weight matrices.
* Decoding: a forward over a prompt returning its state, then one-token
  ``step`` calls, equals one forward over prompt + tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_recurrence_b200 import ESA, esa, esa_scan, inputs
from tests._parity import DT, TOL, assert_close, host64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dt,mode", [("f32", "controlled"), ("f16", "direct"), ("bf16", "controlled")])
def test_esa_scan_autograd_matches_oracle(cuda_device, dt, mode):
    B, T, H, D = 2, 300, 4, 32
    m = 1 if mode == "controlled" else 0
    x = inputs.make_scan_inputs(B, T, H, D, dt, 1.0, 31)
    a, v, q, w = (x[k].to(cuda_device).requires_grad_(k != "dy") for k in ("a", "v", "q", "dy"))
    E0 = inputs.make_state(B, H, D, seed=32, scale=0.5).to(cuda_device).requires_grad_(True)
    u = inputs.make_state(B, H, D, seed=33).to(cuda_device)
    y, Ef = esa_scan(a, v, q, mode, E_init=E0)
    loss = (y.float() * w.float()).sum() + (Ef * u).sum()
    loss.backward()
    f64 = lambda t: host64(t.detach())   # noqa: E731
    y_r, Ef_r = oracle.scan_fwd(f64(a), f64(v), f64(q), m, E_init=f64(E0))
    da_r, dv_r, dq_r, dE0_r = oracle.scan_bwd(f64(a), f64(v), f64(q), f64(w), m, E_init=f64(E0), dE_final=f64(u))
    tol = TOL[DT[dt]]
    assert_close(y, y_r, tol, "y")
    assert_close(Ef, Ef_r, tol, "E_final")
    assert_close(a.grad, da_r, tol, "da")
    assert_close(v.grad, dv_r, tol, "dv")
    assert_close(q.grad, dq_r, tol, "dq")
    assert_close(E0.grad, dE0_r, tol, "dE_init")


def _reference_layer(x, WA, WV, WQ, WO, H, mode, eps=1e-6):
    """Float64 per-token loop: gates, values and queries by projection, the
    recurrence per head, the per-head RMS readout and the output projection."""
    B, T, C = x.shape
    D = C // H
    a = (x @ WA.T).reshape(B, T, H, D)
    v = (x @ WV.T).reshape(B, T, H, D)
    q = (x @ WQ.T).reshape(B, T, H, D)
    E = torch.zeros(B, H, D, dtype=x.dtype)
    ys = []
    for t in range(T):
        A = torch.sigmoid(a[:, t])
        write = v[:, t] if mode == "direct" else (1.0 - A) * v[:, t]
        E = A * E + write
        r = torch.rsqrt(E.pow(2).mean(dim=-1, keepdim=True) + eps)
        ys.append(q[:, t] * E * r)
    y = torch.stack(ys, dim=1).reshape(B, T, C)
    return y @ WO.T


@pytest.mark.parametrize("mode", ["controlled", "direct"])
def test_layer_matches_float64_reference(cuda_device, mode):
    torch.manual_seed(5)
    B, T, C, H = 2, 70, 64, 2
    layer = ESA(C, H, mode=mode, device=cuda_device, dtype=torch.float32)
    x = (torch.randn(B, T, C, device=cuda_device) * 0.5).requires_grad_(True)
    g = torch.randn(B, T, C, device=cuda_device)
    out = layer(x)
    (out * g).sum().backward()

    W = {n: getattr(layer, n).weight.detach().cpu().double().requires_grad_(True) for n in ("W_A", "W_V", "W_Q", "W_O")}
    x64 = x.detach().cpu().double().requires_grad_(True)
    ref = _reference_layer(x64, W["W_A"], W["W_V"], W["W_Q"], W["W_O"], H, mode)
    (ref * g.cpu().double()).sum().backward()
    tol = 1e-4   # float32 projections and scan against float64 (library GEMMs included)
    assert_close(out, ref.detach().numpy(), tol, "out")
    assert_close(x.grad, x64.grad.numpy(), tol, "dx")
    for n in W:
        assert_close(getattr(layer, n).weight.grad, W[n].grad.numpy(), tol, f"d{n}")


def test_layer_decode_matches_full_sequence(cuda_device):
    torch.manual_seed(6)
    B, T, C, H, extra = 3, 100, 128, 4, 6
    layer = ESA(C, H, mode="controlled", scan_dtype=torch.float16, device=cuda_device)
    x = torch.randn(B, T + extra, C, device=cuda_device)
    with torch.no_grad():
        full = layer(x)
        out, state = layer(x[:, :T], return_state=True)
        steps = [layer.step(x[:, T + i], state) for i in range(extra)]
    tol = TOL[torch.float16]
    assert_close(out, host64(full[:, :T]), tol, "prefill")
    assert_close(torch.stack(steps, dim=1), host64(full[:, T:]), tol, "decode")
    assert np.isfinite(host64(state)).all()


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("mode", ["controlled", "direct"])
def test_fused_layer_matches_unfused_layer(cuda_device, dt, mode):
    """16-bit layer: the projections inside the scan kernel (tcgen05) against
    the same layer with linear projections, output and every gradient.  Both
    round a, v, q to the 16-bit type; their GEMMs accumulate in different
    orders, so a few roundings differ by one unit: tolerance 1e-2 (bf16) /
    5e-3 (fp16) relative to (1 + |ref|)."""
    torch.manual_seed(7)
    B, T, C, H = 2, 333, 128, 4
    fused = ESA(C, H, mode=mode, device=cuda_device, dtype=dt)
    plain = ESA(C, H, mode=mode, device=cuda_device, dtype=dt, fused=False)
    plain.load_state_dict(fused.state_dict())
    assert fused._fused_ok(torch.empty(1, 1, C, device=cuda_device, dtype=dt))
    x = torch.randn(B, T, C, device=cuda_device, dtype=dt)
    E0 = torch.randn(B, H, C // H, device=cuda_device) * 0.3
    g = torch.randn(B, T, C, device=cuda_device, dtype=dt)
    res = []
    for layer in (fused, plain):
        xi = x.clone().requires_grad_(True)
        Ei = E0.clone().requires_grad_(True)
        out, E = layer(xi, state=Ei, return_state=True)
        ((out.float() * g.float()).sum() + E.sum()).backward()
        res.append([out.detach(), E.detach(), xi.grad, Ei.grad] +
                   [getattr(layer, n).weight.grad for n in ("W_A", "W_V", "W_Q", "W_O")])
    tol = 1e-2 if dt == torch.bfloat16 else 5e-3
    names = ("out", "E_final", "dx", "dE0", "dW_A", "dW_V", "dW_Q", "dW_O")
    for name, f_, p_ in zip(names, res[0], res[1]):
        scale = float(p_.float().abs().max()) or 1.0
        assert_close(f_.float() / scale, host64(p_.float()) / scale, tol, name)


def test_fused_layer_inference_matches_reference(cuda_device):
    """Inference through the fused path (no projections written) against
    the float64 per-token loop, on the layer's own 16-bit weights."""
    torch.manual_seed(8)
    B, T, C, H = 2, 200, 64, 2
    layer = ESA(C, H, mode="controlled", device=cuda_device, dtype=torch.float16)
    x = torch.randn(B, T, C, device=cuda_device, dtype=torch.float16)
    with torch.no_grad():
        out = layer(x)
    W = {n: getattr(layer, n).weight.detach().cpu().double() for n in ("W_A", "W_V", "W_Q", "W_O")}
    ref = _reference_layer(x.cpu().double(), W["W_A"], W["W_V"], W["W_Q"], W["W_O"], H, "controlled")
    scale = float(ref.abs().max())
    assert_close(out.float() / scale, ref.numpy() / scale, 1e-2, "out")


def test_layer_inference_applies_w_o_inside_the_fused_kernel(cuda_device):
    """At embd = 64 without gradients the layer's output comes from
    esa_fused_layer_fwd (z = y W_O^T in the scan kernel): bit for bit that
    call's z, close to the layer with the output projection as a separate
    GEMM (fused=False), and the returned state equal to the fused scan's."""
    torch.manual_seed(9)
    B, T, C, H = 3, 333, 64, 4
    layer = ESA(C, H, mode="direct", device=cuda_device, dtype=torch.bfloat16)
    x = torch.randn(B, T, C, device=cuda_device, dtype=torch.bfloat16)
    E0 = torch.randn(B, H, C // H, device=cuda_device) * 0.5
    with torch.no_grad():
        out, E = layer(x, state=E0, return_state=True)
        W = torch.cat([layer.W_A.weight, layer.W_V.weight, layer.W_Q.weight], dim=0)
        z, _, E_z, _ = esa.esa_fused_layer_fwd(x, W, layer.W_O.weight, H, mode=esa.DIRECT, E_init=E0)
        layer.fused = False
        out_u, E_u = layer(x, state=E0, return_state=True)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), z.view(torch.int16))
    assert torch.equal(E, E_z)
    # the unfused layer's GEMMs accumulate in other orders, so a few bf16
    # roundings of a, v, q and the output differ by one unit (as in the
    # fused-against-unfused layer test): 1e-2 relative to (1 + |ref|), scaled
    for name, f_, p_ in (("out", out, out_u), ("E_final", E, E_u)):
        scale = float(p_.float().abs().max()) or 1.0
        assert_close(f_.float() / scale, host64(p_.float()) / scale, 1e-2, name)


def test_prefill_and_decode_step_interface(cuda_device):
    """prefill -> (out, state) and decode_step -> (out_t, state) agree with
    one forward over prompt + tokens (fused 16-bit layer)."""
    torch.manual_seed(11)
    B, T, C, H, extra = 2, 150, 128, 4, 5
    layer = ESA(C, H, mode="direct", device=cuda_device, dtype=torch.float16)
    x = torch.randn(B, T + extra, C, device=cuda_device, dtype=torch.float16)
    with torch.no_grad():
        full = layer(x)
    out, state = layer.prefill(x[:, :T])
    steps = []
    for i in range(extra):
        y_t, state = layer.decode_step(x[:, T + i], state)
        steps.append(y_t)
    scale = float(full.float().abs().max())
    assert_close(out.float() / scale, host64(full[:, :T].float()) / scale, 1e-2, "prefill")
    assert_close(torch.stack(steps, dim=1).float() / scale, host64(full[:, T:].float()) / scale, 1e-2, "decode")


@pytest.mark.parametrize("bias,wdt,sdt", [(True, torch.float32, torch.float16), (False, torch.bfloat16, None),
                                          (True, torch.float32, None)])
def test_layer_one_projection_gemm_matches_separate_projections(cuda_device, bias, wdt, sdt):
    """The unfused layer runs its three input projections as one GEMM and
    scans the column blocks of its output in place; its backward writes da,
    dv, dq into one buffer.  Against the same layer written with three
    separate projections feeding esa_scan: output, final state and every
    gradient (input, initial state, weights, biases)."""
    torch.manual_seed(11)
    B, T, C, H = 2, 257, 128, 4
    layer = ESA(C, H, mode="controlled", bias=bias, scan_dtype=sdt, device=cuda_device, dtype=wdt, fused=False)
    x = torch.randn(B, T, C, device=cuda_device, dtype=wdt)
    E0 = torch.randn(B, H, C // H, device=cuda_device) * 0.3
    g = torch.randn(B, T, C, device=cuda_device, dtype=wdt)

    def separate(xi, Ei):
        proj = [lin(xi).reshape(B, T, H, C // H) for lin in (layer.W_A, layer.W_V, layer.W_Q)]
        if sdt is not None:
            proj = [p.to(sdt) for p in proj]
        y, E = esa_scan(*proj, "controlled", E_init=Ei)
        return layer.W_O(y.reshape(B, T, C).to(wdt)), E

    res = []
    for run in (lambda xi, Ei: layer(xi, state=Ei, return_state=True), separate):
        layer.zero_grad(set_to_none=True)
        xi = x.clone().requires_grad_(True)
        Ei = E0.clone().requires_grad_(True)
        out, E = run(xi, Ei)
        ((out.float() * g.float()).sum() + E.sum()).backward()
        grads = [getattr(layer, n).weight.grad for n in ("W_A", "W_V", "W_Q", "W_O")]
        if bias:
            grads += [getattr(layer, n).bias.grad for n in ("W_A", "W_V", "W_Q")]
        res.append([out.detach(), E.detach(), xi.grad, Ei.grad] + grads)
    names = ["out", "E_final", "dx", "dE0", "dW_A", "dW_V", "dW_Q", "dW_O"] + (["db_A", "db_V", "db_Q"] if bias else [])
    # The GEMMs accumulate in different orders; 16-bit roundings may then differ by one unit.
    tol = 1e-2 if torch.bfloat16 in (wdt, sdt) else 5e-3
    for name, one, sep in zip(names, res[0], res[1]):
        scale = float(sep.float().abs().max()) or 1.0
        assert_close(one.float() / scale, host64(sep.float()) / scale, tol, name)
