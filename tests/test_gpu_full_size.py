"""Parity of the widened calls at the benchmark workload's full size.

Workload: controlled mode, B = 64, T = 65536, H = 4, D = 32 (C = 128), gate
logits ~ N(4, 1), v, q, dy ~ N(0, 1), the sizes the benchmark times.  Whole
batch rows are sampled and recomputed by the oracle one by one (every step
and channel of a sampled row is compared):

* fp8 (e4m3) inputs -- the workload's values rounded to e4m3 -- through the
  forward and the backward;
* the fused projection + scan forward with C_in = 128: the sampled rows'
  projections against their float64 products, then the scan of exactly those
  projections against the oracle's;
* the sequence split in 8 time slices of 8192 steps, run one after another on
  one device through the context-parallel functions, against the oracle's
  scan of the whole sequence.
"""
import pytest
import torch

import oracle
from gated_linear_recurrence_b200 import context_parallel as cp, esa, inputs
from tests._parity import DT, TOL, assert_close, compare, host64, oracle_fwd_bwd
from tests.test_gpu_fused import _check_projections

pytestmark = pytest.mark.gpu

W = inputs.WORKLOADS["controlled_f16_B64_T65536_H4_D32"]
ROWS = [0, 37, 63]
GRADS = ("da", "dv", "dq", "dE_init")


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _workload_inputs(dev):
    x = inputs.make_scan_inputs(W.B, W.T, W.H, W.D, W.dtype, W.a_mean, W.seed, device=dev)
    return {k: x[k] for k in ("a", "v", "q", "dy")}


def test_fp8_forward_backward_full_size_sampled_rows(cuda_device):
    x8 = {k: t.to(torch.float8_e4m3fn) for k, t in _workload_inputs(cuda_device).items()}
    _free()
    y, Ef, ws = esa.esa_scan_fwd(x8["a"], x8["v"], x8["q"], mode=W.mode)
    da, dv, dq, dE0 = esa.esa_scan_bwd(x8["a"], x8["v"], x8["q"], x8["dy"], ws, mode=W.mode)
    esa.esa_check(ws)
    gpu = {"y": y, "E_final": Ef, "da": da, "dv": dv, "dq": dq, "dE_init": dE0}
    for b in ROWS:
        sel = slice(b, b + 1)
        widened = {k: t[sel].float() for k, t in x8.items()}   # the e4m3 values, exactly
        ref = oracle_fwd_bwd(widened, W.mode)
        compare(gpu, ref, TOL[torch.float16], ("y", "E_final") + GRADS, rows=sel, prefix=f"row{b}.")
    del gpu, x8, y, da, dv, dq
    _free()


def test_fused_forward_full_size_sampled_rows(cuda_device):
    C = W.H * W.D
    C_in = C
    g = torch.Generator(device=cuda_device).manual_seed(W.seed + 11)
    x = torch.randn(W.B, W.T, C_in, generator=g, device=cuda_device).half()
    Wt = (torch.randn(3 * C, C_in, generator=g, device=cuda_device) / C_in ** 0.5).half()
    y, Ef, ws, avq = esa.esa_fused_fwd(x, Wt, W.H, mode=W.mode, want_avq=True)
    esa.esa_check(ws)
    tol = TOL[torch.float16]
    for b in ROWS:
        sel = slice(b, b + 1)
        _check_projections(x[sel], Wt, [t[sel] for t in avq], C, torch.float16)
        y_r, Ef_r = oracle.scan_fwd(*(host64(t[sel]) for t in avq), W.mode)
        assert_close(y[sel], y_r, tol, f"row{b}.y")
        assert_close(Ef[sel], Ef_r, tol, f"row{b}.E_final")
    del x, y, avq
    _free()


def test_context_parallel_full_size_eight_slices_sampled_rows(cuda_device):
    xd = _workload_inputs(cuda_device)
    n = 8
    Tr = W.T // n
    E0 = inputs.make_state(W.B, W.H, W.D, seed=W.seed + 20, scale=0.5).to(cuda_device)
    dEf = inputs.make_state(W.B, W.H, W.D, seed=W.seed + 21).to(cuda_device)
    ws = [esa.new_workspace(W.B, Tr, W.H, W.D, xd["a"].dtype, cuda_device) for _ in range(n)]
    y = torch.empty_like(xd["a"])
    grads = {k: torch.empty_like(xd["a"]) for k in ("da", "dv", "dq")}

    def piece(k, r):
        return xd[k][:, r * Tr:(r + 1) * Tr].contiguous()

    fmaps = [cp.forward_map(piece("a", r), piece("v", r), W.mode, workspace=ws[r]) for r in range(n)]
    P_all = torch.stack([m[0] for m in fmaps])
    S_all = torch.stack([m[1] for m in fmaps])
    E_ins = []
    for r in range(n):
        E_in, E_final = cp.boundary_state(P_all, S_all, r, E0)
        yr, _, _ = esa.esa_scan_fwd(piece("a", r), piece("v", r), piece("q", r), mode=W.mode, E_init=E_in,
                                    workspace=ws[r])
        y[:, r * Tr:(r + 1) * Tr] = yr
        E_ins.append(E_in)
    bmaps = [cp.backward_map(piece("a", r), piece("v", r), piece("q", r), piece("dy", r), ws[r], W.mode, E_ins[r])
             for r in range(n)]
    Pb = torch.stack([m[0] for m in bmaps])
    Sb = torch.stack([m[1] for m in bmaps])
    dE_init = None
    for r in range(n):
        dE_out = cp.boundary_grad(Pb, Sb, r, dEf)
        da, dv, dq, dE0 = esa.esa_scan_bwd(piece("a", r), piece("v", r), piece("q", r), piece("dy", r), ws[r],
                                           mode=W.mode, E_init=E_ins[r], dE_final=dE_out)
        for k, t in zip(("da", "dv", "dq"), (da, dv, dq)):
            grads[k][:, r * Tr:(r + 1) * Tr] = t
        if r == 0:
            dE_init = dE0
    for w_ in ws:
        esa.esa_check(w_)
    gpu = {"y": y, "E_final": E_final, "dE_init": dE_init, **grads}
    tol = TOL[DT[W.dtype]]
    for b in ROWS:
        sel = slice(b, b + 1)
        ref = oracle_fwd_bwd(xd, W.mode, E_init=E0, dE_final=dEf, rows=sel)
        compare(gpu, ref, tol, ("y", "E_final") + GRADS, rows=sel, prefix=f"row{b}.")
    del gpu, xd, y, grads, ws
    _free()
