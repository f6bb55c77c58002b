"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases span several chunks with a ragged tail, partial channel tiles,
every supported head dimension, both modes, the three I/O dtypes, non-zero
initial states and final-state gradients.  The five specified workloads run
at full size; where the oracle would take long, whole batch rows are sampled
and recomputed by the oracle one by one (every time step and channel of each
sampled row is compared).
"""
import numpy as np
import pytest
import torch

import oracle
from gated_linear_recurrence_b200 import esa, inputs
from tests._parity import DT, TOL, assert_close, compare, gpu_fwd_bwd, host64, oracle_fwd_bwd

pytestmark = pytest.mark.gpu

ALL = ("y", "E_final", "da", "dv", "dq", "dE_init")


def _inputs(B, T, H, D, dtype, a_mean, seed, dev):
    x = inputs.make_scan_inputs(B, T, H, D, dtype, a_mean, seed)
    return {k: x[k].to(dev) for k in ("a", "v", "q", "dy")}


SMALL = [
    # B, T, H, D, mode, dtype, a_mean, nonzero states
    (2, 1000, 4, 32, 1, "f16", 2.0, True),     # 16 chunks, ragged tail
    (1, 1, 4, 32, 0, "f16", 0.0, True),        # a single token
    (3, 200, 3, 32, 1, "f32", 1.0, True),      # C = 96 < one channel tile
    (2, 333, 5, 64, 0, "bf16", 0.0, False),    # C = 320: three channel tiles, last partial
    (1, 130, 2, 128, 1, "f16", 3.0, True),     # D = 128
    (2, 100, 2, 256, 0, "bf16", 0.5, True),    # D = 256 (256-channel tiles)
    (2, 257, 16, 8, 1, "f16", 2.0, False),     # D = 8: one lane per head
    (2, 90, 4, 16, 0, "f32", 0.0, True),       # D = 16
    (1, 20000, 1, 32, 1, "f16", 4.0, True),    # one long chain: 313 chunks of look-back
    (4, 64, 8, 64, 1, "bf16", 3.0, True),      # exactly one chunk
    (2, 129, 4, 32, 0, "f32", 0.0, False),     # fp32 chunks of 32 + 1
    (2, 3000, 2, 128, 1, "f16", 4.0, True),    # D = 128: 128-row forward tiles over 24 chunks, ragged tail
    (1, 2500, 1, 128, 0, "bf16", 2.0, True),   # D = 128 direct: one chain of 20 forward tiles
    (1, 1100, 1, 256, 1, "f16", 3.0, True),    # D = 256: 64-row tiles, one chain of 18 chunks
]


@pytest.mark.parametrize("case", SMALL, ids=[f"B{c[0]}T{c[1]}H{c[2]}D{c[3]}m{c[4]}{c[5]}" for c in SMALL])
def test_small_cases(cuda_device, case):
    B, T, H, D, mode, dt, a_mean, states = case
    x = _inputs(B, T, H, D, dt, a_mean, 100 + T, cuda_device)
    E0 = inputs.make_state(B, H, D, seed=7, scale=0.5).to(cuda_device) if states else None
    dEf = inputs.make_state(B, H, D, seed=8).to(cuda_device) if states else None
    gpu = gpu_fwd_bwd(x, mode, E0, dEf)
    ref = oracle_fwd_bwd(x, mode, E0, dEf)
    compare(gpu, ref, TOL[DT[dt]], ALL)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("mode", [0, 1])
def test_all_modes_and_dtypes(cuda_device, dt, mode):
    B, T, H, D = 2, 300, 4, 32
    x = _inputs(B, T, H, D, dt, 1.5 * mode, 5, cuda_device)
    E0 = inputs.make_state(B, H, D, seed=9).to(cuda_device)
    dEf = inputs.make_state(B, H, D, seed=10).to(cuda_device)
    compare(gpu_fwd_bwd(x, mode, E0, dEf), oracle_fwd_bwd(x, mode, E0, dEf), TOL[DT[dt]], ALL)


def test_deterministic(cuda_device):
    x = _inputs(4, 3000, 4, 32, "f16", 4.0, 3, cuda_device)
    r1 = gpu_fwd_bwd(x, 1)
    r2 = gpu_fwd_bwd(x, 1)
    for k in ALL:
        assert torch.equal(r1[k], r2[k]), k


def test_split_resume(cuda_device):
    x = _inputs(2, 700, 4, 32, "f16", 2.0, 4, cuda_device)
    full = gpu_fwd_bwd(x, 1, with_bwd=False)
    first = {k: v[:, :300].contiguous() for k, v in x.items()}
    second = {k: v[:, 300:].contiguous() for k, v in x.items()}
    r1 = gpu_fwd_bwd(first, 1, with_bwd=False)
    r2 = gpu_fwd_bwd(second, 1, E_init=r1["E_final"], with_bwd=False)
    tol = TOL[torch.float16]
    assert_close(torch.cat([r1["y"], r2["y"]], dim=1), host64(full["y"]), tol, "y")
    assert_close(r2["E_final"], host64(full["E_final"]), tol, "E_final")


def test_empty_inputs(cuda_device):
    B, H, D = 2, 4, 32
    a = torch.zeros(B, 0, H, D, dtype=torch.float16, device=cuda_device)
    E0 = inputs.make_state(B, H, D, seed=1).to(cuda_device)
    y, Ef, ws = esa.esa_scan_fwd(a, a, a, E_init=E0)
    assert y.shape == a.shape and torch.equal(Ef, E0)
    da, dv, dq, dE0 = esa.esa_scan_bwd(a, a, a, a, ws, dE_final=E0)
    assert torch.equal(dE0, E0)
    z = torch.zeros(0, 10, H, D, dtype=torch.float16, device=cuda_device)
    y, Ef, ws = esa.esa_scan_fwd(z, z, z)
    assert y.shape == z.shape and Ef.shape == (0, H, D)


def test_device_argument_errors(cuda_device):
    lib = esa.load_library()
    x = torch.zeros(2, 64, 4, 32, dtype=torch.float16, device=cuda_device)
    ws = esa.new_workspace(2, 64, 4, 32, torch.float16, cuda_device)
    import ctypes
    P = ctypes.c_void_p
    rc = lib.esa_scan_fwd(P(x.data_ptr() + 2), P(x.data_ptr()), P(x.data_ptr()), P(x.data_ptr()), None,
                          2, 63, 4, 32, 1, None, 1, P(ws.data_ptr()), ws.numel(), None)
    assert rc == esa.ESA_ERR_ALIGN
    rc = lib.esa_scan_fwd(P(x.data_ptr()), P(x.data_ptr()), P(x.data_ptr()), P(x.data_ptr()), None,
                          2, 64, 4, 32, 1, None, 1, P(ws.data_ptr()), ws.numel() - 1, None)
    assert rc == esa.ESA_ERR_WORKSPACE


# ---------------------------------------------------------------------------
# The five specified workloads.
# ---------------------------------------------------------------------------

def test_workload_direct_f32_B2_T128_fwd_bwd_and_128_steps(cuda_device):
    w = inputs.WORKLOADS["direct_f32_B2_T128_H4_D32"]
    x = _inputs(w.B, w.T, w.H, w.D, w.dtype, w.a_mean, w.seed, cuda_device)
    tol = TOL[torch.float32]
    gpu = gpu_fwd_bwd(x, w.mode)
    ref = oracle_fwd_bwd(x, w.mode)
    compare(gpu, ref, tol, ALL)
    # 128 esa_step calls reproduce the scan.
    E = torch.zeros(w.B, w.H, w.D, dtype=torch.float32, device=cuda_device)
    E_ref = np.zeros((w.B, w.H, w.D))
    for t in range(w.T):
        yt = esa.esa_step(x["a"][:, t].contiguous(), x["v"][:, t].contiguous(), x["q"][:, t].contiguous(), E,
                          mode=w.mode)
        yt_ref, E_ref = oracle.step(host64(x["a"][:, t]), host64(x["v"][:, t]), host64(x["q"][:, t]), E_ref,
                                    w.mode)
        assert_close(yt, yt_ref, tol, f"step y[{t}]")
        assert_close(yt, ref["y"][:, t], tol, f"step y[{t}] vs scan")
    assert_close(E, E_ref, tol, "step E")
    assert_close(E, ref["E_final"], tol, "step E vs scan E_final")


def test_workload_controlled_f16_B16_T1024_fwd(cuda_device):
    w = inputs.WORKLOADS["controlled_f16_B16_T1024_H4_D32"]
    x = _inputs(w.B, w.T, w.H, w.D, w.dtype, w.a_mean, w.seed, cuda_device)
    gpu = gpu_fwd_bwd(x, w.mode, with_bwd=False)
    ref = oracle_fwd_bwd(x, w.mode, with_bwd=False)
    compare(gpu, ref, TOL[torch.float16], ("y", "E_final"))


def _full_size(w, dev):
    x = inputs.make_scan_inputs(w.B, w.T, w.H, w.D, w.dtype, w.a_mean, w.seed, device=dev)
    return {k: x[k] for k in ("a", "v", "q", "dy")}


@pytest.mark.parametrize("name,rows", [
    ("controlled_bf16_B64_T4096_H8_D64", [0, 21, 63]),
    ("controlled_f16_B64_T65536_H4_D32", [0, 40, 63]),
])
def test_workload_full_size_sampled_rows(cuda_device, name, rows):
    w = inputs.WORKLOADS[name]
    x = _full_size(w, cuda_device)
    gpu = gpu_fwd_bwd(x, w.mode)
    tol = TOL[DT[w.dtype]]
    for b in rows:
        sel = slice(b, b + 1)
        ref = oracle_fwd_bwd(x, w.mode, rows=sel)
        compare(gpu, ref, tol, ALL, rows=sel, prefix=f"row{b}.")
    del gpu, x
    torch.cuda.empty_cache()


def test_workload_prefill_then_256_decode_steps(cuda_device):
    w = inputs.WORKLOADS["direct_f16_B64_H4_D32_prefill_decode"]
    tol = TOL[torch.float16]
    for T in w.prompts:
        g = torch.Generator().manual_seed(w.seed)
        x = inputs.make_scan_inputs(w.B, T, w.H, w.D, w.dtype, w.a_mean, generator=g, with_dy=False)
        steps = [inputs.make_step_inputs(w.B, w.H, w.D, w.dtype, w.a_mean, generator=g) for _ in range(w.steps)]
        xd = {k: x[k].to(cuda_device) for k in ("a", "v", "q")}
        y, E, _ = esa.esa_scan_fwd(xd["a"], xd["v"], xd["q"], mode=w.mode)
        ys = []
        for s in steps:
            ys.append(esa.esa_step(s["a"].to(cuda_device), s["v"].to(cuda_device), s["q"].to(cuda_device), E,
                                   mode=w.mode))
        # Oracle: one scan over prompt + generated tokens.
        cat = {k: torch.cat([x[k], torch.stack([s[k] for s in steps], dim=1)], dim=1) for k in ("a", "v", "q")}
        y_ref, E_ref = oracle.scan_fwd(host64(cat["a"]), host64(cat["v"]), host64(cat["q"]), w.mode)
        assert_close(y, y_ref[:, :T], tol, f"prefill T={T} y")
        assert_close(torch.stack(ys, dim=1), y_ref[:, T:], tol, f"decode after T={T} y")
        assert_close(E, E_ref, tol, f"decode after T={T} E")


def test_prepared_step_matches_esa_step_and_the_oracle(cuda_device):
    """PreparedStep (arguments resolved once) is the same C call as esa_step:
    bitwise-equal outputs and state, and both match the oracle's step."""
    B, H, D = 8, 4, 32
    g = torch.Generator().manual_seed(77)
    E0 = inputs.make_state(B, H, D, seed=78).to(cuda_device)
    E1, E2 = E0.clone(), E0.clone()
    E_ref = host64(E0)
    bufs = {k: torch.empty(B, H, D, dtype=torch.float16, device=cuda_device) for k in ("a", "v", "q")}
    step = esa.PreparedStep(bufs["a"], bufs["v"], bufs["q"], E2, mode=esa.CONTROLLED)
    for t in range(5):
        s = inputs.make_step_inputs(B, H, D, "f16", 1.0, generator=g)
        for k in ("a", "v", "q"):
            bufs[k].copy_(s[k])
        y1 = esa.esa_step(bufs["a"], bufs["v"], bufs["q"], E1, mode=esa.CONTROLLED)
        y2 = step()
        torch.cuda.synchronize()
        assert torch.equal(y1, y2) and torch.equal(E1, E2), t
        y_ref, E_ref = oracle.step(host64(s["a"]), host64(s["v"]), host64(s["q"]), E_ref, esa.CONTROLLED)
        assert_close(y2, y_ref, TOL[torch.float16], f"prepared y[{t}]")
        assert_close(E2, E_ref, TOL[torch.float16], f"prepared E[{t}]")
