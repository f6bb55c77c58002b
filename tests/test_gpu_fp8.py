"""GPU parity of the fp8 (e4m3) input mode of the forward scans.

a, v, q are e4m3 (torch.float8_e4m3fn); the state and the arithmetic are
fp32 and y is fp16.  The oracle scans the same e4m3 values widened to fp64,
so the comparison is the fp16 one (2e-3 (1 + |ref|)).  The backward takes e4m3 dy too and returns fp16 gradients;
the decode step takes e4m3 inputs and returns fp16; the fused forward does
not take fp8 inputs and must say so.
"""
import pytest
import torch

import oracle
from gated_linear_recurrence_b200 import esa, inputs
from tests._parity import TOL, assert_close, host64

pytestmark = pytest.mark.gpu

F8 = torch.float8_e4m3fn
CASES = [
    (2, 300, 4, 32, 1),
    (3, 1000, 2, 64, 0),
    (1, 97, 8, 8, 1),
    (2, 257, 5, 16, 0),    # C = 80: a partial channel tile
    (1, 129, 1, 128, 1),   # 128-channel tiles
    (1, 200, 1, 256, 0),   # 256-channel tiles
    (2, 4100, 4, 32, 1),
]


def _fp8_inputs(B, T, H, D, seed, device):
    x = inputs.make_scan_inputs(B, T, H, D, "f32", 1.5, seed, with_dy=False)
    return {k: x[k].to(F8).to(device) for k in ("a", "v", "q")}


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}T{c[1]}H{c[2]}D{c[3]}m{c[4]}" for c in CASES])
def test_fp8_forward_matches_oracle(cuda_device, case):
    B, T, H, D, mode = case
    x = _fp8_inputs(B, T, H, D, 400 + T, cuda_device)
    E0 = inputs.make_state(B, H, D, seed=401, scale=0.5).to(cuda_device)
    y, Ef, ws = esa.esa_scan_fwd(x["a"], x["v"], x["q"], mode=mode, E_init=E0)
    esa.esa_check(ws)
    assert y.dtype == torch.float16
    f64 = lambda t: t.to(torch.float32).to("cpu", torch.float64).numpy()  # noqa: E731
    y_r, Ef_r = oracle.scan_fwd(f64(x["a"]), f64(x["v"]), f64(x["q"]), mode, E_init=host64(E0))
    assert_close(y, y_r, TOL[torch.float16], "y")
    assert_close(Ef, Ef_r, TOL[torch.float16], "E_final")


def test_fp8_segment_map_matches_oracle(cuda_device):
    B, T, H, D = 2, 700, 4, 32
    x = _fp8_inputs(B, T, H, D, 410, cuda_device)
    P, S, ws = esa.esa_scan_map(x["a"], x["v"], mode=1)
    esa.esa_check(ws)
    f64 = lambda t: t.to(torch.float32).to("cpu", torch.float64).numpy()  # noqa: E731
    P_r, S_r = oracle.scan_map(f64(x["a"]), f64(x["v"]), 1)
    assert_close(P, P_r, TOL[torch.float16], "P")
    assert_close(S, S_r, TOL[torch.float16], "S")


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}T{c[1]}H{c[2]}D{c[3]}m{c[4]}" for c in CASES])
def test_fp8_backward_matches_oracle(cuda_device, case):
    """e4m3 a, v, q and upstream gradient dy; fp16 gradients."""
    B, T, H, D, mode = case
    x = inputs.make_scan_inputs(B, T, H, D, "f32", 1.5, 430 + T)
    xd = {k: x[k].to(F8).to(cuda_device) for k in ("a", "v", "q", "dy")}
    E0 = inputs.make_state(B, H, D, seed=431, scale=0.5).to(cuda_device)
    dEf = inputs.make_state(B, H, D, seed=432).to(cuda_device)
    _, _, ws = esa.esa_scan_fwd(xd["a"], xd["v"], xd["q"], mode=mode, E_init=E0)
    da, dv, dq, dE0 = esa.esa_scan_bwd(xd["a"], xd["v"], xd["q"], xd["dy"], ws, mode=mode, E_init=E0,
                                       dE_final=dEf)
    esa.esa_check(ws)
    assert da.dtype == dv.dtype == dq.dtype == torch.float16
    f64 = lambda t: t.to(torch.float32).to("cpu", torch.float64).numpy()  # noqa: E731
    ref = oracle.scan_bwd(*(f64(xd[k]) for k in ("a", "v", "q", "dy")), mode, E_init=host64(E0),
                          dE_final=host64(dEf))
    for name, g, r in zip(("da", "dv", "dq", "dE_init"), (da, dv, dq, dE0), ref):
        assert_close(g, r, TOL[torch.float16], name)


def test_fp8_decode_steps_match_oracle(cuda_device):
    B, H, D, n = 3, 4, 32, 8
    E = inputs.make_state(B, H, D, seed=440, scale=0.5).to(cuda_device)
    E_r = host64(E)
    f64 = lambda t: t.to(torch.float32).to("cpu", torch.float64).numpy()  # noqa: E731
    for i in range(n):
        st = inputs.make_step_inputs(B, H, D, "f32", 1.0, seed=441 + i)
        a, v, q = (st[k].to(F8).to(cuda_device) for k in ("a", "v", "q"))
        y = esa.esa_step(a, v, q, E, mode=i % 2)
        assert y.dtype == torch.float16
        y_r, E_r = oracle.step(f64(a), f64(v), f64(q), E_r, i % 2)
        assert_close(y, y_r, TOL[torch.float16], f"step{i}.y")
    assert_close(E, E_r, TOL[torch.float16], "E")


def test_fp8_is_refused_by_the_fused_forward(cuda_device):
    B, T, H, D = 1, 64, 2, 32
    xin = torch.zeros(B, T, 128, device=cuda_device).to(F8)
    W = torch.zeros(3 * H * D, 128, device=cuda_device).to(F8)
    with pytest.raises(esa.EsaError) as err:
        esa.esa_fused_fwd(xin, W, H)
    assert err.value.code == esa.ESA_ERR_UNSUPPORTED
