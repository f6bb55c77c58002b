"""The library's calls inside CUDA graphs.

The scans carry no per-call host state: tile tickets, completion counts and
the carry-word epoch live in the workspace and are reset or advanced by the
kernels themselves, so a captured forward + backward (or fused forward) can
be replayed any number of times.  Each replay here runs on new input values
copied into the captured buffers and is checked against the oracle; a
captured run of 16 decode steps is checked the same way.
"""
import pytest
import torch

import oracle
from gated_linear_recurrence_b200 import esa, inputs
from tests._parity import DT, TOL, assert_close, compare, host64, oracle_fwd_bwd

pytestmark = pytest.mark.gpu


def _capture(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()   # warm-up outside the capture (library set-up, allocator)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


@pytest.mark.parametrize("dt,mode", [("f16", 1), ("bf16", 0)])
def test_scan_fwd_bwd_replayed_from_a_graph(cuda_device, dt, mode):
    B, T, H, D = 2, 777, 4, 32
    bufs = {k: torch.empty(B, T, H, D, dtype=DT[dt], device=cuda_device) for k in ("a", "v", "q", "dy")}
    ws = esa.new_workspace(B, T, H, D, DT[dt], cuda_device)
    out = {k: torch.empty(B, T, H, D, dtype=DT[dt], device=cuda_device) for k in ("y", "da", "dv", "dq")}
    st = {k: torch.empty(B, H, D, dtype=torch.float32, device=cuda_device) for k in ("E_final", "dE_init")}

    def step():
        esa.esa_scan_fwd(bufs["a"], bufs["v"], bufs["q"], y=out["y"], E_final=st["E_final"], mode=mode, workspace=ws)
        esa.esa_scan_bwd(bufs["a"], bufs["v"], bufs["q"], bufs["dy"], ws, mode=mode, da=out["da"], dv=out["dv"],
                         dq=out["dq"], dE_init=st["dE_init"])

    for k in range(3):   # the first input set also serves the warm-up and capture
        x = inputs.make_scan_inputs(B, T, H, D, dt, 1.0 + k, 1000 + k)
        for n in bufs:
            bufs[n].copy_(x[n])
        if k == 0:
            g = _capture(step)
        g.replay()
        torch.cuda.synchronize()
        esa.esa_check(ws)
        gpu = {"y": out["y"], "E_final": st["E_final"], "da": out["da"], "dv": out["dv"], "dq": out["dq"],
               "dE_init": st["dE_init"]}
        compare(gpu, oracle_fwd_bwd(bufs, mode), TOL[DT[dt]], tuple(gpu), prefix=f"replay{k}.")
    del g


def test_fused_forward_replayed_from_a_graph(cuda_device):
    B, T, H, D, C_in = 2, 500, 4, 32, 128
    C = H * D
    x = torch.empty(B, T, C_in, dtype=torch.float16, device=cuda_device)
    W = torch.empty(3 * C, C_in, dtype=torch.float16, device=cuda_device)
    y = torch.empty(B, T, H, D, dtype=torch.float16, device=cuda_device)
    Ef = torch.empty(B, H, D, dtype=torch.float32, device=cuda_device)
    avq = tuple(torch.empty(B, T, H, D, dtype=torch.float16, device=cuda_device) for _ in range(3))
    ws = esa.new_workspace(B, T, H, D, torch.float16, cuda_device)

    def step():
        esa.esa_fused_fwd(x, W, H, mode=1, y=y, E_final=Ef, workspace=ws, avq=avq)

    for k in range(3):
        gen = torch.Generator().manual_seed(2000 + k)
        x.copy_(torch.randn(B, T, C_in, generator=gen).half())
        W.copy_((torch.randn(3 * C, C_in, generator=gen) / C_in ** 0.5).half())
        if k == 0:
            g = _capture(step)
        g.replay()
        torch.cuda.synchronize()
        esa.esa_check(ws)
        y_r, Ef_r = oracle.scan_fwd(*(host64(t) for t in avq), 1)
        assert_close(y, y_r, TOL[torch.float16], f"replay{k}.y")
        assert_close(Ef, Ef_r, TOL[torch.float16], f"replay{k}.E_final")
    del g


def test_decode_steps_replayed_from_a_graph(cuda_device):
    B, H, D, n = 3, 4, 32, 16
    steps = [inputs.make_step_inputs(B, H, D, "f16", 1.0, seed=3000 + i) for i in range(n)]
    dev_steps = [{k: s[k].to(cuda_device) for k in ("a", "v", "q")} for s in steps]
    E = torch.zeros(B, H, D, dtype=torch.float32, device=cuda_device)
    ys = [torch.empty(B, H, D, dtype=torch.float16, device=cuda_device) for _ in range(n)]

    def run():
        for s, yt in zip(dev_steps, ys):
            esa.esa_step(s["a"], s["v"], s["q"], E, y_t=yt, mode=0)

    g = _capture(run)
    E0 = inputs.make_state(B, H, D, seed=3100)
    E.copy_(E0)
    g.replay()
    torch.cuda.synchronize()
    E_r = host64(E0)
    for i, s in enumerate(steps):
        y_r, E_r = oracle.step(host64(s["a"]), host64(s["v"]), host64(s["q"]), E_r, 0)
        assert_close(ys[i], y_r, TOL[torch.float16], f"step{i}.y")
    assert_close(E, E_r, TOL[torch.float16], "E")
    del g
