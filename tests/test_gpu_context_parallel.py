"""GPU parity of the segment-map calls and of a sequence split along time.

* ``esa_scan_map`` and ``esa_scan_bwd_map`` against the oracle's maps
  (P = product of the gates, S = the scan from a zero state / gradient), on
  ragged lengths, partial channel tiles, every tile width and an empty slice;
  the backward map leaves the forward's chunk states for ``esa_scan_bwd``.
* ``esa_compose`` against the oracle's composition, both orders, aliasing.
* The slices of one sequence run one after another on one device through the
  same orchestration functions the multi-rank path uses (no collective: the
  maps are stacked in slice order), compared with the oracle's scan of the
  whole sequence.
* The ESA layer with a one-rank NCCL group against the layer without one.
"""
import pytest
import torch

import oracle
from gated_linear_recurrence_b200 import ESA, context_parallel as cp, esa, inputs
from tests._parity import DT, TOL, assert_close, host64, oracle_fwd_bwd

pytestmark = pytest.mark.gpu

MAP_CASES = [
    (2, 300, 4, 32, 1, "f16"),
    (3, 1000, 2, 64, 0, "bf16"),
    (1, 97, 3, 8, 0, "f32"),
    (2, 129, 1, 128, 1, "f16"),
    (1, 200, 2, 256, 0, "bf16"),
    (2, 257, 5, 8, 1, "f16"),      # C = 40: one partial channel tile
    (2, 0, 2, 32, 1, "f16"),       # empty slice: the identity map
    (1, 4100, 1, 32, 1, "f32"),
]


def _ids(c):
    return f"B{c[0]}T{c[1]}H{c[2]}D{c[3]}m{c[4]}{c[5]}"


@pytest.mark.parametrize("case", MAP_CASES, ids=[_ids(c) for c in MAP_CASES])
def test_scan_map_matches_oracle(cuda_device, case):
    B, T, H, D, mode, dt = case
    x = inputs.make_scan_inputs(B, T, H, D, dt, 1.5, 40 + T)
    a, v = x["a"].to(cuda_device), x["v"].to(cuda_device)
    P, S, ws = esa.esa_scan_map(a, v, mode=mode)
    esa.esa_check(ws)
    P_r, S_r = oracle.scan_map(host64(a), host64(v), mode)
    tol = TOL[DT[dt]]
    assert_close(P, P_r, tol, "P")
    assert_close(S, S_r, tol, "S")


@pytest.mark.parametrize("case", MAP_CASES, ids=[_ids(c) for c in MAP_CASES])
def test_scan_bwd_map_matches_oracle_and_keeps_checkpoints(cuda_device, case):
    B, T, H, D, mode, dt = case
    x = inputs.make_scan_inputs(B, T, H, D, dt, 1.5, 60 + T)
    xd = {k: x[k].to(cuda_device) for k in ("a", "v", "q", "dy")}
    E0 = inputs.make_state(B, H, D, seed=61, scale=0.8).to(cuda_device)
    dEf = inputs.make_state(B, H, D, seed=62).to(cuda_device)
    _, _, ws = esa.esa_scan_fwd(xd["a"], xd["v"], xd["q"], mode=mode, E_init=E0)
    P, S = esa.esa_scan_bwd_map(xd["a"], xd["v"], xd["q"], xd["dy"], ws, mode=mode, E_init=E0)
    # the forward's chunk states are still there for the full backward
    da, dv, dq, dE0 = esa.esa_scan_bwd(xd["a"], xd["v"], xd["q"], xd["dy"], ws, mode=mode, E_init=E0,
                                       dE_final=dEf)
    esa.esa_check(ws)
    tol = TOL[DT[dt]]
    P_r, S_r = oracle.scan_bwd_map(*(host64(xd[k]) for k in ("a", "v", "q", "dy")), mode, E_init=host64(E0))
    assert_close(P, P_r, tol, "P")
    assert_close(S, S_r, tol, "S")
    ref = oracle_fwd_bwd(xd, mode, E_init=E0, dE_final=dEf)
    for k, g in (("da", da), ("dv", dv), ("dq", dq), ("dE_init", dE0)):
        assert_close(g, ref[k], tol, k)
    # the map reproduces the backward's own initial-state gradient
    assert_close(P * dEf + S, ref["dE_init"], tol, "P dE_final + S")


@pytest.mark.parametrize("n,reverse,with_x0", [(0, False, True), (1, False, False), (3, False, True),
                                               (3, True, True), (5, True, False)])
def test_compose_matches_oracle(cuda_device, n, reverse, with_x0):
    g = torch.Generator().manual_seed(70 + n)
    shape = (3, 4, 32)
    P = torch.rand((n,) + shape, generator=g) * 1.2
    S = torch.randn((n,) + shape, generator=g)
    x0 = torch.randn(shape, generator=g) if with_x0 else None
    out = esa.esa_compose(P.to(cuda_device), S.to(cuda_device),
                          x0=None if x0 is None else x0.to(cuda_device), reverse=reverse)
    ref = oracle.compose(P.double().numpy(), S.double().numpy(),
                         None if x0 is None else x0.double().numpy(), reverse)
    assert_close(out, ref, 1e-6, "compose")
    if with_x0:   # in place: x0 is also the output
        x = x0.to(cuda_device)
        esa.esa_compose(P.to(cuda_device), S.to(cuda_device), x0=x, reverse=reverse, out=x)
        assert torch.equal(x, out)


SPLIT_CASES = [
    (2, 700, 4, 32, 1, "f16", [0, 256, 300, 700]),
    (2, 1000, 2, 64, 0, "bf16", [0, 129, 1000]),
    (1, 333, 3, 8, 1, "f32", [0, 0, 100, 101, 333]),
    (2, 520, 1, 128, 0, "f16", [0, 200, 400, 520]),
]


@pytest.mark.parametrize("case", SPLIT_CASES, ids=[_ids(c) + f"-{len(c[6]) - 1}sl" for c in SPLIT_CASES])
def test_slices_in_sequence_match_whole_sequence(cuda_device, case):
    B, T, H, D, mode, dt, cuts = case
    x = inputs.make_scan_inputs(B, T, H, D, dt, 1.0, 80 + T)
    xd = {k: x[k].to(cuda_device) for k in ("a", "v", "q", "dy")}
    E0 = inputs.make_state(B, H, D, seed=81, scale=0.6).to(cuda_device)
    dEf = inputs.make_state(B, H, D, seed=82).to(cuda_device)
    n = len(cuts) - 1
    sl = [{k: xd[k][:, cuts[r]:cuts[r + 1]].contiguous() for k in xd} for r in range(n)]
    # forward: every slice's map, then each slice from its boundary state
    fmaps = [cp.forward_map(s["a"], s["v"], mode) for s in sl]
    P_all = torch.stack([m[0] for m in fmaps])
    S_all = torch.stack([m[1] for m in fmaps])
    ys, E_ins, wss = [], [], []
    for r, s in enumerate(sl):
        E_in, E_final = cp.boundary_state(P_all, S_all, r, E0)
        y, _, ws = esa.esa_scan_fwd(s["a"], s["v"], s["q"], mode=mode, E_init=E_in, workspace=fmaps[r][2])
        ys.append(y)
        E_ins.append(E_in)
        wss.append(ws)
    # backward: every slice's reverse map, then each slice with its boundary gradient
    bmaps = [cp.backward_map(s["a"], s["v"], s["q"], s["dy"], wss[r], mode, E_ins[r]) for r, s in enumerate(sl)]
    Pb = torch.stack([m[0] for m in bmaps])
    Sb = torch.stack([m[1] for m in bmaps])
    grads = []
    for r, s in enumerate(sl):
        dE_out = cp.boundary_grad(Pb, Sb, r, dEf)
        grads.append(esa.esa_scan_bwd(s["a"], s["v"], s["q"], s["dy"], wss[r], mode=mode, E_init=E_ins[r],
                                      dE_final=dE_out))
    for ws in wss:
        esa.esa_check(ws)
    ref = oracle_fwd_bwd(xd, mode, E_init=E0, dE_final=dEf)
    tol = TOL[DT[dt]]
    assert_close(torch.cat(ys, dim=1), ref["y"], tol, "y")
    assert_close(E_final, ref["E_final"], tol, "E_final")
    for i, k in enumerate(("da", "dv", "dq")):
        assert_close(torch.cat([g[i] for g in grads], dim=1), ref[k], tol, k)
    assert_close(grads[0][3], ref["dE_init"], tol, "dE_init")


def test_layer_with_one_rank_group_matches_plain_layer(cuda_device):
    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group is already initialised in this process")
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1)
    try:
        torch.manual_seed(9)
        B, T, C, H = 2, 300, 128, 4
        plain = ESA(C, H, mode="controlled", scan_dtype=torch.float16, device=cuda_device)
        cpl = ESA(C, H, mode="controlled", scan_dtype=torch.float16, device=cuda_device,
                  cp_group=dist.group.WORLD)
        cpl.load_state_dict(plain.state_dict())
        x = torch.randn(B, T, C, device=cuda_device)
        E0 = torch.randn(B, H, C // H, device=cuda_device) * 0.3
        g = torch.randn(B, T, C, device=cuda_device)
        outs = []
        for layer in (plain, cpl):
            xi = x.clone().requires_grad_(True)
            Ei = E0.clone().requires_grad_(True)
            out, E = layer(xi, state=Ei, return_state=True)
            ((out * g).sum() + E.sum()).backward()
            outs.append((out.detach(), E.detach(), xi.grad, Ei.grad, layer.W_A.weight.grad))
        tol = TOL[torch.float16]
        for name, p_, c_ in zip(("out", "E_final", "dx", "dE0", "dW_A"), outs[0], outs[1]):
            assert_close(c_, host64(p_), tol, name)
    finally:
        dist.destroy_process_group()
