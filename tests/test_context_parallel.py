"""Host logic of the context-parallel scan, on CPU with the gloo backend.

Two and three gloo ranks each hold one time slice (of unequal lengths) of the
same seeded problem and run ``cp_scan_fwd`` / ``cp_scan_bwd`` with the five
library calls replaced by the double-precision oracle.  The concatenated
slices must equal the oracle's scan of the whole sequence: this checks the
rank order of the gathered maps, the forward and reverse composition ranges,
the summing of the final-state gradients and where the initial-state
gradient is returned.  The ESA layer itself is run the same way over a
gloo group (each rank projecting its own slice) against one layer over the
whole sequence.  The CUDA calls themselves are checked against the oracle in
the GPU tests.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleOps:
    """The library calls of the orchestration, evaluated by the oracle (float64, CPU)."""

    @staticmethod
    def _np(t):
        return None if t is None else t.detach().numpy()

    @staticmethod
    def scan_map(a, v, mode, workspace):
        import oracle
        P, S = oracle.scan_map(a.numpy(), v.numpy(), mode)
        return torch.from_numpy(P), torch.from_numpy(S), None

    @staticmethod
    def scan_bwd_map(a, v, q, dy, workspace, mode, E_init):
        import oracle
        P, S = oracle.scan_bwd_map(a.numpy(), v.numpy(), q.numpy(), dy.numpy(), mode,
                                   E_init=OracleOps._np(E_init))
        return torch.from_numpy(P), torch.from_numpy(S)

    @staticmethod
    def compose(P, S, x0, reverse):
        import oracle
        return torch.from_numpy(np.asarray(oracle.compose(P.numpy(), S.numpy(), OracleOps._np(x0), reverse)))

    @staticmethod
    def scan_fwd(a, v, q, mode, E_init, workspace):
        import oracle
        y, _ = oracle.scan_fwd(a.numpy(), v.numpy(), q.numpy(), mode, E_init=OracleOps._np(E_init))
        return torch.from_numpy(y), None

    @staticmethod
    def scan_bwd(a, v, q, dy, workspace, mode, E_init, dE_final, want_dE_init):
        import oracle
        out = oracle.scan_bwd(a.numpy(), v.numpy(), q.numpy(), dy.numpy(), mode, E_init=OracleOps._np(E_init),
                              dE_final=OracleOps._np(dE_final))
        return tuple(torch.from_numpy(x) for x in out)


def _problem(T, mode_seed):
    r = np.random.default_rng(100 + mode_seed)
    B, H, D = 2, 2, 4
    x = {k: r.normal(0.5 if k == "a" else 0.0, 1.0, (B, T, H, D)) for k in ("a", "v", "q", "dy")}
    x["E0"] = r.normal(0, 1, (B, H, D))
    # each rank's own gradient of the replicated final state; they are summed
    x["dEf"] = [r.normal(0, 1, (B, H, D)) for _ in range(4)]
    return x


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, cuts, mode, out):
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from gated_linear_recurrence_b200 import context_parallel as cp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        x = _problem(cuts[-1], mode)
        s = slice(cuts[rank], cuts[rank + 1])
        a, v, q, dy = (torch.from_numpy(np.ascontiguousarray(x[k][:, s])) for k in ("a", "v", "q", "dy"))
        E0 = torch.from_numpy(x["E0"])
        y, Ef, E_in, ws = cp.cp_scan_fwd(a, v, q, mode, E0, ops=OracleOps)
        da, dv, dq, dE0 = cp.cp_scan_bwd(a, v, q, dy, ws, E_in, mode, torch.from_numpy(x["dEf"][rank]),
                                         ops=OracleOps)
        out[rank] = {"y": y.numpy(), "E_final": Ef.numpy(), "da": da.numpy(), "dv": dv.numpy(),
                     "dq": dq.numpy(), "dE_init": None if dE0 is None else dE0.numpy()}
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts,mode", [([0, 17, 40], 1), ([0, 9, 10, 31], 0), ([0, 0, 12, 30], 1)])
def test_gloo_ranks_match_the_whole_sequence(cuts, mode):
    import oracle
    world = len(cuts) - 1
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, cuts, mode, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
            assert p.exitcode == 0
        res = dict(out)
    x = _problem(cuts[-1], mode)
    dEf = sum(x["dEf"][r] for r in range(world))
    y, Ef = oracle.scan_fwd(x["a"], x["v"], x["q"], mode, E_init=x["E0"])
    da, dv, dq, dE0 = oracle.scan_bwd(x["a"], x["v"], x["q"], x["dy"], mode, E_init=x["E0"], dE_final=dEf)
    for k, ref in (("y", y), ("da", da), ("dv", dv), ("dq", dq)):
        got = np.concatenate([res[r][k] for r in range(world)], axis=1)
        np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12, err_msg=k)
    for r in range(world):
        np.testing.assert_allclose(res[r]["E_final"], Ef, rtol=1e-12, atol=1e-13)
        if r == 0:
            np.testing.assert_allclose(res[r]["dE_init"], dE0, rtol=1e-10, atol=1e-12)
        else:
            assert res[r]["dE_init"] is None


def _layer_problem(T):
    from gated_linear_recurrence_b200 import ESA
    torch.manual_seed(21)
    lay = ESA(16, 2, mode="controlled", bias=True, dtype=torch.float64)
    x = torch.randn(2, T, 16, dtype=torch.float64)
    E0 = torch.randn(2, 2, 8, dtype=torch.float64) * 0.3
    g = torch.randn(2, T, 16, dtype=torch.float64)
    u = torch.randn(2, 2, 8, dtype=torch.float64)
    return lay, x, E0, g, u


def _layer_worker(rank, world, port, cuts, out):
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from gated_linear_recurrence_b200 import context_parallel as cp
    for name in ("scan_map", "scan_bwd_map", "compose", "scan_fwd", "scan_bwd"):   # the oracle stands in
        setattr(cp.LibraryOps, name, staticmethod(getattr(OracleOps, name)))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lay, x, E0, g, u = _layer_problem(cuts[-1])
        lay.cp_group = dist.group.WORLD
        s = slice(cuts[rank], cuts[rank + 1])
        xs = x[:, s].clone().requires_grad_(True)
        E0r = E0.clone().requires_grad_(True)
        o, E = lay(xs, state=E0r, return_state=True)
        loss = (o * g[:, s]).sum()
        if rank == 0:   # the final state is replicated: its loss term is counted once
            loss = loss + (E.double() * u).sum()
        loss.backward()
        grads = [p.grad.clone() for p in lay.parameters()]
        for gr in grads:   # the slices' weight gradients add up (what data parallelism would all-reduce)
            dist.all_reduce(gr)
        out[rank] = {"out": o.detach().numpy(), "E": E.detach().double().numpy(), "dx": xs.grad.numpy(),
                     "dE0": E0r.grad.numpy(), "dW": [gr.numpy() for gr in grads]}
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [[0, 13, 29], [0, 5, 6, 20]])
def test_layer_over_a_gloo_group_matches_the_whole_sequence(cuts, monkeypatch):
    """The ESA layer with a context-parallel group: each rank projects its
    slice, the scan crosses the slices, and the concatenated outputs and
    input gradients, the initial-state gradient (sum over ranks) and the
    summed weight gradients equal one layer over the whole sequence."""
    from gated_linear_recurrence_b200 import esa
    from tests.test_layer_host import _oracle_scan_bwd, _oracle_scan_fwd
    world = len(cuts) - 1
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_layer_worker, args=(r, world, port, cuts, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=180)
            assert p.exitcode == 0
        res = dict(out)

    monkeypatch.setattr(esa, "esa_scan_fwd", _oracle_scan_fwd)
    monkeypatch.setattr(esa, "esa_scan_bwd", _oracle_scan_bwd)
    lay, x, E0, g, u = _layer_problem(cuts[-1])
    x = x.requires_grad_(True)
    E0 = E0.requires_grad_(True)
    o, E = lay(x, state=E0, return_state=True)
    ((o * g).sum() + (E.double() * u).sum()).backward()
    tol = dict(rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(np.concatenate([res[r]["out"] for r in range(world)], axis=1), o.detach().numpy(),
                               **tol)
    np.testing.assert_allclose(np.concatenate([res[r]["dx"] for r in range(world)], axis=1), x.grad.numpy(), **tol)
    for r in range(world):
        np.testing.assert_allclose(res[r]["E"], E.detach().double().numpy(), **tol)
    np.testing.assert_allclose(sum(res[r]["dE0"] for r in range(world)), E0.grad.numpy(), **tol)
    for got, p in zip(res[0]["dW"], lay.parameters()):
        np.testing.assert_allclose(got, p.grad.numpy(), **tol)
