"""Context parallelism: one sequence split along time over the ranks of a group.

Rank r holds the r-th time slice of every sequence (``[B, T_r, H, D]``
contiguous, slices in rank order).  The recurrence of every channel is affine
in the state entering a slice (the associative state composition of the
mlbricks-web.pages.dev/esa page, panel "Long-context throughput"), so one
exchange of 2 B C floats per rank replaces waiting for the earlier slices:

forward
  1. ``esa_scan_map``: the slice's map ``E_end = P E_start + S``.
  2. all-gather of ``(P, S)`` from every rank.
  3. ``esa_compose``: the state entering slice r is the maps of slices
     ``0..r-1`` applied to ``E_init``; the global final state is all of them.
  4. ``esa_scan_fwd`` of the slice from that state.

backward (the same in reverse)
  1. ``esa_scan_bwd_map``: ``dE_start = P dE_end + S`` for the slice.
  2. all-gather of ``(P, S)`` and of each rank's gradient of the final state.
  3. ``esa_compose`` (reverse): the gradient leaving slice r is the maps of
     slices ``N-1..r+1`` applied to the summed final-state gradient.
  4. ``esa_scan_bwd`` of the slice with that gradient.

Each step runs in the CUDA library; this module only orders the calls and the
collective.  The steps are separate functions so that the same code can run
the slices of one device one after another (no collective), and so that the
host logic can be exercised with other implementations of the five library
calls (``ops``).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import esa as _esa

__all__ = ["LibraryOps", "forward_map", "boundary_state", "backward_map", "boundary_grad",
           "cp_scan_fwd", "cp_scan_bwd", "cp_esa_scan", "gather_stacked"]


class LibraryOps:
    """The five library calls the orchestration uses (the CUDA library)."""

    @staticmethod
    def scan_map(a, v, mode, workspace):
        return _esa.esa_scan_map(a, v, mode=mode, workspace=workspace)

    @staticmethod
    def scan_bwd_map(a, v, q, dy, workspace, mode, E_init):
        return _esa.esa_scan_bwd_map(a, v, q, dy, workspace, mode=mode, E_init=E_init)

    @staticmethod
    def compose(P, S, x0, reverse):
        return _esa.esa_compose(P, S, x0=x0, reverse=reverse)

    @staticmethod
    def scan_fwd(a, v, q, mode, E_init, workspace):
        y, _, ws = _esa.esa_scan_fwd(a, v, q, mode=mode, E_init=E_init, workspace=workspace,
                                     want_E_final=False)
        return y, ws

    @staticmethod
    def scan_bwd(a, v, q, dy, workspace, mode, E_init, dE_final, want_dE_init):
        return _esa.esa_scan_bwd(a, v, q, dy, workspace, mode=mode, E_init=E_init, dE_final=dE_final,
                                 want_dE_init=want_dE_init)


def gather_stacked(t, group=None):
    """All-gather ``t`` from every rank of ``group``: ``[world, *t.shape]``
    in rank order."""
    world = dist.get_world_size(group)
    t = t.contiguous()
    out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, t, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), t, group=group)
    return out


def forward_map(a, v, mode, workspace=None, ops=LibraryOps):
    """Step 1 of the forward: ``(P, S, workspace)`` of this slice."""
    return ops.scan_map(a, v, mode, workspace)


def boundary_state(P_all, S_all, rank, E_init=None, ops=LibraryOps):
    """Step 3 of the forward, from the gathered maps ``[world, B, H, D]``:
    ``(E_in, E_final)`` -- the state entering slice ``rank`` and the state
    after the last slice (identical on every rank)."""
    P_all, S_all = P_all.contiguous(), S_all.contiguous()
    E_in = ops.compose(P_all[:rank], S_all[:rank], E_init, False)
    E_final = ops.compose(P_all, S_all, E_init, False)
    return E_in, E_final


def backward_map(a, v, q, dy, workspace, mode, E_in, ops=LibraryOps):
    """Step 1 of the backward: ``(P, S)`` of this slice's reverse map.
    ``workspace`` is the one this slice's forward scan wrote."""
    return ops.scan_bwd_map(a, v, q, dy, workspace, mode, E_in)


def boundary_grad(P_all, S_all, rank, dE_final=None, ops=LibraryOps):
    """Step 3 of the backward: the gradient of the state leaving slice
    ``rank``: the reverse maps of the later slices applied to ``dE_final``."""
    P_all, S_all = P_all.contiguous(), S_all.contiguous()
    return ops.compose(P_all[rank + 1:], S_all[rank + 1:], dE_final, True)


def cp_scan_fwd(a, v, q, mode=_esa.CONTROLLED, E_init=None, group=None, ops=LibraryOps, workspace=None):
    """Forward scan of this rank's slice.  ``E_init`` is the state before the
    first slice (the same on every rank, or None); ``workspace`` is reused
    when given (allocated otherwise).

    Returns ``(y, E_final, E_in, workspace)``: this slice's readout, the state
    after the last slice, the state entering this slice and the workspace
    (keep both for :func:`cp_scan_bwd`).
    """
    rank = dist.get_rank(group)
    P, S, ws = forward_map(a, v, mode, workspace, ops)
    maps = gather_stacked(torch.stack([P, S]), group)
    E_in, E_final = boundary_state(maps[:, 0], maps[:, 1], rank, E_init, ops)
    y, ws = ops.scan_fwd(a, v, q, mode, E_in, ws)
    return y, E_final, E_in, ws


def cp_scan_bwd(a, v, q, dy, workspace, E_in, mode=_esa.CONTROLLED, dE_final=None, group=None,
                ops=LibraryOps):
    """Backward scan of this rank's slice.

    ``dE_final`` is this rank's gradient of the (replicated) final state, or
    None; the gradients of all ranks are summed.  Returns ``(da, dv, dq,
    dE_init)``; ``dE_init`` (the gradient of ``E_init``) is the full gradient
    on rank 0 and None on the other ranks, so that a sum over ranks counts it
    once.
    """
    rank = dist.get_rank(group)
    P, S = backward_map(a, v, q, dy, workspace, mode, E_in, ops)
    dEf = torch.zeros_like(P) if dE_final is None else dE_final.to(P.dtype)
    parts = gather_stacked(torch.stack([P, S, dEf]), group)
    dEf_sum = parts[:, 2].sum(dim=0)
    dE_out = boundary_grad(parts[:, 0], parts[:, 1], rank, dEf_sum, ops)
    da, dv, dq, dE0 = ops.scan_bwd(a, v, q, dy, workspace, mode, E_in, dE_out, rank == 0)
    return da, dv, dq, (dE0 if rank == 0 else None)


class _CpScanFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, a, v, q, E_init, mode, group):
        a, v, q = a.contiguous(), v.contiguous(), q.contiguous()
        E0 = None if E_init is None else E_init.detach().contiguous().float()
        y, E_final, E_in, ws = cp_scan_fwd(a, v, q, mode, E0, group)
        ctx.mode, ctx.group, ctx.ws = mode, group, ws
        ctx.has_E_init = E_init is not None
        ctx.save_for_backward(a, v, q, E_in)
        return y, E_final

    @staticmethod
    def backward(ctx, dy, dE_final):
        a, v, q, E_in = ctx.saved_tensors
        dy = torch.zeros_like(a) if dy is None else dy.to(a.dtype).contiguous()
        dEf = None if dE_final is None else dE_final.float().contiguous()
        da, dv, dq, dE0 = cp_scan_bwd(a, v, q, dy, ctx.ws, E_in, ctx.mode, dEf, ctx.group)
        ctx.ws = None
        if ctx.has_E_init and dE0 is None:
            dE0 = torch.zeros_like(E_in)
        return da, dv, dq, (dE0 if ctx.has_E_init else None), None, None


def cp_esa_scan(a, v, q, mode="controlled", E_init=None, group=None):
    """Differentiable context-parallel scan of this rank's slice.  Returns
    ``(y, E_final)`` with ``E_final`` the state after the last slice on
    every rank.  Every rank of ``group`` must call it (and its backward)."""
    m = {"direct": _esa.DIRECT, "controlled": _esa.CONTROLLED}[mode] if isinstance(mode, str) else int(mode)
    return _CpScanFn.apply(a, v, q, E_init, m, group)
