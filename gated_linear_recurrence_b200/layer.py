"""PyTorch autograd wrapper and an ESA layer over the C ABI.

* :func:`esa_scan` -- differentiable scan ``(a, v, q) -> (y, E_final)``: the
  forward is ``esa_scan_fwd``, the backward ``esa_scan_bwd`` (the forward's
  workspace, which holds the chunk checkpoints, is kept for it).
* :class:`ESA` -- the sequence-mixing layer of "Entangled State Attention
  v2.1", section 1 ("ESA layer": ``ESA(embd, head, ...)`` mapping
  ``[B, T, embd]`` to ``[B, T, embd]``), computed as on the
  "entangled-state-attention 0.1.0" page, section "Core idea":
  gate logits ``a = x W_A``, values ``v = x W_V``, queries ``q = x W_Q``, the
  recurrence (direct or controlled) over each head, and ``y = W_O(q * Norm(E))``
  with Norm the per-head RMS.

When the shapes allow it (16-bit weights and input, no bias, head dimension
<= 64, input width 64 or 128) the input projections run inside the scan
kernel on the tensor cores (``esa_fused_fwd``); in training that call also
writes a, v, q for the library backward, and the projections' own gradients
(dx, dW) are ordinary GEMMs.  Otherwise the three input projections are one
GEMM whose ``[B, T, 3 C]`` output the scan reads in place (a, v, q are its
column blocks, row stride 3 C); the backward writes da, dv, dq into one such
buffer, so dx and dW are single GEMMs over K = 3 C as well.  With a
context-parallel group the projections are separate linear layers feeding
the context-parallel scan.  W_O is a linear layer, except in inference
(no gradient) through the fused path at embd = 64 without bias, where the
same kernel also computes the output projection (``esa_fused_layer_fwd``).
Every step of the recurrence and its readout runs in the CUDA library; there
is no CPU path.
"""
from __future__ import annotations

import torch

from . import esa as _esa

__all__ = ["ESA", "esa_scan"]

_MODES = {"direct": _esa.DIRECT, "controlled": _esa.CONTROLLED}


class _EsaScanFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, a, v, q, E_init, mode):
        a, v, q = a.contiguous(), v.contiguous(), q.contiguous()
        E0 = None if E_init is None else E_init.detach().contiguous().float()
        y, E_final, ws = _esa.esa_scan_fwd(a, v, q, mode=mode, E_init=E0)
        ctx.mode = mode
        ctx.ws = ws
        ctx.has_E_init = E_init is not None
        ctx.save_for_backward(a, v, q, E0 if E0 is not None else torch.empty(0, device=a.device))
        return y, E_final

    @staticmethod
    def backward(ctx, dy, dE_final):
        a, v, q, E0 = ctx.saved_tensors
        E0 = E0 if ctx.has_E_init else None
        if dy is None:
            dy = torch.zeros_like(a)
        dy = dy.to(a.dtype).contiguous()
        dEf = None if dE_final is None else dE_final.float().contiguous()
        da, dv, dq, dE0 = _esa.esa_scan_bwd(a, v, q, dy, ctx.ws, mode=ctx.mode, E_init=E0, dE_final=dEf,
                                            want_dE_init=ctx.has_E_init)
        ctx.ws = None
        return da, dv, dq, (dE0 if ctx.has_E_init else None), None


class _FusedProjScanFn(torch.autograd.Function):
    """(x, W = [W_A; W_V; W_Q]) -> (y, E_final) through esa_fused_fwd; the
    backward is esa_scan_bwd on the projections the forward wrote, then the
    projections' gradients dx = da W_A + dv W_V + dq W_Q and
    dW = [da^T x; dv^T x; dq^T x] (GEMMs, no concatenated copy of the
    gradients)."""

    @staticmethod
    def forward(ctx, x, W, E_init, mode, H):
        x = x.contiguous()
        W = W.contiguous()
        E0 = None if E_init is None else E_init.detach().contiguous().float()
        train = any(ctx.needs_input_grad[:3])
        out = _esa.esa_fused_fwd(x, W, H, mode=mode, E_init=E0, want_avq=train)
        y, E_final, ws = out[:3]
        ctx.mode, ctx.has_E_init = mode, E_init is not None
        if train:
            a, v, q = out[3]
            ctx.ws = ws
            ctx.save_for_backward(x, W, a, v, q, E0 if E0 is not None else torch.empty(0, device=x.device))
        return y, E_final

    @staticmethod
    def backward(ctx, dy, dE_final):
        x, W, a, v, q, E0 = ctx.saved_tensors
        E0 = E0 if ctx.has_E_init else None
        dy = torch.zeros_like(a) if dy is None else dy.to(a.dtype).contiguous()
        dEf = None if dE_final is None else dE_final.float().contiguous()
        G, dE0 = _grads_into_one_buffer(a, v, q, dy, ctx.ws, ctx.mode, E0, dEf, ctx.has_E_init)
        ctx.ws = None
        dx, dW, _ = _projection_grads(G, x, W, ctx.needs_input_grad[0], False)
        return dx, dW, (dE0 if ctx.has_E_init else None), None, None


def _grads_into_one_buffer(a, v, q, dy, ws, mode, E0, dEf, want_dE_init):
    """esa_scan_bwd writing da, dv, dq as the column blocks of one
    ``[B, T, 3 C]`` buffer (row stride 3 C), so that the projections'
    gradients are single GEMMs over K = 3 C."""
    B, T, H, D = a.shape
    G = torch.empty(B, T, 3, H, D, dtype=_esa.out_dtype(a.dtype), device=a.device)
    da, dv, dq = G.unbind(2)
    _, _, _, dE0 = _esa.esa_scan_bwd(a, v, q, dy, ws, mode=mode, E_init=E0, dE_final=dEf, da=da, dv=dv, dq=dq,
                                     want_dE_init=want_dE_init)
    return G, dE0


def _projection_grads(G, x, W, want_dx, want_db):
    """dx = G W, dW = G^T x (and db = column sums of G) for the projection
    P = x W^T (+ b), G = dL/dP as ``[B, T, 3 C]``."""
    B, T = x.shape[:2]
    G2 = G.reshape(B * T, -1)
    if G2.dtype != W.dtype:
        G2 = G2.to(W.dtype)
    x2 = x.reshape(B * T, -1)
    dx = (G2 @ W).reshape(x.shape) if want_dx else None
    dW = G2.t() @ x2
    db = G2.sum(0) if want_db else None
    return dx, dW, db


class _ProjScanFn(torch.autograd.Function):
    """(x, W = [W_A; W_V; W_Q], b) -> (y, E_final) with the three input
    projections as one GEMM: P = x W^T + b is ``[B, T, 3 C]`` and a, v, q are
    its column blocks, scanned in place (row stride 3 C, esa_scan_fwd_ld).
    The backward writes da, dv, dq into one ``[B, T, 3 C]`` buffer
    (esa_scan_bwd_ld), so dx = G W and dW = G^T x are single GEMMs."""

    @staticmethod
    def forward(ctx, x, W, b, E_init, mode, H, scan_dtype):
        B, T, _ = x.shape
        C = W.shape[0] // 3
        P = torch.nn.functional.linear(x, W, b)
        if scan_dtype is not None and P.dtype != scan_dtype:
            P = P.to(scan_dtype)
        a, v, q = P.view(B, T, 3, H, C // H).unbind(2)
        E0 = None if E_init is None else E_init.detach().contiguous().float()
        y, E_final, ws = _esa.esa_scan_fwd(a, v, q, mode=mode, E_init=E0)
        ctx.mode, ctx.has_E_init, ctx.has_b, ctx.H = mode, E_init is not None, b is not None, H
        ctx.ws = ws
        ctx.save_for_backward(x, W, P, E0 if E0 is not None else torch.empty(0, device=x.device))
        return y, E_final

    @staticmethod
    def backward(ctx, dy, dE_final):
        x, W, P, E0 = ctx.saved_tensors
        E0 = E0 if ctx.has_E_init else None
        B, T, _ = x.shape
        C = W.shape[0] // 3
        a, v, q = P.view(B, T, 3, ctx.H, C // ctx.H).unbind(2)
        dy = torch.zeros(a.shape, dtype=a.dtype, device=a.device) if dy is None else dy.to(a.dtype).contiguous()
        dEf = None if dE_final is None else dE_final.float().contiguous()
        G, dE0 = _grads_into_one_buffer(a, v, q, dy, ctx.ws, ctx.mode, E0, dEf, ctx.has_E_init)
        ctx.ws = None
        dx, dW, db = _projection_grads(G, x, W, ctx.needs_input_grad[0], ctx.has_b)
        return dx, dW, db, (dE0 if ctx.has_E_init else None), None, None, None


def esa_scan(a, v, q, mode="controlled", E_init=None):
    """Differentiable scan of ``[B, T, H, D]`` CUDA tensors (float32, float16
    or bfloat16).  Returns ``(y, E_final)``; ``E_final`` is float32
    ``[B, H, D]``.  ``E_init`` (float32 ``[B, H, D]``) may require grad."""
    m = _MODES[mode] if isinstance(mode, str) else int(mode)
    return _EsaScanFn.apply(a, v, q, E_init, m)


class ESA(torch.nn.Module):
    """ESA sequence mixer: ``[B, T, embd] -> [B, T, embd]``.

    Args:
        embd: embedding width C.
        head: number of heads H; the head dimension ``embd // head`` must be
            one of 8, 16, 32, 64, 128, 256 (the library's head dimensions).
        mode: ``"controlled"`` (default) or ``"direct"``.
        bias: bias terms in the four projections.
        scan_dtype: dtype the scan reads and writes (float16, bfloat16 or
            float32); the state is float32 either way.  ``None`` keeps the
            dtype of the projections' output.
        fused: run the input projections inside the scan kernel
            (``esa_fused_fwd``): ``None`` (default) whenever the shapes and
            dtypes allow it, ``True`` to require it, ``False`` never.
        cp_group: a ``torch.distributed`` process group over which each
            sequence is split along time (context parallelism: rank r of the
            group passes the r-th time slice of the sequence); ``None`` runs
            the whole sequence on this device.

    ``forward(x, state=None, return_state=False)`` runs the whole sequence;
    ``state`` (float32 ``[B, H, D]``) is the state before the first token and
    ``return_state`` also returns the state after the last.  ``step(x_t,
    state)`` is the one-token update for decoding: ``x_t`` is ``[B, embd]``,
    ``state`` is updated in place and the output for the token returned.
    """

    def __init__(self, embd: int, head: int, mode: str = "controlled", bias: bool = False,
                 scan_dtype: torch.dtype | None = None, device=None, dtype=None, cp_group=None,
                 fused: bool | None = None):
        super().__init__()
        if embd % head != 0:
            raise ValueError("embd must be a multiple of head")
        if embd // head not in (8, 16, 32, 64, 128, 256):
            raise ValueError("head dimension embd // head must be one of 8, 16, 32, 64, 128, 256")
        if mode not in _MODES:
            raise ValueError("mode must be 'controlled' or 'direct'")
        self.embd, self.head, self.mode = embd, head, mode
        self.head_dim = embd // head
        self.scan_dtype = scan_dtype
        self.cp_group = cp_group
        self.fused = fused
        kw = {"device": device, "dtype": dtype}
        self.W_A = torch.nn.Linear(embd, embd, bias=bias, **kw)
        self.W_V = torch.nn.Linear(embd, embd, bias=bias, **kw)
        self.W_Q = torch.nn.Linear(embd, embd, bias=bias, **kw)
        self.W_O = torch.nn.Linear(embd, embd, bias=bias, **kw)

    def _proj(self, x, shape):
        dt = self.scan_dtype
        out = []
        for lin in (self.W_A, self.W_V, self.W_Q):
            t = lin(x).reshape(shape)
            out.append((t if dt is None else t.to(dt)).contiguous())
        return out

    def _fused_ok(self, x):
        dt = self.W_A.weight.dtype
        return (x.is_cuda and self.cp_group is None and self.W_A.bias is None and dt in (torch.float16, torch.bfloat16)
                and x.dtype == dt and self.scan_dtype in (None, dt) and self.head_dim <= 64
                and self.embd in (64, 128, 256) and -(-self.embd // 64) <= 48)

    def _fused_out_ok(self, x):
        """The fused forward can also apply W_O: 64 channels (one channel tile
        holds whole rows), no output bias, W_O in x's dtype, and no gradient
        wanted (the kernel does not keep y for W_O's gradient)."""
        wants_grad = torch.is_grad_enabled() and (x.requires_grad or any(p.requires_grad for p in self.parameters()))
        return (self.embd == 64 and self.W_O.bias is None and self.W_O.weight.dtype == x.dtype and not wants_grad)

    def forward(self, x, state=None, return_state=False):
        B, T, C = x.shape
        if C != self.embd:
            raise ValueError(f"expected last dimension {self.embd}, got {C}")
        use_fused = self._fused_ok(x) if self.fused is None else bool(self.fused)
        if use_fused:
            if not self._fused_ok(x):
                raise ValueError("fused=True needs 16-bit CUDA input and weights of the same dtype, no bias, "
                                 "head_dim <= 64, embd of 64 or 128 and no context-parallel group")
            W = torch.cat([self.W_A.weight, self.W_V.weight, self.W_Q.weight], dim=0)
            m = _MODES[self.mode]
            if self._fused_out_ok(x):   # inference: the output projection in the same kernel
                z, _, E, _ = _esa.esa_fused_layer_fwd(x.contiguous(), W, self.W_O.weight.contiguous(), self.head,
                                                      mode=m, E_init=state)
                return (z, E) if return_state else z
            y, E = _FusedProjScanFn.apply(x, W, state, m, self.head)
            out = self.W_O(y.reshape(B, T, C).to(self.W_O.weight.dtype))
            return (out, E) if return_state else out
        if self.cp_group is not None:
            from .context_parallel import cp_esa_scan
            a, v, q = self._proj(x, (B, T, self.head, self.head_dim))
            y, E = cp_esa_scan(a, v, q, self.mode, E_init=state, group=self.cp_group)
        else:
            W = torch.cat([self.W_A.weight, self.W_V.weight, self.W_Q.weight], dim=0)
            b = None if self.W_A.bias is None else torch.cat([self.W_A.bias, self.W_V.bias, self.W_Q.bias])
            y, E = _ProjScanFn.apply(x, W, b, state, _MODES[self.mode], self.head, self.scan_dtype)
        out = self.W_O(y.reshape(B, T, C).to(self.W_O.weight.dtype))
        return (out, E) if return_state else out

    @torch.no_grad()
    def step(self, x_t, state):
        B, C = x_t.shape
        if C != self.embd:
            raise ValueError(f"expected last dimension {self.embd}, got {C}")
        a, v, q = self._proj(x_t, (B, self.head, self.head_dim))
        y = _esa.esa_step(a, v, q, state, mode=_MODES[self.mode])
        return self.W_O(y.reshape(B, C).to(self.W_O.weight.dtype))

    def init_state(self, batch: int, device=None):
        """A zero state ``[batch, head, head_dim]`` (float32)."""
        return torch.zeros(batch, self.head, self.head_dim, dtype=torch.float32,
                           device=device if device is not None else self.W_A.weight.device)

    # The generation interface of the pages (mlbricks-web.pages.dev/esa, Quick
    # start: prefill returns the output and the state, decode_step advances
    # one token), on the layer's input and output.
    @torch.no_grad()
    def prefill(self, x, state=None):
        """``(out, state)`` after the whole prompt ``x`` [B, T, embd]."""
        out, E = self.forward(x, state=state, return_state=True)
        return out, E

    @torch.no_grad()
    def decode_step(self, x_t, state):
        """``(out_t, state)`` for one token ``x_t`` [B, embd]; ``state`` is
        updated in place and returned."""
        return self.step(x_t, state), state
