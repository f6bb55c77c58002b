"""Seeded synthetic inputs for the ESA scan workloads.

This module holds no arithmetic of the method: it only draws random numbers
and casts them.  Both the GPU path (tests, bench) and the CPU oracle consume
the tensors it returns, so the two sides always see the same values.

Recipe (the same for every workload): ``torch.Generator('cpu')`` seeded with
the workload's seed, ``torch.randn`` in fp32, drawn in the order a, v, q, dy
(then, for decode workloads, per step a_t, v_t, q_t), the gate logits shifted
by the workload's mean, then each tensor rounded to the I/O dtype with
round-to-nearest-even.  Large workloads that the host should not materialise
are drawn on the device with a seeded ``torch.Generator('cuda')`` instead
(``device='cuda'``); those draws follow the same distributions but not the
same values as the CPU stream.

The workloads mirror the shapes the pages benchmark: batch 64, FP16, contexts
up to 64K tokens, and C = 128 channels (the width that the peak-memory
figures on mlbricks-web.pages.dev/esa imply); the state is [B, H, D].
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
DIRECT = 0
CONTROLLED = 1


@dataclass(frozen=True)
class Workload:
    name: str
    mode: int            # 0 direct, 1 controlled
    dtype: str           # "f32" | "f16" | "bf16"
    B: int
    T: int
    H: int
    D: int
    a_mean: float        # mean of the gate logits a ~ N(a_mean, 1)
    seed: int
    passes: str          # "fwd", "fwd+bwd", "fwd+bwd+step", "prefill+decode"
    prompts: tuple = field(default_factory=tuple)   # prefill lengths (decode workloads)
    steps: int = 0                                   # decode steps per prompt

    @property
    def C(self) -> int:
        return self.H * self.D


# The five workloads the path is specified on.
WORKLOADS = {
    "direct_f32_B2_T128_H4_D32": Workload(
        "direct_f32_B2_T128_H4_D32", DIRECT, "f32", 2, 128, 4, 32, 0.0, 0, "fwd+bwd+step", steps=128),
    "controlled_f16_B16_T1024_H4_D32": Workload(
        "controlled_f16_B16_T1024_H4_D32", CONTROLLED, "f16", 16, 1024, 4, 32, 2.0, 1, "fwd"),
    "controlled_bf16_B64_T4096_H8_D64": Workload(
        "controlled_bf16_B64_T4096_H8_D64", CONTROLLED, "bf16", 64, 4096, 8, 64, 3.0, 2, "fwd+bwd"),
    "controlled_f16_B64_T65536_H4_D32": Workload(
        "controlled_f16_B64_T65536_H4_D32", CONTROLLED, "f16", 64, 65536, 4, 32, 4.0, 3, "fwd+bwd"),
    "direct_f16_B64_H4_D32_prefill_decode": Workload(
        "direct_f16_B64_H4_D32_prefill_decode", DIRECT, "f16", 64, 8192, 4, 32, 0.0, 4,
        "prefill+decode", prompts=(512, 1024, 4096, 8192), steps=256),
}

LONG_CONTEXT = WORKLOADS["controlled_f16_B64_T65536_H4_D32"]


def make_scan_inputs(B, T, H, D, dtype="f16", a_mean=0.0, seed=0, with_dy=True,
                     device="cpu", generator=None):
    """Draw a, v, q (and dy) of shape [B, T, H, D] in the I/O dtype.

    With ``device='cpu'`` the draws come from a CPU generator seeded with
    ``seed`` (the canonical stream).  With a CUDA device they come from a CUDA
    generator seeded with ``seed`` and never touch the host.
    Returns a dict with keys 'a', 'v', 'q' (and 'dy'), plus the generator so
    callers can continue the stream.
    """
    dt = DTYPES[dtype]
    dev = torch.device(device)
    if generator is None:
        generator = torch.Generator(device=dev)
        generator.manual_seed(int(seed))
    shape = (B, T, H, D)
    out = {}
    out["a"] = (torch.randn(shape, generator=generator, device=dev, dtype=torch.float32)
                .add_(a_mean).to(dt))
    out["v"] = torch.randn(shape, generator=generator, device=dev, dtype=torch.float32).to(dt)
    out["q"] = torch.randn(shape, generator=generator, device=dev, dtype=torch.float32).to(dt)
    if with_dy:
        out["dy"] = torch.randn(shape, generator=generator, device=dev, dtype=torch.float32).to(dt)
    out["generator"] = generator
    return out


def make_step_inputs(B, H, D, dtype="f16", a_mean=0.0, generator=None, seed=0, device="cpu"):
    """Draw one decode step's a_t, v_t, q_t of shape [B, H, D], continuing ``generator``."""
    dt = DTYPES[dtype]
    dev = torch.device(device)
    if generator is None:
        generator = torch.Generator(device=dev)
        generator.manual_seed(int(seed))
    shape = (B, H, D)
    a = torch.randn(shape, generator=generator, device=dev, dtype=torch.float32).add_(a_mean).to(dt)
    v = torch.randn(shape, generator=generator, device=dev, dtype=torch.float32).to(dt)
    q = torch.randn(shape, generator=generator, device=dev, dtype=torch.float32).to(dt)
    return {"a": a, "v": v, "q": q, "generator": generator}


def make_state(B, H, D, seed=0, scale=1.0, device="cpu"):
    """Draw an fp32 state [B, H, D] ~ N(0, scale^2) (for non-zero E_init / dE_final cases)."""
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return torch.randn((B, H, D), generator=g, device=torch.device(device),
                       dtype=torch.float32).mul_(scale)


def workload_inputs(w: Workload, device="cpu", T=None):
    """Inputs for workload ``w`` (optionally with a different sequence length)."""
    return make_scan_inputs(w.B, w.T if T is None else T, w.H, w.D, w.dtype, w.a_mean,
                            w.seed, with_dy="bwd" in w.passes, device=device)
