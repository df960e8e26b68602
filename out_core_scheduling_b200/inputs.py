"""Seeded synthetic inputs for the CQS attention workloads.

This module only draws random tensors; it holds none of the method's
arithmetic.  Tests feed the same tensors to the CUDA library and to the fp64
oracle, and the benchmark uses it for its workloads.

Recipe: one ``torch.Generator`` per call, seeded, on the device the tensors
are drawn on; draws in the order Q, K, V; each drawn in fp32 and rounded to
the storage dtype (round-to-nearest-even).  Distributions:
  * ``"normal"``: Q, K, V i.i.d. N(0, 1).
  * ``"half_normal_uniform_v"``: Q, K ~ 0.5 * N(0, 1), V ~ U(-1, 1).
"""
from __future__ import annotations

import torch

DISTRIBUTIONS = ("normal", "half_normal_uniform_v")


def make_qkv(N: int, H: int, d: int, dtype=torch.bfloat16, seed: int = 0,
             device="cpu", dist: str = "normal"):
    """Return (q, k, v), each [N, H, d] contiguous, in ``dtype`` on ``device``."""
    if dist not in DISTRIBUTIONS:
        raise ValueError(f"unknown distribution {dist!r}")
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    shape = (N, H, d)
    out = []
    for name in ("q", "k", "v"):
        if dist == "half_normal_uniform_v" and name == "v":
            x = torch.rand(shape, generator=g, device=device, dtype=torch.float32) * 2.0 - 1.0
        else:
            x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
            if dist == "half_normal_uniform_v":
                x = x * 0.5
        out.append(x.to(dtype).contiguous())
    return tuple(out)


def sample_rows(N: int, count: int = 256, seed: int = 1234):
    """Query rows drawn without replacement: ``randperm(N)[:count]`` from a
    CPU generator with the given seed, sorted."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    rows = torch.randperm(N, generator=g)[:min(count, N)]
    return torch.sort(rows).values
