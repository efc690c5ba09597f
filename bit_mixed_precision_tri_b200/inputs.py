"""Seeded synthetic inputs shared by the tests, the bench and the smoke check.

This module only draws random numbers (torch CPU generator, fixed seeds); it
holds none of the method's arithmetic, so both the CUDA path and the CPU
oracle can consume what it produces without sharing any computation.

Distributions follow the workloads of the ternary-linear-layer pages:
latent weights N(0, 0.02) in float32, activations N(0, 1) rounded to fp16,
and (for format stress) trits drawn i.i.d. with a chosen zero probability and
+1/-1 equally likely, with per-block scales drawn from U(0.01, 0.05).
"""
from __future__ import annotations

import numpy as np
import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def latent_weights(N: int, K: int, seed: int, std: float = 0.02) -> torch.Tensor:
    """float32 (N, K) ~ N(0, std)."""
    return torch.randn(N, K, generator=_gen(seed), dtype=torch.float32) * std


def activations(M: int, K: int, seed: int) -> torch.Tensor:
    """fp16 (M, K) ~ N(0, 1) rounded to fp16."""
    return torch.randn(M, K, generator=_gen(seed), dtype=torch.float32).to(torch.float16)


def random_trits(N: int, K: int, p_zero: float, seed: int) -> torch.Tensor:
    """int8 (N, K) trits: P(0) = p_zero, +1 and -1 equally likely otherwise."""
    g = _gen(seed)
    u = torch.rand(N, K, generator=g)
    s = torch.randint(0, 2, (N, K), generator=g, dtype=torch.int8) * 2 - 1
    return torch.where(u < p_zero, torch.zeros_like(s), s).to(torch.int8)


def block_scales(N: int, K: int, seed: int, lo: float = 0.01, hi: float = 0.05) -> torch.Tensor:
    """float32 (N, K/256) ~ U(lo, hi), one draw per 256-weight block."""
    return lo + (hi - lo) * torch.rand(N, K // 256, generator=_gen(seed), dtype=torch.float32)


def random_bytes(n: int, seed: int) -> torch.Tensor:
    """uint8 (n,) uniformly random bytes (for invalid-code handling)."""
    return torch.randint(0, 256, (n,), generator=_gen(seed), dtype=torch.uint8)


def as_numpy(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def random_trits_on(device, N: int, K: int, p_zero: float, seed: int) -> torch.Tensor:
    """As ``random_trits``, drawn by torch's generator on `device` (for large
    timing-only weights; the parity tests use the CPU draws)."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    u = torch.rand(N, K, generator=g, device=device)
    s = torch.randint(0, 2, (N, K), generator=g, dtype=torch.int8, device=device) * 2 - 1
    return torch.where(u < p_zero, torch.zeros_like(s), s).to(torch.int8)


def fp16_normal_on(device, shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """fp16 tensor ~ N(0, std) drawn on `device` (timing-only caches)."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return (torch.randn(*shape, generator=g, device=device) * std).to(torch.float16)
