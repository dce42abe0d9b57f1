"""Seeded synthetic inputs for the fused Linear + epilogue path.

The one module both the CUDA path's tests/benchmark and the CPU oracle's
callers draw inputs from.  It holds no arithmetic of the method itself: it only
draws random tensors.

Distribution (the nn.Linear problems on the pages): x ~ N(0, 1); W and b ~
U(-1/sqrt(K), 1/sqrt(K)), which is what nn.Linear's default Kaiming-uniform
initialisation with a = sqrt(5) gives for fan_in = K (page "Kimi-K2.6 l2_p98",
its discussion of matching the reference model's initialisation).  Draw order
is x, then W, then b, from one torch.Generator seeded with ``seed``.
"""
from __future__ import annotations

import math

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def linear_inputs(M: int, K: int, N: int, seed: int = 0, device="cpu", x_std: float = 1.0):
    """x [M,K] ~ N(0, x_std^2); W [N,K], b [N] ~ U(-1/sqrt(K), 1/sqrt(K)); all fp32, contiguous."""
    device = torch.device(device)
    g = _gen(seed, device)
    x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    if x_std != 1.0:
        x.mul_(x_std)
    bound = 1.0 / math.sqrt(K) if K > 0 else 1.0
    W = torch.rand(N, K, generator=g, device=device, dtype=torch.float32).mul_(2 * bound).sub_(bound)
    b = torch.rand(N, generator=g, device=device, dtype=torch.float32).mul_(2 * bound).sub_(bound)
    return x, W, b


def integer_inputs(M: int, K: int, N: int, seed: int = 0, device="cpu", lo: int = -4, hi: int = 4):
    """Small-integer fp32 tensors in [lo, hi]: exact in fp32, TF32 and fp64 alike."""
    device = torch.device(device)
    g = _gen(seed, device)
    x = torch.randint(lo, hi + 1, (M, K), generator=g, device=device).to(torch.float32)
    W = torch.randint(lo, hi + 1, (N, K), generator=g, device=device).to(torch.float32)
    b = torch.randint(lo, hi + 1, (N,), generator=g, device=device).to(torch.float32)
    return x, W, b


def sample_rows(M: int, n: int, seed: int = 0):
    """A sorted seeded subset of exactly min(n, M) distinct row indices in
    [0, M) that holds the first and last row (tile edges) when n >= 2."""
    n = min(n, M)
    if n <= 0:
        return []
    if n == M:
        return list(range(M))
    g = _gen(seed + 7919, "cpu")
    picked = [0, M - 1][:n]
    for r in torch.randperm(M, generator=g).tolist():
        if len(picked) == n:
            break
        if r not in (0, M - 1):
            picked.append(r)
    return sorted(set(picked))
