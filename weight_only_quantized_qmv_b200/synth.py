"""Seeded synthetic inputs shared by the tests, the bench and the CPU oracle.

This module holds only random-number generation and reshaping: none of the
quantisation arithmetic.  Every generator takes a ``torch.Generator`` so a
caller draws a workload in one fixed order from one seed:
weights, outlier columns, activations, routing.

Workload shapes and distributions follow the pages' decode problem: weights
~N(0, 0.02) with a few input columns scaled x20 (outlier channels), fp16
activations ~N(0, 1), top-k uniform routing over the experts.
"""
from __future__ import annotations

import torch

WEIGHT_STD = 0.02
OUTLIER_SCALE = 20.0


def generator(seed: int = 0, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights(N: int, K: int, gen: torch.Generator, n_outlier_cols: int = 0, std: float = WEIGHT_STD,
            device=None) -> tuple[torch.Tensor, torch.Tensor]:
    """W float32 [N, K] ~ N(0, std); ``n_outlier_cols`` input columns (picked by
    a seeded permutation) scaled by OUTLIER_SCALE.  Returns (W, cols)."""
    device = device or gen.device
    W = torch.randn(N, K, generator=gen, device=device, dtype=torch.float32)
    W.mul_(std)
    cols = torch.randperm(K, generator=gen, device=device)[:n_outlier_cols]
    if n_outlier_cols:
        W[:, cols] *= OUTLIER_SCALE
    return W, cols


def activations(B: int, K: int, gen: torch.Generator, device=None, extra_shape=()) -> torch.Tensor:
    """x fp16 [B, *extra_shape, K] ~ N(0, 1) (drawn in fp32, rounded to fp16)."""
    device = device or gen.device
    x = torch.randn(B, *extra_shape, K, generator=gen, device=device, dtype=torch.float32)
    return x.to(torch.float16)


def routing(B: int, topk: int, E: int, gen: torch.Generator) -> torch.Tensor:
    """Expert ids int32 [B, topk]: per token the first topk of a random
    permutation of the E experts (uniform, no repeats within a token)."""
    rows = [torch.randperm(E, generator=gen, device=gen.device)[:topk] for _ in range(B)]
    return torch.stack(rows).to(torch.int32)


def palette_tables(N: int, K: int, gen: torch.Generator, std: float = WEIGHT_STD, device=None):
    """Stand-in int4km inputs for throughput runs at sizes where a CPU k-means
    fit is too slow: per row a sorted 16-entry fp16 table drawn ~N(0, std) and
    uniformly random 4-bit indices packed two per byte.  Same shapes and
    bytes as a fitted palette; the values are random, not a fit."""
    device = device or gen.device
    lut = torch.randn(N, 16, generator=gen, device=device, dtype=torch.float32).mul_(std)
    lut = torch.sort(lut, dim=1).values.to(torch.float16)
    idx = torch.randint(0, 256, (N, K // 2), generator=gen, device=device, dtype=torch.int32).to(torch.uint8)
    return lut, idx


def palette_tables8(N: int, K: int, gen: torch.Generator, std: float = WEIGHT_STD, device=None):
    """Stand-in int8km inputs (as palette_tables, 8-bit): per group of 32 rows
    a sorted 256-entry fp16 table drawn ~N(0, std) and uniformly random index
    bytes [N, K].  Same shapes and bytes as a fitted int8km palette."""
    device = device or gen.device
    G = (N + 31) // 32
    lut = torch.randn(G, 256, generator=gen, device=device, dtype=torch.float32).mul_(std)
    lut = torch.sort(lut, dim=1).values.to(torch.float16)
    idx = torch.randint(0, 256, (N, K), generator=gen, device=device, dtype=torch.int32).to(torch.uint8)
    return lut, idx


def int_codes(N: int, K: int, bits: int, gen: torch.Generator, device=None):
    """Uniform random packed codes (uint8 [N, K*bits/8]) for edge-case tests."""
    device = device or gen.device
    return torch.randint(0, 256, (N, K * bits // 8), generator=gen, device=device, dtype=torch.int32).to(torch.uint8)
