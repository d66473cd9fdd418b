"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and packing boundaries; it holds none of
the attention arithmetic.  The pages measure lightning attention on no public
dataset, so these draws stand in for every workload: Q, K and V are i.i.d.
N(0, 1) / sqrt(D) (the 1/sqrt(D) lives in the inputs, since the method has no
score scaling), drawn from a seeded ``torch.Generator`` on the target device
and cast to the compute dtype.  Packed varlen batches cut the token range at
S - 1 seeded uniform points (sorted), as in the data-packing scheme the
jvyan.cn article describes in section 2 ("compute optimisation").
"""
from __future__ import annotations

import math

import numpy as np
import torch


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def normal(shape, D: int, seed: int, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """One tensor of N(0,1)/sqrt(D) values, drawn in fp32 then cast to ``dtype``."""
    g = generator(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    x.mul_(1.0 / math.sqrt(D))
    return x.to(dtype)


def qkv(T: int, H: int, D: int, seed: int = 0, dtype=torch.bfloat16, device="cpu"):
    """q, k, v of shape [T, H, D]; the three draws use seeds 3*seed + {0, 1, 2}."""
    return tuple(normal((T, H, D), D, 3 * seed + i, dtype, device) for i in range(3))


def cu_seqlens_uniform(total: int, num_seqs: int, seed: int = 0) -> np.ndarray:
    """Packed boundaries: S-1 seeded uniform cut points in [0, total], sorted.

    Returns an int32 array of S+1 entries from 0 to ``total``; a repeated cut
    point gives a zero-length sequence, which the method allows.
    """
    rng = np.random.default_rng(seed)
    cuts = np.sort(rng.integers(0, total + 1, size=num_seqs - 1))
    return np.concatenate([[0], cuts, [total]]).astype(np.int32)


def decode_tokens(B: int, H: int, D: int, step: int, seed: int = 0, dtype=torch.bfloat16,
                  device="cpu"):
    """q, k, v of shape [B, H, D] for decode step ``step`` (fresh seeded draws per step)."""
    base = 1_000_003 * (seed + 1) + 3 * step
    return tuple(normal((B, H, D), D, base + i, dtype, device) for i in range(3))


def initial_state(S: int, H: int, D: int, tokens: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """A stand-in for the state a sequence carries after ``tokens`` earlier tokens:
    i.i.d. N(0, 1) * sqrt(tokens) / D in fp32, shape [S, H, D, D] (the entries of a
    sum of ``tokens`` outer products k v^T with k, v ~ N(0, 1/D) have that spread)."""
    g = generator(7_000_003 + int(seed), device)
    x = torch.randn((S, H, D, D), generator=g, device=device, dtype=torch.float32)
    return x * (float(tokens) ** 0.5 / D)
