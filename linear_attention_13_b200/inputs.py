"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This module holds no arithmetic of the method: it only draws random numbers
with a fixed recipe and lays them out.  Both sides consume exactly the tensors
it returns (the oracle widens the already-rounded bf16/fp32 values to fp64).

Recipe (q, k ~ N(0, 1/d), v ~ N(0, 1), drawn in the order q, k, v from one
``torch.Generator`` seeded per call, fp32 draws then a cast to the compute
dtype) follows the workload descriptions of the benchmark configurations.
"""
from __future__ import annotations

import numpy as np
import torch


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def qkv(shape, dtype=torch.bfloat16, device="cpu", seed: int = 0):
    """Draw q, k, v of ``shape`` (last dim d): q,k ~ N(0,1/d), v ~ N(0,1)."""
    d = shape[-1]
    g = _gen(device, seed)
    q = torch.randn(shape, generator=g, dtype=torch.float32, device=device).mul_(d ** -0.5)
    k = torch.randn(shape, generator=g, dtype=torch.float32, device=device).mul_(d ** -0.5)
    v = torch.randn(shape, generator=g, dtype=torch.float32, device=device)
    return q.to(dtype), k.to(dtype), v.to(dtype)


def ternary_qkv(shape, dtype=torch.bfloat16, device="cpu", seed: int = 0):
    """q, k, v with entries in {-1, 0, 1} (small integers, exact in bf16/fp32)."""
    g = _gen(device, seed)
    out = []
    for _ in range(3):
        out.append(torch.randint(-1, 2, shape, generator=g, device=device).to(dtype))
    return tuple(out)


def onehot_k_qkv(shape, dtype=torch.bfloat16, device="cpu", seed: int = 0):
    """Ternary q, v and a k whose rows each hold a single +-1 at a random column.

    With one nonzero per key row, every state entry is a sum of at most about
    N/d unit terms, so all intermediate values stay small integers and are
    exact in bf16 and fp32 even for sequences of several thousand tokens.
    """
    g = _gen(device, seed)
    d = shape[-1]
    q = torch.randint(-1, 2, shape, generator=g, device=device)
    v = torch.randint(-1, 2, shape, generator=g, device=device)
    pos = torch.randint(0, d, shape[:-1], generator=g, device=device)
    sign = torch.randint(0, 2, shape[:-1], generator=g, device=device) * 2 - 1
    k = torch.zeros(shape, dtype=torch.int64, device=device)
    k.scatter_(-1, pos.unsqueeze(-1), sign.unsqueeze(-1))
    return q.to(dtype), k.to(dtype), v.to(dtype)


def varlen_lengths(total_tokens: int, lo: int, hi: int, seed: int = 0):
    """Integer lengths uniform in [lo, hi] (inclusive), drawn until they cover
    ``total_tokens``; the last one is trimmed so the lengths sum exactly to it."""
    rng = np.random.default_rng(seed)
    lens = []
    acc = 0
    while acc < total_tokens:
        n = int(rng.integers(lo, hi, endpoint=True))
        n = min(n, total_tokens - acc)
        lens.append(n)
        acc += n
    return lens


def cu_seqlens_from_lengths(lengths):
    """Prefix offsets [0, l0, l0+l1, ...] as int32."""
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu.astype(np.int32)


def decode_step_inputs(n_seq: int, H: int, d: int, step: int, dtype=torch.bfloat16,
                       device="cpu"):
    """q, k, v of shape [n_seq, H, d] for decode step ``step`` (seed = step)."""
    return qkv((n_seq, H, d), dtype=dtype, device=device, seed=step)
