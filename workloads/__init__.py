"""Seeded synthetic inputs for CSA2 (shared by the CUDA path's tests/bench and the oracle).

This module holds random draws and shapes only -- none of the method's
arithmetic.  Every tensor comes from its own torch.Generator whose seed is a
stable hash of (seed, name, index...), so any one sequence's inputs can be
regenerated alone, on the device that needs them, and copied elsewhere.
"""
import hashlib
import math

import torch


def sub_seed(seed, *names):
    h = hashlib.sha256(repr((int(seed),) + tuple(names)).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def generator(seed, *names, device="cpu"):
    g = torch.Generator(device=device)
    g.manual_seed(sub_seed(seed, *names))
    return g


def normal(shape, seed, *names, device="cpu", dtype=torch.float32, std=1.0, mean=None):
    g = generator(seed, *names, device=device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    if mean is not None:
        x = x + mean
    return x.to(dtype)


def uniform(shape, seed, *names, lo=0.0, hi=1.0, device="cpu", dtype=torch.float32):
    g = generator(seed, *names, device=device)
    x = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    return (lo + (hi - lo) * x).to(dtype)


def choice(n, k, seed, *names):
    """k distinct integers from [0, n), uniform without replacement (CPU int32)."""
    g = generator(seed, *names)
    if k * 8 >= n:
        return torch.randperm(n, generator=g)[:k].to(torch.int32)
    # rejection on a larger draw keeps it O(k) for huge n
    out = []
    seen = set()
    while len(out) < k:
        cand = torch.randint(0, n, (2 * k,), generator=g).tolist()
        for c in cand:
            if c not in seen:
                seen.add(c)
                out.append(c)
                if len(out) == k:
                    break
    return torch.tensor(out, dtype=torch.int32)


def log_uniform_ints(count, lo, hi, seed, *names):
    u = uniform((count,), seed, *names, dtype=torch.float64)
    return torch.floor(torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))).to(torch.int64)


def permutation(n, seed, *names):
    return torch.randperm(n, generator=generator(seed, *names)).to(torch.int32)
