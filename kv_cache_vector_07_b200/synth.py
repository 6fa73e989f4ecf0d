"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no arithmetic of the codec: it only draws input tensors.
Both the CUDA path (through its tests and the benchmark) and the CPU oracle
receive exactly these tensors.

Recipes (head_dim 128, GQA, 32K-262K contexts, per the pages' workload shapes):
  * ``outlier_normal``: iid N(0,1) with a few channels scaled (channels 5 and
    77 scaled x20 in the small single-head check and the decode caches).
  * ``lognormal_channels``: z * s[h, c] with z ~ N(0,1), s ~ lognormal(0,1)
    per (kv-head, channel), plus 4 distinct seeded outlier channels per
    kv-head scaled x15 (the 8B-dense-layer write-path shape).
  * ``unit_normal``: N(0,1) rows normalised to unit length (vector search).

Small inputs use NumPy's PCG64 ``default_rng(seed)`` so they are identical on
every machine; large ones use torch's seeded generator on the target device
(identical for a given device type), and tests hand the very same tensors to
the oracle.
"""
from __future__ import annotations

import numpy as np
import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def np_outlier_normal(rng: np.random.Generator, n: int, d: int,
                      channels=(5, 77), scale: float = 20.0) -> np.ndarray:
    x = rng.standard_normal((n, d))
    for c in channels:
        if c < d:
            x[:, c] *= scale
    return x


def small_check(seed: int = 0, d: int = 128, n_kv: int = 1024, n_q: int = 16):
    """Tiny single-head case: K, V [n_kv, d] and Q [n_q, d], float32."""
    rng = np.random.default_rng(seed)
    K = np_outlier_normal(rng, n_kv, d).astype(np.float32)
    V = np_outlier_normal(rng, n_kv, d).astype(np.float32)
    Q = rng.standard_normal((n_q, d)).astype(np.float32)
    return K, V, Q


def outlier_normal(shape, seed: int, device="cpu", dtype=torch.bfloat16,
                   channels=(5, 77), scale: float = 20.0) -> torch.Tensor:
    """iid N(0,1) over ``shape`` (last dim = channel), chosen channels scaled."""
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    d = shape[-1]
    for c in channels:
        if c < d:
            x[..., c] *= scale
    return x.to(dtype)


def lognormal_channels(n_tokens: int, n_heads: int, d: int, seed: int, device="cpu",
                       dtype=torch.bfloat16, n_outliers: int = 4,
                       outlier_scale: float = 15.0) -> torch.Tensor:
    """[n_tokens, n_heads, d]: z * s[h, c], s ~ lognormal(0, 1) per (head,
    channel), and n_outliers distinct channels per head scaled further."""
    g = _gen(seed, device)
    s = torch.exp(torch.randn((n_heads, d), generator=g, device=device, dtype=torch.float32))
    for h in range(n_heads):
        perm = torch.randperm(d, generator=g, device=device)[:n_outliers]
        s[h, perm] *= outlier_scale
    out = torch.empty((n_tokens, n_heads, d), device=device, dtype=dtype)
    step = 1 << 16
    for t0 in range(0, n_tokens, step):
        t1 = min(n_tokens, t0 + step)
        z = torch.randn((t1 - t0, n_heads, d), generator=g, device=device, dtype=torch.float32)
        out[t0:t1] = (z * s).to(dtype)
    return out


def normal(shape, seed: int, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(dtype)


def unit_normal(n: int, d: int, seed: int, device="cpu") -> torch.Tensor:
    """[n, d] float32 rows drawn N(0,1) then normalised to unit length."""
    g = _gen(seed, device)
    out = torch.empty((n, d), device=device, dtype=torch.float32)
    step = 1 << 16
    for r0 in range(0, n, step):
        r1 = min(n, r0 + step)
        x = torch.randn((r1 - r0, d), generator=g, device=device, dtype=torch.float32)
        out[r0:r1] = x / x.norm(dim=1, keepdim=True)
    return out


def contiguous_block_table(batch: int, seq_len: int, page_tokens: int, device="cpu",
                           shuffle_seed: int | None = None):
    """Block table [batch, blocks_per_seq] (int32) giving each sequence its own
    pages, optionally in a seeded random physical order, and the matching
    slot mapping [batch * seq_len] for tokens laid out sequence-major."""
    bps = -(-seq_len // page_tokens)
    nblk = batch * bps
    if shuffle_seed is None:
        phys = torch.arange(nblk, dtype=torch.int64)
    else:
        g = torch.Generator().manual_seed(int(shuffle_seed))
        phys = torch.randperm(nblk, generator=g)
    bt = phys.view(batch, bps).to(torch.int32)
    tok = torch.arange(seq_len, dtype=torch.int64)
    slots = (bt.to(torch.int64)[:, tok // page_tokens] * page_tokens + (tok % page_tokens)).reshape(-1)
    return bt.to(device), slots.to(torch.int32).to(device), nblk
