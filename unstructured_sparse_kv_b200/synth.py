"""Seeded synthetic KV-cache inputs shared by the CUDA path's tests/bench and the oracle.

This module only draws random numbers; it holds none of the pruning, compression
or attention arithmetic.  Both sides receive the same fp16 bit patterns from it.

Distributions (stand-ins for the Llama-3-8B / Mistral-7B / Llama-2-7B caches the
pages evaluate on, which need model weights that are not available here):

* K ~ N(0, 1) in fp32; for every kv head, 4 distinct channels are drawn uniformly
  and scaled by 10 (outlier channels are a property of the model, so they are
  shared by every batch row and token of that head); then cast to fp16.
  The pages note that the Key cache has prominent outlier elements
  (Mustafar abstract, catalyzex author page).
* V ~ N(0, 1) -> fp16 (the abstract describes the Value cache as uniform in magnitude).
* q ~ N(0, 1) / sqrt(128) -> fp16.
* New decode tokens use the same distributions and the same outlier channels.

Seeds: every tensor kind has its own seed offset from the base seed; big tensors
are drawn batch row by batch row (seed + row) so the generator never needs the
whole tensor in fp32 at once.
"""
from __future__ import annotations

import math

import torch

OUTLIERS_PER_HEAD = 4
OUTLIER_SCALE = 10.0

_OFF_Q, _OFF_K, _OFF_V, _OFF_OUT, _OFF_STEP = 0, 100_000, 200_000, 300_000, 400_000


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def outlier_channels(num_kv_heads: int, head_dim: int, seed: int) -> torch.Tensor:
    """[Hkv, 4] distinct channel indices per kv head (CPU int64)."""
    g = _gen("cpu", seed + _OFF_OUT)
    rows = [torch.randperm(head_dim, generator=g)[:OUTLIERS_PER_HEAD] for _ in range(num_kv_heads)]
    return torch.stack(rows)


def _scale_vector(num_kv_heads: int, head_dim: int, seed: int, device) -> torch.Tensor:
    """[Hkv, d] fp32 multipliers: 10 on each head's outlier channels, 1 elsewhere."""
    s = torch.ones(num_kv_heads, head_dim, dtype=torch.float32)
    idx = outlier_channels(num_kv_heads, head_dim, seed)
    s.scatter_(1, idx, OUTLIER_SCALE)
    return s.to(device)


def keys(B: int, Hkv: int, L: int, d: int, seed: int, device="cpu", capacity: int | None = None) -> torch.Tensor:
    """Dense fp16 K cache, layout [B, Hkv, capacity, d]; tokens >= L are zero."""
    cap = L if capacity is None else capacity
    out = torch.zeros(B, Hkv, cap, d, dtype=torch.float16, device=device)
    sc = _scale_vector(Hkv, d, seed, device)
    for b in range(B):
        g = _gen(device, seed + _OFF_K + b)
        x = torch.randn(Hkv, L, d, generator=g, device=device, dtype=torch.float32)
        x.mul_(sc[:, None, :])
        out[b, :, :L] = x.to(torch.float16)
    return out


def values(B: int, Hkv: int, L: int, d: int, seed: int, device="cpu", capacity: int | None = None) -> torch.Tensor:
    """Dense fp16 V cache, layout [B, Hkv, capacity, d]; tokens >= L are zero."""
    cap = L if capacity is None else capacity
    out = torch.zeros(B, Hkv, cap, d, dtype=torch.float16, device=device)
    for b in range(B):
        g = _gen(device, seed + _OFF_V + b)
        out[b, :, :L] = torch.randn(Hkv, L, d, generator=g, device=device, dtype=torch.float32).to(torch.float16)
    return out


def queries(B: int, Hq: int, d: int, seed: int, device="cpu", step: int = 0) -> torch.Tensor:
    """fp16 q, layout [B, Hq, d], N(0,1)/sqrt(d)."""
    g = _gen(device, seed + _OFF_Q + 7919 * step)
    x = torch.randn(B, Hq, d, generator=g, device=device, dtype=torch.float32) / math.sqrt(d)
    return x.to(torch.float16)


def step_tokens(B: int, Hkv: int, d: int, seed: int, step: int, device="cpu"):
    """One new decode token per (batch, kv head): (k_new, v_new), each [B, Hkv, d] fp16."""
    g = _gen(device, seed + _OFF_STEP + 2 * step)
    k = torch.randn(B, Hkv, d, generator=g, device=device, dtype=torch.float32)
    k.mul_(_scale_vector(Hkv, d, seed, device)[None])
    g2 = _gen(device, seed + _OFF_STEP + 2 * step + 1)
    v = torch.randn(B, Hkv, d, generator=g2, device=device, dtype=torch.float32)
    return k.to(torch.float16), v.to(torch.float16)


def seq_lens(B: int, L: int, ragged: bool, seed: int) -> torch.Tensor:
    """Per-row context lengths (CPU int32): all L, or a seeded mix in [1, L]."""
    if not ragged:
        return torch.full((B,), L, dtype=torch.int32)
    g = _gen("cpu", seed + 999)
    r = torch.randint(1, L + 1, (B,), generator=g, dtype=torch.int64)
    r[0] = L
    return r.to(torch.int32)
