"""Seeded synthetic K / V / q generators, shaped like the paper's models.

This module holds no step of the quantiser or of attention: it only draws
random numbers.  Both the CUDA path and the oracle-based tests take their
inputs from here.

Value recipe (one cache layer):
  K[s, h, t, d] = N(0,1) * f[h, d] * g[s, h, t]
      f[h, d]  per-(layer, kv-head) channel factor, lognormal(0, 1), with a few
               outlier channels multiplied by 15 (chosen per head by a seeded
               draw without replacement, or fixed by the caller)
      g        per-token factor, lognormal(0, sigma_k); the token at absolute
               position 0 is multiplied by 8
  V[s, h, t, d] = N(0,1) * lognormal(0, 0.3) per token
  q[s, hq, d]   = N(0,1)
Values are drawn in fp32 and cast to the requested dtype.
"""
from __future__ import annotations

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def channel_factors(seed: int, num_kv_heads: int, head_dim: int, n_outliers: int,
                    outlier_channels=None, device="cpu") -> torch.Tensor:
    """Per-(kv head, channel) K factor f[h, d] (fp32)."""
    g = _gen(seed, device)
    f = torch.exp(torch.randn(num_kv_heads, head_dim, generator=g, device=device))
    for h in range(num_kv_heads):
        if outlier_channels is not None:
            idx = torch.as_tensor(list(outlier_channels), device=device)
        else:
            idx = torch.randperm(head_dim, generator=g, device=device)[:n_outliers]
        f[h, idx] *= 15.0
    return f


def keys(seed: int, f: torch.Tensor, num_seqs: int, num_tokens: int, sigma_k: float = 0.5,
         first_position: int = 0, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """K of shape [S, Hkv, T, D] for tokens first_position .. first_position+T-1."""
    Hkv, D = f.shape
    g = _gen(seed, device)
    z = torch.randn(num_seqs, Hkv, num_tokens, D, generator=g, device=device)
    tok = torch.exp(sigma_k * torch.randn(num_seqs, Hkv, num_tokens, 1, generator=g, device=device))
    if first_position == 0 and num_tokens > 0:
        tok[:, :, 0] *= 8.0
    z.mul_(f.to(device)[None, :, None, :]).mul_(tok)
    return z.to(dtype)


def values(seed: int, num_seqs: int, num_kv_heads: int, num_tokens: int, head_dim: int,
           dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """V of shape [S, Hkv, T, D]."""
    g = _gen(seed, device)
    z = torch.randn(num_seqs, num_kv_heads, num_tokens, head_dim, generator=g, device=device)
    z.mul_(torch.exp(0.3 * torch.randn(num_seqs, num_kv_heads, num_tokens, 1, generator=g, device=device)))
    return z.to(dtype)


def queries(seed: int, num_seqs: int, num_q_heads: int, head_dim: int, dtype=torch.bfloat16,
            device="cpu") -> torch.Tensor:
    """q of shape [S, Hq, D]."""
    g = _gen(seed, device)
    return torch.randn(num_seqs, num_q_heads, head_dim, generator=g, device=device).to(dtype)


def layer_kv(seed: int, layer: int, num_seqs: int, num_kv_heads: int, num_tokens: int, head_dim: int,
             n_outliers: int = 4, sigma_k: float = 0.5, outlier_channels=None, first_position: int = 0,
             dtype=torch.bfloat16, device="cpu"):
    """(K, V) for one layer; every (seed, layer, first_position) triple draws independent numbers."""
    base = (int(seed) * 1_000_003 + int(layer) * 7919) & 0x7FFFFFFF
    f = channel_factors(base, num_kv_heads, head_dim, n_outliers, outlier_channels, device=device)
    k = keys(base + 1 + 2 * first_position, f, num_seqs, num_tokens, sigma_k, first_position, dtype, device)
    v = values(base + 2 + 2 * first_position, num_seqs, num_kv_heads, num_tokens, head_dim, dtype, device)
    return k, v


def common_component_kv(seed: int, kind: str, num_seqs: int, num_kv_heads: int, num_tokens: int, head_dim: int,
                        amount: float, channel: int = 0, dtype=torch.bfloat16, device="cpu"):
    """(K, V) whose tokens share a large common part, each [S, Hkv, T, D].

    kind "identical": every token of a (sequence, kv head) is one random token x (N(0,1) times a lognormal(0,1)
    channel factor) plus amount * N(0,1) per element (amount 0: exact copies).
    kind "dc": N(0,1) per element with `amount` added to channel `channel` of every token.
    kind "offset": `amount` + N(0,1) in every element (every row and column has mean/std = amount).
    K and V use independent draws of the same recipe.
    """
    g = _gen(seed, device)
    out = []
    for _ in range(2):
        shape = (num_seqs, num_kv_heads, num_tokens, head_dim)
        if kind == "identical":
            x = torch.randn(num_seqs, num_kv_heads, 1, head_dim, generator=g, device=device)
            x = x * torch.exp(torch.randn(num_seqs, num_kv_heads, 1, head_dim, generator=g, device=device))
            z = x.expand(shape) + amount * torch.randn(shape, generator=g, device=device)
        elif kind == "dc":
            z = torch.randn(shape, generator=g, device=device)
            z[..., channel] += amount
        elif kind == "offset":
            z = amount + torch.randn(shape, generator=g, device=device)
        else:
            raise ValueError(kind)
        out.append(z.contiguous().to(dtype))
    return out[0], out[1]
