"""Seeded synthetic looped-Transformer K/V and queries (harness only).

This module draws random numbers and nothing else: it holds none of the
method's arithmetic and serves both the CUDA path (as device inputs) and the
oracle (the exact BF16 arrays are copied back to the host).

Recipe (shapes and structure of the pages' workloads; Ouro-1.4B: 24 layers,
4 loops; Huginn-3.5B: 32 loops in 8 groups of 4):
  * anchor loop (last loop of a group) K/V ~ N(0, 1) per element, with 4
    distinct seeded outlier channels per (layer, group, kv head, K|V) scaled
    by 10;
  * a loop at distance k from its group's anchor is c * anchor + sigma_k *
    N(0, 1) with c ~ U(0.8, 1.2) drawn per (layer, loop, sequence, token,
    head, K|V) and sigma_k from the configuration (Ouro-shaped:
    0.1/0.2/0.3 for distance 1/2/3; deep-recurrence shape: 0.1/0.25/0.4);
  * queries ~ N(0, 1).
Everything is generated in fp32 with torch's seeded generators on the
requested device and rounded to BF16.
"""
from __future__ import annotations

import torch

_M64 = (1 << 64) - 1


def mix_seed(*vals: int) -> int:
    """Deterministic 63-bit seed from integers (a splitmix-style hash)."""
    z = 0x243F6A8885A308D3
    for v in vals:
        z = (z + (int(v) & _M64) + 0x9E3779B97F4A7C15) & _M64
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
        z ^= z >> 31
    return z & ((1 << 63) - 1)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


K, V = 0, 1


def outlier_channels(seed: int, layer: int, group: int, head: int, kv: int, d: int = 128) -> torch.Tensor:
    g = _gen("cpu", mix_seed(seed, 1, layer, group, head, kv))
    return torch.randperm(d, generator=g)[:4]


def anchor_kv(seed: int, layer: int, group: int, kv: int, B: int, T: int, H: int, d: int = 128,
              t0: int = 0, device="cuda") -> torch.Tensor:
    """fp32 [B][T][H][d] anchor values for tokens t0..t0+T-1."""
    g = _gen(device, mix_seed(seed, 2, layer, group, kv, t0))
    x = torch.randn((B, T, H, d), generator=g, device=device, dtype=torch.float32)
    scale = torch.ones((H, d), device=device)
    for h in range(H):
        scale[h, outlier_channels(seed, layer, group, h, kv, d).to(device)] = 10.0
    return x * scale


def loop_kv(anchor: torch.Tensor, seed: int, layer: int, loop: int, kv: int, sigma: float,
            t0: int = 0) -> torch.Tensor:
    """fp32 c * anchor + sigma * N(0, 1), c ~ U(0.8, 1.2) per (b, t, h)."""
    B, T, H, d = anchor.shape
    g = _gen(anchor.device, mix_seed(seed, 3, layer, loop, kv, t0))
    c = 0.8 + 0.4 * torch.rand((B, T, H, 1), generator=g, device=anchor.device)
    noise = torch.randn((B, T, H, d), generator=g, device=anchor.device)
    return c * anchor + sigma * noise


def group_kv(seed: int, layer: int, group: int, Lg: int, sigma_by_distance, B: int, T: int, H: int,
             d: int = 128, t0: int = 0, device="cuda"):
    """BF16 K and V of one loop group: two lists of Lg tensors [B][T][H][d]
    (index j = loop within the group; j = Lg-1 is the anchor)."""
    out = [[None] * Lg, [None] * Lg]
    for kv in (K, V):
        a = anchor_kv(seed, layer, group, kv, B, T, H, d, t0, device)
        out[kv][Lg - 1] = a.to(torch.bfloat16)
        for j in range(Lg - 1):
            dist = Lg - 1 - j
            x = loop_kv(a, seed, layer, group * Lg + j, kv, sigma_by_distance[dist - 1], t0)
            out[kv][j] = x.to(torch.bfloat16)
    return out[K], out[V]


def queries(seed: int, layer: int, loop: int, step: int, B: int, Hq: int, d: int = 128,
            device="cuda") -> torch.Tensor:
    g = _gen(device, mix_seed(seed, 4, layer, loop, step))
    return torch.randn((B, Hq, d), generator=g, device=device).to(torch.bfloat16)


def bf16_to_u16(t: torch.Tensor):
    """BF16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
