"""Seeded synthetic inputs for the sparse-attention path.

This module draws random tensors and lays them out; it holds none of the method's
arithmetic (no pooling, scoring, selection or attention).  The CUDA path and the CPU
oracle both take their inputs from here, and parity always feeds the oracle the exact
bf16 bits the GPU consumed.

Workloads are shaped like the 480p / 720p latent grids of a 14B video DiT and a
122,880-token long-sequence case, with Q/K correlated through a positional signal so
that the block-mean scores carry structure (as real attention maps do):

    f(t,h,w) = [sin 2pi t/T, cos 2pi t/T, sin 2pi h/Hg, cos 2pi h/Hg, sin 2pi w/W, cos 2pi w/W]
    W_h      ~ N(0, 1/d) entries, 6 x d, one per head, shared by Q and K
    Q        = 0.5 * f @ W_h + N(0,1) noise
    K        = 0.5 * f @ W_h + N(0,1) noise   (independent noise)
    V        ~ N(0,1)
    tokens t >= L (padding up to a multiple of the block) are 0
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads: int
    grid: tuple  # (T, Hg, W) latent token grid; L = T*Hg*W
    head_dim: int
    block: int
    keep: float
    kind: str = "positional"  # "positional" or "normal"

    @property
    def seq_len(self) -> int:
        T, Hg, W = self.grid
        return T * Hg * W

    @property
    def seq_len_padded(self) -> int:
        return -(-self.seq_len // self.block) * self.block

    @property
    def num_blocks(self) -> int:
        return self.seq_len_padded // self.block


WORKLOADS = {
    # 1 batch, 2 heads, d=64, 1024 tokens in 16 blocks of 64, keep 25% (4 blocks)
    "tiny": Workload("tiny", 1, 2, (1, 1, 1024), 64, 64, 0.25, kind="normal"),
    # 480p latent grid 21x30x52 = 32,760 tokens (padded to 32,768), keep 20%
    "480p": Workload("480p", 1, 40, (21, 30, 52), 128, 128, 0.20),
    # 720p latent grid 21x45x80 = 75,600 tokens (padded to 75,648), keep 15%
    "720p": Workload("720p", 1, 40, (21, 45, 80), 128, 128, 0.15),
    # long-sequence case: 24x64x80 = 122,880 tokens, 960 blocks, keep 10%
    "long122880": Workload("long122880", 1, 40, (24, 64, 80), 128, 128, 0.10),
}


def sweep_workload(keep: float) -> Workload:
    """L = 32,768 tokens (grid 32x32x32), block 128, 40 heads, d=128 at a given keep."""
    return Workload(f"sweep_keep{int(round(keep * 100))}", 1, 40, (32, 32, 32), 128, 128, keep)


def _gen(device, *ids) -> torch.Generator:
    seed = 0
    for x in ids:
        seed = (seed * 1000003 + int(x)) % (2 ** 62)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def positional_features(grid, device="cpu") -> torch.Tensor:
    """[L, 6] float32 sin/cos features of each token's (t, h, w) grid position."""
    T, Hg, W = grid
    idx = torch.arange(T * Hg * W, device=device, dtype=torch.int64)
    t = (idx // (Hg * W)).to(torch.float64)
    h = ((idx // W) % Hg).to(torch.float64)
    w = (idx % W).to(torch.float64)
    two_pi = 2.0 * math.pi
    f = torch.stack([torch.sin(two_pi * t / T), torch.cos(two_pi * t / T),
                     torch.sin(two_pi * h / Hg), torch.cos(two_pi * h / Hg),
                     torch.sin(two_pi * w / W), torch.cos(two_pi * w / W)], dim=-1)
    return f.to(torch.float32)


def make_qkv(wl: Workload, seed: int = 0, device="cpu", dtype=torch.bfloat16):
    """Q, K, V as [B, H, Lp, d] tensors of ``dtype`` on ``device``."""
    B, H, d = wl.batch, wl.heads, wl.head_dim
    L, Lp = wl.seq_len, wl.seq_len_padded
    q = torch.zeros(B, H, Lp, d, dtype=dtype, device=device)
    k = torch.zeros_like(q)
    v = torch.zeros_like(q)
    f = positional_features(wl.grid, device) if wl.kind == "positional" else None
    for b in range(B):
        for h in range(H):
            if wl.kind == "positional":
                w_h = torch.randn(6, d, generator=_gen(device, seed, 0, h), device=device) / math.sqrt(d)
                pos = 0.5 * (f @ w_h)
                q[b, h, :L] = (pos + torch.randn(L, d, generator=_gen(device, seed, 1, b, h), device=device)).to(dtype)
                k[b, h, :L] = (pos + torch.randn(L, d, generator=_gen(device, seed, 2, b, h), device=device)).to(dtype)
            else:
                q[b, h, :L] = torch.randn(L, d, generator=_gen(device, seed, 1, b, h), device=device).to(dtype)
                k[b, h, :L] = torch.randn(L, d, generator=_gen(device, seed, 2, b, h), device=device).to(dtype)
            v[b, h, :L] = torch.randn(L, d, generator=_gen(device, seed, 3, b, h), device=device).to(dtype)
    return q, k, v


def random_qkv(B, H, Lp, d, L=None, seed=0, device="cpu", dtype=torch.bfloat16, q_scale=1.0):
    """Plain N(0,1) tensors [B,H,Lp,d]; tokens t >= L zeroed.  For parity edge cases."""
    L = Lp if L is None else L
    out = []
    for tid in range(3):
        x = torch.randn(B, H, Lp, d, generator=_gen(device, seed, 10 + tid), device=device)
        if tid == 0:
            x = x * q_scale
        x[:, :, L:] = 0
        out.append(x.to(dtype))
    return tuple(out)


def bf16_bits(x: torch.Tensor):
    """A bf16 tensor's raw 16-bit patterns as a numpy uint16 array (host copy)."""
    assert x.dtype == torch.bfloat16
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
