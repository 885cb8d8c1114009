"""Seeded synthetic inputs for Sol-Attn (shared by the CUDA path's tests, the
benchmark and the oracle's tests).

This module only draws random numbers and arranges them into Q, K, V. It holds
none of the attention method's arithmetic, so both sides of a parity test can
use it without sharing any of the method.

Stand-in for the pages' workloads. The pages ("Sol-Attn: Accelerating Video
Generation Inference via On-the-Fly Attention Sparsification", paithon.it,
sections "Perché l'attenzione pesa tanto nei video" and "Una soglia per ogni
riga") measure trained video diffusion transformers (Wan 2.1, HunyuanVideo,
LTX 2.3) whose weights and prompts are not available here. These inputs keep
their shapes: a raster-flattened (t, h, w) latent grid, 64-token blocks, and
spatially correlated queries and keys, so that neighbouring blocks have related
proxy scores as in a real video model:

    E(p)  : d/2 random Fourier frequencies w_f ~ N(0, 0.3^2 I_3), shared by all
            heads; E_f(p) = [cos(w_f . p), sin(w_f . p)], p = integer (t, h, w)
    Q     = 0.8 * E(p) W_q + N(0, 1)
    K     = 0.8 * E(p) W_k + N(0, 1)
    V     = N(0, 1)
    W_q, W_k ~ N(0, 1) / sqrt(d), independent per head

Everything is drawn in fp32 from torch CPU generators and cast to bf16 with
round-to-nearest-even. Head h of batch b draws from its own generator seeded
from (seed, b, h), so any subset of heads can be regenerated on its own.
Token order is raster with w fastest.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import torch

__all__ = ["Workload", "WORKLOADS", "grid_positions", "make_head", "make_qkv"]


@dataclass(frozen=True)
class Workload:
    """One synthetic attention problem: B x H heads over a T x Hs x Ws grid."""

    name: str
    B: int
    H: int
    d: int
    grid: tuple  # (T, Hs, Ws)
    n_tokens: int | None = None  # take the first n raster tokens (sweep); None = whole grid

    @property
    def N(self) -> int:
        T, Hs, Ws = self.grid
        full = T * Hs * Ws
        return full if self.n_tokens is None else min(full, self.n_tokens)


# Shapes of the pages' workloads (720p Wan2.1 latent grid 21x45x80, HunyuanVideo
# 33x45x80), plus small cases a CPU reference finishes in seconds.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, (4, 16, 32)),
    "mid": Workload("mid", 1, 8, 128, (8, 32, 32)),
    "wan_75k": Workload("wan_75k", 1, 40, 128, (21, 45, 80)),
    "hunyuan_119k": Workload("hunyuan_119k", 1, 24, 128, (33, 45, 80)),
    "sweep_16k": Workload("sweep_16k", 1, 24, 128, (5, 45, 80), 16384),
    "sweep_32k": Workload("sweep_32k", 1, 24, 128, (10, 45, 80), 32768),
    "sweep_64k": Workload("sweep_64k", 1, 24, 128, (19, 45, 80), 65536),
    "sweep_128k": Workload("sweep_128k", 1, 24, 128, (37, 45, 80), 131072),
}


def grid_positions(grid, n_tokens=None) -> torch.Tensor:
    """Integer (t, h, w) of every token in raster order (w fastest), fp32 [N, 3]."""
    T, Hs, Ws = grid
    t = torch.arange(T, dtype=torch.float32)
    h = torch.arange(Hs, dtype=torch.float32)
    w = torch.arange(Ws, dtype=torch.float32)
    tt, hh, ww = torch.meshgrid(t, h, w, indexing="ij")
    p = torch.stack([tt.reshape(-1), hh.reshape(-1), ww.reshape(-1)], dim=1)
    if n_tokens is not None:
        p = p[:n_tokens]
    return p


def _frequencies(seed: int, d: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(int(seed) * 2 + 1)
    return torch.randn(d // 2, 3, generator=g, dtype=torch.float32) * 0.3


def _features(p: torch.Tensor, omega: torch.Tensor) -> torch.Tensor:
    ang = p @ omega.T  # [N, d/2]
    return torch.cat([torch.cos(ang), torch.sin(ang)], dim=1)  # [N, d]


def _head_seed(seed: int, b: int, h: int) -> int:
    return (int(seed) * 1_000_003 + b * 7_919 + h * 104_729 + 17) % (2**62)


def make_head(seed: int, b: int, h: int, d: int, feats: torch.Tensor):
    """Q, K, V (bf16, [N, d]) of head h of batch b; feats = E(p) [N, d] fp32."""
    N = feats.shape[0]
    g = torch.Generator().manual_seed(_head_seed(seed, b, h))
    wq = torch.randn(d, d, generator=g, dtype=torch.float32) / math.sqrt(d)
    wk = torch.randn(d, d, generator=g, dtype=torch.float32) / math.sqrt(d)
    q = torch.randn(N, d, generator=g, dtype=torch.float32)
    k = torch.randn(N, d, generator=g, dtype=torch.float32)
    v = torch.randn(N, d, generator=g, dtype=torch.float32)
    q.add_(0.8 * (feats @ wq))
    k.add_(0.8 * (feats @ wk))
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def make_qkv(wl: Workload, seed: int = 0, heads=None, threads: int = 8):
    """Q, K, V as bf16 CPU tensors [B, H', N, d] for the heads listed in `heads`
    (default: all H heads of every batch; `heads` is a list of (b, h))."""
    if heads is None:
        heads = [(b, h) for b in range(wl.B) for h in range(wl.H)]
    omega = _frequencies(seed, wl.d)
    feats = _features(grid_positions(wl.grid, wl.n_tokens), omega)
    N, d = feats.shape[0], wl.d
    out_shape = (len(heads), N, d)
    q = torch.empty(out_shape, dtype=torch.bfloat16)
    k = torch.empty(out_shape, dtype=torch.bfloat16)
    v = torch.empty(out_shape, dtype=torch.bfloat16)

    def one(idx):
        b, h = heads[idx]
        q[idx], k[idx], v[idx] = make_head(seed, b, h, d, feats)

    if threads > 1 and len(heads) > 1:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(one, range(len(heads))))
    else:
        for i in range(len(heads)):
            one(i)
    if len(heads) == wl.B * wl.H:
        shape = (wl.B, wl.H, N, d)
        return q.view(shape), k.view(shape), v.view(shape)
    return q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0)
