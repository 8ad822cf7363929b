"""Seeded synthetic Q/K/V generators for the block-sparse attention workloads.

This module holds no part of the attention method: it only draws inputs. Both the
CUDA path (tests, bench) and the CPU oracle consume what it produces, so it sits
apart from either.

The shapes stand in for the video DiTs the pages measure on (Wan 2.2 / Wan2.1-14B /
HunyuanVideo-13B latents, "Training-free sparse attention based on cumulative
energy filtering", results paragraph; iCATS abstract), whose weights and prompts
are not available: tokens of a T x H x W latent grid are clustered into
spatio-temporal patches, and each token's Q and K lean towards its patch centroid,
which gives the block-local attention structure those models show.

Recipe (every detail below is fixed here, not on the pages):
  * token order is raster (t, y, x) with x fastest;
  * cluster of token (t, y, x) = (t // pt, y // py, x // px);
  * per (b, h) an independent generator seeded with seed*1000 + b*100 + h;
  * draw order: centroids [n_clusters, d], Q noise [N, d], K noise [N, d], V [N, d],
    then (only if noise_frac > 0) one uniform [N] used to pick pure-noise tokens;
  * Q = w*c + 0.7*zq, K = w*c + 0.7*zk, V = zv  (w = centroid weight);
  * pure-noise tokens (noise_frac of them) take Q = zq, K = zk (no centroid);
  * language-shaped workload: Q = zq + pe, K = zk + pe with
    pe[t, c] = amp*sin(2*pi*t/period + 2*pi*c/d); then K[0] += 4*mean_t(Q[t]);
  * values are drawn in fp32 and rounded once to bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional, Sequence, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    N: int
    causal: bool
    kind: str  # "video" | "lm"
    grid: Optional[Tuple[int, int, int]] = None
    patch: Optional[Tuple[int, int, int]] = None
    centroid_weight: float = 1.5
    noise_frac: float = 0.0
    pe_period: int = 512
    pe_amp: float = 1.0
    sink_gain: float = 4.0
    taus: Tuple[float, ...] = (0.95,)
    lams: Tuple[Optional[float], ...] = (None,)
    centroid_weights: Tuple[float, ...] = ()

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _video(name, H, D, grid, patch, **kw):
    t, y, x = grid
    return Workload(name=name, B=1, H=H, D=D, N=t * y * x, causal=False, kind="video",
                    grid=grid, patch=patch, **kw)


# The five workloads the measurements are quoted on (sizes as stated with them).
WORKLOADS = {
    "tiny": _video("tiny", 2, 64, (4, 16, 16), (2, 4, 4), taus=(0.95,), lams=(None,)),
    "small": _video("small", 24, 128, (16, 16, 16), (2, 4, 4),
                    taus=(0.90, 0.95, 0.99), lams=(None, -12.0)),
    "wan": _video("wan", 40, 128, (21, 45, 80), (3, 5, 5), noise_frac=0.05,
                  taus=(0.95,), lams=(None,)),
    "hunyuan": _video("hunyuan", 24, 128, (33, 45, 80), (3, 5, 5),
                      taus=(0.90, 0.95), lams=(-12.0,), centroid_weights=(0.5, 1.5, 3.0)),
    "lm": Workload(name="lm", B=1, H=32, D=128, N=32768, causal=True, kind="lm",
                   taus=(0.95,), lams=(None,)),
}


def head_seed(seed: int, b: int, h: int) -> int:
    return seed * 1000 + b * 100 + h


def _cluster_ids(grid, patch, device):
    T, Y, X = grid
    pt, py, px = patch
    t = torch.arange(T, device=device).view(T, 1, 1)
    y = torch.arange(Y, device=device).view(1, Y, 1)
    x = torch.arange(X, device=device).view(1, 1, X)
    ny = -(-Y // py)
    nx = -(-X // px)
    cid = ((t // pt) * ny + (y // py)) * nx + (x // px)
    n_clusters = (-(-T // pt)) * ny * nx
    return cid.reshape(-1), n_clusters


def generate(w: Workload, seed: int = 0, device="cpu", heads: Optional[Sequence[int]] = None,
             centroid_weight: Optional[float] = None):
    """Return (Q, K, V) bf16 tensors of shape [B, H', N, D] on `device`.

    `heads` restricts generation to a subset of heads (same values as the full
    tensor's heads, since each head has its own seeded stream)."""
    device = torch.device(device)
    heads = list(range(w.H)) if heads is None else list(heads)
    cw = w.centroid_weight if centroid_weight is None else centroid_weight
    N, D = w.N, w.D
    Q = torch.empty((w.B, len(heads), N, D), dtype=torch.bfloat16, device=device)
    K = torch.empty_like(Q)
    V = torch.empty_like(Q)
    if w.kind == "video":
        cid, n_clusters = _cluster_ids(w.grid, w.patch, device)
        assert cid.numel() == N
    else:
        t = torch.arange(N, device=device, dtype=torch.float64).view(N, 1)
        c = torch.arange(D, device=device, dtype=torch.float64).view(1, D)
        pe = (w.pe_amp * torch.sin(2 * math.pi * t / w.pe_period + 2 * math.pi * c / D)).float()
    for b in range(w.B):
        for hi, h in enumerate(heads):
            g = torch.Generator(device=device)
            g.manual_seed(head_seed(seed, b, h))
            if w.kind == "video":
                cent = torch.randn((n_clusters, D), generator=g, device=device)
                zq = torch.randn((N, D), generator=g, device=device)
                zk = torch.randn((N, D), generator=g, device=device)
                zv = torch.randn((N, D), generator=g, device=device)
                c = cent[cid]
                q = cw * c + 0.7 * zq
                k = cw * c + 0.7 * zk
                if w.noise_frac > 0:
                    u = torch.rand((N,), generator=g, device=device)
                    noisy = (u < w.noise_frac).view(N, 1)
                    q = torch.where(noisy, zq, q)
                    k = torch.where(noisy, zk, k)
            else:
                zq = torch.randn((N, D), generator=g, device=device)
                zk = torch.randn((N, D), generator=g, device=device)
                zv = torch.randn((N, D), generator=g, device=device)
                q = zq + pe
                k = zk + pe
                k[0] += w.sink_gain * q.mean(dim=0)
            Q[b, hi] = q.to(torch.bfloat16)
            K[b, hi] = k.to(torch.bfloat16)
            V[b, hi] = zv.to(torch.bfloat16)
    return Q, K, V


def random_qkv(B, H, N, D, seed=0, device="cpu", scale_qk=1.0):
    """Plain i.i.d. N(0,1) inputs (bf16) for edge-case tests of arbitrary shape."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    shape = (B, H, N, D)
    Q = (scale_qk * torch.randn(shape, generator=g, device=device)).to(torch.bfloat16)
    K = (scale_qk * torch.randn(shape, generator=g, device=device)).to(torch.bfloat16)
    V = torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
    return Q, K, V
