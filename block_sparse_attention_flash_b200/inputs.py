"""Seeded synthetic inputs for block-sparse video attention.

This module is input plumbing only: it draws the tensors that both the CUDA
path and the CPU oracle consume, and holds none of the method's arithmetic
(no pooling, no scores, no softmax, no masks derived from data).  Every
tensor is produced on the CPU from an explicit seed with ``torch.Generator``
so that both sides receive bit-identical bf16 inputs.

Token order is raster (t, h, w): token n = (t*Hh + h)*Ww + w, which is how a
video DiT flattens its (frame x height x width) latent grid (VMoBA page,
"hierarchical cyclic blocking" paragraph, describes the same 3D grid).

Locality generator ("random Fourier features of the grid position"):
per head, D = 256 features phi_k(t,h,w) = sqrt(2/D) cos(w_k.(t,h,w) + b_k)
with w_t ~ N(0, 1/sigma_t^2), w_h, w_w ~ N(0, 1/sigma_s^2), b_k ~ U[0, 2pi);
L = phi @ W with W ~ N(0,1)^{D x d}, so each entry of L has unit variance.
Q = 0.7 L + 0.3 xi_Q, K = 0.7 L + 0.3 xi_K (same L, so nearby tokens attend
to each other), V ~ N(0,1).  Everything is rounded to bf16 at the end.

Denoising drift for the LiteAttention chain: x_{s+1} = bf16(0.98 x_s + 0.2 xi_s)
computed in fp32 from the bf16 x_s.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

RFF_FEATURES = 256


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic video-attention workload (shapes follow the pages' models)."""

    name: str
    B: int
    H: int
    d: int
    T: int
    Hh: int
    Ww: int
    block: int
    kind: str  # "tiny" | "tau" | "radial" | "lite" | "pyramid"
    seed: int
    tau: float = 0.9
    eps: float = 10.0
    steps: int = 1
    level_frac: tuple = (0.1, 0.3, 0.6)
    sigma_t: float = 2.0
    sigma_s: float = 4.0

    @property
    def N(self) -> int:
        return self.T * self.Hh * self.Ww

    @property
    def nblocks(self) -> int:
        return -(-self.N // self.block)


# The five workloads: a tiny parity case and four video-shaped cases whose
# grids match the token counts the pages quote for 480p/720p generation.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, 4, 8, 16, 64, "tiny", seed=1234),
    "wan13b_480p_tau": Workload("wan13b_480p_tau", 1, 12, 128, 21, 30, 52, 64, "tau", seed=2024, tau=0.9),
    "hunyuan_720p_radial": Workload("hunyuan_720p_radial", 1, 24, 128, 33, 45, 80, 128, "radial", seed=3033),
    "wan14b_720p_lite": Workload("wan14b_720p_lite", 1, 40, 128, 21, 45, 80, 128, "lite", seed=4044, eps=10.0, steps=50),
    "psa_480p_pyramid": Workload("psa_480p_pyramid", 1, 12, 128, 21, 30, 52, 64, "pyramid", seed=5055),
}


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def grid_coords(T: int, Hh: int, Ww: int) -> torch.Tensor:
    """(N, 3) float32 tensor of (t, h, w) for raster token order."""
    t = torch.arange(T, dtype=torch.float32).view(T, 1, 1).expand(T, Hh, Ww)
    h = torch.arange(Hh, dtype=torch.float32).view(1, Hh, 1).expand(T, Hh, Ww)
    w = torch.arange(Ww, dtype=torch.float32).view(1, 1, Ww).expand(T, Hh, Ww)
    return torch.stack([t, h, w], dim=-1).reshape(-1, 3)


def rff_qkv(wl: Workload, B: Optional[int] = None, H: Optional[int] = None, device="cpu"):
    """Q, K, V bf16 [B, H, N, d] from the locality generator of ``wl``.

    Heads are drawn in order from one generator, so a run with fewer heads
    (H smaller than wl.H) yields exactly the first H heads of the full draw.
    ``device="cuda"`` draws the same recipe with torch's CUDA generator (fast,
    used for full-size timing runs); its values differ from the CPU draw, and
    any oracle check of such inputs copies them to the host first.
    """
    B = wl.B if B is None else B
    H = wl.H if H is None else H
    N, d, D = wl.N, wl.d, RFF_FEATURES
    coords = grid_coords(wl.T, wl.Hh, wl.Ww).to(device)
    g = _gen(wl.seed, device)
    q = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    sig = torch.tensor([wl.sigma_t, wl.sigma_s, wl.sigma_s], dtype=torch.float32, device=device)
    for b in range(B):
        for h in range(H):
            omega = torch.randn(3, D, generator=g, device=device) / sig.view(3, 1)
            phase = torch.rand(D, generator=g, device=device) * (2.0 * math.pi)
            W = torch.randn(D, d, generator=g, device=device)
            phi = torch.cos(coords @ omega + phase) * math.sqrt(2.0 / D)
            L = phi @ W
            q[b, h] = (0.7 * L + 0.3 * torch.randn(N, d, generator=g, device=device)).to(torch.bfloat16)
            k[b, h] = (0.7 * L + 0.3 * torch.randn(N, d, generator=g, device=device)).to(torch.bfloat16)
            v[b, h] = torch.randn(N, d, generator=g, device=device).to(torch.bfloat16)
    return q, k, v


def normal_qkv(B: int, H: int, N: int, d: int, seed: int):
    """i.i.d. N(0,1) Q, K, V in bf16 (the tiny parity case's distribution)."""
    g = _gen(seed)
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g).to(torch.bfloat16)
    k = torch.randn(shape, generator=g).to(torch.bfloat16)
    v = torch.randn(shape, generator=g).to(torch.bfloat16)
    return q, k, v


def bernoulli_block_mask(B: int, H: int, nqb: int, nkb: int, p: float, seed: int,
                         force_diagonal: bool = True) -> torch.Tensor:
    """uint8 [B, H, nqb, nkb] Bernoulli(p) block mask; optionally keep (i, i)."""
    g = _gen(seed)
    m = (torch.rand(B, H, nqb, nkb, generator=g) < p).to(torch.uint8)
    if force_diagonal:
        n = min(nqb, nkb)
        idx = torch.arange(n)
        m[:, :, idx, idx] = 1
    return m


def drift(x: torch.Tensor, g: torch.Generator) -> torch.Tensor:
    """One denoising-drift step x -> bf16(0.98 x + 0.2 xi), xi ~ N(0,1)."""
    xi = torch.randn(x.shape, generator=g, device=x.device)
    return (0.98 * x.float() + 0.2 * xi).to(torch.bfloat16)


def lite_chain_inputs(wl: Workload, steps: int, H: Optional[int] = None):
    """Yield (q, k, v) for denoising steps 0..steps-1 of the LiteAttention chain.

    Step 0 is the locality draw; each later step applies ``drift`` to Q, K and V
    with noise from a second seeded generator (seed + 1).
    """
    q, k, v = rff_qkv(wl, H=H)
    g = _gen(wl.seed + 1)
    for s in range(steps):
        yield q, k, v
        if s + 1 < steps:
            q, k, v = drift(q, g), drift(k, g), drift(v, g)


def const_group_kv(B: int, H: int, N: int, d: int, group: int, seed: int):
    """K, V bf16 that are constant over every run of ``group`` consecutive tokens.

    Used by the pyramid exactness check: pooling such K/V changes nothing, so a
    distribution-preserving pyramid attention must equal dense attention.
    """
    g = _gen(seed)
    ng = -(-N // group)
    kg = torch.randn(B, H, ng, d, generator=g)
    vg = torch.randn(B, H, ng, d, generator=g)
    k = kg.repeat_interleave(group, dim=2)[:, :, :N].to(torch.bfloat16)
    v = vg.repeat_interleave(group, dim=2)[:, :, :N].to(torch.bfloat16)
    return k, v
