"""Small, self-contained launches of each kernel, for profiler captures.

    python -m block_sparse_attention_flash_b200.profile_case attn   [--heads 4] [--reps 2]
    python -m block_sparse_attention_flash_b200.profile_case tau    [--heads 12] [--reps 2]
    python -m block_sparse_attention_flash_b200.profile_case radial [--reps 2]
    python -m block_sparse_attention_flash_b200.profile_case mask   [--heads 12] [--reps 2]
    python -m block_sparse_attention_flash_b200.profile_case pool   [--heads 12] [--reps 2]
    python -m block_sparse_attention_flash_b200.profile_case pyr    [--heads 2] [--reps 2]
    python -m block_sparse_attention_flash_b200.profile_case bwd    [--heads 2] [--reps 2]
    python -m block_sparse_attention_flash_b200.profile_case perm   [--heads 12] [--reps 2]

Each case uses a workload's real token grid with fewer heads, so one launch
holds a few hundred MB (larger than L2) and a full profiler capture ends in
seconds.  Inputs are drawn on the device from the seeded generator.
  attn    75,600-token LiteAttention grid (block 128, d 128), all kept, skip update on
  tau     32,760-token 480p grid (block 64, d 128): the tau = 0.9 mask, then the attention
  radial  118,800-token HunyuanVideo-like grid, block 128
  mask    32,760-token 480p grid, block 64, tau = 0.9
  pool    32,760-token 480p grid, block 64
  pyr     32,760-token 480p grid, block 64, PSA levels from the GPU level builder
  bwd     32,760-token 480p grid, block 64, all kept: forward once, then the backward
  perm    32,760-token 480p grid: Q, K, V permuted in one launch (per-head orders, 3x5x4 cells)
"""
from __future__ import annotations

import argparse

import torch

from . import build, inputs, ops


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["attn", "tau", "radial", "mask", "pool", "pyr", "bwd", "perm"])
    ap.add_argument("--heads", type=int, default=0)
    ap.add_argument("--reps", type=int, default=2)
    args = ap.parse_args()
    build.build()
    ops.lib()
    dev = torch.device("cuda", 0)
    if args.case == "attn":
        wl = inputs.WORKLOADS["wan14b_720p_lite"]
        q, k, v = inputs.rff_qkv(wl, H=args.heads or 4, device=dev)
        nb = wl.nblocks
        skip = [torch.zeros(1, q.shape[1], nb, nb, dtype=torch.uint8, device=dev) for _ in range(args.reps + 1)]
        for r in range(args.reps):
            ops.sa_sparse_attn_fwd(q, k, v, wl.block, skip_in=skip[r], skip_out=skip[r + 1], eps=wl.eps)
    elif args.case == "tau":
        wl = inputs.WORKLOADS["wan13b_480p_tau"]
        q, k, v = inputs.rff_qkv(wl, H=args.heads or wl.H, device=dev)
        m = ops.sa_build_mask(q, k, wl.block, "tau", tau=wl.tau)
        o = torch.empty_like(q)
        for _ in range(args.reps):
            ops.sa_sparse_attn_fwd(q, k, v, wl.block, mask=m, out=o)
    elif args.case == "radial":
        wl = inputs.WORKLOADS["hunyuan_720p_radial"]
        for _ in range(args.reps):
            ops.sa_radial_mask(wl.T, wl.Hh, wl.Ww, wl.block)
    elif args.case == "mask":
        wl = inputs.WORKLOADS["wan13b_480p_tau"]
        q, k, _ = inputs.rff_qkv(wl, H=args.heads or wl.H, device=dev)
        for _ in range(args.reps):
            ops.sa_build_mask(q, k, wl.block, "tau", tau=wl.tau)
    elif args.case == "pool":
        wl = inputs.WORKLOADS["psa_480p_pyramid"]
        _, k, v = inputs.rff_qkv(wl, H=args.heads or wl.H, device=dev)
        for _ in range(args.reps):
            ops.sa_pyramid_pool(k, v, wl.block)
    elif args.case == "bwd":
        wl = inputs.WORKLOADS["wan13b_480p_tau"]
        q, k, v = inputs.rff_qkv(wl, H=args.heads or 2, device=dev)
        g = torch.Generator(device=dev).manual_seed(wl.seed + 7)
        dout = torch.randn(q.shape, generator=g, device=dev).to(torch.bfloat16)
        lse = torch.empty(q.shape[:3], device=dev)
        o = ops.sa_sparse_attn_fwd(q, k, v, wl.block, lse=lse)
        for _ in range(args.reps):
            ops.sa_sparse_attn_bwd(q, k, v, o, dout, lse, wl.block)
    elif args.case == "perm":
        wl = inputs.WORKLOADS["wan13b_480p_tau"]
        q, k, v = inputs.rff_qkv(wl, H=args.heads or wl.H, device=dev)
        orders = (torch.arange(q.shape[1], device=dev) % 6).to(torch.uint8)
        for _ in range(args.reps):
            ops.sa_token_permute([q, k, v], wl.T, wl.Hh, wl.Ww, head_order=orders, cells=(3, 5, 4))
    else:
        wl = inputs.WORKLOADS["psa_480p_pyramid"]
        q, k, v = inputs.rff_qkv(wl, H=args.heads or 2, device=dev)
        kp, vp = ops.sa_pyramid_pool(k, v, wl.block)
        lv = ops.sa_build_mask(q, k, wl.block, "levels", level_frac=wl.level_frac)
        for _ in range(args.reps):
            ops.sa_pyramid_attn_fwd(q, k, v, wl.block, lv, kp, vp)
    ops.sa_get_device_status()
    print(f"profile case {args.case}: ok")


if __name__ == "__main__":
    main()
