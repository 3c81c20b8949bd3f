"""GPU parity: sa_sparse_attn_bwd (dQ, dK, dV) vs the fp64 oracle.

The CUDA backward takes the CUDA forward's O and LSE as its inputs (as a
training step would); the oracle computes the gradients from q, k, v, dO and
the mask alone, so nothing it uses comes from the CUDA path.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_flash_b200 import build, inputs, ops
from oracle import masked_attention_bwd, masked_attention_bwd_rows
from _parity import check_grad

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    yield
    ops.sa_get_device_status()


def run_bwd(q, k, v, dout, block, mask=None, causal=False):
    """Forward then backward on the GPU; returns (dq, dk, dv) on the host."""
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    B, H, N, d = q.shape
    md = None if mask is None else mask.cuda()
    lse = torch.empty(B, H, N, device="cuda")
    o = ops.sa_sparse_attn_fwd(qd, kd, vd, block, mask=md, lse=lse, causal=causal)
    dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
    ops.sa_sparse_attn_bwd(qd, kd, vd, o, gd, lse, block, mask=md, dq=dq, dk=dk, dv=dv, causal=causal)
    ops.sa_get_device_status()
    return dq.cpu(), dk.cpu(), dv.cpu()


def check_all(got, ref, what):
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        check_grad(g, r, f"{what} {name}")


def test_tiny_dense():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.normal_qkv(wl.B, wl.H, wl.N, wl.d, wl.seed)
    dout = inputs.normal_qkv(wl.B, wl.H, wl.N, wl.d, wl.seed + 1)[0]
    got = run_bwd(q, k, v, dout, wl.block)
    check_all(got, masked_attention_bwd(q, k, v, wl.block, None, dout), "tiny dense")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [64, 128])
def test_ragged_random_mask(d, block):
    """Ragged tail (N = 7 tiles + 40), Bernoulli(0.5) mask, one q-block with no
    kept block and one k-block kept by no q-block: their gradients are zero."""
    B, H, N = 1, 2, 128 * 7 + 40
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=d + block)
    dout = inputs.normal_qkv(B, H, N, d, seed=d + block + 1)[0]
    nb = -(-N // block)
    mask = inputs.bernoulli_block_mask(B, H, nb, nb, 0.5, seed=block)
    mask[:, :, 2, :] = 0
    mask[:, :, :, 5] = 0
    got = run_bwd(q, k, v, dout, block, mask)
    ref = masked_attention_bwd(q, k, v, block, mask, dout)
    check_all(got, ref, f"ragged d={d} block={block}")
    dq, dk, dv = got
    assert torch.all(dq[:, :, 2 * block:3 * block] == 0)
    assert torch.all(dk[:, :, 5 * block:6 * block] == 0) and torch.all(dv[:, :, 5 * block:6 * block] == 0)


@pytest.mark.parametrize("block", [64, 128])
def test_rff_radial_mask(block):
    """Locality inputs (random Fourier features of the grid) under the radial mask."""
    wl = inputs.Workload("br", 1, 2, 128, 6, 10, 24, block, "radial", seed=51)
    q, k, v = inputs.rff_qkv(wl)
    dout = inputs.normal_qkv(1, 2, wl.N, 128, seed=52)[0]
    from oracle import radial_mask
    nb = wl.nblocks
    rm = torch.from_numpy(np.ascontiguousarray(radial_mask(wl.T, wl.Hh, wl.Ww, block))).view(1, 1, nb, nb)
    m = rm.expand(1, 2, nb, nb).contiguous()
    got = run_bwd(q, k, v, dout, block, m)
    check_all(got, masked_attention_bwd(q, k, v, block, m, dout), f"radial block={block}")


def test_uneven_tiles_and_empty_everything():
    """One kv tile kept by every q-tile, one q-tile keeping a single tile, and a
    head whose mask is all zero (every gradient exactly 0)."""
    B, H, N, d, block = 1, 2, 128 * 6, 128, 128
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=61)
    dout = inputs.normal_qkv(B, H, N, d, seed=62)[0]
    nb = N // block
    mask = torch.zeros(B, H, nb, nb, dtype=torch.uint8)
    mask[:, 0, :, 3] = 1
    mask[:, 0, 4, :] = 1
    got = run_bwd(q, k, v, dout, block, mask)
    check_all([g[:, :1] for g in got], [r[:, :1] for r in masked_attention_bwd(q, k, v, block, mask, dout)],
              "uneven head 0")
    for g in got:
        assert torch.all(g[:, 1] == 0)


def test_full_size_480p_sampled_rows():
    """The 480p workload's shape (12 heads, 32,760 tokens, block 64) with a
    seeded Bernoulli(0.87) block mask at the tau mask's density: sampled rows
    of dQ and of dK / dV of the last head against the oracle's row form (the
    oracle visits every query row of the head in fp64: about a minute)."""
    wl = inputs.WORKLOADS["wan13b_480p_tau"]
    q, k, v = inputs.rff_qkv(wl)
    dout = inputs.normal_qkv(wl.B, wl.H, wl.N, wl.d, seed=71)[0]
    nb = wl.nblocks
    mask = inputs.bernoulli_block_mask(wl.B, wl.H, nb, nb, 0.87, seed=72)
    dq, dk, dv = run_bwd(q, k, v, dout, wl.block, mask)
    rows = [0, 1, 63, 64, 4095, 16384, 20001, wl.N - 64, wl.N - 1]
    for h in (wl.H - 1,):
        rq, rk, rv = masked_attention_bwd_rows(q, k, v, wl.block, mask, dout, 0, h, rows, rows, chunk=2048)
        check_grad(dq[0, h, rows], rq, f"480p dQ head {h}")
        check_grad(dk[0, h, rows], rk, f"480p dK head {h}")
        check_grad(dv[0, h, rows], rv, f"480p dV head {h}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [64, 128])
def test_causal_ragged(d, block):
    B, H, N = 1, 2, 128 * 5 + 72
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=d + block + 7)
    dout = inputs.normal_qkv(B, H, N, d, seed=d + block + 8)[0]
    nb = -(-N // block)
    mask = inputs.bernoulli_block_mask(B, H, nb, nb, 0.7, seed=block + 9)
    got = run_bwd(q, k, v, dout, block, mask, causal=True)
    check_all(got, masked_attention_bwd(q, k, v, block, mask, dout, causal=True), f"causal d={d} block={block}")


@pytest.mark.parametrize("layout", ["2d", "3d", "4d"])
def test_batch_two_mask_layouts(layout):
    """B = 2 with the mask given as [Nb, Nb] (broadcast), [H, Nb, Nb] or a full
    [B, H, Nb, Nb] array: the element strides reach the kernels unchanged."""
    B, H, N, d, block = 2, 3, 128 * 4 + 56, 128, 64
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=81)
    dout = inputs.normal_qkv(B, H, N, d, seed=82)[0]
    nb = -(-N // block)
    full = inputs.bernoulli_block_mask(B, H, nb, nb, 0.5, seed=83)
    if layout == "2d":
        m = full[0, 0]
        ref_mask = m.view(1, 1, nb, nb).expand(B, H, nb, nb)
    elif layout == "3d":
        m = full[0]
        ref_mask = m.view(1, H, nb, nb).expand(B, H, nb, nb)
    else:
        m = full
        ref_mask = full
    md = m.cuda()
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    lse = torch.empty(B, H, N, device="cuda")
    o = ops.sa_sparse_attn_fwd(qd, kd, vd, block, mask=md, lse=lse)
    dq, dk, dv = ops.sa_sparse_attn_bwd(qd, kd, vd, o, gd, lse, block, mask=md)
    ops.sa_get_device_status()
    ref = masked_attention_bwd(q, k, v, block, ref_mask.numpy(), dout)
    check_all((dq.cpu(), dk.cpu(), dv.cpu()), ref, f"batch 2 mask {layout}")
