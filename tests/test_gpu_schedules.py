"""GPU parity for the hand-off schedules of the attention and pyramid kernels.

A CTA owns two 128-row q-tiles that share one S buffer in turn; these masks
make the sequence of S computations uneven: one q-tile of a pair with no kept
tile at all, the two q-tiles keeping disjoint kv tiles (every S belongs to one
q-tile, so consecutive S may belong to the same one), and one q-tile keeping a
single tile while the other keeps all.  All are compared with the fp64 oracle.
"""
import math

import pytest
import torch

from block_sparse_attention_flash_b200 import build, inputs, ops
from oracle import masked_attention, pyramid_attention
from _parity import check_o, check_lse

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    yield
    ops.sa_get_device_status()


def run_attn(q, k, v, block, mask):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    B, H, N, d = q.shape
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    ops.sa_sparse_attn_fwd(qd, kd, vd, block, mask=mask.cuda(), out=out, lse=lse)
    ops.sa_get_device_status()
    return out.cpu(), lse.cpu()


def uneven_masks(nb, qpt, seed):
    """Masks over nb x nb blocks (qpt q-blocks per 128-row q-tile), one per pattern."""
    g = torch.Generator().manual_seed(seed)
    ntile = -(-nb // qpt)
    pats = {}
    m = (torch.rand(nb, nb, generator=g) < 0.5).to(torch.uint8)
    for t in range(0, ntile, 2):            # q-tile 0 of every pair keeps nothing
        m[t * qpt:(t + 1) * qpt] = 0
    pats["first_tile_empty"] = m
    m = (torch.rand(nb, nb, generator=g) < 0.5).to(torch.uint8)
    for t in range(1, ntile, 2):            # q-tile 1 of every pair keeps nothing
        m[t * qpt:(t + 1) * qpt] = 0
    pats["second_tile_empty"] = m
    m = torch.zeros(nb, nb, dtype=torch.uint8)
    for t in range(ntile):                   # the pair's q-tiles keep disjoint kv tiles
        for j in range(nb):
            if ((j // qpt) + t) % 2 == 0 and torch.rand(1, generator=g).item() < 0.7:
                m[t * qpt:(t + 1) * qpt, j] = 1
    pats["disjoint"] = m
    m = torch.ones(nb, nb, dtype=torch.uint8)
    for t in range(0, ntile, 2):            # q-tile 0 keeps a single kv block
        m[t * qpt:(t + 1) * qpt] = 0
        m[t * qpt:(t + 1) * qpt, (3 * t) % nb] = 1
    pats["one_vs_all"] = m
    return pats


@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("pattern", ["first_tile_empty", "second_tile_empty", "disjoint", "one_vs_all"])
def test_attention_uneven_pairs(block, pattern):
    B, H, N, d = 1, 2, 128 * 7 + 40, 128   # 8 q-tiles: four pairs, the last one ragged
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=block + len(pattern))
    nb = -(-N // block)
    mask = uneven_masks(nb, 128 // block, seed=block * 31 + len(pattern))[pattern]
    m = mask.view(1, 1, nb, nb).expand(B, H, nb, nb).contiguous()
    O, L = run_attn(q, k, v, block, m)
    Or, Lr = masked_attention(q, k, v, block, m)
    check_o(O, Or, f"{pattern} block={block}")
    check_lse(L, Lr, f"{pattern} block={block}")


@pytest.mark.parametrize("block", [64, 128])
def test_pyramid_unbalanced_tiles(block):
    """One q-tile of each pair at level 0 everywhere (many packed key tiles), the
    other at level 3 on a few blocks (one or two), one q-tile with nothing."""
    B, H, N, d = 1, 2, 128 * 6 + 24, 128
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=block + 5)
    nb = -(-N // block)
    qpt = 128 // block
    codes = torch.zeros(B, H, nb, nb, dtype=torch.uint8)
    ntile = -(-nb // qpt)
    for t in range(ntile):
        rows = slice(t * qpt, min(nb, (t + 1) * qpt))
        if t % 2 == 0:
            codes[:, :, rows, :] = 1                       # level 0, all blocks
        elif t != 3:
            codes[:, :, rows, (t * 5) % nb] = 4            # level 3, a single block
            codes[:, :, rows, (t * 5 + 2) % nb] = 4
    kd, vd = k.cuda(), v.cuda()
    kp, vp = ops.sa_pyramid_pool(kd, vd, block)
    out = torch.full_like(kd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    ops.sa_pyramid_attn_fwd(q.cuda(), kd, vd, block, codes.cuda(), kp, vp, out=out, lse=lse)
    ops.sa_get_device_status()
    Or, Lr = pyramid_attention(q, k, v, block, codes.numpy())
    check_o(out.cpu(), Or, f"pyramid unbalanced block={block}")
    check_lse(lse.cpu(), Lr, f"pyramid unbalanced block={block}")
    rows3 = slice(3 * 128, 4 * 128)                        # q-tile 3 keeps nothing
    assert torch.all(out.cpu()[:, :, rows3] == 0) and torch.all(lse.cpu()[:, :, rows3] == -math.inf)


@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("kernel", ["attention", "pyramid"])
def test_tail_wave_split_is_bit_identical(block, kernel):
    """A launch whose last wave would hold at most half of the SMs runs the
    pairs of that wave as two CTAs each, one per q-tile.  With 148 SMs: 20
    heads of 9 q-tiles (5 pairs each, the last one ragged) make 100 pairs, a
    last wave of more than half the SMs, so no pair is split; the first 3
    heads alone (15 pairs) are all split.  The same heads must give
    bit-identical O, LSE and skip bits both ways, and match the oracle."""
    H, N, d = 20, 128 * 8 + 40, 128
    q, k, v = inputs.normal_qkv(1, H, N, d, seed=block + 91)
    nb = -(-N // block)
    g = torch.Generator().manual_seed(block + 92)
    if kernel == "attention":
        mask = (torch.rand(1, H, nb, nb, generator=g) < 0.6).to(torch.uint8)
        skip_in = (torch.rand(1, H, nb, nb, generator=g) < 0.1).to(torch.uint8)
    else:
        codes = torch.randint(0, 5, (1, H, nb, nb), generator=g, dtype=torch.uint8)

    def run(h):
        qd, kd, vd = q[:, :h].cuda(), k[:, :h].cuda(), v[:, :h].cuda()
        out = torch.full_like(qd, float("nan"))
        lse = torch.full((1, h, N), float("nan"), device="cuda")
        if kernel == "attention":
            so = torch.full((1, h, nb, nb), 7, dtype=torch.uint8, device="cuda")
            ops.sa_sparse_attn_fwd(qd, kd, vd, block, mask=mask[:, :h].contiguous().cuda(),
                                   skip_in=skip_in[:, :h].contiguous().cuda(), skip_out=so, eps=2.0,
                                   out=out, lse=lse)
        else:
            kp, vp = ops.sa_pyramid_pool(kd, vd, block)
            ops.sa_pyramid_attn_fwd(qd, kd, vd, block, codes[:, :h].contiguous().cuda(), kp, vp, out=out, lse=lse)
            so = torch.zeros(1)
        ops.sa_get_device_status()
        return out.cpu(), lse.cpu(), so.cpu()

    O20, L20, S20 = run(H)
    O3, L3, S3 = run(3)
    assert torch.equal(O20[:, :3].view(torch.int16), O3.view(torch.int16))
    assert torch.equal(L20[:, :3], L3)
    if kernel == "attention":
        assert torch.equal(S20[:, :3], S3)
        keep = mask & (1 - skip_in)
        Or, Lr = masked_attention(q, k, v, block, keep)
    else:
        Or, Lr = pyramid_attention(q, k, v, block, codes.numpy())
    check_o(O20, Or, f"{kernel} block={block}")
    check_lse(L20, Lr, f"{kernel} block={block}")
