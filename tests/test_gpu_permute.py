"""GPU parity: sa_token_permute (bit-exact against the oracle's sort-based
permutation) and permuted block-sparse attention end to end."""
import numpy as np
import pytest
import torch

from block_sparse_attention_flash_b200 import build, inputs, ops
from oracle import permute_tokens, masked_attention
from _parity import check_o

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    yield
    ops.sa_get_device_status()


def _bits(t):
    return t.view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("cells", [(1, 1, 1), (3, 1, 1), (6, 4, 6), (2, 2, 3)])
def test_permute_bit_exact_per_head_orders(d, cells):
    T, Hh, Ww, B, H = 6, 8, 12, 2, 6
    N = T * Hh * Ww
    g = torch.Generator().manual_seed(d + sum(cells))
    xs = [torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3)]
    orders = torch.tensor([0, 1, 2, 3, 4, 5], dtype=torch.uint8)
    outs = ops.sa_token_permute([x.cuda() for x in xs], T, Hh, Ww, head_order=orders.cuda(), cells=cells)
    for x, o in zip(xs, outs):
        ref = permute_tokens(_bits(x), T, Hh, Ww, orders.tolist(), cells)
        assert np.array_equal(_bits(o), ref)
    back = ops.sa_token_permute(outs, T, Hh, Ww, head_order=orders.cuda(), cells=cells, inverse=True)
    for x, b in zip(xs, back):
        assert np.array_equal(_bits(b), _bits(x))


def test_uniform_order_and_full_size_grid():
    """One order for all heads on the 480p grid (21 x 30 x 52, 12 heads):
    VMoBA-style 3D cells of 3 x 5 x 4 tokens."""
    wl = inputs.WORKLOADS["wan13b_480p_tau"]
    q, k, v = inputs.rff_qkv(wl)
    outs = ops.sa_token_permute([q.cuda(), k.cuda(), v.cuda()], wl.T, wl.Hh, wl.Ww, order="thw", cells=(3, 5, 4))
    for x, o in zip((q, k, v), outs):
        assert np.array_equal(_bits(o), permute_tokens(_bits(x), wl.T, wl.Hh, wl.Ww, "thw", (3, 5, 4)))


@pytest.mark.parametrize("block", [64, 128])
def test_permuted_attention_end_to_end(block):
    """Permute Q, K, V (per-head PARO orders), block-sparse attention on the
    permuted sequence, inverse-permute O: equals the oracle's masked attention
    of the permuted inputs, brought back to raster order."""
    wl = inputs.Workload("pm", 1, 3, 128, 4, 12, 16, block, "tau", seed=91)
    q, k, v = inputs.rff_qkv(wl)
    nb = wl.nblocks
    mask = inputs.bernoulli_block_mask(1, wl.H, nb, nb, 0.6, seed=92)
    orders = torch.tensor([3, 1, 5], dtype=torch.uint8)
    qp, kp, vp = ops.sa_token_permute([q.cuda(), k.cuda(), v.cuda()], wl.T, wl.Hh, wl.Ww, head_order=orders.cuda())
    o_perm = ops.sa_sparse_attn_fwd(qp, kp, vp, block, mask=mask.cuda())
    (o,) = ops.sa_token_permute([o_perm], wl.T, wl.Hh, wl.Ww, head_order=orders.cuda(), inverse=True)
    pq, pk, pv = (permute_tokens(x.float().numpy(), wl.T, wl.Hh, wl.Ww, orders.tolist()) for x in (q, k, v))
    ref, _ = masked_attention(pq, pk, pv, block, mask)
    ref = permute_tokens(ref, wl.T, wl.Hh, wl.Ww, orders.tolist(), inverse=True)
    check_o(o.cpu(), ref, f"permuted attention block={block}")
