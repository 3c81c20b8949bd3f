"""Pins for the oracle's block-masked attention (CPU only).

Each check ties the oracle to something other than itself: torch's own SDPA
(a library routine the oracle does not call), a pure-Python token-level
brute force, and invariants of softmax attention (rows sum to one, a single
kept block is attention over that block, empty rows are defined).
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from block_sparse_attention_flash_b200 import inputs
from oracle import masked_attention, dense_attention


def _sdpa64(q, k, v, scale=None):
    return torch.nn.functional.scaled_dot_product_attention(
        q.double(), k.double(), v.double(), scale=scale).numpy()


def _brute(q, k, v, mask, block, scale):
    """Token-level masked softmax with plain Python loops (tiny inputs)."""
    q, k, v = q.double().tolist(), k.double().tolist(), v.double().tolist()
    N, d = len(q), len(q[0])
    O = [[0.0] * d for _ in range(N)]
    L = [-math.inf] * N
    for r in range(N):
        logits = []
        for c in range(N):
            if mask[r // block][c // block]:
                logits.append((c, scale * sum(q[r][t] * k[c][t] for t in range(d))))
        if not logits:
            continue
        mx = max(s for _, s in logits)
        z = sum(math.exp(s - mx) for _, s in logits)
        for c, s in logits:
            w = math.exp(s - mx) / z
            for t in range(d):
                O[r][t] += w * v[c][t]
        L[r] = mx + math.log(z)
    return np.array(O), np.array(L)


def test_all_ones_mask_equals_dense_sdpa_tiny_config():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.normal_qkv(wl.B, wl.H, wl.N, wl.d, wl.seed)
    O, L = masked_attention(q, k, v, wl.block, mask=None)
    ref = _sdpa64(q, k, v)
    assert np.max(np.abs(O - ref)) < 1e-12
    Od, Ld = dense_attention(q, k, v)
    assert np.max(np.abs(Od - ref)) < 1e-12
    assert np.max(np.abs(L - Ld)) < 1e-12


@pytest.mark.parametrize("N,block", [(24, 8), (21, 8), (9, 4)])
def test_brute_force_token_level_matches_block_path(N, block):
    g = torch.Generator().manual_seed(7 + N)
    d = 4
    q = torch.randn(1, 1, N, d, generator=g)
    k = torch.randn(1, 1, N, d, generator=g)
    v = torch.randn(1, 1, N, d, generator=g)
    nb = -(-N // block)
    mask = (torch.rand(nb, nb, generator=g) < 0.5).to(torch.uint8).numpy()
    mask[0, :] = 0                      # one row with no kept block
    mask[1, 1] = 1
    scale = 1.0 / math.sqrt(d)
    O, L = masked_attention(q, k, v, block, mask=mask)
    Ob, Lb = _brute(q[0, 0], k[0, 0], v[0, 0], mask, block, scale)
    assert np.allclose(O[0, 0], Ob, atol=1e-12, rtol=0)
    fin = np.isfinite(Lb)
    assert np.array_equal(np.isfinite(L[0, 0]), fin)
    assert np.allclose(L[0, 0][fin], Lb[fin], atol=1e-12)
    assert np.all(O[0, 0][:block] == 0.0) and np.all(L[0, 0][:block] == -np.inf)


def test_rows_sum_to_one_with_unit_values():
    wl = inputs.WORKLOADS["tiny"]
    q, k, _ = inputs.normal_qkv(wl.B, wl.H, wl.N, wl.d, wl.seed)
    v = torch.ones_like(q)
    m = inputs.bernoulli_block_mask(wl.B, wl.H, wl.nblocks, wl.nblocks, 0.5, wl.seed + 1)
    O, _ = masked_attention(q, k, v, wl.block, mask=m)
    assert np.max(np.abs(O - 1.0)) < 1e-12


def test_single_kept_block_is_attention_over_that_block():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.normal_qkv(1, 1, wl.N, wl.d, wl.seed)
    nb = wl.nblocks
    mask = np.zeros((nb, nb), dtype=np.uint8)
    j = 5
    mask[2, j] = 1
    O, _ = masked_attention(q, k, v, wl.block, mask=mask)
    blk = slice(j * wl.block, (j + 1) * wl.block)
    rows = slice(2 * wl.block, 3 * wl.block)
    ref = _sdpa64(q[:, :, rows], k[:, :, blk], v[:, :, blk])
    assert np.max(np.abs(O[0, 0, rows] - ref[0, 0])) < 1e-12


def test_lse_matches_scipy_logsumexp_on_kept_columns():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.normal_qkv(1, 1, wl.N, wl.d, wl.seed)
    nb = wl.nblocks
    m = inputs.bernoulli_block_mask(1, 1, nb, nb, 0.5, 99)
    _, L = masked_attention(q, k, v, wl.block, mask=m)
    qd, kd = q[0, 0].double().numpy(), k[0, 0].double().numpy()
    s = qd @ kd.T / math.sqrt(wl.d)
    tok = np.repeat(np.repeat(m[0, 0].numpy() != 0, wl.block, 0), wl.block, 1)
    s = np.where(tok, s, -np.inf)
    assert np.allclose(L[0, 0], logsumexp(s, axis=1), atol=1e-12)


def test_sampled_qblocks_equal_full_computation():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.normal_qkv(wl.B, wl.H, wl.N, wl.d, wl.seed)
    m = inputs.bernoulli_block_mask(wl.B, wl.H, wl.nblocks, wl.nblocks, 0.5, 3)
    O, L = masked_attention(q, k, v, wl.block, mask=m)
    part = masked_attention(q, k, v, wl.block, mask=m, qblocks=[(0, 1, 3), (0, 0, 7)])
    for (b, h, i), (o, l) in part.items():
        sl = slice(i * wl.block, (i + 1) * wl.block)
        assert np.array_equal(o, O[b, h, sl]) and np.array_equal(l, L[b, h, sl])


# ------------------------------------------------------------------ causal ---

def test_causal_all_ones_equals_sdpa_is_causal():
    g = torch.Generator().manual_seed(21)
    B, H, N, d, block = 1, 2, 200, 32, 64
    q, k, v = (torch.randn(B, H, N, d, generator=g, dtype=torch.float64) for _ in range(3))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    O, L = masked_attention(q.numpy(), k.numpy(), v.numpy(), block, None, causal=True)
    assert np.max(np.abs(O - ref.numpy())) < 1e-12
    s = (q @ k.transpose(-1, -2)).numpy() / math.sqrt(d)
    s = np.where(np.tri(N, dtype=bool), s, -np.inf)
    assert np.max(np.abs(L - logsumexp(s, axis=-1))) < 1e-12


def test_causal_block_mask_equals_token_level_brute_force():
    """Causal with a block mask (diagonal kept or not, empty rows included)
    against a per-row loop over the visible keys written out directly."""
    g = np.random.default_rng(22)
    N, d, block = 150, 8, 32
    q, k, v = (g.normal(size=(1, 1, N, d)) for _ in range(3))
    nb = -(-N // block)
    mask = (g.random((1, 1, nb, nb)) < 0.5).astype(np.uint8)
    mask[0, 0, 1, :] = 0
    mask[0, 0, 1, 3] = 1                      # q-block 1 keeps only a future block: no visible key
    mask[0, 0, 2, 2] = 0                      # q-block 2 without its diagonal block
    O, L = masked_attention(q, k, v, block, mask, causal=True)
    for r in range(N):
        vis = [c for c in range(N) if mask[0, 0, r // block, c // block] and c <= r]
        if not vis:
            assert np.all(O[0, 0, r] == 0) and L[0, 0, r] == -np.inf
            continue
        s = np.array([q[0, 0, r] @ k[0, 0, c] for c in vis]) / math.sqrt(d)
        p = np.exp(s - s.max())
        assert np.max(np.abs(O[0, 0, r] - (p / p.sum()) @ v[0, 0, vis])) < 1e-12
        assert abs(L[0, 0, r] - (s.max() + math.log(p.sum()))) < 1e-12
