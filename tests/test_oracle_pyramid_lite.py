"""Pins for the oracle's PSA pyramid attention and LiteAttention skip update (CPU only)."""
import math

import numpy as np
import torch

from block_sparse_attention_flash_b200 import inputs
from oracle import (masked_attention, dense_attention, pyramid_pool, pyramid_attention,
                    lite_step, lite_chain, visit_order)


# ---------------------------------------------------------------- pyramid ---

def test_pool_partial_group_and_progressive_equals_direct():
    N = 22
    x = torch.arange(N, dtype=torch.float64).view(1, 1, N, 1)
    p2 = pyramid_pool(x, 2)[0, 0, :, 0]
    assert np.allclose(p2, np.arange(11) * 2 + 0.5)
    p8 = pyramid_pool(x, 8)[0, 0, :, 0]
    assert np.allclose(p8, [3.5, 11.5, 18.5])            # last group = tokens 16..21
    g = torch.Generator().manual_seed(5)
    y = torch.randn(2, 3, 64, 5, generator=g, dtype=torch.float64)
    assert np.allclose(pyramid_pool(torch.from_numpy(pyramid_pool(y, 2)), 2), pyramid_pool(y, 4))


def test_all_level_zero_equals_block_attention():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.normal_qkv(wl.B, wl.H, wl.N, wl.d, wl.seed)
    nb = wl.nblocks
    O1, L1 = pyramid_attention(q, k, v, wl.block, np.ones((nb, nb), np.uint8))
    O2, L2 = masked_attention(q, k, v, wl.block, None)
    assert np.max(np.abs(O1 - O2)) < 1e-12 and np.max(np.abs(L1 - L2)) < 1e-12
    m = inputs.bernoulli_block_mask(wl.B, wl.H, nb, nb, 0.5, 8).numpy()
    O1, _ = pyramid_attention(q, k, v, wl.block, m)
    O2, _ = masked_attention(q, k, v, wl.block, m)
    assert np.max(np.abs(O1 - O2)) < 1e-12


def test_constant_groups_make_any_level_mix_exact():
    """If K and V are constant over every 8-token group, pooling loses nothing
    and the +ln(count) correction makes pyramid attention equal full attention."""
    N, d, block = 64 * 5 + 24, 16, 64        # partial last block of 24 tokens
    g = torch.Generator().manual_seed(21)
    q = torch.randn(1, 2, N, d, generator=g).to(torch.bfloat16)
    k, v = inputs.const_group_kv(1, 2, N, d, 8, seed=22)
    nb = -(-N // block)
    codes = torch.randint(1, 5, (1, 2, nb, nb), generator=g).numpy().astype(np.uint8)
    O, L = pyramid_attention(q, k, v, block, codes)
    Od, Ld = dense_attention(q, k, v)
    assert np.max(np.abs(O - Od)) < 1e-12
    assert np.max(np.abs(L - Ld)) < 1e-12
    Oc, _ = pyramid_attention(q, k, v, block, np.full_like(codes, 4))
    assert np.max(np.abs(Oc - Od)) < 1e-12


def test_causal_constant_groups_equal_causal_attention():
    """Causal option with K/V constant over 8-token groups: earlier blocks at
    any level are exact, so pyramid attention equals causal masked attention
    with the same kept blocks; all-level-0 codes equal it for any K/V."""
    N, d, block = 64 * 5 + 24, 16, 64
    g = torch.Generator().manual_seed(23)
    q = torch.randn(1, 2, N, d, generator=g).to(torch.bfloat16)
    k, v = inputs.const_group_kv(1, 2, N, d, 8, seed=24)
    nb = -(-N // block)
    codes = torch.randint(0, 5, (1, 2, nb, nb), generator=g).numpy().astype(np.uint8)
    O, L = pyramid_attention(q, k, v, block, codes, causal=True)
    Om, Lm = masked_attention(q, k, v, block, (codes != 0).astype(np.uint8), causal=True)
    assert np.max(np.abs(O - Om)) < 1e-12
    fin = np.isfinite(Lm)
    assert np.array_equal(fin, np.isfinite(L)) and np.max(np.abs(L[fin] - Lm[fin])) < 1e-12
    q2, k2, v2 = inputs.normal_qkv(1, 2, N, d, seed=25)
    O1, _ = pyramid_attention(q2, k2, v2, block, np.ones_like(codes), causal=True)
    Om1, _ = masked_attention(q2, k2, v2, block, None, causal=True)
    assert np.max(np.abs(O1 - Om1)) < 1e-12


def test_exactness_pin_catches_a_wrong_correction(monkeypatch):
    """Plant a sign error in the oracle's ln(count) bias: the pin must fail."""
    import oracle.pyramid as pyr
    real = pyr._level_keys

    def flipped(*a, **kw):
        kk, vv, bb = real(*a, **kw)
        return kk, vv, -bb
    N, d, block = 128, 16, 64
    g = torch.Generator().manual_seed(23)
    q = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    k, v = inputs.const_group_kv(1, 1, N, d, 8, seed=24)
    Od, _ = dense_attention(q, k, v)
    monkeypatch.setattr(pyr, "_level_keys", flipped)
    # mixed levels: a uniform bias would cancel in the softmax
    Ow, _ = pyramid_attention(q, k, v, block, np.array([[1, 3], [4, 2]], np.uint8))
    assert np.max(np.abs(Ow - Od)) > 1e-3


def test_dropped_level_code_removes_block():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.normal_qkv(1, 1, wl.N, wl.d, wl.seed)
    nb = wl.nblocks
    codes = np.ones((nb, nb), np.uint8)
    codes[:, 3] = 0
    mask = (codes != 0).astype(np.uint8)
    O1, _ = pyramid_attention(q, k, v, wl.block, codes)
    O2, _ = masked_attention(q, k, v, wl.block, mask)
    assert np.max(np.abs(O1 - O2)) < 1e-12


# ------------------------------------------------------------------- lite ---

def test_infinite_eps_never_skips_and_equals_block_attention():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.normal_qkv(wl.B, wl.H, wl.N, wl.d, wl.seed)
    nb = wl.nblocks
    m = inputs.bernoulli_block_mask(wl.B, wl.H, nb, nb, 0.5, 4)
    skip_in = inputs.bernoulli_block_mask(wl.B, wl.H, nb, nb, 0.2, 5, force_diagonal=False)
    skip_in[:, :, torch.arange(nb), torch.arange(nb)] = 0
    O, L, S, _ = lite_step(q, k, v, wl.block, m, skip_in, eps=math.inf)
    assert np.array_equal(S, skip_in.numpy())
    eff = m.numpy() & (1 - skip_in.numpy())
    O2, L2 = masked_attention(q, k, v, wl.block, eff)
    assert np.max(np.abs(O - O2)) < 1e-12 and np.max(np.abs(L - L2)) < 1e-12


def _aligned_case(a, b, d=16, block=8, nb=4):
    u = np.zeros(d)
    u[3] = 1.0
    N = block * nb
    q = np.tile(a * u, (N, 1))
    k = np.tile(-b * u, (N, 1))
    k[:block] = b * u
    v = np.random.default_rng(0).normal(size=(N, d))
    return (q[None, None], k[None, None], v[None, None], block)


def test_hand_built_gap_of_twelve():
    d = 16
    a = b = math.sqrt(6.0 * math.sqrt(d))     # every logit in block 0 is +6, elsewhere -6
    q, k, v, block = _aligned_case(a, b, d=d)
    _, _, S, M = lite_step(q, k, v, block, None, None, eps=10.0)
    assert S[0, 0].tolist() == [[0, 1, 1, 1]] * 4
    assert np.allclose(M[0, 0, :, 1:], -2.0)
    _, _, S, _ = lite_step(q, k, v, block, None, None, eps=1e6)
    assert S.sum() == 0
    _, _, S, _ = lite_step(q, k, v, block, None, None, eps=12.5)
    assert S.sum() == 0


def test_skipped_blocks_are_exponentially_suppressed():
    """Every new bit at a step marks a block whose probabilities, under the
    same step's full row softmax over visited blocks, are all <= exp(-eps)."""
    wl = inputs.Workload("t", 1, 2, 32, 6, 8, 16, 32, "lite", seed=77, sigma_s=2.0)
    q, k, v = inputs.rff_qkv(wl)
    block, eps = wl.block, 0.6
    nb = wl.nblocks
    _, _, S, _ = lite_step(q, k, v, block, None, None, eps=eps)
    assert S.sum() > 0
    qd, kd = q.double().numpy(), k.double().numpy()
    for h in range(wl.H):
        s = qd[0, h] @ kd[0, h].T / math.sqrt(wl.d)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        for i, j in zip(*np.nonzero(S[0, h])):
            blk = p[i * block:(i + 1) * block, j * block:(j + 1) * block]
            assert blk.max() <= math.exp(-eps)


def test_first_visited_block_never_skipped_and_chain_monotone():
    wl = inputs.Workload("t", 1, 2, 32, 6, 8, 16, 32, "lite", seed=78, sigma_s=2.0)
    steps = list(inputs.lite_chain_inputs(wl, 4))
    res = lite_chain(steps, wl.block, eps=1.0)
    prev = np.zeros_like(res[0][2])
    for O, L, S, M in res:
        assert np.all(S >= prev)
        prev = S
        assert np.all(np.isfinite(O))
    nb = wl.nblocks
    first = res[0][2]
    assert np.all(first[..., 0] == 0)       # block 0 is always visited first at step 0
    # a fully skipped row cannot happen: the first visited block is never skipped
    assert np.all(prev.sum(axis=-1) < nb)


def test_running_max_before_or_after_j_is_equivalent():
    wl = inputs.Workload("t", 1, 1, 32, 6, 8, 16, 32, "lite", seed=79, sigma_s=2.0)
    q, k, v = inputs.rff_qkv(wl)
    _, _, S, M = lite_step(q, k, v, wl.block, None, None, eps=1.2)
    qd, kd = q[0, 0].double().numpy(), k[0, 0].double().numpy()
    s = qd @ kd.T / math.sqrt(wl.d)
    nb, block = wl.nblocks, wl.block
    for i in range(nb):
        rows = s[i * block:(i + 1) * block]
        run = np.full(rows.shape[0], -np.inf)
        for j in range(nb):
            loc = rows[:, j * block:(j + 1) * block].max(axis=1)
            after = np.maximum(run, loc)
            bit = j > 0 and bool(np.all(loc < after - 1.2))
            assert bit == bool(S[0, 0, i, j])
            run = after


# ------------------------------------------------------ radial-centric order ---

def test_radial_visit_order_hand_listed():
    """Orders listed by hand from the reading: 128-key tiles, 256-row bands,
    ascending distance from the band's two diagonal tiles, ties by tile index."""
    assert visit_order(2, 8, 128, "radial") == [2, 3, 1, 4, 0, 5, 6, 7]
    assert visit_order(3, 8, 128, "radial") == [2, 3, 1, 4, 0, 5, 6, 7]
    assert visit_order(0, 5, 128, "radial") == [0, 1, 2, 3, 4]
    assert visit_order(6, 7, 128, "radial") == [6, 5, 4, 3, 2, 1, 0]
    assert visit_order(5, 12, 64, "radial") == [4, 5, 6, 7, 2, 3, 8, 9, 0, 1, 10, 11]
    assert visit_order(9, 11, 64, "radial") == [8, 9, 10, 6, 7, 4, 5, 2, 3, 0, 1]
    assert visit_order(1, 4, 64, "ascending") == [0, 1, 2, 3]
    for nkb, block in ((13, 64), (9, 128), (1, 64)):
        for i in range(nkb):
            assert sorted(visit_order(i, nkb, block, "radial")) == list(range(nkb))


def test_radial_order_changes_no_output_and_keeps_suppression():
    """The order decides only which blocks are skipped next step: with eps = inf
    the step equals block attention, and with a finite eps every new bit still
    marks a block whose probabilities are all <= exp(-eps)."""
    wl = inputs.Workload("t", 1, 2, 8, 8, 8, 64, 16, "lite", seed=81, sigma_s=2.0)
    q, k, v = inputs.rff_qkv(wl)
    block, nb = wl.block, wl.nblocks
    m = inputs.bernoulli_block_mask(wl.B, wl.H, nb, nb, 0.7, 6)
    O, L, S, _ = lite_step(q, k, v, block, m, None, eps=math.inf, order="radial")
    O2, L2 = masked_attention(q, k, v, block, m)
    assert S.sum() == 0 and np.max(np.abs(O - O2)) < 1e-12 and np.max(np.abs(L - L2)) < 1e-12
    eps = 0.5
    _, _, S, _ = lite_step(q, k, v, block, None, None, eps=eps, order="radial")
    assert S.sum() > 0
    qd, kd = q.double().numpy(), k.double().numpy()
    for h in range(wl.H):
        s = qd[0, h] @ kd[0, h].T / math.sqrt(wl.d)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        for i, j in zip(*np.nonzero(S[0, h])):
            assert p[i * block:(i + 1) * block, j * block:(j + 1) * block].max() <= math.exp(-eps)


def test_radial_order_reaches_the_row_max_first():
    """Keys of k-blocks 4 and 5 give logit +6, all others -6; q-block 4 sits in
    the band whose diagonal tiles hold k-blocks 4-7.  Ascending order meets
    blocks 0-3 before any +6 block and can skip only 6 and 7; radial order
    starts at block 4 and skips every -6 block."""
    d, block, nb = 16, 64, 8
    a = b = math.sqrt(6.0 * math.sqrt(d))
    u = np.zeros(d)
    u[3] = 1.0
    N = block * nb
    q = np.tile(a * u, (N, 1))
    k = np.tile(-b * u, (N, 1))
    k[4 * block:6 * block] = b * u
    v = np.random.default_rng(1).normal(size=(N, d))
    q, k, v = q[None, None], k[None, None], v[None, None]
    _, _, Sa, _ = lite_step(q, k, v, block, None, None, eps=10.0)
    _, _, Sr, _ = lite_step(q, k, v, block, None, None, eps=10.0, order="radial")
    assert Sa[0, 0, 4].tolist() == [0, 0, 0, 0, 0, 0, 1, 1]
    assert Sr[0, 0, 4].tolist() == [1, 1, 1, 1, 0, 0, 1, 1]
    # the skip bits of a radial step equal a re-walk of the hand-listed order
    s = q[0, 0] @ k[0, 0].T / math.sqrt(d)
    for i in range(nb):
        rows = s[i * block:(i + 1) * block]
        order = [4, 5, 6, 7, 2, 3, 0, 1] if 4 <= i < 8 else [0, 1, 2, 3, 4, 5, 6, 7]
        run = np.full(block, -np.inf)
        for n_vis, j in enumerate(order):
            loc = rows[:, j * block:(j + 1) * block].max(axis=1)
            assert bool(n_vis > 0 and np.all(loc < run - 10.0)) == bool(Sr[0, 0, i, j])
            run = np.maximum(run, loc)


def test_sampled_qblocks_equal_full_for_lite_and_pyramid():
    """The q-block samplers that the full-size GPU tests use (``qblocks=``) return exactly the
    full computation's rows, for the skip update (with a carried skip mask and a block mask) and
    for pyramid attention over a mixed level map; the samples include the partial last q-block."""
    wl = inputs.Workload("s", 1, 2, 16, 3, 5, 7, 16, "lite", seed=91)   # 105 tokens, 7 blocks
    q, k, v = inputs.rff_qkv(wl)
    nb, N = wl.nblocks, wl.N
    g = np.random.default_rng(92)
    mask = (g.random((1, 2, nb, nb)) < 0.8).astype(np.uint8)
    skip0 = (g.random((1, 2, nb, nb)) < 0.2).astype(np.uint8)
    picks = [(0, 1, 0), (0, 0, 3), (0, 1, nb - 1)]
    O, L, S, M = lite_step(q, k, v, wl.block, mask, skip0, eps=2.0)
    part = lite_step(q, k, v, wl.block, mask, skip0, eps=2.0, qblocks=picks)
    assert list(part) == picks
    for (b, h, i), (o, l, srow, mrow) in part.items():
        sl = slice(i * wl.block, min(N, (i + 1) * wl.block))
        assert np.array_equal(o, O[b, h, sl]) and np.array_equal(l, L[b, h, sl])
        assert np.array_equal(srow, S[b, h, i]) and np.array_equal(mrow, M[b, h, i], equal_nan=True)
    codes = g.integers(0, 5, size=(1, 2, nb, nb)).astype(np.uint8)
    Op, Lp = pyramid_attention(q, k, v, wl.block, codes)
    pp = pyramid_attention(q, k, v, wl.block, codes, qblocks=picks)
    for (b, h, i), (o, l) in pp.items():
        sl = slice(i * wl.block, min(N, (i + 1) * wl.block))
        assert np.array_equal(o, Op[b, h, sl]) and np.array_equal(l, Lp[b, h, sl])
