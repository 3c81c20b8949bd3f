"""Pins for the oracle's block masks: tau-mass, PSA levels, static radial (CPU only)."""
import itertools
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_flash_b200 import inputs
from oracle import block_means, block_scores, tau_mask, level_map, radial_mask
from oracle.masks import tau_row, level_counts


def test_block_means_closed_form_with_partial_tail():
    N, block = 21, 8
    x = torch.arange(N, dtype=torch.float64).view(1, 1, N, 1).repeat(1, 1, 1, 3)
    m = block_means(x, block)
    # mean of r0..r1-1 is (r0 + r1 - 1) / 2; the last block holds 16..20
    assert np.allclose(m[0, 0, :, 0], [3.5, 11.5, 18.0])


def test_block_scores_closed_form():
    d, block, nb = 8, 4, 3
    N = block * nb
    q = torch.zeros(1, 1, N, d, dtype=torch.float64)
    k = torch.zeros_like(q)
    alpha, beta = [1.0, -2.0, 3.0], [0.5, 4.0, -1.0]
    for i in range(nb):
        q[0, 0, i * block:(i + 1) * block, 2] = alpha[i]
        k[0, 0, i * block:(i + 1) * block, 2] = beta[i]
        k[0, 0, i * block:(i + 1) * block, 5] = 7.0   # orthogonal to q: no effect
    S = block_scores(q, k, block)
    assert np.allclose(S[0, 0], np.outer(alpha, beta) / math.sqrt(d))


def test_tau_uniform_scores_keep_first_ceil_tau_n():
    nkb, tau = 10, 0.75
    keep, _, _, _ = tau_row(np.zeros(nkb), tau)
    assert keep.tolist() == [True] * 8 + [False] * 2
    # through the full path: Q == 0 gives uniform probabilities on every row
    q = torch.zeros(1, 2, 70, 4)
    k = torch.randn(1, 2, 70, 4, generator=torch.Generator().manual_seed(0))
    m = tau_mask(q, k, 7, 0.75)
    assert (m[..., :8] == 1).all() and (m[..., 8:] == 0).all()


def test_tau_block_exactly_at_the_threshold_is_dropped():
    """Keep a block iff the mass strictly before it is < tau, checked where the
    mass before a block equals tau exactly: four equal blocks (p = 1/4, sums
    exact in binary) and tau = 1/2 keep two blocks, not three."""
    keep, _, p, mass_before = tau_row(np.zeros(4), 0.5)
    assert p.tolist() == [0.25] * 4 and mass_before.tolist() == [0.0, 0.25, 0.5, 0.75]
    assert keep.tolist() == [True, True, False, False]


def test_tau_to_zero_keeps_only_argmax():
    g = np.random.default_rng(1)
    for _ in range(20):
        s = g.normal(size=13)
        keep, _, _, _ = tau_row(s, 1e-12)
        assert keep.sum() == 1 and keep[np.argmax(s)]


def test_tau_brute_force_minimum_cardinality_prefix():
    g = np.random.default_rng(2)
    for trial in range(40):
        n = int(g.integers(2, 9))
        s = g.normal(size=n) * 2
        tau = float(g.uniform(0.05, 0.99))
        keep, _, p, _ = tau_row(s, tau)
        best = None
        for r in range(1, n + 1):
            masses = [sum(p[list(c)]) for c in itertools.combinations(range(n), r)]
            if max(masses) >= tau - 1e-15:
                best = r
                break
        kept = np.nonzero(keep)[0]
        # smallest number of blocks whose mass reaches tau ...
        assert len(kept) == best
        # ... and they are the highest-probability ones
        assert p[kept].min() >= np.max(p[~keep], initial=-1.0)


def test_tau_monotone():
    g = np.random.default_rng(3)
    s = g.normal(size=40)
    prev = None
    for tau in np.linspace(0.01, 0.99, 30):
        keep, _, _, _ = tau_row(s, tau)
        if prev is not None:
            assert np.all(keep >= prev)
        prev = keep


def test_level_quotas_and_order():
    assert level_counts(512, (0.1, 0.3, 0.6)) == [52, 154, 308]
    g = torch.Generator().manual_seed(11)
    q = torch.randn(1, 2, 64 * 512 // 8, 16, generator=g)
    k = torch.randn_like(q)
    lv, _, S = level_map(q, k, 8, return_info=True)
    assert lv.shape[-1] == 512
    for row_l, row_s in zip(lv.reshape(-1, 512), S.reshape(-1, 512)):
        counts = np.bincount(row_l, minlength=5)
        assert counts.tolist() == [0, 52, 102, 154, 204]
        order = np.argsort(-row_s, kind="stable")
        assert np.all(np.diff(row_l[order].astype(int)) >= 0)


def test_level_ties_break_by_index():
    q = torch.zeros(1, 1, 40, 4)
    k = torch.randn(1, 1, 40, 4)
    lv = level_map(q, k, 4)          # Nkb = 10 -> quotas 1, 3, 6
    assert lv[0, 0, 0].tolist() == [1, 2, 2, 3, 3, 3, 4, 4, 4, 4]


def _radial_bruteforce(T, Hh, Ww, block):
    """Independent restatement: decode each block's first token to (t, h, w),
    halve the window in a loop while the frame distance reaches the next
    power of two, compare in floating point."""
    N, F = T * Hh * Ww, Hh * Ww
    nb = -(-N // block)
    S = math.ceil(F / block)
    info = []
    for i in range(nb):
        n = i * block
        t = n // F
        rem = n - t * F
        info.append((t, rem // block))
    out = np.zeros((nb, nb), dtype=np.uint8)
    for i in range(nb):
        for j in range(nb):
            dt = abs(info[i][0] - info[j][0])
            if dt <= 1:
                out[i, j] = 1
                continue
            window, reach = float(S), 1
            while reach * 2 <= dt:
                window /= 2.0
                reach *= 2
            out[i, j] = 1 if abs(info[i][1] - info[j][1]) < window else 0
    return out


@pytest.mark.parametrize("T,Hh,Ww,block", [(9, 8, 16, 16), (17, 4, 9, 8), (33, 3, 5, 4), (6, 5, 7, 64)])
def test_radial_matches_bruteforce(T, Hh, Ww, block):
    assert np.array_equal(radial_mask(T, Hh, Ww, block), _radial_bruteforce(T, Hh, Ww, block))


def test_radial_structure():
    m = radial_mask(20, 8, 16, 16)       # 8 blocks per frame, frame-aligned
    assert np.array_equal(m, m.T)
    assert np.all(np.diag(m) == 1)
    S = 8
    for i in range(m.shape[0]):
        for j in range(m.shape[0]):
            dt, dp = abs(i // S - j // S), abs(i % S - j % S)
            if dt <= 1:
                assert m[i, j] == 1
            elif dp == 0:
                assert m[i, j] == 1          # window never closes on the same position
    # window halves when the frame distance doubles: kept blocks per row at
    # dt = 2..3 (window 4) is 7, at dt = 4..7 (window 2) is 3, at dt >= 8 is 1
    i = 3                                 # frame 0, in-frame position 3
    per_dt = {dt: int(m[i, dt * S:(dt + 1) * S].sum()) for dt in range(2, 20)}
    assert all(per_dt[dt] == 7 for dt in (2, 3))
    assert all(per_dt[dt] == 3 for dt in range(4, 8))
    assert all(per_dt[dt] == 1 for dt in range(8, 20))


def test_radial_density_hunyuan_720p_grid():
    wl = inputs.WORKLOADS["hunyuan_720p_radial"]
    m = radial_mask(wl.T, wl.Hh, wl.Ww, wl.block)
    assert m.shape == (929, 929)
    assert abs(m.mean() - 0.3707) < 5e-5


# ------------------------------------------------------- global selection ---

def test_global_single_row_equals_tau_row():
    from oracle.masks import global_head, tau_row
    g = np.random.default_rng(3)
    for tau in (0.3, 0.5, 0.9):
        s = g.normal(size=(1, 37)) * 2.0
        keep, _ = global_head(s, tau)
        keep_t, _, _, _ = tau_row(s[0], tau)
        assert np.array_equal(keep[0], keep_t)


def test_global_hand_built_peaked_and_uniform_rows():
    """Row 0 has one dominant block, row 1 is uniform: the head's mass (2) is
    reached with the peak and then row 1's blocks in index order."""
    from oracle.masks import global_head
    s = np.array([[20.0, 0.0, 0.0, 0.0], [0.0, 0.0, 0.0, 0.0]])
    keep, _ = global_head(s, 0.5)                  # target mass 1.0
    assert keep.astype(int).tolist() == [[1, 0, 0, 0], [1, 0, 0, 0]]
    keep, _ = global_head(s, 0.7)                  # target mass 1.4
    assert keep.astype(int).tolist() == [[1, 0, 0, 0], [1, 1, 0, 0]]
    keep, _ = global_head(s, 1.0)
    assert keep.all()


def test_global_pair_exactly_at_the_threshold_is_dropped():
    """Two uniform rows of two blocks (every P = 1/2 exactly) and tau = 1/2:
    the head's target mass is 1, reached exactly before the third pair in
    index order, so two pairs are kept."""
    from oracle.masks import global_head
    keep, _ = global_head(np.zeros((2, 2)), 0.5)
    assert keep.astype(int).tolist() == [[1, 1], [0, 0]]


def test_global_brute_force_shortest_prefix():
    """Pure-Python brute force: the kept pairs are the shortest prefix of the
    pairs sorted by (descending P, index) whose mass reaches tau * Nqb."""
    from oracle.masks import global_head
    g = np.random.default_rng(4)
    s = g.normal(size=(5, 7)) * 1.5
    for tau in (0.2, 0.55, 0.8):
        keep, _ = global_head(s, tau)
        rows = []
        for i in range(5):
            e = [math.exp(x - max(s[i])) for x in s[i]]
            z = sum(e)
            rows.append([x / z for x in e])
        pairs = sorted(((rows[i][j], -(i * 7 + j), i, j) for i in range(5) for j in range(7)), reverse=True)
        acc, want = 0.0, np.zeros((5, 7), dtype=bool)
        for p, _, i, j in pairs:
            if acc >= tau * 5:
                break
            want[i, j] = True
            acc += p
        assert np.array_equal(keep, want)
