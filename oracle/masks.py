"""Block masks, fp64 / exact integer (oracle; test infrastructure only).

* ``block_means`` / ``block_scores``: the cheap block-importance score the
  VMoBA write-up describes (mean-pooled query and key blocks, all pairs scored
  with one matrix product: "global block selection" and implementation
  paragraphs) and the PSA page's importance evaluation.  Reading: the score is
  the dot product of the block means scaled by 1/sqrt(d), the same scale as the
  attention logits; a partial last block is averaged over its valid tokens.
* ``tau_mask``: the "threshold dynamic selection" paragraph of the VMoBA
  write-up: per q-block row, softmax over the k-block scores, visit k-blocks
  by descending probability (ties: lower k-block index first) and keep a block
  iff the mass of the blocks ranked strictly before it is < tau.  The block
  that crosses tau is kept, so every row keeps at least one block.
* ``global_mask``: the "global block selection" paragraph (pairs of a head
  compete with each other instead of within a row) with the threshold of the
  "threshold dynamic selection" paragraph (the head's concentration sets the
  count).  Reading: P = per-row softmax of the scores as above; all (i, j) of
  the head are visited by descending P (ties: lower i * Nkb + j first) and a
  pair is kept iff the mass visited before it is < tau * Nqb, the head's
  total mass.  A row may keep nothing.
* ``level_map``: the PSA page's multi-level mask generator with the fixed
  level quotas: ranks (same order as above, on the scores) below
  ceil(f1*Nkb) get level 0, below ceil(f2*Nkb) level 1, below ceil(f3*Nkb)
  level 2, the rest level 3; encoded as level+1 (0 would mean dropped).
* ``radial_mask``: the static mask of the Radial Attention page (spatial
  window halves each time the frame distance doubles, O(n log n) density).
  Reading: a block's frame and in-frame position are those of its first
  token; S = ceil(F / block) blocks per frame; keep (i, j) iff
  |dt| <= 1 or |dp| < S / 2^floor(log2 |dt|).
"""
from __future__ import annotations

import math

import numpy as np

from .attention import _f64, _nblocks

MARGIN = 1e-3


def level_counts(nkb: int, fracs):
    """Cumulative rank quotas ceil(f * nkb) for the three level boundaries."""
    return [int(math.ceil(f * nkb - 1e-9)) for f in fracs]


def block_means(x, block):
    """Mean of the rows of each block, [B, H, N, d] -> [B, H, Nb, d] (fp64)."""
    x = _f64(x)
    B, H, N, d = x.shape
    nb = _nblocks(N, block)
    out = np.zeros((B, H, nb, d))
    for i in range(nb):
        r0, r1 = i * block, min(N, (i + 1) * block)
        out[:, :, i] = x[:, :, r0:r1].sum(axis=2) / (r1 - r0)
    return out


def block_scores(q, k, block, scale=None):
    """S[b,h,i,j] = scale * mean(Q block i) . mean(K block j)."""
    qm, km = block_means(q, block), block_means(k, block)
    d = qm.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    return np.einsum("bhid,bhjd->bhij", qm, km) * scale


def _order(row):
    """k-block indices by descending value, ties broken by lower index."""
    return np.lexsort((np.arange(row.shape[0]), -row))


def tau_row(scores_row, tau):
    """Keep bits, flags, probabilities and mass-before for one score row."""
    s = scores_row
    p = np.exp(s - s.max())
    p = p / p.sum()
    order = _order(p)
    mass_before = np.empty_like(p)
    acc = 0.0
    for j in order:
        mass_before[j] = acc
        acc += p[j]
    keep = mass_before < tau
    flag = np.abs(mass_before - tau) < MARGIN
    kept_p, dropped_p = p[keep], p[~keep]
    if kept_p.size and dropped_p.size:
        p_in, p_out = kept_p.min(), dropped_p.max()
        flag |= keep & (np.abs(p - p_out) <= MARGIN * p_out)
        flag |= (~keep) & (np.abs(p - p_in) <= MARGIN * p_in)
    return keep, flag, p, mass_before


def tau_mask(q, k, block, tau, scale=None, return_info=False):
    """uint8 [B,H,Nqb,Nkb] tau-mass mask (and per-bit margin flags)."""
    S = block_scores(q, k, block, scale)
    B, H, nqb, nkb = S.shape
    mask = np.zeros(S.shape, dtype=np.uint8)
    flags = np.zeros(S.shape, dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(nqb):
                keep, flag, _, _ = tau_row(S[b, h, i], tau)
                mask[b, h, i] = keep
                flags[b, h, i] = flag
    if return_info:
        return mask, flags, S
    return mask


def level_row(scores_row, counts):
    """Level code (level+1) and boundary flags for one score row."""
    s = scores_row
    order = _order(s)
    rank = np.empty(s.shape[0], dtype=np.int64)
    rank[order] = np.arange(s.shape[0])
    code = np.full(s.shape[0], 4, dtype=np.uint8)
    for lvl in (2, 1, 0):
        code[rank < counts[lvl]] = lvl + 1
    flag = np.zeros(s.shape[0], dtype=bool)
    for c in counts:
        if 0 < c < s.shape[0]:
            s_in, s_out = s[order[c - 1]], s[order[c]]
            flag |= (rank < c) & (s - s_out < MARGIN)
            flag |= (rank >= c) & (s_in - s < MARGIN)
    return code, flag


def level_map(q, k, block, fracs=(0.1, 0.3, 0.6), scale=None, return_info=False):
    """uint8 [B,H,Nqb,Nkb] PSA level map, code = level + 1 (all blocks kept)."""
    S = block_scores(q, k, block, scale)
    B, H, nqb, nkb = S.shape
    counts = level_counts(nkb, fracs)
    out = np.zeros(S.shape, dtype=np.uint8)
    flags = np.zeros(S.shape, dtype=bool)
    for b in range(B):
        for h in range(H):
            for i in range(nqb):
                out[b, h, i], flags[b, h, i] = level_row(S[b, h, i], counts)
    if return_info:
        return out, flags, S
    return out


def radial_mask(T, Hh, Ww, block):
    """uint8 [Nb, Nb] static radial mask for a T x Hh x Ww raster grid."""
    N = T * Hh * Ww
    F = Hh * Ww
    nb = _nblocks(N, block)
    S = -(-F // block)
    first = np.arange(nb, dtype=np.int64) * block
    f = first // F
    p = (first % F) // block
    dt = np.abs(f[:, None] - f[None, :])
    dp = np.abs(p[:, None] - p[None, :])
    out = np.zeros((nb, nb), dtype=np.uint8)
    for i in range(nb):
        for j in range(nb):
            t = int(dt[i, j])
            if t <= 1:
                out[i, j] = 1
            else:
                kexp = t.bit_length() - 1          # floor(log2 t)
                out[i, j] = 1 if int(dp[i, j]) * (1 << kexp) < S else 0
    return out


def global_head(scores_head, tau):
    """Keep bits and margin flags of one head's [Nqb, Nkb] scores, global selection."""
    s = np.asarray(scores_head, dtype=np.float64)
    nqb, nkb = s.shape
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)
    flat = p.ravel()
    order = np.lexsort((np.arange(flat.size), -flat))     # descending P, lower index first
    mass_before = np.empty_like(flat)
    mass_before[order] = np.concatenate(([0.0], np.cumsum(flat[order])[:-1]))
    target = tau * nqb
    keep = mass_before < target
    flag = np.abs(mass_before - target) < MARGIN * nqb
    if keep.any() and (~keep).any():
        p_in, p_out = flat[keep].min(), flat[~keep].max()
        flag |= keep & (np.abs(flat - p_out) <= MARGIN * p_out)
        flag |= (~keep) & (np.abs(flat - p_in) <= MARGIN * p_in)
    return keep.reshape(nqb, nkb), flag.reshape(nqb, nkb)


def global_mask(q, k, block, tau, scale=None, return_info=False):
    """uint8 [B,H,Nqb,Nkb] mask of the global (per-head) top-mass selection."""
    S = block_scores(q, k, block, scale)
    B, H = S.shape[:2]
    mask = np.zeros(S.shape, dtype=np.uint8)
    flags = np.zeros(S.shape, dtype=bool)
    for b in range(B):
        for h in range(H):
            keep, flag = global_head(S[b, h], tau)
            mask[b, h] = keep
            flags[b, h] = flag
    if return_info:
        return mask, flags, S
    return mask

