"""LiteAttention skip update over a denoising chain, fp64 (oracle only).

Follows the LiteAttention write-up (arXiv 2511.11062):
* section 5: a block whose local maximum lies far below the accumulated
  (running) maximum contributes an exponentially suppressed amount, the test
  is local to each block;
* sections 2, 3 and 6: the decision is recorded in a persistent tile-level
  skip mask that later denoising steps reuse; a skipped tile is not loaded,
  multiplied or exponentiated at all.

Readings (stated because the page gives prose only):
* k-blocks of q-block i are visited in ascending j among those with
  mask[i, j] != 0 and skip_in[i, j] == 0;
* m_r is the running maximum of the logits of row r over the blocks visited
  before j; l_r(j) is the maximum of row r over block j's valid columns;
* block j (not the first visited) gets a new skip bit iff l_r(j) < m_r - eps
  for every valid row r of the q-block; eps is in natural-log logit units;
* the output of the detecting step still includes block j; the bit takes
  effect from the next step: skip_out = skip_in | new_bits;
* causal option: blocks j > i are not visited; in the diagonal block a row's
  maximum is over the columns at or before it.
* radial-centric order (section 5 names it, section 10 expects 10-20 % more
  sparsity from it; neither defines it): the key axis is cut into tiles of
  128 tokens and the query axis into bands of 256 rows; the k-blocks of
  q-block i are visited by ascending distance of their tile from the band's
  two diagonal tiles (distance 0 for both), ties by ascending tile index, and
  in ascending j inside a tile.  The band holding q-block i is the one that
  holds its first row.  Only the order in which blocks are visited changes;
  the output is the same up to rounding.
"""
from __future__ import annotations

import math

import numpy as np

from .attention import _f64, _nblocks, _mask4
from .masks import MARGIN


RADIAL_TILE = 128     # keys per tile of the radial-centric order
RADIAL_BAND = 256     # query rows per band of the radial-centric order


def visit_order(i, nkb, block, order="ascending"):
    """k-block indices 0..nkb-1 in the order q-block i visits them."""
    if order == "ascending":
        return list(range(nkb))
    if order != "radial":
        raise ValueError(f"unknown visit order {order!r}")
    per_tile = RADIAL_TILE // block
    n_tiles = -(-nkb // per_tile)
    c = (i * block // RADIAL_BAND) * (RADIAL_BAND // RADIAL_TILE)   # first diagonal tile of the band
    last = c + RADIAL_BAND // RADIAL_TILE - 1                      # last diagonal tile

    def dist(t):
        return c - t if t < c else (t - last if t > last else 0)

    tiles = sorted(range(n_tiles), key=lambda t: (dist(t), t))
    return [j for t in tiles for j in range(t * per_tile, min(nkb, (t + 1) * per_tile))]


def lite_qblock(qh, kh, vh, block, keep_row, i, eps, scale, order="ascending", causal=False):
    """(O rows, LSE rows, new-bit row, margin row) for one q-block.

    margin[j] = max_r (l_r(j) - m_r + eps) for tested blocks (NaN elsewhere);
    the new bit is set iff margin[j] < 0.
    """
    N = qh.shape[0]
    d = vh.shape[1]
    nkb = keep_row.shape[0]
    r0, r1 = i * block, min(N, (i + 1) * block)
    visited = np.array([j for j in visit_order(i, nkb, block, order) if keep_row[j] and (not causal or j <= i)],
                       dtype=np.int64)
    new = np.zeros(nkb, dtype=np.uint8)
    margin = np.full(nkb, np.nan)
    if visited.size == 0:
        return np.zeros((r1 - r0, d)), np.full(r1 - r0, -np.inf), new, margin
    cols = [np.arange(j * block, min(N, (j + 1) * block)) for j in visited]
    c = np.concatenate(cols)
    s = (qh[r0:r1] @ kh[c].T) * scale
    if causal:
        s = np.where(c[None, :] <= np.arange(r0, r1)[:, None], s, -np.inf)
    running = np.full(r1 - r0, -np.inf)
    off = 0
    for n_vis, j in enumerate(visited):
        w = cols[n_vis].shape[0]
        local = s[:, off:off + w].max(axis=1)
        if n_vis > 0:
            mg = np.max(local - running + eps)
            margin[j] = mg
            if mg < 0:
                new[j] = 1
        running = np.maximum(running, local)
        off += w
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    return (e / z) @ vh[c], (m + np.log(z))[:, 0], new, margin


def skip_flags(margin):
    """Skip decisions within MARGIN of the cut, from lite_step's margin rows.

    The comparison rule for skip bits is bit-exact except where the decision
    margin max_r (l_r(j) - m_r + eps) lies within 1e-3 of 0 (absolute, in
    natural-log logit units): there fp32 and fp64 may decide differently.
    Untested blocks (NaN margin) are never flagged.
    """
    m = np.asarray(margin, dtype=np.float64)
    return np.isfinite(m) & (np.abs(m) < MARGIN)


def lite_step(q, k, v, block, mask=None, skip_in=None, eps=10.0, scale=None, qblocks=None,
              order="ascending", causal=False):
    """One denoising step of block attention with the LiteAttention skip update.

    Effective keep = mask & ~skip_in; ``order`` is "ascending" or "radial".  Returns (O, LSE, skip_out, margin) with
    skip_out = skip_in | new bits, or a dict {(b,h,i): (O, LSE, skip_out_row,
    margin_row)} when ``qblocks`` is given.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    nqb = nkb = _nblocks(N, block)
    m4 = _mask4(mask, B, H, nqb, nkb)
    if skip_in is None:
        s4 = np.zeros((B, H, nqb, nkb), dtype=np.uint8)
    else:
        s4 = np.asarray(skip_in.detach().cpu().numpy() if hasattr(skip_in, "detach") else skip_in)
        s4 = np.broadcast_to(s4, (B, H, nqb, nkb))

    def one(b, h, i):
        keep = (m4[b, h, i] != 0) & (s4[b, h, i] == 0)
        o, lse, new, mg = lite_qblock(q[b, h], k[b, h], v[b, h], block, keep, i, eps, scale, order, causal)
        return o, lse, (s4[b, h, i] | new).astype(np.uint8), mg

    if qblocks is not None:
        return {key: one(*key) for key in qblocks}
    O = np.zeros((B, H, N, d))
    L = np.zeros((B, H, N))
    S = np.zeros((B, H, nqb, nkb), dtype=np.uint8)
    M = np.full((B, H, nqb, nkb), np.nan)
    for b in range(B):
        for h in range(H):
            for i in range(nqb):
                r0, r1 = i * block, min(N, (i + 1) * block)
                O[b, h, r0:r1], L[b, h, r0:r1], S[b, h, i], M[b, h, i] = one(b, h, i)
    return O, L, S, M


def lite_chain(steps_inputs, block, eps, mask=None, skip0=None, feed=None, order="ascending"):
    """Run lite_step over a sequence of (q, k, v) denoising inputs.

    ``feed(s, skip_out)`` may replace the skip mask handed to step s+1 (used
    for teacher forcing against another implementation).  Returns a list of
    per-step (O, LSE, skip_out, margin).
    """
    out = []
    skip = skip0
    for s, (q, k, v) in enumerate(steps_inputs):
        O, L, S, M = lite_step(q, k, v, block, mask, skip, eps, order=order)
        out.append((O, L, S, M))
        skip = S if feed is None else feed(s, S)
    return out
