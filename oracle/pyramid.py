"""Pyramid (PSA) pooling and multi-level attention, fp64 (oracle only).

Follows the PSA page ("浙江大学突破视频AI瓶颈:金字塔方法提升视频AI效率10倍"):
the pyramid KV keeps the original keys and values at the bottom level and
average-pools them more coarsely at each level up; every (q-block, k-block)
pair is assigned a level; attention over pooled keys keeps the probability
distribution consistent with full attention.

Readings:
* level l pools groups of c = 2^l consecutive tokens; groups never cross a
  block edge (the block size is a multiple of 8) and a partial last group is
  the mean of its valid tokens;
* a pooled key stands for the n_g tokens of its group, so its logit gets
  + ln(n_g): if the n_g keys were equal, full attention would weight them
  n_g * exp(s), which is exactly exp(s + ln n_g);
* level codes: 0 = dropped, 1 + l = attend at level l;
* causal option (the page: PSA serves causal generation too): k-blocks j > i
  are dropped; block i itself, if kept, is attended at level 0 (a pooled key
  of that block would mix in later tokens) with key c visible to row r only
  if c <= r; blocks j < i keep their codes (all their tokens are earlier).
"""
from __future__ import annotations

import math

import numpy as np

from .attention import _f64, _nblocks, _mask4


def pyramid_pool(x, c):
    """Mean over groups of c consecutive tokens: [B,H,N,d] -> [B,H,ceil(N/c),d]."""
    x = _f64(x)
    B, H, N, d = x.shape
    ng = -(-N // c)
    out = np.zeros((B, H, ng, d))
    for g in range(ng):
        r0, r1 = g * c, min(N, (g + 1) * c)
        out[:, :, g] = x[:, :, r0:r1].sum(axis=2) / (r1 - r0)
    return out


def _level_keys(kh, vh, pooled_k, pooled_v, N, block, j, level):
    """Keys, values and logit bias for k-block j attended at ``level``."""
    r0, r1 = j * block, min(N, (j + 1) * block)
    if level == 0:
        return kh[r0:r1], vh[r0:r1], np.zeros(r1 - r0)
    c = 1 << level
    g0, g1 = r0 // c, -(-r1 // c)
    counts = np.array([min(N, (g + 1) * c) - g * c for g in range(g0, g1)], dtype=np.float64)
    return pooled_k[level][g0:g1], pooled_v[level][g0:g1], np.log(counts)


def pyramid_attention(q, k, v, block, levels, scale=None, qblocks=None, causal=False):
    """Multi-level block attention over [B,H,N,d] with a level-code map.

    levels: anything broadcastable to uint8 [B,H,Nqb,Nkb] (0 drop, 1+l level l).
    Returns (O, LSE) like ``masked_attention`` (or a dict when qblocks given).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    nqb = nkb = _nblocks(N, block)
    lv = _mask4(levels, B, H, nqb, nkb)
    pk = {l: pyramid_pool(k, 1 << l) for l in (1, 2, 3)}
    pv = {l: pyramid_pool(v, 1 << l) for l in (1, 2, 3)}

    def one(b, h, i):
        r0, r1 = i * block, min(N, (i + 1) * block)
        ks, vs, bs, ids = [], [], [], []
        for j in range(nkb):
            code = int(lv[b, h, i, j])
            if causal and j > i:
                code = 0
            if causal and j == i and code:
                code = 1
            if code == 0:
                continue
            kk, vv, bb = _level_keys(k[b, h], v[b, h],
                                     {l: pk[l][b, h] for l in pk},
                                     {l: pv[l][b, h] for l in pv}, N, block, j, code - 1)
            ks.append(kk), vs.append(vv), bs.append(bb)
            # key index of level-0 columns of the diagonal block, -1 elsewhere
            ids.append(np.arange(j * block, j * block + kk.shape[0]) if (causal and j == i) else
                       np.full(kk.shape[0], -1))
        if not ks:
            return np.zeros((r1 - r0, d)), np.full(r1 - r0, -np.inf)
        K, V, bias = np.concatenate(ks), np.concatenate(vs), np.concatenate(bs)
        s = (q[b, h, r0:r1] @ K.T) * scale + bias[None, :]
        if causal:
            kid = np.concatenate(ids)
            s = np.where(kid[None, :] > np.arange(r0, r1)[:, None], -np.inf, s)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        return (e / z) @ V, (m + np.log(z))[:, 0]

    if qblocks is not None:
        return {key: one(*key) for key in qblocks}
    O = np.zeros((B, H, N, d))
    L = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            for i in range(nqb):
                r0, r1 = i * block, min(N, (i + 1) * block)
                O[b, h, r0:r1], L[b, h, r0:r1] = one(b, h, i)
    return O, L
