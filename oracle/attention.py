"""Block-masked softmax attention, fp64 (oracle; test infrastructure only).

Definition (non-causal block-sparse attention, the "keep or drop each block"
scheme the PSA page names as the mainstream block-sparse method, and the
full-attention special case every page compares against):

    for a query row r in q-block i of head (b, h):
        s_rc   = scale * q_r . k_c          for every key column c in a kept
                                            k-block j (mask[b,h,i,j] != 0)
        O_r    = sum_c softmax_c(s_r.) v_c
        LSE_r  = log sum_c exp(s_rc)

Blocks are consecutive runs of ``block`` tokens in raster (t,h,w) order; the
last block may be partial and then holds only its valid tokens.  A row with
no kept column gets O_r = 0 and LSE_r = -inf.  ``scale`` defaults to
1/sqrt(d) (natural-log units).

Causal option (the PSA page says the method serves causal video generation
as well as bidirectional understanding; reading): key column c is visible to
row r only if it is kept by the block mask and c <= r.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().float().cpu().numpy()
    return np.asarray(x, dtype=np.float64)


def _nblocks(n: int, block: int) -> int:
    return -(-n // block)


def _mask4(mask, B, H, nqb, nkb):
    if mask is None:
        return np.ones((B, H, nqb, nkb), dtype=np.uint8)
    if hasattr(mask, "detach"):
        mask = mask.detach().cpu().numpy()
    m = np.asarray(mask)
    return np.broadcast_to(m, (B, H, nqb, nkb))


def attention_qblock(qh, kh, vh, block, keep_row, i, scale, causal=False):
    """O (rows x d) and LSE (rows,) for q-block ``i`` of one head.

    ``keep_row`` is the boolean row of the block mask for q-block ``i``.
    The kept key columns are gathered in ascending order and one fp64 matmul
    gives the logits; softmax is the textbook max-subtracted form.  With
    ``causal``, logits of columns after the row are -inf.
    """
    N = qh.shape[0]
    r0, r1 = i * block, min(N, (i + 1) * block)
    cols = [np.arange(j * block, min(N, (j + 1) * block))
            for j in np.nonzero(keep_row)[0]]
    d = vh.shape[1]
    if not cols:
        return np.zeros((r1 - r0, d)), np.full(r1 - r0, -np.inf)
    c = np.concatenate(cols)
    s = (qh[r0:r1] @ kh[c].T) * scale
    if causal:
        s = np.where(c[None, :] <= np.arange(r0, r1)[:, None], s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    o = np.divide(e, z, out=np.zeros_like(e), where=z > 0) @ vh[c]
    with np.errstate(divide="ignore"):
        lse = (m + np.log(z))[:, 0]
    return o, lse


def masked_attention(q, k, v, block, mask=None, scale=None, qblocks=None, causal=False):
    """Block-masked attention over [B, H, N, d] inputs.

    mask: None (all kept) or anything broadcastable to uint8 [B, H, Nqb, Nkb].
    qblocks: optional list of (b, h, i); then only those q-blocks are computed
    and a dict {(b, h, i): (O_rows, LSE_rows)} is returned.  Otherwise returns
    (O [B,H,N,d] fp64, LSE [B,H,N] fp64).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    nqb = _nblocks(N, block)
    nkb = _nblocks(k.shape[2], block)
    m4 = _mask4(mask, B, H, nqb, nkb)
    if qblocks is not None:
        out = {}
        for (b, h, i) in qblocks:
            out[(b, h, i)] = attention_qblock(q[b, h], k[b, h], v[b, h], block,
                                              m4[b, h, i] != 0, i, scale, causal)
        return out
    O = np.zeros((B, H, N, d))
    L = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            for i in range(nqb):
                r0, r1 = i * block, min(N, (i + 1) * block)
                O[b, h, r0:r1], L[b, h, r0:r1] = attention_qblock(
                    q[b, h], k[b, h], v[b, h], block, m4[b, h, i] != 0, i, scale, causal)
    return O, L


def dense_attention(q, k, v, scale=None):
    """Textbook softmax(Q K^T * scale) V over all keys (no mask)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    s = np.einsum("bhnd,bhmd->bhnm", q, k) * scale
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=-1, keepdims=True)
    return np.einsum("bhnm,bhmd->bhnd", e / z, v), (m + np.log(z))[..., 0]


def block_mask_to_token_mask(mask_bh, N, block):
    """Expand one head's [Nqb, Nkb] block mask to a boolean [N, N] token mask."""
    m = np.asarray(mask_bh) != 0
    idx = np.arange(N) // block
    return m[idx][:, idx]
