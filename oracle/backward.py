"""Backward pass of block-masked softmax attention, fp64 (oracle; test infrastructure only).

Why a backward pass: the Radial Attention write-up ("MIT实验室推出Radial
Attention", arXiv 2506.19852) extends pretrained video models to 4x longer
videos by LoRA fine-tuning through the sparse attention (its training-cost
paragraph: 4.4x lower), which needs the gradients of the masked attention
with respect to Q, K and V over the same block masks.

The gradient is the derivative of the forward definition in
``oracle/attention.py`` (no page states it; it follows from the chain rule
through the row softmax).  For one head, with M the token keep matrix
expanded from the block mask (and, with the causal option, restricted to
key c <= row r) and dO the incoming gradient of O:

    S    = scale * Q K^T,  S_rc = -inf where M_rc = 0
    P    = row softmax of S (a row with no kept column is all zero)
    dV   = P^T dO
    dP   = dO V^T
    D_r  = sum_c P_rc dP_rc            (= dO_r . O_r)
    dS   = P * (dP - D)                (elementwise, D broadcast over c)
    dQ   = scale * dS K
    dK   = scale * dS^T Q
"""
from __future__ import annotations

import math

import numpy as np

from .attention import _f64, _nblocks, _mask4, block_mask_to_token_mask


def _softmax_rows(s):
    """Row softmax of s; rows whose entries are all -inf give zeros."""
    m = s.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    return np.divide(e, z, out=np.zeros_like(e), where=z > 0)


def attention_bwd_head(qh, kh, vh, doh, keep, scale):
    """(dQ, dK, dV) of one head: qh [N,d], kh/vh [Nk,d], doh [N,d], keep [N,Nk] bool."""
    s = np.where(keep, (qh @ kh.T) * scale, -np.inf)
    p = _softmax_rows(s)
    dv = p.T @ doh
    dp = doh @ vh.T
    dr = np.sum(p * dp, axis=1, keepdims=True)
    ds = p * (dp - dr)
    return scale * (ds @ kh), scale * (ds.T @ qh), dv


def masked_attention_bwd(q, k, v, block, mask, dout, scale=None, causal=False):
    """Gradients (dQ, dK, dV), fp64 [B,H,N,d] each, of block-masked attention.

    mask: None (all kept) or anything broadcastable to uint8 [B, H, Nb, Nb];
    dout: the gradient of the loss with respect to O, [B, H, N, d].
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    nb = _nblocks(N, block)
    m4 = _mask4(mask, B, H, nb, nb)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            keep = block_mask_to_token_mask(m4[b, h], N, block)
            if causal:
                keep = keep & np.tri(N, dtype=bool)
            dq[b, h], dk[b, h], dv[b, h] = attention_bwd_head(q[b, h], k[b, h], v[b, h], do[b, h], keep, scale)
    return dq, dk, dv


def masked_attention_bwd_rows(q, k, v, block, mask, dout, b, h, q_rows, k_rows, scale=None, chunk=1024,
                              causal=False):
    """Selected rows of dQ (query rows ``q_rows``) and of dK, dV (key rows
    ``k_rows``) of head (b, h), for sizes where the full N x N matrices do not
    fit.  The same formulas as ``attention_bwd_head``, evaluated over chunks of
    query rows: every query row's softmax and D_r are needed for the key rows'
    gradients, so all rows are visited; only the selected outputs are kept.
    Returns (dQ [len(q_rows), d], dK [len(k_rows), d], dV [len(k_rows), d]).
    """
    B, H = q.shape[0], q.shape[1]
    qh, kh, vh, doh = (_f64(x[b, h]) for x in (q, k, v, dout))
    N, d = qh.shape
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    nb = _nblocks(N, block)
    m = np.asarray(_mask4(mask, B, H, nb, nb)[b, h]) != 0
    q_rows = np.asarray(q_rows, dtype=np.int64)
    k_rows = np.asarray(k_rows, dtype=np.int64)
    kblk = np.arange(N) // block
    dq = np.zeros((q_rows.size, d))
    dk = np.zeros((k_rows.size, d))
    dv = np.zeros((k_rows.size, d))
    for r0 in range(0, N, chunk):
        r1 = min(N, r0 + chunk)
        rows = np.arange(r0, r1)
        keep = m[(rows // block)[:, None], kblk[None, :]]
        if causal:
            keep = keep & (np.arange(N)[None, :] <= rows[:, None])
        s = np.where(keep, (qh[r0:r1] @ kh.T) * scale, -np.inf)
        p = _softmax_rows(s)
        o = p @ vh
        dr = np.sum(doh[r0:r1] * o, axis=1, keepdims=True)          # D_r = dO_r . O_r
        # key rows: the columns k_rows of P and dS for every query row
        pc = p[:, k_rows]
        dsc = pc * (doh[r0:r1] @ vh[k_rows].T - dr)
        dk += scale * (dsc.T @ qh[r0:r1])
        dv += pc.T @ doh[r0:r1]
        # query rows that fall in this chunk: full rows of dS
        sel = np.nonzero((q_rows >= r0) & (q_rows < r1))[0]
        if sel.size:
            loc = q_rows[sel] - r0
            ds = p[loc] * (doh[q_rows[sel]] @ vh.T - dr[loc])
            dq[sel] = scale * (ds @ kh)
    return dq, dk, dv
