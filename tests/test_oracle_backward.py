"""Pins for the oracle's attention backward pass (CPU only).

The gradient formulas are checked against things other than themselves:
central finite differences of the (separately pinned) forward oracle,
torch autograd of the textbook dense formula, and the translation invariance
of the keys (a shift of every key by one vector changes each row's logits by
a constant, so the key gradients sum to zero).
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_flash_b200 import inputs
from oracle import masked_attention, masked_attention_bwd, masked_attention_bwd_rows


def _case(N=40, d=8, block=16, seed=3):
    g = np.random.default_rng(seed)
    q, k, v = (g.normal(size=(1, 1, N, d)) for _ in range(3))
    dout = g.normal(size=(1, 1, N, d))
    nb = -(-N // block)
    mask = (g.random((1, 1, nb, nb)) < 0.6).astype(np.uint8)
    mask[0, 0, 0, :] = 0          # q-block 0 keeps nothing
    mask[0, 0, 1:, 1] = 0         # k-block 1 is kept by no q-block
    mask[0, 0, 1:, 2] = 1
    return q, k, v, dout, block, mask


def test_finite_differences_every_entry():
    """dL/dX for L = sum(O * dO), every entry of Q, K and V, by central
    differences of the forward oracle (h = 1e-5)."""
    q, k, v, dout, block, mask = _case()
    dq, dk, dv = masked_attention_bwd(q, k, v, block, mask, dout)
    h = 1e-5

    def loss(q_, k_, v_):
        o, _ = masked_attention(q_, k_, v_, block, mask)
        return float(np.sum(o * dout))

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        assert np.max(np.abs(num - g)) < 1e-7, name


def test_dense_case_equals_torch_autograd():
    g = torch.Generator().manual_seed(5)
    B, H, N, d = 1, 2, 70, 16
    q, k, v, do = (torch.randn(B, H, N, d, generator=g, dtype=torch.float64) for _ in range(4))
    qa, ka, va = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = torch.softmax(qa @ ka.transpose(-1, -2) / math.sqrt(d), dim=-1) @ va
    o.backward(do)
    dq, dk, dv = masked_attention_bwd(q.numpy(), k.numpy(), v.numpy(), 32, None, do.numpy())
    for ref, got in ((qa.grad, dq), (ka.grad, dk), (va.grad, dv)):
        assert np.max(np.abs(ref.numpy() - got)) < 1e-12


def test_empty_rows_and_columns_and_key_shift_invariance():
    q, k, v, dout, block, mask = _case(N=72, d=16, block=16, seed=8)
    dq, dk, dv = masked_attention_bwd(q, k, v, block, mask, dout)
    assert np.all(dq[0, 0, :block] == 0)                  # q-block 0 keeps nothing
    assert np.all(dk[0, 0, block:2 * block] == 0) and np.all(dv[0, 0, block:2 * block] == 0)
    assert np.max(np.abs(dk.sum(axis=2))) < 1e-12         # key gradients sum to zero
    assert np.max(np.abs(dv.sum(axis=2) - dout[0, 0, block:].sum(axis=0))) < 1e-12  # rows of P sum to 1


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_rows_equal_full_gradients(causal):
    """The chunked row sampler agrees with the full backward (itself pinned by finite
    differences and autograd), on a random block mask with and without the causal cut; the
    sampled rows include block edges (63, 64, 127) and the last, partial block's rows."""
    wl = inputs.Workload("b", 1, 2, 32, 3, 10, 10, 64, "tau", seed=11)
    q, k, v = inputs.rff_qkv(wl)
    do = inputs.normal_qkv(1, 2, wl.N, 32, seed=12)[0]
    nb = wl.nblocks
    mask = inputs.bernoulli_block_mask(1, 2, nb, nb, 0.5, seed=13)
    dq, dk, dv = masked_attention_bwd(q, k, v, wl.block, mask, do, causal=causal)
    qr = [0, 5, 63, 64, 200, wl.N - 1]
    kr = [1, 64, 127, 150, wl.N - 1]
    for h in range(2):
        sq, sk, sv = masked_attention_bwd_rows(q, k, v, wl.block, mask, do, 0, h, qr, kr, chunk=96, causal=causal)
        assert np.max(np.abs(sq - dq[0, h, qr])) < 1e-12
        assert np.max(np.abs(sk - dk[0, h, kr])) < 1e-12
        assert np.max(np.abs(sv - dv[0, h, kr])) < 1e-12


def test_pins_catch_planted_mistakes(monkeypatch):
    """Each planted mistake (dropped D term, missing scale in dQ) must break
    the key-shift invariance or the finite-difference pin."""
    import oracle.backward as ob

    q, k, v, dout, block, mask = _case(N=24, d=4, block=8, seed=21)
    good = ob.attention_bwd_head

    def no_d(qh, kh, vh, doh, keep, scale):
        s = np.where(keep, (qh @ kh.T) * scale, -np.inf)
        p = ob._softmax_rows(s)
        ds = p * (doh @ vh.T)
        return scale * (ds @ kh), scale * (ds.T @ qh), p.T @ doh

    def no_scale_dq(qh, kh, vh, doh, keep, scale):
        dq, dk, dv = good(qh, kh, vh, doh, keep, scale)
        return dq / scale, dk, dv

    def fd_q(i):
        h = 1e-5
        xp, xm = q.copy(), q.copy()
        xp[0, 0, i, 0] += h
        xm[0, 0, i, 0] -= h
        op, _ = masked_attention(xp, k, v, block, mask)
        om, _ = masked_attention(xm, k, v, block, mask)
        return float(np.sum((op - om) * dout)) / (2 * h)

    for bad in (no_d, no_scale_dq):
        monkeypatch.setattr(ob, "attention_bwd_head", bad)
        dq, dk, _ = ob.masked_attention_bwd(q, k, v, block, mask, dout)
        shift_ok = np.max(np.abs(dk.sum(axis=2))) < 1e-12
        fd_ok = all(abs(fd_q(i) - dq[0, 0, i, 0]) < 1e-7 for i in range(block, 24))
        assert not (shift_ok and fd_ok), bad.__name__
    monkeypatch.setattr(ob, "attention_bwd_head", good)


def test_causal_finite_differences():
    q, k, v, dout, block, mask = _case(N=24, d=4, block=8, seed=31)
    mask[:] = 1
    mask[0, 0, 2, 1] = 0
    dq, dk, dv = masked_attention_bwd(q, k, v, block, mask, dout, causal=True)
    h = 1e-5

    def loss(q_, k_, v_):
        o, _ = masked_attention(q_, k_, v_, block, mask, causal=True)
        return float(np.sum(o * dout))

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in [(0, 0, 0, 0), (0, 0, 5, 1), (0, 0, 13, 2), (0, 0, 23, 3), (0, 0, 17, 0)]:
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": lambda y: (y, k, v), "k": lambda y: (q, y, v), "v": lambda y: (q, k, y)}[name]
            num = (loss(*args(xp)) - loss(*args(xm))) / (2 * h)
            assert abs(num - g[idx]) < 1e-7, (name, idx)
    # the last key takes part only in the last row: its gradients come from that row alone
    assert np.max(np.abs(dk[0, 0, :23].sum(axis=0) + dk[0, 0, 23])) < 1e-12
