"""The seeded input generators (CPU only): the recipe the design states for
the synthetic workloads, checked on small grids.

Locality generator: random Fourier features of the (t, h, w) coordinates,
one shared projection L per head, Q = 0.7 L + 0.3 xi_Q, K = 0.7 L + 0.3 xi_K,
V ~ N(0, 1), all bf16; denoising drift x -> bf16(0.98 x + 0.2 xi).
"""
import math

import torch

from block_sparse_attention_flash_b200 import inputs


def _wl(**kw):
    base = dict(name="t", B=1, H=3, d=64, T=6, Hh=8, Ww=10, block=64, kind="tau", seed=123)
    base.update(kw)
    return inputs.Workload(base.pop("name"), base.pop("B"), base.pop("H"), base.pop("d"), base.pop("T"),
                           base.pop("Hh"), base.pop("Ww"), base.pop("block"), base.pop("kind"), **base)


def test_raster_coordinates():
    c = inputs.grid_coords(2, 3, 4)
    assert c.shape == (24, 3)
    n = 17                                  # (t, h, w) = (1, 1, 1): n = (t*3 + h)*4 + w
    assert c[n].tolist() == [1.0, 1.0, 1.0]
    assert c[:, 2].tolist()[:5] == [0.0, 1.0, 2.0, 3.0, 0.0]


def test_seeded_bf16_and_head_prefix():
    wl = _wl()
    q, k, v = inputs.rff_qkv(wl)
    assert q.dtype == torch.bfloat16 and q.shape == (1, 3, wl.N, wl.d)
    q2, k2, v2 = inputs.rff_qkv(wl)
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    q1, k1, v1 = inputs.rff_qkv(wl, H=1)          # fewer heads: the first heads of the full draw
    assert torch.equal(q1[:, 0], q[:, 0]) and torch.equal(v1[:, 0], v[:, 0])
    assert not torch.equal(q[:, 0], q[:, 1])       # heads differ
    q3, _, _ = inputs.rff_qkv(_wl(seed=124))
    assert not torch.equal(q3, q)                  # the seed matters


def test_variances_and_shared_projection():
    """Var(L) is about 1 (sqrt(2/D)-scaled cosines times an N(0,1) matrix), so
    Var(Q) = Var(K) = 0.49 + 0.09 = 0.58, Cov(Q, K) = 0.49 per entry, Var(V) = 1."""
    q, k, v = (x.float() for x in inputs.rff_qkv(_wl(H=4, T=8, Hh=16, Ww=16)))
    assert abs(v.var().item() - 1.0) < 0.02
    assert abs(q.var().item() - 0.58) < 0.08 and abs(k.var().item() - 0.58) < 0.08
    cov = ((q - q.mean()) * (k - k.mean())).mean().item()
    assert abs(cov - 0.49) < 0.08
    assert abs((q * v).mean().item()) < 0.02        # V independent of Q


def test_locality_nearby_tokens_score_higher():
    """The shared L makes q_r . k_c larger for tokens close in (t, h, w) than
    for distant ones: the structure the block masks are built on."""
    wl = _wl(H=2, T=8, Hh=16, Ww=16)
    q, k, _ = (x.float()[0] for x in inputs.rff_qkv(wl))
    c = inputs.grid_coords(wl.T, wl.Hh, wl.Ww)
    g = torch.Generator().manual_seed(0)
    r = torch.randint(0, wl.N, (400,), generator=g)
    dist = torch.cdist(c[r], c)                     # (400, N)
    for h in range(2):
        s = (q[h, r] @ k[h].T) / math.sqrt(wl.d)
        near = s[(dist > 0) & (dist <= 1.5)].mean().item()
        far = s[dist > 12].mean().item()
        assert near > far + 1.0, (h, near, far)


def test_drift_step():
    g = torch.Generator().manual_seed(5)
    x = torch.randn(4, 1000, generator=g).to(torch.bfloat16)
    g1, g2 = torch.Generator().manual_seed(9), torch.Generator().manual_seed(9)
    y = inputs.drift(x, g1)
    xi = torch.randn(x.shape, generator=g2)
    assert y.dtype == torch.bfloat16
    assert torch.equal(y, (0.98 * x.float() + 0.2 * xi).to(torch.bfloat16))


def test_chain_inputs_start_at_the_locality_draw():
    wl = _wl(H=1, T=2, Hh=4, Ww=8)
    steps = list(inputs.lite_chain_inputs(wl, 3, H=1))
    assert len(steps) == 3
    q0, _, _ = inputs.rff_qkv(wl, H=1)
    assert torch.equal(steps[0][0], q0)
    assert not torch.equal(steps[1][0], steps[0][0])


def test_bernoulli_mask_and_constant_groups():
    m = inputs.bernoulli_block_mask(1, 2, 9, 9, 0.3, seed=4)
    assert m.dtype == torch.uint8 and torch.all(m[:, :, range(9), range(9)] == 1)
    k, v = inputs.const_group_kv(1, 1, 21, 8, 8, seed=2)
    assert torch.equal(k[0, 0, 0], k[0, 0, 7]) and torch.equal(v[0, 0, 16], v[0, 0, 20])
    assert not torch.equal(k[0, 0, 7], k[0, 0, 8])
