"""GPU parity: PSA pyramid attention (sa_pyramid_pool + sa_pyramid_attn_fwd) vs the oracle.

The oracle pools K/V in fp64 and the GPU pools in fp32 and stores bf16; the
difference is absorbed by the O tolerance.  Level maps handed to the oracle
come from the oracle itself or from seeded draws, never from the GPU mask
builder; the end-to-end case runs the GPU attention on the GPU-built map and
compares only q-blocks whose GPU row equals the oracle's row.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_flash_b200 import build, inputs, ops
from oracle import pyramid_attention, masked_attention, dense_attention, level_map
from _parity import check_o, check_lse, check_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    yield
    ops.sa_get_device_status()


def run_pyr(q, k, v, block, codes, causal=False):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    B, H, N, d = q.shape
    kp, vp = ops.sa_pyramid_pool(kd, vd, block)
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda")
    ops.sa_pyramid_attn_fwd(qd, kd, vd, block, codes.cuda(), kp, vp, out=out, lse=lse, causal=causal)
    ops.sa_get_device_status()
    return out.cpu(), lse.cpu()


def _codes(B, H, nb, seed, p_drop=0.1):
    g = torch.Generator().manual_seed(seed)
    c = torch.randint(1, 5, (B, H, nb, nb), generator=g)
    drop = torch.rand(B, H, nb, nb, generator=g) < p_drop
    c[drop] = 0
    return c.to(torch.uint8)


@pytest.mark.parametrize("block", [64, 128])
def test_level_zero_only_equals_block_attention(block):
    B, H, N, d = 1, 2, 1000, 128
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=block)
    nb = -(-N // block)
    m = inputs.bernoulli_block_mask(B, H, nb, nb, 0.6, seed=block + 1)
    O, L = run_pyr(q, k, v, block, m)                 # codes 0/1 only
    Or, Lr = masked_attention(q, k, v, block, m)
    check_o(O, Or, "pyramid level 0")
    check_lse(L, Lr, "pyramid level 0")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("N", [200, 1000, 1031, 2048 + 64 * 3 + 8])
def test_random_levels_ragged(d, block, N):
    B, H = 1, 2
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=N + d + block)
    nb = -(-N // block)
    codes = _codes(B, H, nb, seed=N * 3 + block)
    if nb > 2:
        codes[0, 1, 2, :] = 0                          # a q-block that drops everything
    O, L = run_pyr(q, k, v, block, codes)
    Or, Lr = pyramid_attention(q, k, v, block, codes.numpy())
    check_o(O, Or, f"pyramid N={N} d={d} block={block}")
    check_lse(L, Lr, f"pyramid N={N} d={d} block={block}")
    if nb > 2:
        rows = slice(2 * block, min(N, 3 * block))
        assert torch.all(O[0, 1, rows] == 0) and torch.all(L[0, 1, rows] == -np.inf)


@pytest.mark.parametrize("block", [64, 128])
def test_constant_groups_match_dense_attention(block):
    """K/V constant over 8-token groups: any level mix must reproduce full attention."""
    B, H, N, d = 1, 2, 64 * 9 + 40, 128
    q = torch.randn(B, H, N, d, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    k, v = inputs.const_group_kv(B, H, N, d, 8, seed=4)
    nb = -(-N // block)
    codes = _codes(B, H, nb, seed=5, p_drop=0.0)
    O, L = run_pyr(q, k, v, block, codes)
    Od, Ld = dense_attention(q, k, v)
    check_o(O, Od, "pyramid exactness")
    check_lse(L, Ld, "pyramid exactness")


def test_psa_480p_full_sampled():
    """The PSA workload at full size: 12 heads, 32,760 tokens, block 64,
    oracle level quotas 10/20/30/40 %, sampled q-blocks checked."""
    wl = inputs.WORKLOADS["psa_480p_pyramid"]
    q, k, v = inputs.rff_qkv(wl, device="cuda")
    nb = wl.nblocks
    heads = [0, 6, 11]
    qh, kh, vh = (t[:, heads].cpu() for t in (q, k, v))
    lv = level_map(qh, kh, wl.block, wl.level_frac)
    codes = torch.ones(1, wl.H, nb, nb, dtype=torch.uint8)
    codes[:, heads] = torch.from_numpy(lv)
    kp, vp = ops.sa_pyramid_pool(k, v, wl.block)
    lse = torch.empty(1, wl.H, wl.N, device="cuda")
    O = ops.sa_pyramid_attn_fwd(q, k, v, wl.block, codes.cuda(), kp, vp, lse=lse)
    ops.sa_get_device_status()
    g = np.random.default_rng(7)
    samples = []
    for hh in range(len(heads)):
        rows = sorted(set([0, nb - 1] + list(g.choice(nb, size=4, replace=False))))
        samples += [(0, hh, int(i)) for i in rows]
    ref = pyramid_attention(qh, kh, vh, wl.block, lv, qblocks=samples)
    Oh, Lh = O[:, heads].cpu(), lse[:, heads].cpu()
    got_o, got_l, want_o, want_l = [], [], [], []
    for (b, hh, i), (o, l) in ref.items():
        r0, r1 = i * wl.block, min(wl.N, (i + 1) * wl.block)
        got_o.append(Oh[b, hh, r0:r1]), got_l.append(Lh[b, hh, r0:r1])
        want_o.append(o), want_l.append(l)
    check_o(torch.cat(got_o), np.concatenate(want_o), "psa 480p")
    check_lse(torch.cat(got_l), np.concatenate(want_l), "psa 480p")


def test_psa_480p_gpu_pipeline():
    """The PSA workload as the bench runs it, all on the GPU: level map from
    sa_build_mask (12 heads x 512 x 512, the E = 16 warp selection), pooling,
    then pyramid attention on that map.  The map is checked against the
    oracle's for every head (flag-aware); the attention on sampled q-blocks of
    three heads whose GPU level row is identical to the oracle's row, against
    the oracle's attention on its own map."""
    wl = inputs.WORKLOADS["psa_480p_pyramid"]
    q, k, v = inputs.rff_qkv(wl, device="cuda")
    nb = wl.nblocks
    lv = ops.sa_build_mask(q, k, wl.block, "levels", level_frac=wl.level_frac)
    kp, vp = ops.sa_pyramid_pool(k, v, wl.block)
    lse = torch.empty(1, wl.H, wl.N, device="cuda")
    O = ops.sa_pyramid_attn_fwd(q, k, v, wl.block, lv, kp, vp, lse=lse)
    ops.sa_get_device_status()
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    lv_ref, flags, _ = level_map(qc, kc, wl.block, wl.level_frac, return_info=True)
    lv_gpu = lv.cpu().numpy()
    check_bits(lv_gpu, lv_ref, flags, "levels 480p, 12 heads")
    heads = [0, 6, 11]
    same = (lv_gpu == lv_ref).all(axis=-1)[0]              # [H, nb]: rows the two maps agree on
    g = np.random.default_rng(17)
    samples = []
    for hh, h in enumerate(heads):
        ok = np.nonzero(same[h])[0]
        assert ok.size >= nb - 8, f"head {h}: {nb - ok.size} level rows differ"
        pick = set(g.choice(ok, size=4, replace=False).tolist())
        pick |= {i for i in (0, nb - 1) if same[h, i]}
        samples += [(0, hh, int(i)) for i in sorted(pick)]
    ref = pyramid_attention(qc[:, heads], kc[:, heads], vc[:, heads], wl.block, lv_ref[:, heads], qblocks=samples)
    Oh, Lh = O[:, heads].cpu(), lse[:, heads].cpu()
    got_o, got_l, want_o, want_l = [], [], [], []
    for (b, hh, i), (o, l) in ref.items():
        r0, r1 = i * wl.block, min(wl.N, (i + 1) * wl.block)
        got_o.append(Oh[b, hh, r0:r1]), got_l.append(Lh[b, hh, r0:r1])
        want_o.append(o), want_l.append(l)
    check_o(torch.cat(got_o), np.concatenate(want_o), "psa 480p GPU pipeline")
    check_lse(torch.cat(got_l), np.concatenate(want_l), "psa 480p GPU pipeline")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("N", [1031, 2048 + 64 * 3 + 8])
def test_causal_random_levels_ragged(d, block, N):
    """Causal option: future blocks dropped, the diagonal block at level 0 with
    the per-row cut, earlier blocks at their levels; one q-block whose
    diagonal block is dropped by the map."""
    B, H = 1, 2
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=N + d + block + 1)
    nb = -(-N // block)
    codes = _codes(B, H, nb, seed=N * 5 + block)
    codes[0, 0, 3, 3] = 0
    O, L = run_pyr(q, k, v, block, codes, causal=True)
    Or, Lr = pyramid_attention(q, k, v, block, codes.numpy(), causal=True)
    check_o(O, Or, f"causal pyramid N={N} d={d} block={block}")
    check_lse(L, Lr, f"causal pyramid N={N} d={d} block={block}")


def test_batch_two_broadcast_levels():
    """B = 2, H = 3 with one [Nb, Nb] level map broadcast over batch and heads."""
    B, H, N, d, block = 2, 3, 64 * 11 + 40, 128, 64
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=84)
    nb = -(-N // block)
    codes = _codes(1, 1, nb, seed=85)[0, 0]
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kp, vp = ops.sa_pyramid_pool(kd, vd, block)
    lse = torch.empty(B, H, N, device="cuda")
    out = ops.sa_pyramid_attn_fwd(qd, kd, vd, block, codes.cuda(), kp, vp, lse=lse)
    ops.sa_get_device_status()
    Or, Lr = pyramid_attention(q, k, v, block, codes.numpy())
    check_o(out.cpu(), Or, "pyramid batch 2")
    check_lse(lse.cpu(), Lr, "pyramid batch 2")
