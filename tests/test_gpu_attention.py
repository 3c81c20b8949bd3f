"""GPU parity: sa_sparse_attn_fwd (binary masks, LiteAttention skip update) vs the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_flash_b200 import build, inputs, ops
from oracle import masked_attention, lite_step, radial_mask
from _parity import check_o, check_lse, check_bits, skip_flags

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    yield
    ops.sa_get_device_status()


def run_attn(q, k, v, block, mask=None, skip_in=None, skip_out=None, eps=math.inf, with_lse=True,
             order="ascending", causal=False):
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    B, H, N, d = q.shape
    # poison the output so unwritten rows show up
    out = torch.full_like(qd, float("nan"))
    lse = torch.full((B, H, N), float("nan"), device="cuda") if with_lse else None
    ops.sa_sparse_attn_fwd(qd, kd, vd, block, mask=None if mask is None else mask.cuda(),
                           skip_in=skip_in, skip_out=skip_out, eps=eps, out=out, lse=lse, order=order,
                           causal=causal)
    ops.sa_get_device_status()
    return out.cpu(), (lse.cpu() if lse is not None else None)


def test_tiny_all_ones_equals_dense():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.normal_qkv(wl.B, wl.H, wl.N, wl.d, wl.seed)
    O, L = run_attn(q, k, v, wl.block)
    Or, Lr = masked_attention(q, k, v, wl.block, None)
    check_o(O, Or, "tiny dense")
    check_lse(L, Lr, "tiny dense")


def test_tiny_bernoulli_mask():
    wl = inputs.WORKLOADS["tiny"]
    q, k, v = inputs.normal_qkv(wl.B, wl.H, wl.N, wl.d, wl.seed)
    m = inputs.bernoulli_block_mask(wl.B, wl.H, wl.nblocks, wl.nblocks, 0.5, wl.seed + 1)
    O, L = run_attn(q, k, v, wl.block, m)
    Or, Lr = masked_attention(q, k, v, wl.block, m)
    check_o(O, Or, "tiny bernoulli")
    check_lse(L, Lr, "tiny bernoulli")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("N", [1, 77, 130, 1000, 2065])
def test_ragged_random_masks(d, block, N):
    B, H = 2, 2
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=N * 7 + d + block)
    nb = -(-N // block)
    m = inputs.bernoulli_block_mask(B, H, nb, nb, 0.45, seed=N + 3, force_diagonal=True)
    if nb > 2:
        m[0, 1, 1, :] = 0                      # a q-block with no kept block
    O, L = run_attn(q, k, v, block, m)
    Or, Lr = masked_attention(q, k, v, block, m)
    check_o(O, Or, f"N={N} d={d} block={block}")
    check_lse(L, Lr, f"N={N} d={d} block={block}")
    if nb > 2:
        rows = slice(block, min(N, 2 * block))
        assert torch.all(O[0, 1, rows] == 0)
        assert torch.all(L[0, 1, rows] == -math.inf)


def test_unit_values_rows_sum_to_one():
    B, H, N, d, block = 1, 3, 1500, 128, 128
    q, k, _ = inputs.normal_qkv(B, H, N, d, seed=5)
    v = torch.ones_like(q)
    nb = -(-N // block)
    m = inputs.bernoulli_block_mask(B, H, nb, nb, 0.3, seed=6)
    O, _ = run_attn(q, k, v, block, m, with_lse=False)
    assert torch.all((O.float() - 1.0).abs() <= 8e-3)


def test_radial_mask_broadcast_over_heads():
    T, Hh, Ww, block = 12, 8, 16, 128
    wl = inputs.Workload("r", 1, 3, 128, T, Hh, Ww, block, "radial", seed=31)
    q, k, v = inputs.rff_qkv(wl)
    rm = torch.from_numpy(radial_mask(T, Hh, Ww, block))
    O, L = run_attn(q, k, v, block, rm)             # [Nb, Nb] mask: strides (0, 0, Nb)
    Or, Lr = masked_attention(q, k, v, block, rm.numpy())
    check_o(O, Or, "radial broadcast")
    check_lse(L, Lr, "radial broadcast")


# ------------------------------------------------------------------ skip ---

def _skip_run(q, k, v, block, mask, skip_in, eps, alias=False, order="ascending", causal=False):
    B, H, N, d = q.shape
    nb = -(-N // block)
    si = skip_in.cuda() if skip_in is not None else None
    if alias:
        so = si
    else:
        so = torch.full((B, H, nb, nb), 77, dtype=torch.uint8, device="cuda")
    O, L = run_attn(q, k, v, block, mask, skip_in=si, skip_out=so, eps=eps, order=order, causal=causal)
    return O, L, so.cpu()


def _check_skip_step(q, k, v, block, mask, skip_in, eps, alias=False, order="ascending", causal=False):
    O, L, S = _skip_run(q, k, v, block, mask, skip_in, eps, alias, order, causal)
    Or, Lr, Sr, M = lite_step(q, k, v, block, None if mask is None else mask.numpy(),
                              None if skip_in is None else skip_in.numpy(), eps, order=order, causal=causal)
    check_o(O, Or, f"skip step eps={eps}")
    check_lse(L, Lr, f"skip step eps={eps}")
    nflag = check_bits(S, Sr, skip_flags(M), f"skip bits eps={eps}")
    return S, Sr, nflag


@pytest.mark.parametrize("d", [64, 128])
def test_hand_built_gap_of_twelve(d):
    block, nb = 128, 5
    N = block * nb
    a = math.sqrt(6.0 * math.sqrt(d))
    u = torch.zeros(d)
    u[3] = 1.0
    q = (a * u).repeat(N, 1).view(1, 1, N, d).to(torch.bfloat16)
    k = (-a * u).repeat(N, 1)
    k[:block] = a * u
    k = k.view(1, 1, N, d).to(torch.bfloat16)
    v = torch.randn(1, 1, N, d, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    S, Sr, _ = _check_skip_step(q, k, v, block, None, None, eps=10.0)
    assert S[0, 0, :, 1:].all() and not S[0, 0, :, 0].any()
    S, _, _ = _check_skip_step(q, k, v, block, None, None, eps=1e6)
    assert S.sum() == 0


@pytest.mark.parametrize("block", [64, 128])
def test_rff_skips_small_eps(block):
    wl = inputs.Workload("s", 1, 3, 128, 8, 16, 24, block, "lite", seed=41, sigma_s=2.0, sigma_t=1.5)
    q, k, v = inputs.rff_qkv(wl)
    S, Sr, nflag = _check_skip_step(q, k, v, block, None, None, eps=1.0)
    assert Sr.sum() > 0


@pytest.mark.parametrize("block", [64, 128])
def test_teacher_forced_chain_with_carry_and_alias(block):
    """Four denoising steps.  Each step's skip_in is the oracle's skip_out of
    the step before, handed to both sides, so a flagged bit cannot cascade and
    no oracle input comes from the GPU."""
    wl = inputs.Workload("c", 1, 2, 128, 6, 16, 24, block, "lite", seed=43, sigma_s=2.0, sigma_t=1.5)
    steps = list(inputs.lite_chain_inputs(wl, 4))
    nb = wl.nblocks
    mask = inputs.bernoulli_block_mask(1, wl.H, nb, nb, 0.8, seed=44)
    skip = None
    total = 0
    for s, (q, k, v) in enumerate(steps):
        S, Sr, _ = _check_skip_step(q, k, v, block, mask, skip, eps=1.2, alias=(s % 2 == 1 and skip is not None))
        if skip is not None:
            assert np.all(S.numpy() >= skip.numpy())      # monotone carry
        skip = torch.from_numpy(np.ascontiguousarray(Sr))
        total = int(Sr.sum())
    assert total > 0


def test_skip_in_blocks_are_not_visited():
    B, H, N, d, block = 1, 2, 1024, 128, 128
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=9)
    nb = N // block
    skip_in = inputs.bernoulli_block_mask(B, H, nb, nb, 0.3, seed=10, force_diagonal=False)
    skip_in[:, :, torch.arange(nb), torch.arange(nb)] = 0
    O, L, S = _skip_run(q, k, v, block, None, skip_in, eps=math.inf)
    Or, Lr = masked_attention(q, k, v, block, (1 - skip_in.numpy()))
    check_o(O, Or, "skip_in honoured")
    check_lse(L, Lr, "skip_in honoured")
    assert torch.equal(S, skip_in)                     # eps = inf: carry only


# ------------------------------------------------- radial-centric visit order ---

@pytest.mark.parametrize("block", [64, 128])
def test_radial_order_skip_step(block):
    """Radial-centric order on an RFF grid of 24 kv tiles (12 q-tile pairs):
    O, LSE and skip bits against the oracle walking the same order."""
    wl = inputs.Workload("r", 1, 3, 128, 8, 16, 24, block, "lite", seed=45, sigma_s=2.0, sigma_t=1.5)
    q, k, v = inputs.rff_qkv(wl)
    S, Sr, _ = _check_skip_step(q, k, v, block, None, None, eps=1.0, order="radial")
    _, Sa, _ = _check_skip_step(q, k, v, block, None, None, eps=1.0)
    assert Sr.sum() > 0 and not np.array_equal(Sr, Sa)   # the order changes the decisions


@pytest.mark.parametrize("block", [64, 128])
def test_radial_order_ragged_masked_chain(block):
    """Ragged tail (an odd q-tile count, a partial last tile), a random mask and
    a two-step teacher-forced chain with skip_out aliasing skip_in."""
    wl = inputs.Workload("rc", 1, 2, 128, 5, 13, 17, block, "lite", seed=46, sigma_s=2.0, sigma_t=1.5)
    steps = list(inputs.lite_chain_inputs(wl, 2))
    nb = wl.nblocks
    mask = inputs.bernoulli_block_mask(1, wl.H, nb, nb, 0.8, seed=47)
    skip = None
    for s, (q, k, v) in enumerate(steps):
        S, Sr, _ = _check_skip_step(q, k, v, block, mask, skip, eps=1.2, alias=skip is not None, order="radial")
        skip = torch.from_numpy(np.ascontiguousarray(Sr))
    assert int(skip.sum()) > 0


@pytest.mark.parametrize("d", [64, 128])
def test_radial_order_reaches_the_row_max_first(d):
    """Keys of k-blocks 4 and 5 give logit +6, the rest -6: q-blocks 4-7 skip
    every -6 block under the radial order, only blocks 6 and 7 in ascending order."""
    block, nb = 64, 8
    N = block * nb
    a = math.sqrt(6.0 * math.sqrt(d))
    u = torch.zeros(d)
    u[3] = 1.0
    q = (a * u).repeat(N, 1).view(1, 1, N, d).to(torch.bfloat16)
    k = (-a * u).repeat(N, 1)
    k[4 * block:6 * block] = a * u
    k = k.view(1, 1, N, d).to(torch.bfloat16)
    v = torch.randn(1, 1, N, d, generator=torch.Generator().manual_seed(2)).to(torch.bfloat16)
    S, _, _ = _check_skip_step(q, k, v, block, None, None, eps=10.0, order="radial")
    assert S[0, 0, 4].tolist() == [1, 1, 1, 1, 0, 0, 1, 1]
    S, _, _ = _check_skip_step(q, k, v, block, None, None, eps=10.0)
    assert S[0, 0, 4].tolist() == [0, 0, 0, 0, 0, 0, 1, 1]


# ------------------------------------------------------------------ causal ---

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [64, 128])
def test_causal_ragged_masks(d, block):
    """Causal option on a ragged sequence: all kept, then a Bernoulli mask with
    one q-block keeping only future blocks (no visible key) and one without
    its diagonal block."""
    B, H, N = 1, 2, 128 * 5 + 72
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=d * 3 + block)
    nb = -(-N // block)
    O, L = run_attn(q, k, v, block, None, causal=True)
    Or, Lr = masked_attention(q, k, v, block, None, causal=True)
    check_o(O, Or, f"causal all d={d} block={block}")
    check_lse(L, Lr, f"causal all d={d} block={block}")
    mask = inputs.bernoulli_block_mask(B, H, nb, nb, 0.6, seed=block + 3)
    mask[:, :, 1, :] = 0
    mask[:, :, 1, 4] = 1
    mask[:, :, 3, 3] = 0
    O, L = run_attn(q, k, v, block, mask, causal=True)
    Or, Lr = masked_attention(q, k, v, block, mask, causal=True)
    check_o(O, Or, f"causal masked d={d} block={block}")
    check_lse(L, Lr, f"causal masked d={d} block={block}")


@pytest.mark.parametrize("block", [64, 128])
def test_causal_skip_step_and_radial(block):
    wl = inputs.Workload("cs", 1, 2, 128, 4, 16, 24, block, "lite", seed=47, sigma_s=2.0, sigma_t=1.5)
    q, k, v = inputs.rff_qkv(wl)
    for order in ("ascending", "radial"):
        S, Sr, _ = _check_skip_step(q, k, v, block, None, None, eps=1.0, order=order, causal=True)
        nb = wl.nblocks
        iu = np.triu_indices(nb, 1)
        assert not S.numpy()[0, :, iu[0], iu[1]].any()        # future blocks never marked
        assert Sr.sum() > 0


# ------------------------------------------------------ host-buffer entry ---

@pytest.mark.parametrize("hc", [1, 2, 5])
def test_host_buffers_equal_device_path(hc):
    """Q, K, V, O in pinned host memory, streamed in chunks of hc heads (B = 2,
    H = 5, chunks that do not divide H): O, LSE and skip_out are identical to
    one device-path call, with a mask, a skip chain and the radial order."""
    B, H, N, d, block = 2, 5, 128 * 4 + 40, 128, 64
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=95)
    nb = -(-N // block)
    mask = inputs.bernoulli_block_mask(B, H, nb, nb, 0.7, seed=96).cuda()
    skip_in = inputs.bernoulli_block_mask(B, H, nb, nb, 0.2, seed=97, force_diagonal=False).cuda()
    lse_d = torch.empty(B, H, N, device="cuda")
    so_d = torch.zeros(B, H, nb, nb, dtype=torch.uint8, device="cuda")
    o_d = ops.sa_sparse_attn_fwd(q.cuda(), k.cuda(), v.cuda(), block, mask=mask, skip_in=skip_in, skip_out=so_d,
                                 eps=1.0, lse=lse_d, order="radial")
    hq, hk, hv = (t.pin_memory() for t in (q, k, v))
    ho = torch.empty_like(hq).pin_memory()
    lse_h = torch.empty(B, H, N, device="cuda")
    so_h = torch.zeros(B, H, nb, nb, dtype=torch.uint8, device="cuda")
    ops.sa_sparse_attn_fwd_host(hq, hk, hv, block, out=ho, mask=mask, skip_in=skip_in, skip_out=so_h, eps=1.0,
                                lse=lse_h, heads_per_chunk=hc, order="radial")
    torch.cuda.synchronize()
    ops.sa_get_device_status()
    assert torch.equal(ho, o_d.cpu())
    assert torch.equal(lse_h, lse_d)
    assert torch.equal(so_h, so_d)


def test_maximum_sequence_sampled_qblocks():
    """The longest supported sequence (4096 kv tiles: N = 524,288 - 40 tokens,
    d = 64, block 128) with a 5 % Bernoulli mask: sampled q-blocks (first,
    middle, last, ragged) against the oracle."""
    B, H, d, block = 1, 1, 64, 128
    N = 128 * 4096 - 40
    q, k, v = inputs.normal_qkv(B, H, N, d, seed=4097)
    nb = -(-N // block)
    mask = inputs.bernoulli_block_mask(B, H, nb, nb, 0.05, seed=4098)
    O, L = run_attn(q, k, v, block, mask)
    picks = [(0, 0, 0), (0, 0, 1), (0, 0, 2047), (0, 0, nb - 1)]
    ref = masked_attention(q, k, v, block, mask, qblocks=picks)
    for (b, h, i), (Or, Lr) in ref.items():
        r0, r1 = i * block, min(N, (i + 1) * block)
        check_o(O[b, h, r0:r1], Or, f"max N q-block {i}")
        check_lse(L[b, h, r0:r1], Lr, f"max N q-block {i}")
