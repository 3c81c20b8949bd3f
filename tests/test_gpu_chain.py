"""GPU parity of the LiteAttention denoising chain at its full size: the
Wan2.1-14B-like 720p workload (40 heads, 21 x 45 x 80 = 75,600 tokens, block
128), 50 denoising steps with the drift x <- bf16(0.98 x + 0.2 xi) applied to
Q, K and V and the skip mask carried from each step to the next (LiteAttention
write-up, sections 2, 3 and 6: the persistent tile-level skip mask).

The GPU runs the whole chain, every head and every q-block, exactly as the
bench does.  The oracle runs its own chain for a fixed sample of q-blocks of
heads 0, 13, 26 and 39 (a q-block's skip row depends only on its own rows, so
the sample is exact for those rows): at every step O, LSE and the new skip row
of each sampled q-block are compared.  The oracle's skip rows are then written
into the GPU's next skip mask at those positions (they agree except on
flagged bits), so a flagged bit cannot make the two chains drift apart; no
oracle input ever comes from the GPU.

eps = 10 is the workload's threshold (on this generator it skips nothing, so
the chain is 50 steps of full attention on drifting inputs); eps = 2 makes
roughly half the pairs skip after the first step, so the carried bits, the
skipped tiles and the growing skip mask are exercised at full size.
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_flash_b200 import build, inputs, ops
from oracle import lite_step
from _parity import check_o, check_lse, check_bits, skip_flags

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

HEADS = [0, 13, 26, 39]
STEPS = 50


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    yield
    ops.sa_get_device_status()


def _samples(nb, per_head, seed):
    g = np.random.default_rng(seed)
    out = []
    for hh in range(len(HEADS)):
        rows = set(g.choice(nb - 1, size=per_head, replace=False).tolist())
        if hh == len(HEADS) - 1:
            rows.add(nb - 1)                 # the partial last q-block (80 rows)
        out += [(0, hh, int(i)) for i in sorted(rows)]
    return out


@pytest.mark.parametrize("eps,per_head", [(10.0, 1), (2.0, 2)])
def test_wan14b_720p_lite_chain_50_steps(eps, per_head):
    wl = inputs.WORKLOADS["wan14b_720p_lite"]
    nb, block, N = wl.nblocks, wl.block, wl.N
    samples = _samples(nb, per_head, seed=int(eps * 7))
    q, k, v = inputs.rff_qkv(wl, device="cuda")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(wl.seed + 1)
    skip = torch.zeros(1, wl.H, nb, nb, dtype=torch.uint8, device="cuda")
    state = {key: np.zeros(nb, dtype=np.uint8) for key in samples}       # the oracle's skip rows
    lse = torch.empty(1, wl.H, N, device="cuda")
    n_flag, n_bits, density = 0, 0, []
    for s in range(STEPS):
        nxt = torch.empty_like(skip)
        O = ops.sa_sparse_attn_fwd(q, k, v, block, skip_in=skip, skip_out=nxt, eps=eps, lse=lse)
        ops.sa_get_device_status()
        density.append(1.0 - skip.float().mean().item())
        qh, kh, vh = (t[:, HEADS].cpu() for t in (q, k, v))
        skip_in = np.zeros((1, len(HEADS), nb, nb), dtype=np.uint8)
        for (b, hh, i), row in state.items():
            skip_in[b, hh, i] = row
        ref = lite_step(qh, kh, vh, block, None, skip_in, eps, qblocks=samples)
        Oh, Lh, Sh = O[:, HEADS].cpu(), lse[:, HEADS].cpu(), nxt[:, HEADS].cpu().numpy()
        got_o, got_l, want_o, want_l, got_s, want_s, flags = [], [], [], [], [], [], []
        for (b, hh, i), (o, l, srow, mrow) in ref.items():
            r0, r1 = i * block, min(N, (i + 1) * block)
            got_o.append(Oh[b, hh, r0:r1]), got_l.append(Lh[b, hh, r0:r1])
            want_o.append(o), want_l.append(l)
            got_s.append(Sh[b, hh, i]), want_s.append(srow), flags.append(skip_flags(mrow))
        what = f"lite chain eps={eps} step {s}"
        check_o(torch.cat(got_o), np.concatenate(want_o), what)
        check_lse(torch.cat(got_l), np.concatenate(want_l), what)
        n_flag += check_bits(np.stack(got_s), np.stack(want_s), np.stack(flags), what)
        for (b, hh, i), (_, _, srow, _) in ref.items():
            assert np.all(srow >= state[(b, hh, i)]), f"{what}: the skip mask must only grow"
            state[(b, hh, i)] = srow
            nxt[b, HEADS[hh], i] = torch.from_numpy(srow).to(nxt.device)
        n_bits += int(sum(r.sum() for r in state.values()))
        skip = nxt
        if s + 1 < STEPS:
            q, k, v = inputs.drift(q, gen), inputs.drift(k, gen), inputs.drift(v, gen)
    print(f"[chain] eps={eps}: {len(samples)} q-blocks x {STEPS} steps checked, {n_flag} flagged skip bits, "
          f"density of the GPU chain per step: first {density[0]:.3f}, last {density[-1]:.3f}")
    if eps == 10.0:
        assert n_bits == 0 and min(density) == 1.0
    else:
        assert n_bits > 0 and density[-1] < 0.7
