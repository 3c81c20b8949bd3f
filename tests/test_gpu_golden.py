"""GPU pins against the hand-worked fixtures in tests/golden/: the CUDA
path's radial mask rows, token permutations, tau / global keep bits and
LiteAttention skip bits against values worked out by hand from the rules the
pages state (the oracle is not involved)."""
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_flash_b200 import build, ops
from _golden import floats, ints, matrix, records

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    yield
    ops.sa_get_device_status()


@pytest.mark.parametrize("rec", records("radial_rows.txt"), ids=lambda r: f"{r['grid']}/{r['block']}/{r['row']}")
def test_radial_rows(rec):
    T, Hh, Ww = ints(rec["grid"])
    m = ops.sa_radial_mask(T, Hh, Ww, int(rec["block"])).cpu().numpy()
    assert np.nonzero(m[int(rec["row"])])[0].tolist() == ints(rec["keep"])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("rec", records("axis_orders.txt"), ids=lambda r: f"{r['grid']}/{r['cells']}/{r['order']}")
def test_axis_orders(rec, d):
    """Row n of the input holds the value n in every element (exact in bf16
    for n < 256): output row n' must hold the fixture's raster index."""
    T, Hh, Ww = ints(rec["grid"])
    N = T * Hh * Ww
    x = torch.arange(N, dtype=torch.float32).view(1, 1, N, 1).expand(1, 1, N, d).to(torch.bfloat16).cuda()
    (y,) = ops.sa_token_permute([x], T, Hh, Ww, order=rec["order"], cells=tuple(ints(rec["cells"])))
    y = y.float().cpu()[0, 0]
    assert torch.all(y == y[:, :1])
    assert y[:, 0].long().tolist() == rec["list"]
    (back,) = ops.sa_token_permute([y.to(torch.bfloat16).view(1, 1, N, d).cuda()], T, Hh, Ww, order=rec["order"],
                                   cells=tuple(ints(rec["cells"])), inverse=True)
    assert back.float().cpu()[0, 0, :, 0].long().tolist() == list(range(N))


def _scores_qk(P, block=64, d=64):
    """bf16 Q, K of one head whose block scores are ln P[i, j]: q-block i's rows
    are 8 e_i and k-block j's rows carry ln P[i, j] in dimension i, so the
    scaled dot product of the block means is (1/8) * 8 * ln P[i, j] (ln P
    rounded to bf16; equal entries of P stay exactly equal)."""
    nb = P.shape[0]
    assert P.shape == (nb, nb) and nb <= d
    q = torch.zeros(1, 1, nb * block, d)
    k = torch.zeros(1, 1, nb * block, d)
    for i in range(nb):
        q[0, 0, i * block:(i + 1) * block, i] = 8.0
        for j in range(nb):
            k[0, 0, j * block:(j + 1) * block, i] = math.log(P[i, j])
    return q.to(torch.bfloat16).cuda(), k.to(torch.bfloat16).cuda()


@pytest.mark.parametrize("rec", records("tau_rows.txt"), ids=lambda r: f"{r['p']}@{r['tau']}")
def test_tau_rows(rec):
    p = np.array(matrix(rec["p"])[0])
    P = np.tile(p, (p.size, 1))                 # every q-block sees the fixture's row
    q, k = _scores_qk(P)
    m = ops.sa_build_mask(q, k, 64, mode="tau", tau=float(rec["tau"])).cpu().numpy()[0, 0]
    for i in range(p.size):
        assert np.nonzero(m[i])[0].tolist() == ints(rec["keep"]), i


@pytest.mark.parametrize("rec", records("level_rows.txt"), ids=lambda r: f"{r['p']}@{r['fr']}")
def test_level_rows(rec):
    p = np.array(floats(rec["p"]))
    P = np.tile(p, (p.size, 1))                 # every q-block sees the fixture's row
    q, k = _scores_qk(P)
    m = ops.sa_build_mask(q, k, 64, mode="levels", level_frac=tuple(floats(rec["fr"]))).cpu().numpy()[0, 0]
    for i in range(p.size):
        assert m[i].tolist() == ints(rec["code"]), i


@pytest.mark.parametrize("rec", [r for r in records("global_heads.txt") if len(matrix(r["p"])) == len(matrix(r["p"])[0])],
                         ids=lambda r: f"{r['p']}@{r['tau']}")
def test_global_heads(rec):
    """The square fixtures (the library's masks are Nb x Nb)."""
    P = np.array(matrix(rec["p"]))
    q, k = _scores_qk(P)
    m = ops.sa_build_mask(q, k, 64, mode="global", tau=float(rec["tau"])).cpu().numpy()[0, 0]
    assert m.astype(np.int64).tolist() == matrix(rec["keep"], ints)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("rec", records("lite_skip.txt"), ids=lambda r: f"q{r['q']}/eps{r['eps']}")
def test_lite_skip(rec, d):
    """The fixture's six tokens (blocks of 2) blown up to blocks of 64: fixture
    token 2b + w becomes every token 64b + u with u % 2 == w, which leaves each
    row's block maxima unchanged.  Q carries 8 q in dimension 0 and K carries k
    there, so with the scale 1/8 every logit is q * k exactly."""
    qf, kf = floats(rec["q"]), floats(rec["k"])
    block, N = 64, 3 * 64
    src = [2 * (n // block) + (n % block) % 2 for n in range(N)]
    q = torch.zeros(1, 1, N, d)
    k = torch.zeros(1, 1, N, d)
    q[0, 0, :, 0] = torch.tensor([8.0 * qf[s] for s in src])
    k[0, 0, :, 0] = torch.tensor([kf[s] for s in src])
    v = torch.randn(1, 1, N, d, generator=torch.Generator().manual_seed(1))
    q, k, v = (t.to(torch.bfloat16).cuda() for t in (q, k, v))
    skip_in = torch.zeros(1, 1, 3, 3, dtype=torch.uint8, device="cuda")
    skip_out = torch.full_like(skip_in, 7)
    ops.sa_sparse_attn_fwd(q, k, v, block, skip_in=skip_in, skip_out=skip_out, eps=float(rec["eps"]),
                           scale=1.0 / 8.0)
    ops.sa_get_device_status()
    got = skip_out.cpu()[0, 0]
    assert got[0].tolist() == ints(rec["bits"])
    assert torch.all(got[1:] == 0)               # q = 0: every logit 0, nothing far below the running max
