"""GPU parity: radial mask, tau / level mask builder and pyramid pooling vs the oracle."""
import numpy as np
import pytest
import torch

from block_sparse_attention_flash_b200 import build, inputs, ops
from oracle import radial_mask, tau_mask, level_map, pyramid_pool, global_mask
from _parity import check_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    yield
    ops.sa_get_device_status()


@pytest.mark.parametrize("T,Hh,Ww,block", [(4, 8, 16, 64), (21, 30, 52, 64), (33, 45, 80, 128),
                                           (21, 45, 80, 128), (7, 5, 9, 64), (1, 1, 1, 128)])
def test_radial_mask_bit_exact(T, Hh, Ww, block):
    m = ops.sa_radial_mask(T, Hh, Ww, block)
    ops.sa_get_device_status()
    check_bits(m.cpu(), radial_mask(T, Hh, Ww, block), what=f"radial {T}x{Hh}x{Ww}/{block}")


def _small_rff(block, d=128, H=3, seed=61):
    wl = inputs.Workload("m", 1, H, d, 9, 20, 24, block, "tau", seed=seed)
    return inputs.rff_qkv(wl)


@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("tau", [0.5, 0.9])
def test_tau_mask_small(block, d, tau):
    q, k, _ = _small_rff(block, d)
    m = ops.sa_build_mask(q.cuda(), k.cuda(), block, "tau", tau=tau)
    ops.sa_get_device_status()
    mr, flags, _ = tau_mask(q, k, block, tau, return_info=True)
    check_bits(m.cpu(), mr, flags, f"tau block={block} d={d} tau={tau}")


@pytest.mark.parametrize("block", [64, 128])
def test_level_map_small(block):
    q, k, _ = _small_rff(block)
    m = ops.sa_build_mask(q.cuda(), k.cuda(), block, "levels", level_frac=(0.1, 0.3, 0.6))
    ops.sa_get_device_status()
    lr, flags, _ = level_map(q, k, block, (0.1, 0.3, 0.6), return_info=True)
    check_bits(m.cpu(), lr, flags, f"levels block={block}")


@pytest.mark.parametrize("grid,block,width", [((4, 16, 20), 64, 1), ((8, 40, 40), 64, 8), ((21, 30, 52), 64, 16)])
def test_level_map_each_select_width(grid, block, width):
    """LEVELS rows through the warp selection kernel at E = 1, 8 and 16 keys
    per lane (20, 200 and 512 blocks per row; the last is the PSA 480p grid)."""
    T, Hh, Ww = grid
    wl = inputs.Workload("w", 1, 2, 128, T, Hh, Ww, block, "pyramid", seed=70 + width)
    assert 32 * width // 2 < wl.nblocks <= 32 * width
    q, k, _ = inputs.rff_qkv(wl)
    m = ops.sa_build_mask(q.cuda(), k.cuda(), block, "levels", level_frac=wl.level_frac)
    ops.sa_get_device_status()
    lr, flags, _ = level_map(q, k, block, wl.level_frac, return_info=True)
    check_bits(m.cpu(), lr, flags, f"levels nb={wl.nblocks} E={width}")


def test_scores_out_matches_oracle_scores():
    q, k, _ = _small_rff(64)
    nb = -(-q.shape[2] // 64)
    sc = torch.empty(1, q.shape[1], nb, nb, device="cuda")
    ops.sa_build_mask(q.cuda(), k.cuda(), 64, "tau", tau=0.9, scores_out=sc)
    ops.sa_get_device_status()
    _, _, S = tau_mask(q, k, 64, 0.9, return_info=True)
    assert np.abs(sc.cpu().numpy() - S).max() < 1e-4


def test_block_scores_480p_accuracy():
    """The block scores at the 480p size (2 heads, Nb = 512) against the oracle's fp64 scores.

    The GPU forms the means in fp32 and the scores on tensor cores from three
    tf32 passes of a hi / lo split of the means.  Per score the error is
    bounded by the magnitude m = scale * sum_a |qbar_a| |kbar_a| times: the
    fp32 means (at most 64 additions of 2^-24 each, for both factors), the
    split (the dropped lo * lo term and the tf32 rounding of lo, below 2^-20
    per product) and the fp32 accumulation over d = 128 terms (128 * 2^-24):
    about 2 * 64 * 2^-24 + 2^-20 + 128 * 2^-24 = 1.6e-5.  The test asserts
    2e-5 * m."""
    wl = inputs.WORKLOADS["wan13b_480p_tau"]
    q, k, _ = inputs.rff_qkv(wl, H=2)
    nb = wl.nblocks
    sc = torch.empty(1, 2, nb, nb, device="cuda")
    ops.sa_build_mask(q.cuda(), k.cuda(), wl.block, "tau", tau=wl.tau, scores_out=sc)
    ops.sa_get_device_status()
    _, _, S = tau_mask(q, k, wl.block, wl.tau, return_info=True)
    d = q.shape[-1]
    pad = nb * wl.block - q.shape[2]
    qa = np.pad(q.double().numpy(), ((0, 0), (0, 0), (0, pad), (0, 0)))
    ka = np.pad(k.double().numpy(), ((0, 0), (0, 0), (0, pad), (0, 0)))
    cnt = np.minimum(wl.block, q.shape[2] - np.arange(nb) * wl.block)[None, None, :, None]
    qbar = qa.reshape(1, 2, nb, wl.block, d).sum(3) / cnt
    kbar = ka.reshape(1, 2, nb, wl.block, d).sum(3) / cnt
    mag = np.einsum("bhid,bhjd->bhij", np.abs(qbar), np.abs(kbar)) / np.sqrt(d)
    err = np.abs(sc.cpu().double().numpy() - S)
    worst = float((err / np.maximum(mag, 1e-30)).max())
    print(f"480p block scores: max |error| / magnitude = {worst:.2e}")
    assert np.all(err <= 2e-5 * mag + 1e-12), worst


def test_uniform_scores_keep_first_blocks():
    """Q == 0 makes every score equal: the GPU must break ties by index."""
    N, block = 64 * 42, 64            # tau * Nb = 31.5: no exact tie with the threshold
    q = torch.zeros(1, 2, N, 128, dtype=torch.bfloat16)
    k = torch.randn(1, 2, N, 128, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    m = ops.sa_build_mask(q.cuda(), k.cuda(), block, "tau", tau=0.75).cpu()
    nb = N // block
    keep = int(np.ceil(0.75 * nb))
    assert torch.all(m[..., :keep] == 1) and torch.all(m[..., keep:] == 0)
    lv = ops.sa_build_mask(q.cuda(), k.cuda(), block, "levels", level_frac=(0.1, 0.3, 0.6)).cpu()
    assert lv[0, 0, 0].tolist() == level_map(q[:, :1, :block * nb], k[:, :1], block)[0, 0, 0].tolist()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [64 * 5 + 24, 1000, 1003, 7])
def test_pyramid_pool(d, N):
    g = torch.Generator().manual_seed(N + d)
    k = torch.randn(2, 2, N, d, generator=g).to(torch.bfloat16)
    v = torch.randn(2, 2, N, d, generator=g).to(torch.bfloat16)
    kp, vp = ops.sa_pyramid_pool(k.cuda(), v.cuda(), 64)
    ops.sa_get_device_status()
    for lvl, c in enumerate((2, 4, 8)):
        for got, src in ((kp[lvl], k), (vp[lvl], v)):
            ref = pyramid_pool(src, c)
            err = np.abs(got.float().cpu().numpy() - ref)
            # fp32 sum then one bf16 rounding: within half a bf16 ulp of the mean
            assert np.all(err <= np.abs(ref) * 2.0 ** -8 + 1e-6), (c, float(err.max()))


@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("d", [64, 128])
def test_mask_builder_batch2_ragged(block, d):
    """B = 2 (every mask kernel folds the batch into B*H) with a ragged last block (4,320 tokens):
    the block scores against the oracle's fp64 scores, and the tau and level masks flag-aware."""
    wl = inputs.Workload("b2", 2, 2, d, 9, 20, 24, block, "tau", seed=83 + d + block)
    q, k, _ = inputs.rff_qkv(wl)
    nb = wl.nblocks
    assert q.shape[0] == 2 and q.shape[2] % block != 0
    fr = (0.1, 0.3, 0.6)
    sc = torch.empty(2, 2, nb, nb, device="cuda")
    m = ops.sa_build_mask(q.cuda(), k.cuda(), block, "tau", tau=0.9, scores_out=sc)
    lv = ops.sa_build_mask(q.cuda(), k.cuda(), block, "levels", level_frac=fr)
    ops.sa_get_device_status()
    mr, flags, S = tau_mask(q, k, block, 0.9, return_info=True)
    assert np.abs(sc.cpu().numpy() - S).max() < 1e-4
    check_bits(m.cpu(), mr, flags, f"tau B=2 d={d} block={block}")
    lr, lflags, _ = level_map(q, k, block, fr, return_info=True)
    check_bits(lv.cpu(), lr, lflags, f"levels B=2 d={d} block={block}")


@pytest.mark.parametrize("mode", ["tau", "levels"])
def test_mask_builder_on_a_non_default_stream(mode):
    """Three heads built on a non-default stream and read back on it right after the call, with
    no synchronisation in between: every launch must go to the caller's stream; against the
    oracle, flag-aware."""
    wl = inputs.Workload("h3", 1, 3, 128, 9, 20, 24, 64, "tau", seed=97)
    q, k, _ = inputs.rff_qkv(wl)
    nb = wl.nblocks
    fr = (0.1, 0.3, 0.6)
    qd, kd = q.cuda(), k.cuda()
    m = torch.full((1, 3, nb, nb), 0xFF, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        ops.sa_build_mask(qd, kd, 64, mode, tau=0.9, level_frac=fr, mask_out=m)
        got = m.clone()
    torch.cuda.synchronize()
    ops.sa_get_device_status()
    if mode == "tau":
        ref, flags, _ = tau_mask(q, k, 64, 0.9, return_info=True)
    else:
        ref, flags, _ = level_map(q, k, 64, fr, return_info=True)
    check_bits(got.cpu(), ref, flags, f"{mode} H=3 on a side stream")


@pytest.mark.parametrize("mode", ["tau", "levels"])
def test_mask_builder_graph_capture_matches_eager(mode):
    """A CUDA-graph capture of the builder (caller's workspace and output) replays to the same
    bytes as an eager call; 12 heads, 8,192 tokens."""
    wl = inputs.Workload("g12", 1, 12, 128, 8, 32, 32, 64, "tau", seed=101)
    q, k, _ = inputs.rff_qkv(wl, device="cuda")
    B, H, N, d = q.shape
    nb = wl.nblocks
    fr = (0.1, 0.3, 0.6)
    ws = torch.empty(ops.sa_build_mask_workspace(B, H, N, d, 64), dtype=torch.uint8, device="cuda")
    eager = ops.sa_build_mask(q, k, 64, mode, tau=0.9, level_frac=fr, workspace=ws)
    m = torch.zeros(B, H, nb, nb, dtype=torch.uint8, device="cuda")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ops.sa_build_mask(q, k, 64, mode, tau=0.9, level_frac=fr, mask_out=m, workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    ops.sa_get_device_status()
    assert torch.equal(m, eager)
    del g


def test_tau_mask_wan13b_480p_full():
    """Full-size tau mask of the 480p Wan2.1-1.3B-like workload (12 heads, 512 x 512 blocks)."""
    wl = inputs.WORKLOADS["wan13b_480p_tau"]
    q, k, _ = inputs.rff_qkv(wl)
    m = ops.sa_build_mask(q.cuda(), k.cuda(), wl.block, "tau", tau=wl.tau)
    ops.sa_get_device_status()
    mr, flags, _ = tau_mask(q, k, wl.block, wl.tau, return_info=True)
    nflag = check_bits(m.cpu(), mr, flags, "tau 480p full")
    assert nflag <= 0.001 * mr.size


@pytest.mark.parametrize("nb,mode", [(700, "tau"), (1000, "levels"), (1500, "tau"), (1500, "levels")])
def test_select_paths_for_long_rows(nb, mode):
    """Rows of 513-1024 blocks (widest register sort) and of more than 1024
    blocks (shared-memory sort) against the oracle."""
    block, d = 64, 64
    N = block * nb - 17
    g = torch.Generator().manual_seed(nb)
    q = (torch.randn(1, 1, N, d, generator=g) * 0.5).to(torch.bfloat16)
    k = (torch.randn(1, 1, N, d, generator=g) * 0.5).to(torch.bfloat16)
    m = ops.sa_build_mask(q.cuda(), k.cuda(), block, mode, tau=0.6)
    ops.sa_get_device_status()
    if mode == "tau":
        ref, flags, _ = tau_mask(q, k, block, 0.6, return_info=True)
    else:
        ref, flags, _ = level_map(q, k, block, (0.1, 0.3, 0.6), return_info=True)
    check_bits(m.cpu(), ref, flags, f"{mode} nb={nb}")


@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("tau", [0.3, 0.9])
def test_global_mask_small(block, d, tau):
    q, k, _ = _small_rff(block, d)
    m = ops.sa_build_mask(q.cuda(), k.cuda(), block, "global", tau=tau)
    ops.sa_get_device_status()
    mr, flags, _ = global_mask(q, k, block, tau, return_info=True)
    check_bits(m.cpu(), mr, flags, f"global block={block} d={d} tau={tau}")


def test_global_mask_480p_grid():
    """The 480p workload (12 heads, 512 x 512 block pairs per head), tau 0.9."""
    wl = inputs.WORKLOADS["wan13b_480p_tau"]
    q, k, _ = inputs.rff_qkv(wl)
    m = ops.sa_build_mask(q.cuda(), k.cuda(), wl.block, "global", tau=wl.tau)
    ops.sa_get_device_status()
    mr, flags, _ = global_mask(q, k, wl.block, wl.tau, return_info=True)
    nflag = check_bits(m.cpu(), mr, flags, "global 480p")
    assert nflag <= 0.001 * mr.size


@pytest.mark.parametrize("mode", ["tau", "global"])
def test_maximum_rows_4096_blocks(mode):
    """The largest supported row (Nb = 4096 blocks of 64 tokens, N = 262,144 -
    17): the shared-memory select path (tau) and the many-CTA global search."""
    from oracle import global_mask
    block, d, nb = 64, 64, 4096
    N = block * nb - 17
    g = torch.Generator().manual_seed(4096)
    q = (torch.randn(1, 1, N, d, generator=g) * 0.5).to(torch.bfloat16)
    k = (torch.randn(1, 1, N, d, generator=g) * 0.5).to(torch.bfloat16)
    m = ops.sa_build_mask(q.cuda(), k.cuda(), block, mode, tau=0.6)
    ops.sa_get_device_status()
    if mode == "tau":
        ref, flags, _ = tau_mask(q, k, block, 0.6, return_info=True)
    else:
        ref, flags, _ = global_mask(q, k, block, 0.6, return_info=True)
    nflag = check_bits(m.cpu(), ref, flags, f"{mode} nb=4096")
    assert nflag <= 0.001 * ref.size
