"""CUDA-graph capture of the device entry points.

The device entry points only launch kernels on the caller's stream: no
allocation, no copy, no synchronisation (the mask builder's first call on a
device sets kernel attributes, so each test makes one eager call first).  A
serving loop can therefore capture a step once and replay it.  Each test
captures a chain of calls with its static buffers and checks that a replay
writes the same bytes as the same calls made eagerly.  Replays run twice, so
that nothing in the graph depends on state that the first replay changed.
"""
import pytest
import torch

from block_sparse_attention_flash_b200 import build, inputs, ops

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.lib()
    yield
    ops.sa_get_device_status()


def _capture(fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()                                   # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        fn()
    return g


def test_lite_chain_and_backward_graph_replay():
    """Three LiteAttention steps with the skip mask carried from step to step (eps = 2: about a
    fifth of the pairs skip after the first step), then the backward of the last step, on 4
    heads of a ragged 1,955-token grid (block 128)."""
    wl = inputs.Workload("gl", 1, 4, 128, 5, 17, 23, 128, "lite", seed=131)
    q, k, v = inputs.rff_qkv(wl, device="cuda")
    B, H, N, d = q.shape
    nb = wl.nblocks
    dout = torch.randn(q.shape, generator=torch.Generator(device="cuda").manual_seed(7), device="cuda")
    dout = dout.to(torch.bfloat16)
    zero = torch.zeros(B, H, nb, nb, dtype=torch.uint8, device="cuda")
    ws = torch.empty(max(16, ops.sa_sparse_attn_bwd_workspace(B, H, N)), dtype=torch.uint8, device="cuda")

    def buffers():
        return ([torch.empty_like(q) for _ in range(3)], [torch.empty(B, H, N, device="cuda") for _ in range(3)],
                [torch.empty_like(zero) for _ in range(3)], [torch.empty_like(q) for _ in range(3)])

    def chain(O, L, S, G):
        prev = zero
        for s in range(3):
            ops.sa_sparse_attn_fwd(q, k, v, 128, skip_in=prev, skip_out=S[s], eps=2.0, out=O[s], lse=L[s])
            prev = S[s]
        ops.sa_sparse_attn_bwd(q, k, v, O[2], dout, L[2], 128, dq=G[0], dk=G[1], dv=G[2], workspace=ws)

    eager = buffers()
    chain(*eager)
    torch.cuda.synchronize()
    ops.sa_get_device_status()
    assert eager[2][0].any() and not eager[2][0].all()
    graphed = buffers()
    g = _capture(lambda: chain(*graphed))
    for _ in range(2):
        for bufs in graphed:
            for t in bufs:
                t.zero_()
        g.replay()
        torch.cuda.synchronize()
        ops.sa_get_device_status()
        for want, got in zip(eager, graphed):
            for a, b in zip(want, got):
                assert torch.equal(a, b)
    del g


def test_psa_pipeline_graph_replay():
    """Level map, pyramid pooling and pyramid attention of one PSA step, captured as one graph;
    3 heads, 2,880 tokens, block 64."""
    wl = inputs.Workload("gp", 1, 3, 128, 5, 24, 24, 64, "pyramid", seed=137)
    q, k, v = inputs.rff_qkv(wl, device="cuda")
    B, H, N, d = q.shape
    nb = wl.nblocks
    ws = torch.empty(ops.sa_build_mask_workspace(B, H, N, d, 64), dtype=torch.uint8, device="cuda")

    def buffers():
        lv = torch.empty(B, H, nb, nb, dtype=torch.uint8, device="cuda")
        kp = [torch.empty(B, H, ops.pool_rows(N, c), d, dtype=torch.bfloat16, device="cuda") for c in (2, 4, 8)]
        vp = [torch.empty(B, H, ops.pool_rows(N, c), d, dtype=torch.bfloat16, device="cuda") for c in (2, 4, 8)]
        return lv, kp, vp, torch.empty_like(q)

    def step(lv, kp, vp, o):
        ops.sa_build_mask(q, k, 64, "levels", level_frac=wl.level_frac, mask_out=lv, workspace=ws)
        ops.sa_pyramid_pool(k, v, 64, k_pool=kp, v_pool=vp)
        ops.sa_pyramid_attn_fwd(q, k, v, 64, lv, kp, vp, out=o)

    eager = buffers()
    step(*eager)
    torch.cuda.synchronize()
    ops.sa_get_device_status()
    graphed = buffers()
    g = _capture(lambda: step(*graphed))
    for _ in range(2):
        graphed[0].zero_()
        graphed[3].zero_()
        g.replay()
        torch.cuda.synchronize()
        ops.sa_get_device_status()
        assert torch.equal(graphed[0], eager[0])
        for a, b in zip(graphed[1] + graphed[2], eager[1] + eager[2]):
            assert torch.equal(a, b)
        assert torch.equal(graphed[3], eager[3])
    del g
