"""GPU test of sa_build_mask_noalloc, the mask builder for callers that cannot
allocate device memory (code inside stream capture, runtimes that own every
allocation, loops that must not wait on an allocator).

It calls the entry point through the C ABI twice in a row on different inputs
and modes and checks that each result equals what sa_build_mask (the entry
point that takes a caller-allocated workspace) produces for the same inputs.
Both run the same kernels, so masks must match bit for bit and scores to fp32
rounding.  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_flash_b200 import build, inputs, ops

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 32 << 20


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.lib()


def _noalloc(lib, q, k, block, mode, tau, level_frac, mask_out, scores_out):
    B, H, N, d = q.shape
    fr = (ctypes.c_float * 3)(*level_frac)
    return lib.sa_build_mask_noalloc(q.data_ptr(), k.data_ptr(), B, H, N, d, block, mode, tau,
                                     ctypes.cast(fr, ctypes.c_void_p), mask_out.data_ptr(),
                                     scores_out.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_entry_point_on_two_calls(lib):
    block = 64
    calls = [(ops.SA_MASK_TAU, 0.9, 81), (ops.SA_MASK_LEVELS, 0.0, 82)]
    fr = (0.1, 0.3, 0.6)
    for mode, tau, seed in calls:
        wl = inputs.Workload("n", 1, 4, 128, 9, 20, 24, block, "tau", seed=seed)
        q, k, _ = inputs.rff_qkv(wl)
        q, k = q.cuda(), k.cuda()
        nb = wl.nblocks
        ref_scores = torch.empty(1, 4, nb, nb, device="cuda")
        ref = ops.sa_build_mask(q, k, block, "tau" if mode == ops.SA_MASK_TAU else "levels", tau=tau or 0.9,
                                level_frac=fr, scores_out=ref_scores)
        got = torch.full((1, 4, nb, nb), 255, dtype=torch.uint8, device="cuda")
        got_scores = torch.full((1, 4, nb, nb), float("nan"), device="cuda")
        st = _noalloc(lib, q, k, block, mode, tau or 0.9, fr, got, got_scores)
        assert st == ops.SA_OK, ops.status_string(st)
        ops.sa_get_device_status()
        assert torch.equal(got, ref), f"mode {mode}: mask differs"
        assert np.abs(got_scores.cpu().numpy() - ref_scores.cpu().numpy()).max() <= 1e-6


def test_noalloc_rejects_sizes_beyond_the_scratch(lib):
    # 12 heads, 118,800 tokens, block 64: the workspace would be ~220 MB
    B, H, N, d, block = 1, 12, 118800, 128, 64
    assert ops.sa_build_mask_workspace(B, H, N, d, block) > SCRATCH_LIMIT
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    fr = (ctypes.c_float * 3)(0.1, 0.3, 0.6)
    st = lib.sa_build_mask_noalloc(dummy.data_ptr(), dummy.data_ptr(), B, H, N, d, block, ops.SA_MASK_TAU, 0.9,
                                   ctypes.cast(fr, ctypes.c_void_p), dummy.data_ptr(), None, None)
    assert st == ops.SA_ERR_UNSUPPORTED
