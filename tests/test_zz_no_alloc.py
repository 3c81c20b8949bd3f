"""GPU tests of sa_build_mask_noalloc, the mask builder for callers that cannot
allocate device memory when they need a mask (serving runtimes that reserve
all device memory up front in their own pool, latency-critical loops that
cannot afford cudaMalloc / cudaFree because those can synchronise the device).

Each test calls the entry point through the C ABI several times in a row on
different inputs and modes, so later calls run on scratch that an earlier
call left behind, and checks every result bit for bit against sa_build_mask
(the entry point that takes a caller-allocated workspace): both run the same
kernels, so masks must match exactly and scores to fp32 rounding.  The masks
are also checked against the fp64 oracle, with the margin-flag rule of the
other mask tests.  The modes cover every use of the shared array: block means
and scores (scores_out given or NULL), and the global selection's row
statistics, histograms and search state (more than 64 blocks per row).  The
file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from _parity import check_bits
from block_sparse_attention_flash_b200 import build, inputs, ops

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 32 << 20
FRACS = (0.1, 0.3, 0.6)
MODES = {ops.SA_MASK_TAU: "tau", ops.SA_MASK_LEVELS: "levels", ops.SA_MASK_GLOBAL: "global"}


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.lib()


def _noalloc(lib, q, k, block, mode, tau, mask_out, scores_out):
    B, H, N, d = q.shape
    fr = (ctypes.c_float * 3)(*FRACS)
    return lib.sa_build_mask_noalloc(q.data_ptr(), k.data_ptr(), B, H, N, d, block, mode, tau,
                                     ctypes.cast(fr, ctypes.c_void_p), mask_out.data_ptr(),
                                     None if scores_out is None else scores_out.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)


def _oracle_mask(q, k, block, mode, tau):
    if mode == ops.SA_MASK_TAU:
        return oracle.tau_mask(q, k, block, tau, return_info=True)[:2]
    if mode == ops.SA_MASK_GLOBAL:
        return oracle.global_mask(q, k, block, tau, return_info=True)[:2]
    return oracle.level_map(q, k, block, FRACS, return_info=True)[:2]


def _run_calls(lib, calls):
    for mode, tau, seed, grid, block, with_scores in calls:
        T, Hh, Ww = grid
        wl = inputs.Workload("n", 1, 4, 128, T, Hh, Ww, block, "tau", seed=seed)
        q, k, _ = inputs.rff_qkv(wl)
        qd, kd = q.cuda(), k.cuda()
        nb = wl.nblocks
        ref_scores = torch.empty(1, 4, nb, nb, device="cuda")
        ref = ops.sa_build_mask(qd, kd, block, MODES[mode], tau=tau, level_frac=FRACS, scores_out=ref_scores)
        got = torch.full((1, 4, nb, nb), 255, dtype=torch.uint8, device="cuda")
        got_scores = torch.full((1, 4, nb, nb), float("nan"), device="cuda") if with_scores else None
        st = _noalloc(lib, qd, kd, block, mode, tau, got, got_scores)
        assert st == ops.SA_OK, ops.status_string(st)
        ops.sa_get_device_status()
        what = f"{MODES[mode]} nb={nb} scores={'out' if with_scores else 'scratch'}"
        assert torch.equal(got, ref), f"{what}: mask differs from sa_build_mask"
        if with_scores:
            assert np.abs(got_scores.cpu().numpy() - ref_scores.cpu().numpy()).max() <= 1e-6, what
        want, flags = _oracle_mask(q, k, block, mode, tau)
        n_flag = check_bits(got.cpu(), want, flags, f"{what} vs oracle")
        print(f"{what}: {n_flag} flagged bits differ from the oracle")


def test_noalloc_matches_workspace_entry_point_on_two_calls(lib):
    _run_calls(lib, [(ops.SA_MASK_TAU, 0.9, 81, (9, 20, 24), 64, True),
                     (ops.SA_MASK_LEVELS, 0.9, 82, (9, 20, 24), 64, True)])


def test_noalloc_global_mode_and_scores_in_scratch(lib):
    # 8 x 20 x 40 = 6,400 tokens, block 64: 100 blocks per row, so the global
    # selection takes its multi-CTA path (row statistics, histograms and search
    # state in the shared array); scores_out NULL puts the scores there too.
    _run_calls(lib, [(ops.SA_MASK_GLOBAL, 0.8, 83, (8, 20, 40), 64, False),
                     (ops.SA_MASK_TAU, 0.9, 84, (8, 20, 40), 64, False),
                     (ops.SA_MASK_GLOBAL, 0.6, 85, (8, 20, 40), 64, True)])


def test_noalloc_rejects_sizes_beyond_the_scratch(lib):
    # 12 heads, 118,800 tokens, block 64: the workspace would be ~220 MB
    B, H, N, d, block = 1, 12, 118800, 128, 64
    assert ops.sa_build_mask_workspace(B, H, N, d, block) > SCRATCH_LIMIT
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    fr = (ctypes.c_float * 3)(*FRACS)
    st = lib.sa_build_mask_noalloc(dummy.data_ptr(), dummy.data_ptr(), B, H, N, d, block, ops.SA_MASK_TAU, 0.9,
                                   ctypes.cast(fr, ctypes.c_void_p), dummy.data_ptr(), None, None)
    assert st == ops.SA_ERR_UNSUPPORTED
