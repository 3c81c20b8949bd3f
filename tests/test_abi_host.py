"""Host-side checks of the C-ABI library (no GPU needed).

The library must load, export every entry point the public header declares,
and reject bad arguments on the host before touching the GPU.
"""
import ctypes
import math
import os
import re

import pytest

from block_sparse_attention_flash_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.lib()


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "sparse_attn.h")).read()
    return sorted(set(re.findall(r"SA_API\s+[\w\s\*]*?\b(sa_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared_symbols()
    for n in ("sa_build_mask", "sa_radial_mask", "sa_pyramid_pool", "sa_sparse_attn_fwd",
              "sa_pyramid_attn_fwd", "sa_get_device_status", "sa_build_mask_workspace",
              "sa_sparse_attn_bwd", "sa_sparse_attn_bwd_workspace", "sa_token_permute",
              "sa_sparse_attn_fwd_host", "sa_sparse_attn_fwd_host_workspace", "sa_self_test_timeout",
              "sa_build_mask_noalloc"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_symbols():
        assert hasattr(lib, name), name
        assert name in ops._SIGNATURES, name


def test_status_strings_and_version(lib):
    assert ops.status_string(0) == "SA_OK"
    assert ops.status_string(4) == "SA_ERR_TIMEOUT"
    assert lib.sa_version() >= 100


def test_self_test_timeout_argument_validation(lib):
    assert lib.sa_self_test_timeout(0, None) == ops.SA_ERR_INVALID_ARG
    assert lib.sa_self_test_timeout(1_000_000_001, None) == ops.SA_ERR_INVALID_ARG
    assert lib.sa_self_test_timeout(2**64 - 1, None) == ops.SA_ERR_INVALID_ARG


def test_workspace_size(lib):
    B, H, N, d, block = 1, 12, 32760, 128, 64
    nb = -(-N // block)
    assert ops.sa_build_mask_workspace(B, H, N, d, block) == 4 * (4 * B * H * nb * d + B * H * nb * nb)
    assert ops.sa_build_mask_workspace(0, H, N, d, block) == 0


def _attn(lib, **kw):
    a = dict(q=16, k=16, v=16, B=1, H=1, N=256, d=128, block=128, mask=None, sb=0, sh=0, si=0,
             skip_in=None, skip_out=None, eps=math.inf, scale=0.0, order=0, causal=0, o=16, lse=None, stream=None)
    a.update(kw)
    return lib.sa_sparse_attn_fwd(a["q"], a["k"], a["v"], a["B"], a["H"], a["N"], a["d"], a["block"],
                                  a["mask"], a["sb"], a["sh"], a["si"], a["skip_in"], a["skip_out"],
                                  a["eps"], a["scale"], a["order"], a["causal"], a["o"], a["lse"], a["stream"])


def test_attention_argument_validation(lib):
    assert _attn(lib, d=96) == ops.SA_ERR_UNSUPPORTED
    assert _attn(lib, block=32) == ops.SA_ERR_UNSUPPORTED
    assert _attn(lib, q=None) == ops.SA_ERR_INVALID_ARG
    assert _attn(lib, k=24) == ops.SA_ERR_INVALID_ARG          # not 16-byte aligned
    assert _attn(lib, eps=float("nan")) == ops.SA_ERR_INVALID_ARG
    assert _attn(lib, eps=-1.0) == ops.SA_ERR_INVALID_ARG
    assert _attn(lib, order=2) == ops.SA_ERR_INVALID_ARG
    assert _attn(lib, order=-1) == ops.SA_ERR_INVALID_ARG
    assert _attn(lib, causal=2) == ops.SA_ERR_INVALID_ARG
    assert _attn(lib, scale=-0.5) == ops.SA_ERR_INVALID_ARG
    assert _attn(lib, N=128 * 4097) == ops.SA_ERR_UNSUPPORTED
    assert _attn(lib, B=256, H=256) == ops.SA_ERR_UNSUPPORTED
    assert _attn(lib, N=0) == ops.SA_OK                       # empty input: nothing to do
    assert _attn(lib, B=0) == ops.SA_OK
    assert _attn(lib, mask=16, sb=-1) == ops.SA_ERR_INVALID_ARG


def test_mask_builder_argument_validation(lib):
    fr = (ctypes.c_float * 3)(0.1, 0.3, 0.6)
    bad = (ctypes.c_float * 3)(0.5, 0.3, 0.6)
    f = lib.sa_build_mask
    assert f(16, 16, 1, 1, 512, 64, 64, 0, 1.5, None, 16, None, 256, 1 << 20, None) == ops.SA_ERR_INVALID_ARG
    assert f(16, 16, 1, 1, 512, 64, 64, 7, 0.9, None, 16, None, 256, 1 << 20, None) == ops.SA_ERR_INVALID_ARG
    assert f(16, 16, 1, 1, 512, 64, 64, 1, 0.9, ctypes.cast(bad, ctypes.c_void_p), 16, None, 256, 1 << 20,
             None) == ops.SA_ERR_INVALID_ARG
    assert f(16, 16, 1, 1, 512, 64, 64, 1, 0.9, ctypes.cast(fr, ctypes.c_void_p), 16, None, 256, 16,
             None) == ops.SA_ERR_INVALID_ARG                   # workspace too small
    assert f(16, 16, 1, 1, 512, 64, 64, 0, 0.9, None, 16, None, 200, 1 << 20, None) == ops.SA_ERR_INVALID_ARG
    assert f(16, 16, 1, 1, 512, 80, 64, 0, 0.9, None, 16, None, 256, 1 << 20, None) == ops.SA_ERR_UNSUPPORTED
    assert f(16, 16, 1, 1, 512, 64, 64, 0, 0.9, None, 16, 20, 256, 1 << 20, None) == ops.SA_ERR_INVALID_ARG  # scores_out
    assert f(16, 16, 1, 1, 0, 64, 64, 0, 0.9, None, 16, None, 256, 0, None) == ops.SA_OK



def test_noalloc_mask_builder_checks_arguments_before_its_scratch_lookup(lib):
    """Argument errors of sa_build_mask_noalloc keep sa_build_mask's codes.

    The checks run on the host before the entry point asks the runtime for
    its scratch array's address, so they come back the same with no GPU
    present (where that lookup would fail with SA_ERR_CUDA)."""
    fr = (ctypes.c_float * 3)(0.1, 0.3, 0.6)
    bad = (ctypes.c_float * 3)(0.5, 0.3, 0.6)
    f = lib.sa_build_mask_noalloc
    frp, badp = ctypes.cast(fr, ctypes.c_void_p), ctypes.cast(bad, ctypes.c_void_p)
    assert f(16, 16, 1, 1, 512, 64, 64, 0, 1.5, None, 16, None, None) == ops.SA_ERR_INVALID_ARG   # tau
    assert f(16, 16, 1, 1, 512, 64, 64, 7, 0.9, None, 16, None, None) == ops.SA_ERR_INVALID_ARG   # mode
    assert f(16, 16, 1, 1, 512, 64, 64, 1, 0.9, badp, 16, None, None) == ops.SA_ERR_INVALID_ARG   # fractions
    assert f(16, 16, 1, 1, 512, 64, 64, 1, 0.9, None, 16, None, None) == ops.SA_ERR_INVALID_ARG   # no fractions
    assert f(16, 16, 1, 1, 512, 80, 64, 0, 0.9, None, 16, None, None) == ops.SA_ERR_UNSUPPORTED   # d
    assert f(16, 16, 1, 1, 512, 64, 32, 0, 0.9, None, 16, None, None) == ops.SA_ERR_UNSUPPORTED   # block
    assert f(24, 16, 1, 1, 512, 64, 64, 0, 0.9, None, 16, None, None) == ops.SA_ERR_INVALID_ARG   # alignment
    assert f(16, 16, 1, 1, 512, 64, 64, 0, 0.9, None, 16, 20, None) == ops.SA_ERR_INVALID_ARG     # scores_out
    assert f(16, 16, 1, 1, 512, 64, 64, 0, 0.9, None, None, None, None) == ops.SA_ERR_INVALID_ARG  # no mask
    assert f(16, 16, -1, 1, 512, 64, 64, 0, 0.9, None, 16, None, None) == ops.SA_ERR_INVALID_ARG
    assert f(16, 16, 1, 1, 0, 64, 64, 0, 0.9, frp, 16, None, None) == ops.SA_OK                   # empty
    # beyond the 32 MiB scratch: 12 heads, 118,800 tokens, block 64
    assert f(16, 16, 1, 12, 118800, 128, 64, 0, 0.9, None, 16, None, None) == ops.SA_ERR_UNSUPPORTED

def test_pool_and_radial_argument_validation(lib):
    three = (ctypes.c_void_p * 3)(16, 32, 48)
    holes = (ctypes.c_void_p * 3)(16, None, 48)
    f = lib.sa_pyramid_pool
    assert f(16, 16, 1, 1, 64, 128, 64, ctypes.cast(holes, ctypes.c_void_p), ctypes.cast(three, ctypes.c_void_p),
             None) == ops.SA_ERR_INVALID_ARG
    assert f(16, 16, 1, 1, 64, 100, 64, ctypes.cast(three, ctypes.c_void_p), ctypes.cast(three, ctypes.c_void_p),
             None) == ops.SA_ERR_UNSUPPORTED
    assert lib.sa_radial_mask(4, 8, 16, 0, 16, None) == ops.SA_ERR_INVALID_ARG
    assert lib.sa_radial_mask(4, 8, 16, 64, None, None) == ops.SA_ERR_INVALID_ARG
    assert lib.sa_radial_mask(0, 8, 16, 64, None, None) == ops.SA_OK


def test_ops_refuse_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises((ValueError, RuntimeError)):
        ops.sa_sparse_attn_fwd(q, q, q, 64, out=q.clone())


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the built library every op raises; nothing falls back to another implementation."""
    import torch
    monkeypatch.setattr(ops, "LIB_PATH", str(tmp_path / "libsparse_attn.so"))
    monkeypatch.setattr(ops, "_lib", None)
    with pytest.raises(RuntimeError, match="is missing"):
        ops.lib()
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError, match="is missing"):
        ops.sa_build_mask_workspace(1, 1, 128, 64, 64)
    with pytest.raises((RuntimeError, ValueError)):
        ops.sa_sparse_attn_fwd(q, q, q, 64)


def _bwd(lib, **kw):
    a = dict(q=16, k=16, v=16, o=16, dout=16, lse=16, B=1, H=1, N=256, d=128, block=128, mask=None, sb=0, sh=0,
             si=0, scale=0.0, causal=0, dq=16, dk=16, dv=16, ws=16, ws_bytes=1 << 20, stream=None)
    a.update(kw)
    return lib.sa_sparse_attn_bwd(a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["B"], a["H"], a["N"],
                                  a["d"], a["block"], a["mask"], a["sb"], a["sh"], a["si"], a["scale"], a["causal"], a["dq"],
                                  a["dk"], a["dv"], a["ws"], a["ws_bytes"], a["stream"])


def test_backward_workspace_and_argument_validation(lib):
    assert ops.sa_sparse_attn_bwd_workspace(2, 3, 100) == 2 * 3 * 100 * 4
    assert ops.sa_sparse_attn_bwd_workspace(0, 3, 100) == 0
    assert _bwd(lib, B=0) == ops.SA_OK                          # nothing to do
    assert _bwd(lib, N=-1) == ops.SA_ERR_INVALID_ARG
    assert _bwd(lib, d=96) == ops.SA_ERR_UNSUPPORTED
    assert _bwd(lib, block=256) == ops.SA_ERR_UNSUPPORTED
    assert _bwd(lib, lse=None) == ops.SA_ERR_INVALID_ARG
    assert _bwd(lib, dout=None) == ops.SA_ERR_INVALID_ARG
    assert _bwd(lib, dk=24) == ops.SA_ERR_INVALID_ARG           # not 16-byte aligned
    assert _bwd(lib, lse=18) == ops.SA_ERR_INVALID_ARG          # not 4-byte aligned
    assert _bwd(lib, ws_bytes=256 * 4 - 1) == ops.SA_ERR_INVALID_ARG
    assert _bwd(lib, scale=float("nan")) == ops.SA_ERR_INVALID_ARG
    assert _bwd(lib, mask=16, si=-1) == ops.SA_ERR_INVALID_ARG
    assert _bwd(lib, causal=3) == ops.SA_ERR_INVALID_ARG


def test_permute_argument_validation(lib):
    import ctypes
    src = (ctypes.c_void_p * 4)(16, 32, 48, 64)
    dst = (ctypes.c_void_p * 4)(80, 96, 112, 128)
    same = (ctypes.c_void_p * 4)(16, 32, 48, 64)

    def call(n=1, B=1, H=1, T=2, Hh=3, Ww=4, d=128, order=0, ct=1, ch=1, cw=1, inverse=0, s=src, t=dst):
        return lib.sa_token_permute(ctypes.cast(s, ctypes.c_void_p), ctypes.cast(t, ctypes.c_void_p), n, B, H, T,
                                    Hh, Ww, d, order, None, ct, ch, cw, inverse, None)
    assert call(B=0) == ops.SA_OK
    assert call(n=0) == ops.SA_ERR_INVALID_ARG and call(n=5) == ops.SA_ERR_INVALID_ARG
    assert call(order=6) == ops.SA_ERR_INVALID_ARG and call(order=-1) == ops.SA_ERR_INVALID_ARG
    assert call(inverse=2) == ops.SA_ERR_INVALID_ARG
    assert call(ch=2) == ops.SA_ERR_INVALID_ARG                 # 2 does not divide Hh = 3
    assert call(cw=0) == ops.SA_ERR_INVALID_ARG
    assert call(d=96) == ops.SA_ERR_UNSUPPORTED
    assert call(t=same) == ops.SA_ERR_INVALID_ARG               # dst == src



def test_host_entry_workspace_and_validation(lib):
    assert ops.sa_sparse_attn_fwd_host_workspace(1000, 128, 4) == 2 * 4 * 4 * 1000 * 128 * 2
    assert ops.sa_sparse_attn_fwd_host_workspace(1000, 128, 0) == 0

    def call(q=16, o=16, B=1, H=2, N=256, d=128, block=128, ws=16, ws_bytes=1 << 30, hc=1):
        return lib.sa_sparse_attn_fwd_host(q, 16, 16, B, H, N, d, block, None, 0, 0, 0, None, None, math.inf, 0.0,
                                           0, 0, o, None, ws, ws_bytes, hc, None)
    assert call(B=0) == ops.SA_OK
    assert call(hc=0) == ops.SA_ERR_INVALID_ARG
    assert call(q=None) == ops.SA_ERR_INVALID_ARG
    assert call(o=None) == ops.SA_ERR_INVALID_ARG
    assert call(d=96) == ops.SA_ERR_UNSUPPORTED
    assert call(ws_bytes=100) == ops.SA_ERR_INVALID_ARG
    assert call(ws=24) == ops.SA_ERR_INVALID_ARG


def test_default_heads_per_chunk():
    """Host-buffer forward: the fewest heads whose q-tile pairs fill two waves of 148 SMs."""
    from block_sparse_attention_flash_b200.ops import default_heads_per_chunk
    assert default_heads_per_chunk(75600, 40) == 1      # 296 pairs a head: two waves already
    assert default_heads_per_chunk(32760, 12) == 3      # 128 pairs a head
    assert default_heads_per_chunk(256, 8) == 8         # one pair a head: capped at H
    assert default_heads_per_chunk(1, 1) == 1
