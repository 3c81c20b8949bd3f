"""Thin ctypes binding over libsparse_attn.so (argument marshalling only).

Every function here has the name of the C entry point it calls, takes torch
CUDA tensors, checks dtype / device / contiguity, passes raw device pointers
and the current CUDA stream, and raises ``SparseAttnError`` on a non-OK
status.  There is no CPU path: if the library is missing, or a tensor is not
on a CUDA device, the call fails loudly.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsparse_attn.so")

SA_OK, SA_ERR_INVALID_ARG, SA_ERR_UNSUPPORTED, SA_ERR_CUDA, SA_ERR_TIMEOUT = range(5)
VISIT_ORDERS = {"ascending": 0, "radial": 1}   # sa_visit_order
SA_MASK_TAU, SA_MASK_LEVELS, SA_MASK_GLOBAL = 0, 1, 2

_vp, _i32, _i64, _f32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t

_SIGNATURES = {
    "sa_status_string": (ctypes.c_char_p, [_i32]),
    "sa_version": (_i32, []),
    "sa_get_device_status": (_i32, [_vp]),
    "sa_self_test_timeout": (_i32, [ctypes.c_uint64, _vp]),
    "sa_build_mask_workspace": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "sa_build_mask": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "sa_build_mask_noalloc": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _vp]),
    "sa_radial_mask": (_i32, [_i32, _i32, _i32, _i32, _vp, _vp]),
    "sa_pyramid_pool": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "sa_sparse_attn_fwd": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _i64, _i64,
                                  _vp, _vp, _f32, _f32, _i32, _i32, _vp, _vp, _vp]),
    "sa_pyramid_attn_fwd": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _i64, _i64,
                                   _vp, _vp, _f32, _i32, _vp, _vp, _vp]),
    "sa_sparse_attn_bwd_workspace": (_sz, [_i32, _i32, _i32]),
    "sa_sparse_attn_fwd_host_workspace": (_sz, [_i32, _i32, _i32]),
    "sa_sparse_attn_fwd_host": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _i64, _i64,
                                       _vp, _vp, _f32, _f32, _i32, _i32, _vp, _vp, _vp, _sz, _i32, _vp]),
    "sa_token_permute": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _i32, _i32, _i32,
                                _i32, _vp]),
    "sa_sparse_attn_bwd": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _i64, _i64, _i64,
                                  _f32, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
}

_lib = None


class SparseAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """Load libsparse_attn.so once (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m block_sparse_attention_flash_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def status_string(status: int) -> str:
    return lib().sa_status_string(status).decode()


def _check(status: int, where: str) -> None:
    if status != SA_OK:
        raise SparseAttnError(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _opt(t: Optional[torch.Tensor], name: str, dtype: torch.dtype) -> Optional[int]:
    return None if t is None else _dev(t, name, dtype)


def _mask_strides(m: torch.Tensor, B: int, H: int, nb: int):
    """(sb, sh, si) element strides for a [Nb,Nb], [H,Nb,Nb] or [B,H,Nb,Nb] mask."""
    if m.shape[-1] != nb or m.shape[-2] != nb or m.stride(-1) != 1:
        raise ValueError(f"mask must end in [{nb}, {nb}] with unit stride, got {tuple(m.shape)}")
    if m.dim() == 2:
        return 0, 0, m.stride(0)
    if m.dim() == 3:
        if m.shape[0] != H:
            raise ValueError("3D mask must be [H, Nb, Nb]")
        return 0, m.stride(0), m.stride(1)
    if m.dim() == 4 and m.shape[0] == B and m.shape[1] == H:
        return m.stride(0), m.stride(1), m.stride(2)
    raise ValueError(f"mask shape {tuple(m.shape)} does not broadcast to [{B}, {H}, {nb}, {nb}]")


def nblocks(N: int, block: int) -> int:
    return -(-N // block)


def sa_get_device_status(stream=None) -> None:
    """Synchronise the stream and raise if a kernel recorded a device-side error."""
    _check(lib().sa_get_device_status(_stream(stream)), "sa_get_device_status")


def sa_self_test_timeout(wait_ns: int, stream=None) -> None:
    """Queue the failure-path self-test: one bounded device wait that runs out
    after wait_ns; the next sa_get_device_status reports SA_ERR_TIMEOUT."""
    _check(lib().sa_self_test_timeout(int(wait_ns), _stream(stream)), "sa_self_test_timeout")


def sa_radial_mask(T: int, Hh: int, Ww: int, block: int, out: Optional[torch.Tensor] = None,
                   device=None, stream=None) -> torch.Tensor:
    nb = nblocks(T * Hh * Ww, block)
    if out is None:
        out = torch.empty(nb, nb, dtype=torch.uint8, device=device or "cuda")
    ptr = _dev(out, "out", torch.uint8)
    _check(lib().sa_radial_mask(T, Hh, Ww, block, ptr, _stream(stream)), "sa_radial_mask")
    return out


def sa_build_mask_workspace(B: int, H: int, N: int, d: int, block: int) -> int:
    return int(lib().sa_build_mask_workspace(B, H, N, d, block))


def sa_build_mask(q: torch.Tensor, k: torch.Tensor, block: int, mode: str = "tau", tau: float = 0.9,
                  level_frac: Sequence[float] = (0.1, 0.3, 0.6), mask_out: Optional[torch.Tensor] = None,
                  scores_out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    B, H, N, d = q.shape
    nb = nblocks(N, block)
    if mask_out is None:
        mask_out = torch.empty(B, H, nb, nb, dtype=torch.uint8, device=q.device)
    ws_bytes = sa_build_mask_workspace(B, H, N, d, block)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=q.device)
    fr = (ctypes.c_float * 3)(*[float(x) for x in level_frac])
    modes = {"tau": SA_MASK_TAU, "levels": SA_MASK_LEVELS, "global": SA_MASK_GLOBAL}
    if mode not in modes:
        raise ValueError(f"mode must be one of {sorted(modes)}")
    m = modes[mode]
    st = lib().sa_build_mask(_dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16), B, H, N, d, block, m,
                             float(tau), ctypes.cast(fr, ctypes.c_void_p), _dev(mask_out, "mask_out", torch.uint8),
                             _opt(scores_out, "scores_out", torch.float32), _dev(workspace, "workspace", torch.uint8),
                             workspace.numel(), _stream(stream))
    _check(st, "sa_build_mask")
    return mask_out


def pool_rows(N: int, c: int) -> int:
    return -(-N // c)


def sa_pyramid_pool(k: torch.Tensor, v: torch.Tensor, block: int, k_pool=None, v_pool=None, stream=None):
    B, H, N, d = k.shape
    if k_pool is None:
        k_pool = [torch.empty(B, H, pool_rows(N, c), d, dtype=k.dtype, device=k.device) for c in (2, 4, 8)]
    if v_pool is None:
        v_pool = [torch.empty(B, H, pool_rows(N, c), d, dtype=v.dtype, device=v.device) for c in (2, 4, 8)]
    kp = (ctypes.c_void_p * 3)(*[_dev(t, "k_pool", torch.bfloat16) for t in k_pool])
    vp = (ctypes.c_void_p * 3)(*[_dev(t, "v_pool", torch.bfloat16) for t in v_pool])
    st = lib().sa_pyramid_pool(_dev(k, "k", torch.bfloat16), _dev(v, "v", torch.bfloat16), B, H, N, d, block,
                               ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p), _stream(stream))
    _check(st, "sa_pyramid_pool")
    return k_pool, v_pool


def sa_sparse_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int,
                       mask: Optional[torch.Tensor] = None, skip_in: Optional[torch.Tensor] = None,
                       skip_out: Optional[torch.Tensor] = None, eps: float = math.inf, scale: float = 0.0,
                       out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                       stream=None, order: str = "ascending", causal: bool = False) -> torch.Tensor:
    """Block-sparse attention forward; returns O (and fills lse / skip_out if given).

    ``order`` ("ascending" or "radial") is the k-block visit order of the skip update."""
    if order not in VISIT_ORDERS:
        raise ValueError(f"order must be one of {sorted(VISIT_ORDERS)}")
    B, H, N, d = q.shape
    nb = nblocks(N, block)
    if out is None:
        out = torch.empty_like(q)
    sb = sh = si = 0
    mptr = None
    if mask is not None:
        if mask.dtype != torch.uint8 or not mask.is_cuda:
            raise ValueError("mask must be a CUDA uint8 tensor")
        sb, sh, si = _mask_strides(mask, B, H, nb)
        mptr = mask.data_ptr()
    for name, t in (("skip_in", skip_in), ("skip_out", skip_out)):
        if t is not None and tuple(t.shape) != (B, H, nb, nb):
            raise ValueError(f"{name} must be [{B}, {H}, {nb}, {nb}]")
    st = lib().sa_sparse_attn_fwd(
        _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16), _dev(v, "v", torch.bfloat16),
        B, H, N, d, block, mptr, sb, sh, si,
        _opt(skip_in, "skip_in", torch.uint8), _opt(skip_out, "skip_out", torch.uint8),
        float(eps), float(scale), VISIT_ORDERS[order], int(bool(causal)), _dev(out, "out", torch.bfloat16),
        _opt(lse, "lse", torch.float32), _stream(stream))
    _check(st, "sa_sparse_attn_fwd")
    return out


def sa_pyramid_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int, levels: torch.Tensor,
                        k_pool, v_pool, scale: float = 0.0, out: Optional[torch.Tensor] = None,
                        lse: Optional[torch.Tensor] = None, stream=None, causal: bool = False) -> torch.Tensor:
    """PSA multi-level attention forward over a level-code map (0 drop, 1+l level l)."""
    B, H, N, d = q.shape
    nb = nblocks(N, block)
    if out is None:
        out = torch.empty_like(q)
    if levels.dtype != torch.uint8 or not levels.is_cuda:
        raise ValueError("levels must be a CUDA uint8 tensor")
    sb, sh, si = _mask_strides(levels, B, H, nb)
    kp = (ctypes.c_void_p * 3)(*[_dev(t, "k_pool", torch.bfloat16) for t in k_pool])
    vp = (ctypes.c_void_p * 3)(*[_dev(t, "v_pool", torch.bfloat16) for t in v_pool])
    st = lib().sa_pyramid_attn_fwd(
        _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16), _dev(v, "v", torch.bfloat16),
        B, H, N, d, block, levels.data_ptr(), sb, sh, si,
        ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p), float(scale), int(bool(causal)),
        _dev(out, "out", torch.bfloat16), _opt(lse, "lse", torch.float32), _stream(stream))
    _check(st, "sa_pyramid_attn_fwd")
    return out


def sa_sparse_attn_bwd_workspace(B: int, H: int, N: int) -> int:
    return int(lib().sa_sparse_attn_bwd_workspace(B, H, N))


def sa_sparse_attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, dout: torch.Tensor,
                       lse: torch.Tensor, block: int, mask: Optional[torch.Tensor] = None, scale: float = 0.0,
                       dq: Optional[torch.Tensor] = None, dk: Optional[torch.Tensor] = None,
                       dv: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                       stream=None, causal: bool = False):
    """Gradients (dQ, dK, dV) of sa_sparse_attn_fwd given dO and the forward's O and LSE."""
    B, H, N, d = q.shape
    nb = nblocks(N, block)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(max(16, sa_sparse_attn_bwd_workspace(B, H, N)), dtype=torch.uint8, device=q.device)
    sb = sh = si = 0
    mptr = None
    if mask is not None:
        if mask.dtype != torch.uint8 or not mask.is_cuda:
            raise ValueError("mask must be a CUDA uint8 tensor")
        sb, sh, si = _mask_strides(mask, B, H, nb)
        mptr = mask.data_ptr()
    st = lib().sa_sparse_attn_bwd(
        _dev(q, "q", torch.bfloat16), _dev(k, "k", torch.bfloat16), _dev(v, "v", torch.bfloat16),
        _dev(o, "o", torch.bfloat16), _dev(dout, "dout", torch.bfloat16), _dev(lse, "lse", torch.float32),
        B, H, N, d, block, mptr, sb, sh, si, float(scale), int(bool(causal)),
        _dev(dq, "dq", torch.bfloat16), _dev(dk, "dk", torch.bfloat16), _dev(dv, "dv", torch.bfloat16),
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream(stream))
    _check(st, "sa_sparse_attn_bwd")
    return dq, dk, dv


AXIS_ORDERS = ("thw", "twh", "htw", "hwt", "wth", "wht")   # the library's order codes 0..5


def sa_token_permute(tensors, T: int, Hh: int, Ww: int, order="thw", head_order: Optional[torch.Tensor] = None,
                     cells=(1, 1, 1), inverse: bool = False, out=None, stream=None):
    """Reorder the tokens of up to four [B,H,N,d] bf16 tensors in one launch
    (PARO axis orders / VMoBA cell partitions); returns the list of outputs."""
    tensors = list(tensors)
    if not 1 <= len(tensors) <= 4:
        raise ValueError("one to four tensors")
    B, H, N, d = tensors[0].shape
    if N != T * Hh * Ww:
        raise ValueError("N must equal T * Hh * Ww")
    for t in tensors:
        if tuple(t.shape) != (B, H, N, d):
            raise ValueError("all tensors must have the same shape")
    code = AXIS_ORDERS.index(order) if isinstance(order, str) else int(order)
    hptr = None
    if head_order is not None:
        if head_order.dtype != torch.uint8 or not head_order.is_cuda or head_order.numel() != H:
            raise ValueError("head_order must be a CUDA uint8 tensor of H codes")
        hptr = head_order.data_ptr()
    out = [torch.empty_like(t) for t in tensors] if out is None else list(out)
    src = (ctypes.c_void_p * 4)(*[_dev(t, "tensor", torch.bfloat16) for t in tensors])
    dst = (ctypes.c_void_p * 4)(*[_dev(t, "out", torch.bfloat16) for t in out])
    st = lib().sa_token_permute(ctypes.cast(src, ctypes.c_void_p), ctypes.cast(dst, ctypes.c_void_p), len(tensors),
                                B, H, T, Hh, Ww, d, code, hptr, int(cells[0]), int(cells[1]), int(cells[2]),
                                int(bool(inverse)), _stream(stream))
    _check(st, "sa_token_permute")
    return out


def _host(t: torch.Tensor, name: str, dtype: torch.dtype) -> int:
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor")
    return t.data_ptr()


def sa_sparse_attn_fwd_host_workspace(N: int, d: int, heads_per_chunk: int) -> int:
    return int(lib().sa_sparse_attn_fwd_host_workspace(N, d, heads_per_chunk))


def default_heads_per_chunk(N: int, H: int, n_sm: int = 148) -> int:
    """Heads per chunk for sa_sparse_attn_fwd_host: the fewest heads whose
    q-tile pairs (ceil(N / 256) per head) fill two waves of the SMs.  The
    first chunk's copy in and the last chunk's copy out are not overlapped, so
    smaller chunks hide more; one 75,600-token head is already 296 pairs."""
    pairs = -(-N // 256)
    return max(1, min(H, -(-2 * n_sm // max(pairs, 1))))


def sa_sparse_attn_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int, out: torch.Tensor,
                            mask: Optional[torch.Tensor] = None, skip_in: Optional[torch.Tensor] = None,
                            skip_out: Optional[torch.Tensor] = None, eps: float = math.inf, scale: float = 0.0,
                            lse: Optional[torch.Tensor] = None, heads_per_chunk: Optional[int] = None,
                            workspace: Optional[torch.Tensor] = None, stream=None, order: str = "ascending",
                            causal: bool = False, device=None) -> torch.Tensor:
    """sa_sparse_attn_fwd with q, k, v and out in host memory (pin them for overlap).
    heads_per_chunk None: default_heads_per_chunk(N, H)."""
    B, H, N, d = q.shape
    nb = nblocks(N, block)
    hc = min(heads_per_chunk if heads_per_chunk is not None else default_heads_per_chunk(N, H), H)
    if workspace is None:
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        workspace = torch.empty(sa_sparse_attn_fwd_host_workspace(N, d, hc), dtype=torch.uint8, device=dev)
    sb = sh = si = 0
    mptr = None
    if mask is not None:
        if mask.dtype != torch.uint8 or not mask.is_cuda:
            raise ValueError("mask must be a CUDA uint8 tensor")
        sb, sh, si = _mask_strides(mask, B, H, nb)
        mptr = mask.data_ptr()
    for name, t in (("skip_in", skip_in), ("skip_out", skip_out)):
        if t is not None and tuple(t.shape) != (B, H, nb, nb):
            raise ValueError(f"{name} must be [{B}, {H}, {nb}, {nb}]")
    st = lib().sa_sparse_attn_fwd_host(
        _host(q, "q", torch.bfloat16), _host(k, "k", torch.bfloat16), _host(v, "v", torch.bfloat16),
        B, H, N, d, block, mptr, sb, sh, si, _opt(skip_in, "skip_in", torch.uint8),
        _opt(skip_out, "skip_out", torch.uint8), float(eps), float(scale), VISIT_ORDERS[order], int(bool(causal)),
        _host(out, "out", torch.bfloat16), _opt(lse, "lse", torch.float32), _dev(workspace, "workspace", torch.uint8),
        workspace.numel(), hc, _stream(stream))
    _check(st, "sa_sparse_attn_fwd_host")
    return out

