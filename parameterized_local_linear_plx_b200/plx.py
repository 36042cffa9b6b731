"""Python binding of libplx.so (include/plx.h): argument marshalling only.

Every function here has the name of the C entry point it calls.  Tensors are
PyTorch CUDA tensors (PyTorch provides device memory and the current
stream); every step of the computation runs in the library's kernels.
Importing this module loads the library and raises ImportError if it has not
been built (``python -m parameterized_local_linear_plx_b200.build``): there is
no fallback implementation.
"""
from __future__ import annotations

import ctypes
import functools
import math
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libplx.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python -m parameterized_local_linear_plx_b200.build` "
        "(the library has no CPU fallback)")
_lib = ctypes.CDLL(_LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t

_lib.plx_version.restype = _I
_lib.plx_version.argtypes = []
_lib.plx_status_string.restype = ctypes.c_char_p
_lib.plx_status_string.argtypes = [_I]
_lib.plx_fwd.restype = _I
_lib.plx_fwd.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]
_lib.plx_fwd_varlen.restype = _I
_lib.plx_fwd_varlen.argtypes = [_P] * 7 + [_I] * 7 + [_F, _P]
_lib.plx_fwd_train.restype = _I
_lib.plx_fwd_train.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]
_lib.plx_fwd_partial_size.restype = _SZ
_lib.plx_fwd_partial_size.argtypes = [_I] * 4
_lib.plx_fwd_partial.restype = _I
_lib.plx_fwd_partial.argtypes = [_P] * 5 + [_SZ] + [_I] * 6 + [_F, _P]
_lib.plx_fwd_merge.restype = _I
_lib.plx_fwd_merge.argtypes = [_P] + [_I] * 5 + [_P, _P, _P]
_lib.plx_bwd_workspace_size.restype = _SZ
_lib.plx_bwd_workspace_size.argtypes = [_I, _I, _I, _I, _I]
_lib.plx_bwd.restype = _I
_lib.plx_bwd.argtypes = [_P] * 13 + [_I, _I, _I, _I, _I, _I, _F, _P, _SZ, _P]
_lib.plx_decode_num_splits.restype = _I
_lib.plx_decode_num_splits.argtypes = [_I, _I, _I, _I, _I]
_lib.plx_decode_workspace_size.restype = _SZ
_lib.plx_decode_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I]
_lib.plx_decode.restype = _I
_lib.plx_decode.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _SZ, _P]
_lib.plx_decode_paged.restype = _I
_lib.plx_decode_paged.argtypes = [_P] * 8 + [_I] * 7 + [_F, _I, _P, _SZ, _P]
_lib.plx_kv_append.restype = _I
_lib.plx_kv_append.argtypes = [_P] * 5 + [_I] * 5 + [_P]
_lib.plx_kv_append_paged.restype = _I
_lib.plx_kv_append_paged.argtypes = [_P] * 6 + [_I] * 7 + [_P]
_lib.plx_qkvr_proj.restype = _I
_lib.plx_qkvr_proj.argtypes = [_P] * 6 + [_I] * 6 + [_P]
_lib.plx_qkvr_proj_decode.restype = _I
_lib.plx_qkvr_proj_decode.argtypes = [_P] * 8 + [_I] * 6 + [_P]
_lib.plx_qkvr_proj_decode_paged.restype = _I
_lib.plx_qkvr_proj_decode_paged.argtypes = [_P] * 9 + [_I] * 8 + [_P]
_lib.plx_decode_partial_size.restype = _SZ
_lib.plx_decode_partial_size.argtypes = [_I] * 6
_lib.plx_decode_partial.restype = _I
_lib.plx_decode_partial.argtypes = [_P] * 5 + [_I] * 6 + [_F, _I, _P, _SZ, _P]
_lib.plx_decode_merge.restype = _I
_lib.plx_decode_merge.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P]
_lib.plx_decode_noalloc.restype = _I
_lib.plx_decode_noalloc.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P]
_lib.plx_check_device_status.restype = _I
_lib.plx_check_device_status.argtypes = [_P]
_lib.plx_selftest_wait_timeout.restype = _I
_lib.plx_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, _P]

PLX_OK = 0
PLX_ERR_NULL = -1
PLX_ERR_SHAPE = -2
PLX_ERR_HEADDIM = -3
PLX_ERR_GQA = -4
PLX_ERR_ALIGN = -5
PLX_ERR_WORKSPACE = -6
PLX_ERR_CUDA = -7
PLX_ERR_DEVICE_TIMEOUT = -8
PLX_ERR_ARCH = -9

LIB_PATH = _LIB_PATH
lib = _lib  # the raw ctypes handle, for callers that pass their own pointers


class PlxError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {plx_status_string(status)} ({status})")


def plx_version() -> int:
    return _lib.plx_version()


def plx_status_string(status: int) -> str:
    return _lib.plx_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t, name, dtype, ndim):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def plx_fwd(q, k, v, r=None, causal=True, scale=None, out=None, lse=None, return_lse=True, stream=None):
    """Parallax forward over full sequences.

    q [B, Hq, N, d], k/v [B, Hkv, N, d], r [B, Hq, N, d] or None (rho = 0), all
    bf16 CUDA.  Returns (out [B, Hq, N, d] bf16, lse [B, Hq, N] fp32 or None).
    """
    _check(q, "q", torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    if r is not None:
        _check(r, "r", torch.bfloat16, 4)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape or (r is not None and r.shape != q.shape):
        raise ValueError("shape mismatch between q, k, v, r")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, N), device=q.device, dtype=torch.float32)
    st = _lib.plx_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(r), _ptr(out), _ptr(lse), B, Hq, Hkv, N, d,
                      1 if causal else 0, float(scale), _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_fwd")
    return out, lse


def plx_fwd_partial_size(B, Hq, N, d) -> int:
    return int(_lib.plx_fwd_partial_size(B, Hq, N, d))


def plx_fwd_partial(q, k, v, r=None, causal=True, scale=None, partial=None, stream=None):
    """Partial states of the queries q against one chunk of keys k, v.

    q, r [B, Hq, N, d], k/v [B, Hkv, N, d] bf16 CUDA.  Returns partial
    [B, Hq, N, 2d + 4] fp32: per row m (log2 units), l, c, pad, O1[d], O2[d].
    """
    _check(q, "q", torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    if r is not None:
        _check(r, "r", torch.bfloat16, 4)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape or (r is not None and r.shape != q.shape):
        raise ValueError("shape mismatch between q, k, v, r")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if partial is None:
        partial = torch.empty((B, Hq, N, 2 * d + 4), device=q.device, dtype=torch.float32)
    else:
        _check(partial, "partial", torch.float32, 4)
    st = _lib.plx_fwd_partial(_ptr(q), _ptr(k), _ptr(v), _ptr(r), _ptr(partial), partial.numel() * 4, B, Hq, Hkv, N,
                              d, 1 if causal else 0, float(scale), _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_fwd_partial")
    return partial


def plx_fwd_merge(partials, out=None, lse=None, return_lse=True, stream=None):
    """Merge blocks of partial states [blocks, B, Hq, N, 2d + 4] into (out, lse)."""
    _check(partials, "partials", torch.float32, 5)
    blocks, B, Hq, N, pf = partials.shape
    d = (pf - 4) // 2
    if out is None:
        out = torch.empty((B, Hq, N, d), device=partials.device, dtype=torch.bfloat16)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq, N), device=partials.device, dtype=torch.float32)
    st = _lib.plx_fwd_merge(_ptr(partials), blocks, B, Hq, N, d, _ptr(out), _ptr(lse), _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_fwd_merge")
    return out, lse


def plx_fwd_varlen(q, k, v, cu_seqlens, max_seqlen, r=None, causal=True, scale=None, out=None, lse=None,
                   return_lse=True, stream=None):
    """Packed variable-length forward.  q, r [total, Hq, d], k, v [total, Hkv, d]
    bf16; cu_seqlens [B+1] int32 on the device; max_seqlen (host int) >= every
    length.  Returns (out [total, Hq, d] bf16, lse [Hq, total] fp32 or None)."""
    _check(q, "q", torch.bfloat16, 3)
    _check(k, "k", torch.bfloat16, 3)
    _check(v, "v", torch.bfloat16, 3)
    _check(cu_seqlens, "cu_seqlens", torch.int32, 1)
    if r is not None:
        _check(r, "r", torch.bfloat16, 3)
    total, Hq, d = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.shape[0] - 1
    if k.shape != (total, Hkv, d) or v.shape != k.shape or (r is not None and r.shape != q.shape) or B < 1:
        raise ValueError("shape mismatch between q, k, v, r, cu_seqlens")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((Hq, total), device=q.device, dtype=torch.float32)
    st = _lib.plx_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(r), _ptr(out), _ptr(lse), _ptr(cu_seqlens), B, Hq,
                             Hkv, total, int(max_seqlen), d, 1 if causal else 0, float(scale), _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_fwd_varlen")
    return out, lse


def plx_fwd_train(q, k, v, r=None, causal=True, scale=None, out=None, lse=None, obar=None, sbar=None,
                  stream=None):
    """plx_fwd that also returns the per-row values the backward needs.
    Returns (out, lse, obar [B, Hq, N, d] bf16, sbar [B, Hq, N] fp32 or None when r is None)."""
    _check(q, "q", torch.bfloat16, 4)
    _check(k, "k", torch.bfloat16, 4)
    _check(v, "v", torch.bfloat16, 4)
    if r is not None:
        _check(r, "r", torch.bfloat16, 4)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape or (r is not None and r.shape != q.shape):
        raise ValueError("shape mismatch between q, k, v, r")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, Hq, N), device=q.device, dtype=torch.float32) if lse is None else lse
    obar = torch.empty_like(q) if obar is None else obar
    if r is not None and sbar is None:
        sbar = torch.empty((B, Hq, N), device=q.device, dtype=torch.float32)
    st = _lib.plx_fwd_train(_ptr(q), _ptr(k), _ptr(v), _ptr(r), _ptr(out), _ptr(lse), _ptr(obar),
                            _ptr(sbar if r is not None else None), B, Hq, Hkv, N, d, 1 if causal else 0,
                            float(scale), _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_fwd_train")
    return out, lse, obar, (sbar if r is not None else None)


def plx_bwd_workspace_size(B, Hq, Hkv, N, d) -> int:
    return int(_lib.plx_bwd_workspace_size(B, Hq, Hkv, N, d))


def plx_bwd(q, k, v, r, out, dout, lse, obar, sbar=None, causal=True, scale=None, dq=None, dk=None, dv=None,
            dr=None, want_dr=True, workspace=None, stream=None):
    """Gradients of sum(dout * out) for the forward of plx_fwd_train with the same
    arguments.  Returns (dq, dk, dv, dr); dr is None when want_dr is False."""
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout"), (obar, "obar")):
        _check(t, name, torch.bfloat16, 4)
    _check(lse, "lse", torch.float32, 3)
    if r is not None:
        _check(r, "r", torch.bfloat16, 4)
        _check(sbar, "sbar", torch.float32, 3)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if (k.shape != (B, Hkv, N, d) or v.shape != k.shape or out.shape != q.shape or dout.shape != q.shape
            or obar.shape != q.shape or lse.shape != (B, Hq, N) or (r is not None and r.shape != q.shape)):
        raise ValueError("shape mismatch between the backward's arguments")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if want_dr and dr is None:
        dr = torch.empty_like(q)
    need = plx_bwd_workspace_size(B, Hq, Hkv, N, d)
    if workspace is None:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.plx_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(r), _ptr(out), _ptr(dout), _ptr(lse), _ptr(obar),
                      _ptr(sbar if r is not None else None), _ptr(dq), _ptr(dk), _ptr(dv),
                      _ptr(dr if want_dr else None), B, Hq, Hkv, N, d, 1 if causal else 0, float(scale),
                      _ptr(workspace), ws_bytes, _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_bwd")
    return dq, dk, dv, (dr if want_dr else None)


def plx_decode_num_splits(B, Hq, Hkv, S_max, d) -> int:
    """The number of work partitions (persistent CTAs) plx_decode uses with num_splits = 0."""
    return _lib.plx_decode_num_splits(B, Hq, Hkv, S_max, d)


@functools.lru_cache(maxsize=256)
def _decode_ws_size(B, Hq, Hkv, S_max, d, num_splits, dev):
    # cached per shape so that a steady decode loop makes one library call per step
    return int(_lib.plx_decode_workspace_size(B, Hq, Hkv, S_max, d, num_splits))


def plx_decode_workspace_size(B, Hq, Hkv, S_max, d, num_splits=0) -> int:
    return int(_lib.plx_decode_workspace_size(B, Hq, Hkv, S_max, d, num_splits))


def plx_decode(q, kcache, vcache, seqlens, r=None, scale=None, num_splits=0, out=None, lse=None,
               workspace=None, return_lse=True, stream=None):
    """One decode step.  q/r [B, Hq, d] bf16, caches [B, Hkv, S_max, d] bf16,
    seqlens [B] int32 (device).  Returns (out [B, Hq, d] bf16, lse [B, Hq] fp32 or None).
    workspace: optional uint8 CUDA tensor of at least plx_decode_workspace_size bytes."""
    _check(q, "q", torch.bfloat16, 3)
    _check(kcache, "kcache", torch.bfloat16, 4)
    _check(vcache, "vcache", torch.bfloat16, 4)
    _check(seqlens, "seqlens", torch.int32, 1)
    if r is not None:
        _check(r, "r", torch.bfloat16, 3)
    B, Hq, d = q.shape
    Hkv, S_max = kcache.shape[1], kcache.shape[2]
    if kcache.shape != (B, Hkv, S_max, d) or vcache.shape != kcache.shape or seqlens.shape != (B,) \
            or (r is not None and r.shape != q.shape):
        raise ValueError("shape mismatch between q, caches, seqlens, r")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), device=q.device, dtype=torch.float32)
    if workspace is None:
        need = _decode_ws_size(B, Hq, Hkv, S_max, d, int(num_splits), q.device.index)
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.plx_decode(_ptr(q), _ptr(r), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(out), _ptr(lse),
                         B, Hq, Hkv, S_max, d, float(scale), int(num_splits), _ptr(workspace), ws_bytes,
                         _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_decode")
    return out, lse


def plx_decode_paged(q, kpool, vpool, block_table, seqlens, r=None, scale=None, num_splits=0, out=None, lse=None,
                     workspace=None, return_lse=True, stream=None):
    """One decode step against paged caches.  q/r [B, Hq, d] bf16; kpool/vpool
    [num_pages, Hkv, page_size, d] bf16; block_table [B, max_pages] int32 and
    seqlens [B] int32 on the device.  Returns (out, lse) as plx_decode."""
    _check(q, "q", torch.bfloat16, 3)
    _check(kpool, "kpool", torch.bfloat16, 4)
    _check(vpool, "vpool", torch.bfloat16, 4)
    _check(block_table, "block_table", torch.int32, 2)
    _check(seqlens, "seqlens", torch.int32, 1)
    if r is not None:
        _check(r, "r", torch.bfloat16, 3)
    B, Hq, d = q.shape
    num_pages, Hkv, page_size = kpool.shape[0], kpool.shape[1], kpool.shape[2]
    max_pages = block_table.shape[1]
    if (kpool.shape != (num_pages, Hkv, page_size, d) or vpool.shape != kpool.shape or block_table.shape[0] != B
            or seqlens.shape != (B,) or (r is not None and r.shape != q.shape)):
        raise ValueError("shape mismatch between q, pools, block_table, seqlens, r")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), device=q.device, dtype=torch.float32)
    if workspace is None:
        need = _decode_ws_size(B, Hq, Hkv, max_pages * page_size, d, int(num_splits), q.device.index)
        workspace = torch.empty(max(need, 16), device=q.device, dtype=torch.uint8)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.plx_decode_paged(_ptr(q), _ptr(r), _ptr(kpool), _ptr(vpool), _ptr(block_table), _ptr(seqlens),
                               _ptr(out), _ptr(lse), B, Hq, Hkv, num_pages, page_size, max_pages, d, float(scale),
                               int(num_splits), _ptr(workspace), ws_bytes, _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_decode_paged")
    return out, lse


def plx_kv_append(knew, vnew, kcache, vcache, seqlens, advance=True, stream=None):
    """Write knew/vnew [B, Hkv, d] at row seqlens[b] of the caches [B, Hkv, S_max, d];
    advance seqlens (in place) when asked."""
    for t, n in ((knew, "knew"), (vnew, "vnew")):
        _check(t, n, torch.bfloat16, 3)
    for t, n in ((kcache, "kcache"), (vcache, "vcache")):
        _check(t, n, torch.bfloat16, 4)
    _check(seqlens, "seqlens", torch.int32, 1)
    B, Hkv, d = knew.shape
    S_max = kcache.shape[2]
    if vnew.shape != knew.shape or kcache.shape != (B, Hkv, S_max, d) or vcache.shape != kcache.shape \
            or seqlens.shape != (B,):
        raise ValueError("shape mismatch between knew, vnew, caches, seqlens")
    st = _lib.plx_kv_append(_ptr(knew), _ptr(vnew), _ptr(kcache), _ptr(vcache), _ptr(seqlens), B, Hkv, S_max, d,
                            1 if advance else 0, _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_kv_append")


def plx_kv_append_paged(knew, vnew, kpool, vpool, block_table, seqlens, advance=True, stream=None):
    """plx_kv_append for page pools [num_pages, Hkv, page_size, d] and a block table [B, max_pages]."""
    for t, n in ((knew, "knew"), (vnew, "vnew")):
        _check(t, n, torch.bfloat16, 3)
    for t, n in ((kpool, "kpool"), (vpool, "vpool")):
        _check(t, n, torch.bfloat16, 4)
    _check(block_table, "block_table", torch.int32, 2)
    _check(seqlens, "seqlens", torch.int32, 1)
    B, Hkv, d = knew.shape
    num_pages, page_size = kpool.shape[0], kpool.shape[2]
    max_pages = block_table.shape[1]
    if vnew.shape != knew.shape or kpool.shape != (num_pages, Hkv, page_size, d) or vpool.shape != kpool.shape \
            or block_table.shape[0] != B or seqlens.shape != (B,):
        raise ValueError("shape mismatch between knew, vnew, pools, block_table, seqlens")
    st = _lib.plx_kv_append_paged(_ptr(knew), _ptr(vnew), _ptr(kpool), _ptr(vpool), _ptr(block_table),
                                  _ptr(seqlens), B, Hkv, num_pages, page_size, max_pages, d, 1 if advance else 0,
                                  _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_kv_append_paged")


def _proj_shapes(x, w, Hq, Hkv, d, with_r):
    _check(x, "x", torch.bfloat16, 2)
    _check(w, "w", torch.bfloat16, 2)
    nout = (2 * Hkv + (2 if with_r else 1) * Hq) * d
    if w.shape != (nout, x.shape[1]):
        raise ValueError(f"w must be [{nout}, {x.shape[1]}] ([W_Q; W_K; W_V{'; W_R' if with_r else ''}]), "
                         f"got {tuple(w.shape)}")


def plx_qkvr_proj(x, w, B, N, Hq, Hkv, d, with_r=True, q=None, k=None, v=None, r=None, stream=None):
    """q, k, v, rho of every token from one GEMM: x [B*N, d_model] bf16 (token
    m = b*N + t), w = [W_Q; W_K; W_V; W_R] [Nout, d_model] bf16.  Returns
    (q [B, Hq, N, d], k [B, Hkv, N, d], v, r [B, Hq, N, d] or None)."""
    _proj_shapes(x, w, Hq, Hkv, d, with_r)
    if x.shape[0] != B * N:
        raise ValueError("x must have B * N rows")
    dev = x.device
    q = torch.empty((B, Hq, N, d), device=dev, dtype=torch.bfloat16) if q is None else q
    k = torch.empty((B, Hkv, N, d), device=dev, dtype=torch.bfloat16) if k is None else k
    v = torch.empty((B, Hkv, N, d), device=dev, dtype=torch.bfloat16) if v is None else v
    if with_r and r is None:
        r = torch.empty((B, Hq, N, d), device=dev, dtype=torch.bfloat16)
    for t, n in ((q, "q"), (k, "k"), (v, "v")) + (((r, "r"),) if with_r else ()):
        _check(t, n, torch.bfloat16, 4)
    st = _lib.plx_qkvr_proj(_ptr(x), _ptr(w), _ptr(q), _ptr(k), _ptr(v), _ptr(r if with_r else None), B, N,
                            x.shape[1], Hq, Hkv, d, _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_qkvr_proj")
    return q, k, v, (r if with_r else None)


def plx_qkvr_proj_decode(x, w, kcache, vcache, seqlens, Hq, with_r=True, seqlens_out=None, q=None, r=None,
                         stream=None):
    """One decode step's projection with the KV append fused in: x [B, d_model]
    bf16 (each sequence's new token); k, v go into kcache / vcache
    [B, Hkv, S_max, d] at row seqlens[b].  Returns (q [B, Hq, d], r or None,
    seqlens_out [B] int32 = seqlens + 1 where the token was written)."""
    _check(kcache, "kcache", torch.bfloat16, 4)
    _check(vcache, "vcache", torch.bfloat16, 4)
    _check(seqlens, "seqlens", torch.int32, 1)
    B = x.shape[0]
    Hkv, S_max, d = kcache.shape[1], kcache.shape[2], kcache.shape[3]
    _proj_shapes(x, w, Hq, Hkv, d, with_r)
    if kcache.shape[0] != B or vcache.shape != kcache.shape or seqlens.shape != (B,):
        raise ValueError("shape mismatch between x, caches, seqlens")
    dev = x.device
    q = torch.empty((B, Hq, d), device=dev, dtype=torch.bfloat16) if q is None else q
    if with_r and r is None:
        r = torch.empty((B, Hq, d), device=dev, dtype=torch.bfloat16)
    if seqlens_out is None:
        seqlens_out = torch.empty_like(seqlens)
    st = _lib.plx_qkvr_proj_decode(_ptr(x), _ptr(w), _ptr(q), _ptr(r if with_r else None), _ptr(kcache),
                                   _ptr(vcache), _ptr(seqlens), _ptr(seqlens_out), B, x.shape[1], Hq, Hkv, S_max, d,
                                   _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_qkvr_proj_decode")
    return q, (r if with_r else None), seqlens_out


def plx_qkvr_proj_decode_paged(x, w, kpool, vpool, block_table, seqlens, Hq, with_r=True, seqlens_out=None, q=None,
                               r=None, stream=None):
    """plx_qkvr_proj_decode for page pools [num_pages, Hkv, page_size, d] and a
    block table [B, max_pages] int32."""
    _check(kpool, "kpool", torch.bfloat16, 4)
    _check(vpool, "vpool", torch.bfloat16, 4)
    _check(block_table, "block_table", torch.int32, 2)
    _check(seqlens, "seqlens", torch.int32, 1)
    B = x.shape[0]
    num_pages, Hkv, page_size, d = kpool.shape
    _proj_shapes(x, w, Hq, Hkv, d, with_r)
    if vpool.shape != kpool.shape or block_table.shape[0] != B or seqlens.shape != (B,):
        raise ValueError("shape mismatch between x, pools, block_table, seqlens")
    dev = x.device
    q = torch.empty((B, Hq, d), device=dev, dtype=torch.bfloat16) if q is None else q
    if with_r and r is None:
        r = torch.empty((B, Hq, d), device=dev, dtype=torch.bfloat16)
    if seqlens_out is None:
        seqlens_out = torch.empty_like(seqlens)
    st = _lib.plx_qkvr_proj_decode_paged(_ptr(x), _ptr(w), _ptr(q), _ptr(r if with_r else None), _ptr(kpool),
                                         _ptr(vpool), _ptr(block_table), _ptr(seqlens), _ptr(seqlens_out), B,
                                         x.shape[1], Hq, Hkv, num_pages, page_size, block_table.shape[1], d,
                                         _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_qkvr_proj_decode_paged")
    return q, (r if with_r else None), seqlens_out


def plx_decode_partial_size(B, Hq, Hkv, S_max, d, num_splits=0) -> int:
    return int(_lib.plx_decode_partial_size(B, Hq, Hkv, S_max, d, num_splits))


def plx_decode_partial(q, kcache, vcache, seqlens, r=None, key_offset=0, scale=None, num_splits=0, partial=None,
                       stream=None):
    """The state record of a slice of the keys (keys key_offset .. key_offset + S_max - 1
    of each sequence; seqlens are the full lengths) per (b, h): fp32 [B, Hq, 2d + 4]
    (m in log2 units, l, c, pad, O1[d], O2[d]).  The records are the head of a
    buffer of plx_decode_partial_size bytes whose tail is the kernels' scratch;
    `partial` may be a record view returned by an earlier call (its buffer is reused)."""
    _check(q, "q", torch.bfloat16, 3)
    _check(kcache, "kcache", torch.bfloat16, 4)
    _check(vcache, "vcache", torch.bfloat16, 4)
    _check(seqlens, "seqlens", torch.int32, 1)
    if r is not None:
        _check(r, "r", torch.bfloat16, 3)
    B, Hq, d = q.shape
    Hkv, S_max = kcache.shape[1], kcache.shape[2]
    if kcache.shape != (B, Hkv, S_max, d) or vcache.shape != kcache.shape or seqlens.shape != (B,):
        raise ValueError("shape mismatch between q, caches, seqlens")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = plx_decode_partial_size(B, Hq, Hkv, S_max, d, num_splits)
    if partial is None:
        buf = torch.empty((need + 3) // 4, device=q.device, dtype=torch.float32)
        partial = buf[:B * Hq * (2 * d + 4)].view(B, Hq, 2 * d + 4)
    else:
        _check(partial, "partial", torch.float32, 3)
        if partial.shape != (B, Hq, 2 * d + 4):
            raise ValueError("partial must be [B, Hq, 2d + 4]")
    avail = partial.untyped_storage().nbytes() - partial.storage_offset() * 4
    st = _lib.plx_decode_partial(_ptr(q), _ptr(r), _ptr(kcache), _ptr(vcache), _ptr(seqlens), int(key_offset), B, Hq,
                                 Hkv, S_max, d, float(scale), int(num_splits), _ptr(partial), avail, _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_decode_partial")
    return partial


def plx_decode_merge(partials, out=None, lse=None, return_lse=True, stream=None):
    """Merge gathered state records [ranks, B, Hq, 2d + 4] into (out, lse)."""
    _check(partials, "partials", torch.float32, 4)
    ranks, B, Hq, pf = partials.shape
    d = (pf - 4) // 2
    if out is None:
        out = torch.empty((B, Hq, d), device=partials.device, dtype=torch.bfloat16)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), device=partials.device, dtype=torch.float32)
    st = _lib.plx_decode_merge(_ptr(partials), ranks, B, Hq, d, _ptr(out), _ptr(lse), _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_decode_merge")
    return out, lse


PLX_NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


def plx_decode_noalloc(q, kcache, vcache, seqlens, r=None, scale=None, num_splits=0, out=None, lse=None,
                       return_lse=True, stream=None):
    """plx_decode without a workspace: for callers that cannot allocate device
    memory.  The partial states go to the library's fixed device scratch array
    (PLX_NOALLOC_SCRATCH_BYTES), shared by every call; calls that overlap on
    the GPU race on it.  out / lse are allocated here only when not given."""
    _check(q, "q", torch.bfloat16, 3)
    _check(kcache, "kcache", torch.bfloat16, 4)
    _check(vcache, "vcache", torch.bfloat16, 4)
    _check(seqlens, "seqlens", torch.int32, 1)
    if r is not None:
        _check(r, "r", torch.bfloat16, 3)
    B, Hq, d = q.shape
    Hkv, S_max = kcache.shape[1], kcache.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and return_lse:
        lse = torch.empty((B, Hq), device=q.device, dtype=torch.float32)
    st = _lib.plx_decode_noalloc(_ptr(q), _ptr(r), _ptr(kcache), _ptr(vcache), _ptr(seqlens), _ptr(out),
                                 _ptr(lse), B, Hq, Hkv, S_max, d, float(scale), int(num_splits), _stream(stream))
    if st != PLX_OK:
        raise PlxError(st, "plx_decode_noalloc")
    return out, lse


def plx_check_device_status(stream=None) -> int:
    """Synchronise the stream, read and clear the device error word; returns the status."""
    return _lib.plx_check_device_status(_stream(stream))


def plx_selftest_wait_timeout(limit_cycles: int, stream=None) -> int:
    return _lib.plx_selftest_wait_timeout(int(limit_cycles), _stream(stream))
