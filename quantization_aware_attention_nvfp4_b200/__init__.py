"""Attn-QAT (NVFP4 fake-quantized training attention) for NVIDIA B200 (sm_100a).

A thin Python binding over the C ABI of ``libattnqat.so`` (``include/attnqat.h``).
It only marshals arguments: PyTorch supplies device memory and the current CUDA
stream, and every step of the computation runs in the library's kernels.  There
is no CPU or library fallback: if the library cannot be loaded or the device is
not sm_100, the calls raise.

Entry points (same names as the C ABI):

* ``attnqat_quantize(x2d)`` -- NVFP4 codes, E4M3 scales and dequantized values
  of a bf16 view, blocks of 16 along the last axis (a strided/transposed view is
  allowed).
* ``attnqat_fwd(q, k, v, sm_scale=None, flags=QUANT_ALL)`` -- forward; returns
  ``(o, lse, m, ws)``.
* ``attnqat_bwd(q, k, v, lse, m, dO, ws, sm_scale=None, flags=QUANT_ALL)`` --
  straight-through backward; returns ``(dq, dk, dv)``.
* ``attnqat_sparse_fwd(q, k, v, tile_mask, ...)`` and
  ``attnqat_sparse_bwd(q, k, v, lse, m, dO, ws, tile_mask, ...)`` -- the
  block-sparse (VSA fine attention) variants: ``tile_mask`` is a uint8 CUDA
  tensor [B, H, ceil(Lq/128), ceil(Lk/128)], nonzero where a 128-query tile
  attends a 128-key tile.
* ``attnqat_vsa_select(q, k, topk)`` -- that mask from the coarse scores of
  the tiles' means: the ``topk`` best key tiles per query tile.
* ``tile=64`` on these three selects the tile-64 profile: masks of 64-token
  blocks [B, H, ceil(Lq/64), ceil(Lk/64)].

``sm_scale=None`` means 1/sqrt(D), chosen here and passed explicitly; the
library itself never substitutes a default (FastVideo PR #1457 review, F1).
"""
from __future__ import annotations

import ctypes
import math
import re
import threading

from . import build as _build

QUANT_Q = 1
QUANT_K = 2
QUANT_V = 4
QUANT_P = 8
QUANT_ALL = 15
CAUSAL = 32  # causal masking (attnqat_fwd / attnqat_bwd; Lq == Lk)
TILE64 = 64  # 64-token tile masks on the sparse calls (set by their tile=64 argument)

OK = 0
EINVAL = -1
EUNSUPPORTED = -2
ENOSPC = -3
ECUDA = -4
ETIMEOUT = -5

_lock = threading.Lock()
_lib = None


class AttnQatError(RuntimeError):
    def __init__(self, status: int, what: str):
        lib = load()
        msg = lib.attnqat_strerror(status).decode()
        if status == ECUDA:
            msg += " (cudaError %d)" % lib.attnqat_last_cuda_error()
        super().__init__("%s failed: %s [status %d]" % (what, msg, status))
        self.status = status


def load(build_if_needed: bool = True):
    """Loads libattnqat.so (building it with nvcc first if it is missing or
    stale).  Raises if it cannot be built or loaded."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build() if build_if_needed else _build.LIB
            lib = ctypes.CDLL(path)
            P, I, I64, U32, SZ, F = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                     ctypes.c_uint32, ctypes.c_size_t, ctypes.c_float)
            lib.attnqat_strerror.restype = ctypes.c_char_p
            lib.attnqat_strerror.argtypes = [I]
            lib.attnqat_last_cuda_error.restype = I
            lib.attnqat_last_cuda_error.argtypes = []
            lib.attnqat_device_status.restype = I
            lib.attnqat_device_status.argtypes = []
            lib.attnqat_selftest_wait_timeout.restype = I
            lib.attnqat_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, P, P]
            lib.attnqat_profile_enable.restype = I
            lib.attnqat_profile_enable.argtypes = [I]
            lib.attnqat_profile_read.restype = I
            lib.attnqat_profile_read.argtypes = [P, P, I]
            lib.attnqat_quantize.restype = I
            lib.attnqat_quantize.argtypes = [P, I64, I64, I64, I64, I64, I64, P, P, P, P]
            lib.attnqat_quantize_gs.restype = I
            lib.attnqat_quantize_gs.argtypes = [P, I64, I64, I64, I64, I64, I64, P, P, P, P, P]
            lib.attnqat_workspace_size.restype = SZ
            lib.attnqat_workspace_size.argtypes = [I, I, I, I, I, U32]
            lib.attnqat_fwd.restype = I
            lib.attnqat_fwd.argtypes = [P, P, P, I, I, I, I, I, F, U32, P, P, P, P, SZ, P]
            lib.attnqat_bwd.restype = I
            lib.attnqat_bwd.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, U32, P, P, P, P, SZ, P]
            lib.attnqat_vsa_select_workspace_size.restype = SZ
            lib.attnqat_vsa_select_workspace_size.argtypes = [I, I, I, I, I]
            lib.attnqat_vsa_select.restype = I
            lib.attnqat_vsa_select.argtypes = [P, P, I, I, I, I, I, I, P, P, SZ, P]
            lib.attnqat_vsa_select_tiles_workspace_size.restype = SZ
            lib.attnqat_vsa_select_tiles_workspace_size.argtypes = [I, I, I, I, I, I]
            lib.attnqat_vsa_select_tiles.restype = I
            lib.attnqat_vsa_select_tiles.argtypes = [P, P, I, I, I, I, I, I, I, P, P, SZ, P]
            lib.attnqat_sparse_workspace_size.restype = SZ
            lib.attnqat_sparse_workspace_size.argtypes = [I, I, I, I, I, U32]
            lib.attnqat_sparse_fwd.restype = I
            lib.attnqat_sparse_fwd.argtypes = [P, P, P, I, I, I, I, I, F, U32, P, P, P, P, P, SZ, P]
            lib.attnqat_sparse_bwd.restype = I
            lib.attnqat_sparse_bwd.argtypes = [P, P, P, P, P, P, I, I, I, I, I, F, U32, P, P, P, P, P, SZ,
                                               P]
            _lib = lib
    return _lib


def header_symbols() -> list:
    """Names of the functions include/attnqat.h declares."""
    import os
    text = open(os.path.join(_build.INCLUDE, "attnqat.h")).read()
    return sorted(set(re.findall(r"\b(attnqat_[a-z0-9_]+)\s*\(", text)))


def _torch():
    import torch
    return torch


def _stream_ptr(stream=None, device=None):
    """The cudaStream_t of `stream` (default: the current stream of `device`),
    which must belong to `device` when both are given."""
    torch = _torch()
    s = torch.cuda.current_stream(device) if stream is None else stream
    if device is not None and s.device != device:
        raise ValueError("stream is on %s, the tensors on %s" % (s.device, device))
    return ctypes.c_void_p(s.cuda_stream)


def _on(device):
    """Context that makes `device` the current CUDA device for a library call
    (the library launches on the current device)."""
    import contextlib
    if device.type != "cuda":
        return contextlib.nullcontext()
    return _torch().cuda.device(device)


def _check(status: int, what: str):
    if status != OK:
        raise AttnQatError(status, what)


def _require_bf16_cuda(name, t, ndim=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype != torch.bfloat16:
        raise ValueError("%s must be bfloat16" % name)
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims" % (name, ndim))


def _require_buffer(name, t, shape, dtype, device):
    """A caller-supplied tensor the library reads or writes densely: it must
    have exactly this shape and dtype, be contiguous and sit on `device` (the
    C ABI receives a bare pointer and cannot check its extent)."""
    torch = _torch()
    if not isinstance(t, torch.Tensor) or t.device != device or t.dtype != dtype or \
            tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError("%s must be a contiguous %s tensor of shape %s on %s"
                         % (name, str(dtype).replace("torch.", ""), tuple(shape), device))
    return t


def _require_workspace(ws, device):
    """A caller-supplied workspace: contiguous, on `device` (its size is
    checked by the library against the call's need)."""
    torch = _torch()
    if not isinstance(ws, torch.Tensor) or ws.device != device or not ws.is_contiguous():
        raise ValueError("ws must be a contiguous tensor on %s" % device)
    return ws


def _fwd_outputs(out, q, B, H, Lq):
    """(o, lse, m): new tensors, or the caller's after checking them."""
    torch = _torch()
    if out is None:
        return (torch.empty_like(q), torch.empty((B, H, Lq), dtype=torch.float32, device=q.device),
                torch.empty((B, H, Lq), dtype=torch.float32, device=q.device))
    o, lse, m = out
    _require_buffer("o", o, q.shape, torch.bfloat16, q.device)
    _require_buffer("lse", lse, (B, H, Lq), torch.float32, q.device)
    _require_buffer("m", m, (B, H, Lq), torch.float32, q.device)
    return o, lse, m


def _bwd_buffers(q, k, v, lse, m, dO, ws, out, B, H, Lq):
    """Checks the backward's inputs from the forward (lse, m, ws) and dO;
    returns (dq, dk, dv): new tensors, or the caller's after checking them."""
    torch = _torch()
    _require_bf16_cuda("dO", dO, 4)
    _require_buffer("dO", dO, q.shape, torch.bfloat16, q.device)
    _require_buffer("lse", lse, (B, H, Lq), torch.float32, q.device)
    _require_buffer("m", m, (B, H, Lq), torch.float32, q.device)
    _require_workspace(ws, q.device)
    if out is None:
        return torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dq, dk, dv = out
    _require_buffer("dq", dq, q.shape, torch.bfloat16, q.device)
    _require_buffer("dk", dk, k.shape, torch.bfloat16, q.device)
    _require_buffer("dv", dv, v.shape, torch.bfloat16, q.device)
    return dq, dk, dv


def attnqat_quantize(x, stream=None):
    """NVFP4 fq of a 2-D (or 3-D batched) bf16 CUDA view, blocks of 16 along
    the last axis.  Strides may be arbitrary (e.g. ``v.transpose(-1, -2)``).

    Returns ``(codes uint8 [..., cols/2], scales uint8 [..., cols/16],
    deq bf16 with x's shape and strides)``."""
    torch = _torch()
    _require_bf16_cuda("x", x)
    if x.dim() == 2:
        batch, (rows, cols) = 1, x.shape
        sb, (sr, sc) = 0, x.stride()
    elif x.dim() == 3:
        batch, rows, cols = x.shape
        sb, sr, sc = x.stride()
    else:
        raise ValueError("x must be 2-D or 3-D")
    codes = torch.empty((batch, rows, cols // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((batch, rows, cols // 16), dtype=torch.uint8, device=x.device)
    deq = torch.empty_strided(x.shape, x.stride(), dtype=torch.bfloat16, device=x.device)
    with _on(x.device):
        st = load().attnqat_quantize(ctypes.c_void_p(x.data_ptr()), batch, rows, cols, sb, sr, sc,
                                     ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                                     ctypes.c_void_p(deq.data_ptr()), _stream_ptr(stream, x.device))
    _check(st, "attnqat_quantize")
    if x.dim() == 2:
        codes, scales = codes[0], scales[0]
    return codes, scales, deq


def attnqat_quantize_gs(x, stream=None):
    """NVFP4 with an FP32 global scale (G = 2688 / max|x|) of a 2-D (or 3-D
    batched) bf16 CUDA view, blocks of 16 along the last axis.

    Returns ``(codes uint8 [..., cols/2], scales uint8 [..., cols/16],
    deq bf16 with x's shape and strides, gscale float32 CUDA tensor [1])``."""
    torch = _torch()
    _require_bf16_cuda("x", x)
    if x.dim() == 2:
        batch, (rows, cols) = 1, x.shape
        sb, (sr, sc) = 0, x.stride()
    elif x.dim() == 3:
        batch, rows, cols = x.shape
        sb, sr, sc = x.stride()
    else:
        raise ValueError("x must be 2-D or 3-D")
    codes = torch.empty((batch, rows, cols // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty((batch, rows, cols // 16), dtype=torch.uint8, device=x.device)
    deq = torch.empty_strided(x.shape, x.stride(), dtype=torch.bfloat16, device=x.device)
    gscale = torch.empty(1, dtype=torch.float32, device=x.device)
    with _on(x.device):
        st = load().attnqat_quantize_gs(ctypes.c_void_p(x.data_ptr()), batch, rows, cols, sb, sr, sc,
                                        ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
                                        ctypes.c_void_p(deq.data_ptr()), ctypes.c_void_p(gscale.data_ptr()),
                                        _stream_ptr(stream, x.device))
    _check(st, "attnqat_quantize_gs")
    if x.dim() == 2:
        codes, scales = codes[0], scales[0]
    return codes, scales, deq, gscale


def attnqat_workspace_size(B, H, Lq, Lk, D, flags=QUANT_ALL) -> int:
    return int(load().attnqat_workspace_size(B, H, Lq, Lk, D, flags))


def _shape(q, k, v):
    for n, t in (("q", q), ("k", k), ("v", v)):
        _require_bf16_cuda(n, t, 4)
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous [B, H, L, D]" % n)
    B, H, Lq, D = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[1] != H or k.shape[3] != D:
        raise ValueError("k and v must be [B, H, Lk, D] matching q [B, H, Lq, D]")
    if k.device != q.device or v.device != q.device:
        raise ValueError("q, k and v must be on one device")
    return B, H, Lq, k.shape[2], D


def attnqat_fwd(q, k, v, sm_scale=None, flags=QUANT_ALL, ws=None, out=None, stream=None):
    """Attn-QAT forward.  Returns ``(o, lse, m, ws)``; pass ``ws`` unchanged
    to :func:`attnqat_bwd`."""
    torch = _torch()
    B, H, Lq, Lk, D = _shape(q, k, v)
    c = 1.0 / math.sqrt(D) if sm_scale is None else float(sm_scale)
    need = attnqat_workspace_size(B, H, Lq, Lk, D, flags)
    if need == 0:
        _check(EINVAL, "attnqat_workspace_size")
    ws = torch.empty(need, dtype=torch.uint8, device=q.device) if ws is None else _require_workspace(ws, q.device)
    o, lse, m = _fwd_outputs(out, q, B, H, Lq)
    with _on(q.device):
        st = load().attnqat_fwd(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                ctypes.c_void_p(v.data_ptr()), B, H, Lq, Lk, D, c, flags,
                                ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
                                ctypes.c_void_p(m.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                                ws.numel() * ws.element_size(), _stream_ptr(stream, q.device))
    _check(st, "attnqat_fwd")
    return o, lse, m, ws


def attnqat_bwd(q, k, v, lse, m, dO, ws, sm_scale=None, flags=QUANT_ALL, out=None, stream=None):
    """Attn-QAT backward (straight-through).  ``ws`` is the workspace the
    forward returned.  Returns ``(dq, dk, dv)``."""
    B, H, Lq, Lk, D = _shape(q, k, v)
    dq, dk, dv = _bwd_buffers(q, k, v, lse, m, dO, ws, out, B, H, Lq)
    c = 1.0 / math.sqrt(D) if sm_scale is None else float(sm_scale)
    with _on(q.device):
        st = load().attnqat_bwd(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                ctypes.c_void_p(v.data_ptr()),
                                ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(m.data_ptr()),
                                ctypes.c_void_p(dO.data_ptr()), B, H, Lq, Lk, D, c, flags,
                                ctypes.c_void_p(dq.data_ptr()), ctypes.c_void_p(dk.data_ptr()),
                                ctypes.c_void_p(dv.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                                ws.numel() * ws.element_size(), _stream_ptr(stream, q.device))
    _check(st, "attnqat_bwd")
    return dq, dk, dv


SPARSE_TILE = 128


def attnqat_sparse_workspace_size(B, H, Lq, Lk, D, flags=QUANT_ALL) -> int:
    return int(load().attnqat_sparse_workspace_size(B, H, Lq, Lk, D, flags))


def _check_tile(tile):
    if tile not in (64, 128):
        raise ValueError("tile must be 64 or 128")
    return TILE64 if tile == 64 else 0


def _tile_mask(tile_mask, B, H, Lq, Lk, device, tile=SPARSE_TILE):
    torch = _torch()
    want = (B, H, -(-Lq // tile), -(-Lk // tile))
    if not isinstance(tile_mask, torch.Tensor) or tile_mask.dtype != torch.uint8 or \
            tile_mask.device != device or tuple(tile_mask.shape) != want or not tile_mask.is_contiguous():
        raise ValueError("tile_mask must be a contiguous uint8 tensor %s on %s" % (want, device))
    return ctypes.c_void_p(tile_mask.data_ptr())


def attnqat_vsa_select(q, k, topk, out=None, ws=None, stream=None, tile=SPARSE_TILE):
    """Key tiles per query tile for the block-sparse attention: the ``topk``
    key tiles whose mean row scores highest against the query tile's mean row
    (ties to the lower tile), over ``tile``-token tiles (128, or 64 for the
    tile-64 profile).  ``q`` [B, H, Lq, D], ``k`` [B, H, Lk, D] bf16 CUDA
    tensors.  Returns the uint8 tile mask [B, H, ceil(Lq/tile),
    ceil(Lk/tile)] (``out`` if given)."""
    torch = _torch()
    _check_tile(tile)
    for n, t in (("q", q), ("k", k)):
        _require_bf16_cuda(n, t, 4)
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous [B, H, L, D]" % n)
    B, H, Lq, D = q.shape
    Lk = k.shape[2]
    if k.shape[0] != B or k.shape[1] != H or k.shape[3] != D:
        raise ValueError("k must be [B, H, Lk, D] matching q [B, H, Lq, D]")
    if k.device != q.device:
        raise ValueError("q and k must be on one device")
    need = int(load().attnqat_vsa_select_tiles_workspace_size(B, H, Lq, Lk, D, tile))
    if need == 0:
        _check(EINVAL, "attnqat_vsa_select_tiles_workspace_size")
    ws = torch.empty(need, dtype=torch.uint8, device=q.device) if ws is None else _require_workspace(ws, q.device)
    if out is None:
        out = torch.empty((B, H, -(-Lq // tile), -(-Lk // tile)), dtype=torch.uint8, device=q.device)
    else:
        _tile_mask(out, B, H, Lq, Lk, q.device, tile)
    with _on(q.device):
        st = load().attnqat_vsa_select_tiles(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), B, H, Lq,
                                             Lk, D, tile, int(topk), ctypes.c_void_p(out.data_ptr()),
                                             ctypes.c_void_p(ws.data_ptr()), ws.numel() * ws.element_size(),
                                             _stream_ptr(stream, q.device))
    _check(st, "attnqat_vsa_select_tiles")
    return out


def attnqat_sparse_fwd(q, k, v, tile_mask, sm_scale=None, flags=QUANT_ALL, ws=None, out=None, stream=None,
                       tile=SPARSE_TILE):
    """Block-sparse Attn-QAT forward (VSA fine attention): each ``tile``-token
    query tile (128, or 64 for the tile-64 profile) attends only the key tiles
    ``tile_mask`` selects.  Returns ``(o, lse, m, ws)``; pass ``ws``, the same
    mask and the same tile to :func:`attnqat_sparse_bwd`."""
    torch = _torch()
    B, H, Lq, Lk, D = _shape(q, k, v)
    flags = (flags & ~TILE64) | _check_tile(tile)
    mp = _tile_mask(tile_mask, B, H, Lq, Lk, q.device, tile)
    c = 1.0 / math.sqrt(D) if sm_scale is None else float(sm_scale)
    need = attnqat_sparse_workspace_size(B, H, Lq, Lk, D, flags)
    if need == 0:
        _check(EINVAL, "attnqat_sparse_workspace_size")
    ws = torch.empty(need, dtype=torch.uint8, device=q.device) if ws is None else _require_workspace(ws, q.device)
    o, lse, m = _fwd_outputs(out, q, B, H, Lq)
    with _on(q.device):
        st = load().attnqat_sparse_fwd(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                       ctypes.c_void_p(v.data_ptr()), B, H, Lq, Lk, D, c, flags, mp,
                                       ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
                                       ctypes.c_void_p(m.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                                       ws.numel() * ws.element_size(), _stream_ptr(stream, q.device))
    _check(st, "attnqat_sparse_fwd")
    return o, lse, m, ws


def attnqat_sparse_bwd(q, k, v, lse, m, dO, ws, tile_mask, sm_scale=None, flags=QUANT_ALL, out=None,
                       stream=None, tile=SPARSE_TILE):
    """Block-sparse Attn-QAT backward (straight-through) with the forward's
    ``ws``, ``tile_mask`` and ``tile``.  Returns ``(dq, dk, dv)``."""
    B, H, Lq, Lk, D = _shape(q, k, v)
    flags = (flags & ~TILE64) | _check_tile(tile)
    mp = _tile_mask(tile_mask, B, H, Lq, Lk, q.device, tile)
    dq, dk, dv = _bwd_buffers(q, k, v, lse, m, dO, ws, out, B, H, Lq)
    c = 1.0 / math.sqrt(D) if sm_scale is None else float(sm_scale)
    with _on(q.device):
        st = load().attnqat_sparse_bwd(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                       ctypes.c_void_p(v.data_ptr()),
                                       ctypes.c_void_p(lse.data_ptr()), ctypes.c_void_p(m.data_ptr()),
                                       ctypes.c_void_p(dO.data_ptr()), B, H, Lq, Lk, D, c, flags, mp,
                                       ctypes.c_void_p(dq.data_ptr()), ctypes.c_void_p(dk.data_ptr()),
                                       ctypes.c_void_p(dv.data_ptr()), ctypes.c_void_p(ws.data_ptr()),
                                       ws.numel() * ws.element_size(), _stream_ptr(stream, q.device))
    _check(st, "attnqat_sparse_bwd")
    return dq, dk, dv


def attnqat_profile_enable(on: bool = True) -> None:
    """Start (or stop) recording CUDA events around each kernel the library
    launches; see attnqat_profile_read."""
    _check(load().attnqat_profile_enable(1 if on else 0), "attnqat_profile_enable")


def attnqat_profile_read(max_records: int = 4096) -> list:
    """[(kernel name, milliseconds)] for the kernels launched since the last
    read (waits for their events)."""
    names = (ctypes.c_char_p * max_records)()
    ms = (ctypes.c_float * max_records)()
    n = load().attnqat_profile_read(names, ms, max_records)
    if n < 0:
        _check(n, "attnqat_profile_read")
    return [(names[i].decode(), float(ms[i])) for i in range(min(n, max_records))]


def attnqat_device_status() -> int:
    """Synchronizes the device; raises if a bounded device-side wait timed out."""
    st = load().attnqat_device_status()
    _check(st, "attnqat_device_status")
    return st


def attnqat_selftest_wait_timeout(limit_ns: int = 1000000, stream=None) -> int:
    """Runs the library's timed-out-wait path on purpose (see attnqat.h) and
    returns how many waits ended without their barrier (2 when it works).
    Leaves the device status raised: the next attnqat_device_status() call
    raises ETIMEOUT and clears it."""
    torch = _torch()
    ended = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(load().attnqat_selftest_wait_timeout(int(limit_ns), ctypes.c_void_p(ended.data_ptr()),
                                                _stream_ptr(stream)), "attnqat_selftest_wait_timeout")
    return int(ended.item())
