"""Torch-facing entry points: argument checks and marshalling onto the C ABI.

PyTorch supplies device memory (the output and the workspace, from its caching
allocator) and the current stream; the forward pass itself runs entirely in
the library's CUDA kernels.
"""
from __future__ import annotations

import torch

from . import _lib

_DTYPES = {torch.float32: _lib.F32, torch.bfloat16: _lib.BF16}


def _shape_args(q, f, h, w, b1, b2, tiles, iters):
    if q.dim() != 4:
        raise ValueError("expected [B, H, N, d] tensors")
    B, H, N, d = q.shape
    if N != f * h * w:
        raise ValueError("N = %d but f*h*w = %d" % (N, f * h * w))
    return (B, H, f, h, w, d, b1, b2, tiles, iters)


def _check_tensors(*ts):
    dev = ts[0].device
    for t in ts:
        if not t.is_cuda or t.device != dev:
            raise ValueError("all tensors must be on the same CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous [B, H, N, d]")
        if t.dtype != ts[0].dtype or t.shape != ts[0].shape:
            raise ValueError("q, k, v and out must share dtype and shape")
    if ts[0].dtype not in _DTYPES:
        raise ValueError("dtype must be float32 or bfloat16")


def workspace_bytes(q, *, f, h, w, b1, b2, tiles=1, iters=1) -> int:
    args = _shape_args(q, f, h, w, b1, b2, tiles, iters)
    return _lib.monarch_attn_workspace_bytes(*args, _DTYPES[q.dtype])


def kernel_path(q, *, f, h, w, b1, b2, tiles=1, iters=1) -> int:
    """0 = generic SIMT kernels, 1 = sm_100a tensor-core kernels."""
    args = _shape_args(q, f, h, w, b1, b2, tiles, iters)
    return _lib.monarch_attn_path(*args, _DTYPES[q.dtype])


def monarch_attention(q, k, v, *, f, h, w, b1, b2, tiles=1, iters=1, out=None, workspace=None):
    """Y = M V with M the tiled Monarch approximation of softmax(Q K^T / sqrt(d))."""
    if out is None:
        out = torch.empty_like(q)
    _check_tensors(q, k, v, out)
    args = _shape_args(q, f, h, w, b1, b2, tiles, iters)
    dt = _DTYPES[q.dtype]
    need = _lib.monarch_attn_workspace_bytes(*args, dt)
    if need == 0:
        # validation failed: let the library report why
        _lib.check(_lib.monarch_attn_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            out.data_ptr(), *args, dt, 0, 0, 0),
                   "monarch_attn_fwd_ws")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    _lib.check(_lib.monarch_attn_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                        *args, dt, workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(), stream),
               "monarch_attn_fwd_ws")
    return out


def monarch_attention_kv(q, k, v, *, fq, fk, h, w, b1, b1k, b2, tiles=1, iters=1, out=None):
    """Queries of a chunk of fq frames [B, H, fq*h*w, d] against keys and values of
    fk frames [B, H, fk*h*w, d] (a cache of earlier frames and the chunk's own)."""
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape:
        raise ValueError("expected [B, H, N, d] tensors, k and v alike")
    B, H, nq, d = q.shape
    if nq != fq * h * w or k.shape != (B, H, fk * h * w, d):
        raise ValueError("query or key/value lengths do not match the frame counts")
    if out is None:
        out = torch.empty_like(q)
    for t in (q, k, v, out):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != q.dtype:
            raise ValueError("contiguous CUDA tensors of one dtype expected")
    dt = _DTYPES[q.dtype]
    args = (B, H, fq, fk, h, w, d, b1, b1k, b2, tiles, iters)
    need = _lib.monarch_attn_kv_workspace_bytes(*args, dt)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    _lib.check(_lib.monarch_attn_fwd_kv_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                           out.data_ptr(), *args, dt, ws.data_ptr(), need,
                                           stream), "monarch_attn_fwd_kv_ws")
    return out


def monarch_attention_units(q, k, v, out, *, f, h, w, b1, b2, tiles=1, iters=1, unit_begin=0,
                            unit_end=None):
    """Computes only the (head, tile) units [unit_begin, unit_end) of the forward pass
    (unit = (b*H + h)*tiles + g) into their rows of `out`; other rows are untouched."""
    _check_tensors(q, k, v, out)
    args = _shape_args(q, f, h, w, b1, b2, tiles, iters)
    if unit_end is None:
        unit_end = q.shape[0] * q.shape[1] * tiles
    dt = _DTYPES[q.dtype]
    need = _lib.monarch_attn_workspace_bytes(*args, dt)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    _lib.check(_lib.monarch_attn_fwd_units_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                              out.data_ptr(), *args, dt, unit_begin, unit_end,
                                              ws.data_ptr(), need, stream),
               "monarch_attn_fwd_units_ws")
    return out


def monarch_attention_backward(q, k, v, dy, *, f, h, w, b1, b2, tiles=1, iters=1, workspace=None):
    """Gradients (dq, dk, dv) of a loss whose gradient with respect to
    monarch_attention(q, k, v, ...) is dy (one iteration)."""
    _check_tensors(q, k, v, dy)
    args = _shape_args(q, f, h, w, b1, b2, tiles, iters)
    dt = _DTYPES[q.dtype]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    need = _lib.monarch_attn_bwd_workspace_bytes(*args, dt)
    if need == 0:
        # validation failed or iters != 1: let the library report why
        _lib.check(_lib.monarch_attn_bwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            dy.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                            dv.data_ptr(), *args, dt, 0, 0, 0),
                   "monarch_attn_bwd_ws")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    _lib.check(_lib.monarch_attn_bwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), dy.data_ptr(),
                                        dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), *args, dt,
                                        workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(), stream),
               "monarch_attn_bwd_ws")
    return dq, dk, dv


def monarch_attention_bnhd(q, k, v, *, f, h, w, b1, b2, tiles=1, iters=1, out=None,
                           workspace=None):
    """monarch_attention on [B, N, H, d] tensors (the heads of each token
    contiguous); the kernels read the strided rows directly."""
    if out is None:
        out = torch.empty_like(q)
    _check_tensors(q, k, v, out)
    if q.dim() != 4:
        raise ValueError("expected [B, N, H, d] tensors")
    B, N, H, d = q.shape
    if N != f * h * w:
        raise ValueError("N = %d but f*h*w = %d" % (N, f * h * w))
    args = (B, H, f, h, w, d, b1, b2, tiles, iters)
    dt = _DTYPES[q.dtype]
    need = _lib.monarch_attn_workspace_bytes(*args, dt)
    if need == 0:
        _lib.check(_lib.monarch_attn_fwd_layout_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                   out.data_ptr(), *args, dt, _lib.BNHD, 0, 0, 0),
                   "monarch_attn_fwd_layout_ws")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    _lib.check(_lib.monarch_attn_fwd_layout_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                               out.data_ptr(), *args, dt, _lib.BNHD,
                                               workspace.data_ptr(),
                                               workspace.numel() * workspace.element_size(),
                                               stream),
               "monarch_attn_fwd_layout_ws")
    return out


_AXES = {"query_rows": _lib.TILE_QUERY_ROWS, "key_columns": _lib.TILE_KEY_COLUMNS}
_LAYOUTS = {"bhnd": _lib.BHND, "bnhd": _lib.BNHD}


def monarch_attention_tiled(q, k, v, *, f, h, w, b1, b2, tiles=1, iters=1, axis="query_rows",
                            layout="bhnd", out=None, workspace=None):
    """monarch_attention with the tiles on either axis: axis="query_rows" (tiles in
    [1, b1], every other entry point) or "key_columns" (the key columns of every
    block split into tiles in [1, b2]; each query row's L runs over the b1*t
    (block, key tile) super-keys).  layout "bhnd" ([B, H, N, d]) or "bnhd"
    ([B, N, H, d])."""
    if out is None:
        out = torch.empty_like(q)
    _check_tensors(q, k, v, out)
    if q.dim() != 4:
        raise ValueError("expected 4-D tensors")
    if axis not in _AXES or layout not in _LAYOUTS:
        raise ValueError("axis must be one of %s and layout one of %s" % (list(_AXES),
                                                                          list(_LAYOUTS)))
    if layout == "bhnd":
        B, H, N, d = q.shape
    else:
        B, N, H, d = q.shape
    if N != f * h * w:
        raise ValueError("N = %d but f*h*w = %d" % (N, f * h * w))
    args = (B, H, f, h, w, d, b1, b2, tiles, iters)
    dt, ax, lay = _DTYPES[q.dtype], _AXES[axis], _LAYOUTS[layout]
    need = _lib.monarch_attn_tiled_workspace_bytes(*args, dt, ax)
    if need == 0:
        _lib.check(_lib.monarch_attn_fwd_tiled_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                  out.data_ptr(), *args, dt, ax, lay, 0, 0, 0),
                   "monarch_attn_fwd_tiled_ws")
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    stream = torch.cuda.current_stream(q.device).cuda_stream
    _lib.check(_lib.monarch_attn_fwd_tiled_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                              out.data_ptr(), *args, dt, ax, lay,
                                              workspace.data_ptr(),
                                              workspace.numel() * workspace.element_size(),
                                              stream),
               "monarch_attn_fwd_tiled_ws")
    return out
