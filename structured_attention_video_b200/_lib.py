"""ctypes binding of libmonarch.so: the C ABI of include/monarch_attn.h, same names.

Argument marshalling only.  Every step of the forward pass runs in the CUDA
kernels of the library; there is no Python or CPU fallback.  Importing this
module fails with an ImportError when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

LIB_PATH = _build.LIB

if not os.path.exists(LIB_PATH):
    raise ImportError("libmonarch.so is not built (%s); run "
                      "`python -m structured_attention_video_b200.build`" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

F32, BF16 = 0, 1
STATUS = {0: "MONARCH_OK", 1: "MONARCH_ERR_INVALID_ARG", 2: "MONARCH_ERR_SHAPE",
          3: "MONARCH_ERR_ALIGN", 4: "MONARCH_ERR_UNSUPPORTED", 5: "MONARCH_ERR_NO_MEMORY",
          6: "MONARCH_ERR_CUDA", 7: "MONARCH_ERR_TIMEOUT", 8: "MONARCH_ERR_SCRATCH_LIMIT"}
NOALLOC_SCRATCH_BYTES = 64 << 20

_vp, _i, _sz, _ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_longlong
_ip = ctypes.POINTER(ctypes.c_int32)
_SHAPE = [_i] * 10          # B, H, f, h, w, d, b1, b2, tiles, iters

SIGNATURES = {
    "monarch_attn_fwd": ([_vp, _vp, _vp, _vp] + _SHAPE + [_i, _vp], _i),
    "monarch_attn_workspace_bytes": (_SHAPE + [_i], _sz),
    "monarch_attn_fwd_ws": ([_vp, _vp, _vp, _vp] + _SHAPE + [_i, _vp, _sz, _vp], _i),
    "monarch_attn_fwd_host": ([_vp, _vp, _vp, _vp] + _SHAPE + [_i, _vp], _i),
    "monarch_attn_kv_workspace_bytes": ([_i] * 12 + [_i], _sz),
    "monarch_attn_kv_path": ([_i] * 12 + [_i], _i),
    "monarch_attn_fwd_kv_ws": ([_vp, _vp, _vp, _vp] + [_i] * 12 + [_i, _vp, _sz, _vp], _i),
    "monarch_attn_fwd_units_ws": ([_vp, _vp, _vp, _vp] + _SHAPE + [_i, _i, _i, _vp, _sz, _vp], _i),
    "monarch_attn_fwd_noalloc": ([_vp, _vp, _vp, _vp] + _SHAPE + [_i, _vp], _i),
    "monarch_attn_fwd_layout_ws": ([_vp, _vp, _vp, _vp] + _SHAPE + [_i, _i, _vp, _sz, _vp], _i),
    "monarch_attn_tiled_workspace_bytes": (_SHAPE + [_i, _i], _sz),
    "monarch_attn_tiled_path": (_SHAPE + [_i, _i], _i),
    "monarch_attn_fwd_tiled_ws": ([_vp, _vp, _vp, _vp] + _SHAPE + [_i, _i, _i, _vp, _sz, _vp],
                                  _i),
    "monarch_attn_bwd_workspace_bytes": (_SHAPE + [_i], _sz),
    "monarch_attn_bwd_ws": ([_vp] * 7 + _SHAPE + [_i, _vp, _sz, _vp], _i),
    "monarch_attn_bwd": ([_vp] * 7 + _SHAPE + [_i, _vp], _i),
    "monarch_index_maps": ([_i] * 6 + [_ip, _ip, _ip, _ip], _i),
    "monarch_index_maps_device": ([_i] * 6 + [_vp, _vp, _vp, _vp, _vp], _i),
    "monarch_last_device_status": ([_vp], _i),
    "monarch_set_wait_limit": ([_ll], _ll),
    "monarch_debug_inject_stall": ([_i], _i),
    "monarch_status_string": ([_i], ctypes.c_char_p),
    "monarch_attn_path": (_SHAPE + [_i], _i),
    "monarch_profile_enable": ([_i], _i),
    "monarch_profile_collect": ([ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_ll), _i], _i),
    "monarch_profile_kernel_name": ([_i], ctypes.c_char_p),
}

for _name, (_args, _res) in SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


class MonarchError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.monarch_status_string(status).decode()
        super().__init__("%s: %s (%s)" % (where, STATUS.get(status, status), msg))


def check(status: int, where: str) -> None:
    if status != 0:
        raise MonarchError(status, where)


# Same names as the C ABI; pointers and streams are passed as integers.
def monarch_attn_fwd(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters, dtype, stream):
    return _lib.monarch_attn_fwd(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters, dtype,
                                 stream)


def monarch_attn_workspace_bytes(B, H, f, h, w, d, b1, b2, tiles, iters, dtype):
    return _lib.monarch_attn_workspace_bytes(B, H, f, h, w, d, b1, b2, tiles, iters, dtype)


def monarch_attn_fwd_ws(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters, dtype, workspace,
                        ws_bytes, stream):
    return _lib.monarch_attn_fwd_ws(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters, dtype,
                                    workspace, ws_bytes, stream)


def monarch_attn_kv_workspace_bytes(B, H, fq, fk, h, w, d, b1, b1k, b2, tiles, iters, dtype):
    return _lib.monarch_attn_kv_workspace_bytes(B, H, fq, fk, h, w, d, b1, b1k, b2, tiles, iters,
                                                dtype)


def monarch_attn_kv_path(B, H, fq, fk, h, w, d, b1, b1k, b2, tiles, iters, dtype):
    return _lib.monarch_attn_kv_path(B, H, fq, fk, h, w, d, b1, b1k, b2, tiles, iters, dtype)


def monarch_attn_fwd_kv_ws(q, k, v, out, B, H, fq, fk, h, w, d, b1, b1k, b2, tiles, iters, dtype,
                           workspace, ws_bytes, stream):
    return _lib.monarch_attn_fwd_kv_ws(q, k, v, out, B, H, fq, fk, h, w, d, b1, b1k, b2, tiles,
                                       iters, dtype, workspace, ws_bytes, stream)


def monarch_attn_fwd_units_ws(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters, dtype,
                              unit_begin, unit_end, workspace, ws_bytes, stream):
    return _lib.monarch_attn_fwd_units_ws(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters,
                                          dtype, unit_begin, unit_end, workspace, ws_bytes,
                                          stream)


def monarch_attn_fwd_host(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters, dtype, stream):
    return _lib.monarch_attn_fwd_host(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters,
                                      dtype, stream)


def monarch_attn_fwd_noalloc(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters, dtype,
                             stream):
    return _lib.monarch_attn_fwd_noalloc(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters,
                                         dtype, stream)


BHND, BNHD = 0, 1   # monarch_layout


def monarch_attn_fwd_layout_ws(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters, dtype,
                               layout, workspace, ws_bytes, stream):
    return _lib.monarch_attn_fwd_layout_ws(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters,
                                           dtype, layout, workspace, ws_bytes, stream)


TILE_QUERY_ROWS, TILE_KEY_COLUMNS = 0, 1   # monarch_tile_axis


def monarch_attn_tiled_workspace_bytes(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, axis):
    return _lib.monarch_attn_tiled_workspace_bytes(B, H, f, h, w, d, b1, b2, tiles, iters, dtype,
                                                   axis)


def monarch_attn_tiled_path(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, axis):
    return _lib.monarch_attn_tiled_path(B, H, f, h, w, d, b1, b2, tiles, iters, dtype, axis)


def monarch_attn_fwd_tiled_ws(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters, dtype, axis,
                              layout, workspace, ws_bytes, stream):
    return _lib.monarch_attn_fwd_tiled_ws(q, k, v, out, B, H, f, h, w, d, b1, b2, tiles, iters,
                                          dtype, axis, layout, workspace, ws_bytes, stream)


def monarch_attn_bwd_workspace_bytes(B, H, f, h, w, d, b1, b2, tiles, iters, dtype):
    return _lib.monarch_attn_bwd_workspace_bytes(B, H, f, h, w, d, b1, b2, tiles, iters, dtype)


def monarch_attn_bwd_ws(q, k, v, dy, dq, dk, dv, B, H, f, h, w, d, b1, b2, tiles, iters, dtype,
                        workspace, ws_bytes, stream):
    return _lib.monarch_attn_bwd_ws(q, k, v, dy, dq, dk, dv, B, H, f, h, w, d, b1, b2, tiles,
                                    iters, dtype, workspace, ws_bytes, stream)


def monarch_attn_bwd(q, k, v, dy, dq, dk, dv, B, H, f, h, w, d, b1, b2, tiles, iters, dtype,
                     stream):
    return _lib.monarch_attn_bwd(q, k, v, dy, dq, dk, dv, B, H, f, h, w, d, b1, b2, tiles, iters,
                                 dtype, stream)


def monarch_index_maps(f, h, w, b1, b2, tiles, u_of_n, v_of_n, perm, tile_begin):
    def ptr(a):
        return None if a is None else a.ctypes.data_as(_ip)
    return _lib.monarch_index_maps(f, h, w, b1, b2, tiles, ptr(u_of_n), ptr(v_of_n), ptr(perm),
                                   ptr(tile_begin))


def monarch_index_maps_device(f, h, w, b1, b2, tiles, u_of_n, v_of_n, perm, tile_begin, stream):
    return _lib.monarch_index_maps_device(f, h, w, b1, b2, tiles, u_of_n, v_of_n, perm,
                                          tile_begin, stream)


def monarch_last_device_status(stream):
    return _lib.monarch_last_device_status(stream)


def monarch_set_wait_limit(spins):
    return _lib.monarch_set_wait_limit(spins)


def monarch_debug_inject_stall(on):
    return _lib.monarch_debug_inject_stall(1 if on else 0)


def monarch_status_string(status):
    return _lib.monarch_status_string(status).decode()


def monarch_attn_path(B, H, f, h, w, d, b1, b2, tiles, iters, dtype):
    return _lib.monarch_attn_path(B, H, f, h, w, d, b1, b2, tiles, iters, dtype)


def monarch_profile_enable(on):
    return _lib.monarch_profile_enable(1 if on else 0)


def monarch_profile_collect():
    """{kernel name: (total ms, launches)} since the previous collect."""
    n = 16
    ms = (ctypes.c_double * n)()
    cnt = (_ll * n)()
    k = _lib.monarch_profile_collect(ms, cnt, n)
    if k < 0:
        raise MonarchError(6, "monarch_profile_collect")
    return {_lib.monarch_profile_kernel_name(i).decode(): (ms[i], cnt[i]) for i in range(k)}


def monarch_profile_kernel_name(k):
    name = _lib.monarch_profile_kernel_name(k)
    return None if name is None else name.decode()
