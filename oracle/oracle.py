"""ctypes wrapper of the float64 CPU oracle (monarch_oracle.c).

Test infrastructure: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  It never imports the
CUDA package, and the CUDA package never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "monarch_oracle.c")
LIB = os.path.join(HERE, "_build", "liboracle.so")

_libs = {}


def build(force: bool = False, src: str = SRC, out: str = LIB) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, IEEE float: no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        os.makedirs(os.path.dirname(out), exist_ok=True)
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.run(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", src,
                        "-o", tmp, "-lm"], check=True)
        os.replace(tmp, out)
    return out


def _load(path: str | None = None):
    """The oracle library (default build), or another build of it at `path`."""
    key = path or LIB
    if key not in _libs:
        lib = ctypes.CDLL(build() if path is None else path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        i = ctypes.c_int
        lib.oracle_index_maps.argtypes = [i, i, i, i, i, i, ip, ip, ip, ip, ip]
        lib.oracle_index_maps.restype = i
        lib.oracle_monarch_attn.argtypes = [dp, dp, dp, dp, i, i, i, i, i, i, i, dp, dp, i]
        lib.oracle_monarch_attn.restype = i
        lib.oracle_monarch_problems.argtypes = [dp, dp, dp, dp, i, i, i, i, i, i, i, i, ip, i]
        lib.oracle_monarch_problems.restype = i
        lib.oracle_monarch_attn_kv.argtypes = [dp, dp, dp, dp, i, i, i, i, i, i, i, dp, dp, i]
        lib.oracle_monarch_attn_kv.restype = i
        lib.oracle_monarch_attn_keytiles.argtypes = [dp, dp, dp, dp, i, i, i, i, i, i, i, dp,
                                                     dp, i, ip, i]
        lib.oracle_monarch_attn_keytiles.restype = i
        lib.oracle_monarch_attn_bwd.argtypes = [dp] * 7 + [i] * 7
        lib.oracle_monarch_attn_bwd.restype = i
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = i
        _libs[key] = lib
    return _libs[key]


def _dptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if a is not None else None


def _iptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def max_threads() -> int:
    return _load().oracle_max_threads()


def index_maps(f, h, w, b1, b2, tiles):
    """u(n), v(n), P(n) = v*b1 + u, tile boundaries and tile of each block row."""
    N = f * h * w
    u = np.zeros(N, np.int32)
    v = np.zeros(N, np.int32)
    p = np.zeros(N, np.int32)
    lo = np.zeros(tiles + 1, np.int32)
    tu = np.zeros(max(b1, 1), np.int32)
    rc = _load().oracle_index_maps(f, h, w, b1, b2, tiles, _iptr(u), _iptr(v), _iptr(p),
                                   _iptr(lo), _iptr(tu))
    if rc != 0:
        raise ValueError("oracle_index_maps: invalid arguments")
    return {"u_of_n": u, "v_of_n": v, "perm": p, "tile_lo": lo, "tile_of_u": tu}


def _heads(x):
    x = np.ascontiguousarray(x, dtype=np.float64)
    return x.reshape(-1, x.shape[-2], x.shape[-1]), x.shape


def monarch_attn(q, k, v, b1, b2, tiles=1, iters=1, half_steps=None, factors=False,
                 nthreads=0, lib=None):
    """Forward pass on float64 arrays [..., N, d].  Returns y (and L, R if factors)."""
    qh, shape = _heads(q)
    kh, _ = _heads(k)
    vh, _ = _heads(v)
    BH, N, d = qh.shape
    hs = 2 * iters if half_steps is None else half_steps
    y = np.zeros_like(qh)
    L = np.zeros((BH, b2, b1, b1)) if factors else None
    R = np.zeros((BH, b1, tiles, b2, b2)) if factors else None
    rc = _load(lib).oracle_monarch_attn(_dptr(qh), _dptr(kh), _dptr(vh), _dptr(y), BH, N, d, b1,
                                     b2, tiles, hs, _dptr(L), _dptr(R), nthreads)
    if rc != 0:
        raise ValueError("oracle_monarch_attn failed with code %d" % rc)
    y = y.reshape(shape)
    if factors:
        return y, L.reshape(shape[:-2] + L.shape[1:]), R.reshape(shape[:-2] + R.shape[1:])
    return y


def monarch_attn_kv(q, k, v, b1, b1k, b2, tiles=1, iters=1, half_steps=None, factors=False,
                    nthreads=0, lib=None):
    """Queries [..., b1*b2, d] against keys and values [..., b1k*b2, d] (a chunk of
    frames attending to a cache that also holds earlier frames).  Returns y (and L
    [..., b2, b1, b1k], R [..., b1k, tiles, b2, b2] if factors)."""
    qh, shape = _heads(q)
    kh, _ = _heads(k)
    vh, _ = _heads(v)
    BH, Nq, d = qh.shape
    if Nq != b1 * b2 or kh.shape != (BH, b1k * b2, d) or vh.shape != kh.shape:
        raise ValueError("monarch_attn_kv: shapes do not match the blocks")
    hs = 2 * iters if half_steps is None else half_steps
    y = np.zeros_like(qh)
    L = np.zeros((BH, b2, b1, b1k)) if factors else None
    R = np.zeros((BH, b1k, tiles, b2, b2)) if factors else None
    rc = _load(lib).oracle_monarch_attn_kv(_dptr(qh), _dptr(kh), _dptr(vh), _dptr(y), BH, d, b1,
                                           b1k, b2, tiles, hs, _dptr(L), _dptr(R), nthreads)
    if rc != 0:
        raise ValueError("oracle_monarch_attn_kv failed with code %d" % rc)
    y = y.reshape(shape)
    if factors:
        return y, L.reshape(shape[:-2] + L.shape[1:]), R.reshape(shape[:-2] + R.shape[1:])
    return y


def monarch_attn_keytiles(q, k, v, b1, b2, tiles=1, iters=1, half_steps=None, factors=False,
                          probs=None, nthreads=0, lib=None, y=None):
    """The tiles split the key columns v' of every block (the other reading of the
    tiled parameterisation); float64 arrays [..., N, d], tiles in [1, b2].  Returns y
    (and L [..., b2, b1, tiles*b1] with super-key j = g'*b1 + u', R [..., b1, tiles,
    b2, b2] if factors).  With probs, a list of (bh, c) pairs, only the rows (u, c) of
    those problems are written (the rest of y is NaN, or taken from `y`)."""
    qh, shape = _heads(q)
    kh, _ = _heads(k)
    vh, _ = _heads(v)
    BH, N, d = qh.shape
    hs = 2 * iters if half_steps is None else half_steps
    if probs is None:
        pr, npr = None, -1
        out = np.zeros_like(qh)
    else:
        pr = np.ascontiguousarray(np.asarray(probs, dtype=np.int32).reshape(-1, 2))
        npr = pr.shape[0]
        out = np.full_like(qh, np.nan) if y is None else y.reshape(qh.shape)
    full = factors and probs is None
    L = np.zeros((BH, b2, b1, tiles * b1)) if full else None
    R = np.zeros((BH, b1, tiles, b2, b2)) if full else None
    rc = _load(lib).oracle_monarch_attn_keytiles(
        _dptr(qh), _dptr(kh), _dptr(vh), _dptr(out), BH, N, d, b1, b2, tiles, hs, _dptr(L),
        _dptr(R), npr, _iptr(pr) if pr is not None else None, nthreads)
    if rc != 0:
        raise ValueError("oracle_monarch_attn_keytiles failed with code %d" % rc)
    out = out.reshape(shape)
    if full:
        return out, L.reshape(shape[:-2] + L.shape[1:]), R.reshape(shape[:-2] + R.shape[1:])
    return out


def key_tile_cols(b2, tiles, g):
    """Key columns of key tile g: [floor(g*b2/t), floor((g+1)*b2/t))."""
    return np.arange((g * b2) // tiles, ((g + 1) * b2) // tiles)


def monarch_attn_bwd(q, k, v, dy, b1, b2, tiles=1, nthreads=0, lib=None):
    """Gradients (dq, dk, dv) of sum(dy * y) for one iteration of the forward pass
    (the chain rule through the output, the L-step, the R-step and the query
    aggregation); float64 arrays [..., N, d]."""
    qh, shape = _heads(q)
    kh, _ = _heads(k)
    vh, _ = _heads(v)
    dyh, _ = _heads(dy)
    BH, N, d = qh.shape
    dq, dk, dv = (np.zeros_like(qh) for _ in range(3))
    rc = _load(lib).oracle_monarch_attn_bwd(_dptr(qh), _dptr(kh), _dptr(vh), _dptr(dyh),
                                            _dptr(dq), _dptr(dk), _dptr(dv), BH, N, d, b1, b2,
                                            tiles, nthreads)
    if rc != 0:
        raise ValueError("oracle_monarch_attn_bwd failed with code %d" % rc)
    return dq.reshape(shape), dk.reshape(shape), dv.reshape(shape)


def monarch_problems(q, k, v, b1, b2, tiles, iters, probs, nthreads=0, y=None):
    """Selected (bh, g, c) problems; q, k, v float64 [BH, N, d].  Returns y [BH, N, d]
    with only the rows (u, c), u in tile g, of each listed problem written."""
    qh, _ = _heads(q)
    kh, _ = _heads(k)
    vh, _ = _heads(v)
    BH, N, d = qh.shape
    pr = np.ascontiguousarray(np.asarray(probs, dtype=np.int32).reshape(-1, 3))
    if y is None:
        y = np.full_like(qh, np.nan)
    rc = _load().oracle_monarch_problems(_dptr(qh), _dptr(kh), _dptr(vh), _dptr(y), BH, N, d,
                                         b1, b2, tiles, 2 * iters, pr.shape[0], _iptr(pr),
                                         nthreads)
    if rc != 0:
        raise ValueError("oracle_monarch_problems failed with code %d" % rc)
    return y


def tile_rows(b1, tiles, g):
    """Block rows of tile g (the floor partition, as the oracle's index maps give it)."""
    lo = index_maps(1, 1, b1, b1, 1, tiles)["tile_lo"]
    return np.arange(lo[g], lo[g + 1])
