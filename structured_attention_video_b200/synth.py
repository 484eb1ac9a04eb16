"""Seeded synthetic video-attention inputs and the workload table.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It holds shapes, random numbers and the synthetic data recipe
only: nothing of the Monarch attention arithmetic lives here.

Random numbers
    A counter-based SplitMix64 stream (Steele, Lea and Flood, "Fast splittable
    pseudorandom number generators", OOPSLA 2014; the 64-bit finaliser of
    Vigna's public-domain splitmix64) feeds the Box-Muller transform (Box and
    Muller, 1958).  Element i of a stream with key K is mix(K + (i + 1) * GAMMA),
    so any element can be produced independently and in any order.  The
    streams and the bfloat16 rounding run in synth_gen.c (OpenMP).

Data recipe (MonarchRT, "Block alignment" and "Tiled Monarch" sections of the
explainer page; the (f, h, w) video layout with N = f*h*w tokens)
    * Tokens are ordered (frame, row, column) row-major: n = (fi*h + hi)*w + wi.
    * A sinusoidal positional code p(fi, hi, wi) in R^d splits d into three axis
      groups (f, h, w) of sizes g, g, d - 2g with g = floor(d/3) rounded down to
      even; inside a group of n pairs, p[2j] = sin(omega_j * pos) and
      p[2j+1] = cos(omega_j * pos) with omega_j = 10000^(-j/n).
    * "tiny" workloads: Q, K, V = z + 1.0 * p with z ~ N(0, 1) i.i.d.
    * "wan" workloads: Q, K = z + A * p with A = sqrt(6 / sqrt(d)) (a
      same-position logit about 3 sigma above the noise at scale 1/sqrt(d)),
      V = z / sqrt(d); then 8 planted query-key pairs per (b, h) in different
      frames and more than 2 tokens apart in h and w, each receiving +beta*e on
      the query and the key (e a random unit vector, beta = sqrt(4 * sqrt(d)),
      a +4 sigma logit boost at scale 1/sqrt(d)).
    * Values are generated in float64 and rounded once, round-to-nearest-even,
      to the working dtype (float32 or bfloat16).  The rounded values are
      exactly representable in float64, which is what the oracle consumes.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
import subprocess

import numpy as np

GAMMA = 0x9E3779B97F4A7C15

TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "pairs": 4}


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    f: int
    h: int
    w: int
    b1: int
    b2: int
    tiles: int
    iters: int
    dtype: str          # "f32" or "bf16"
    seed: int
    kind: str           # "tiny" or "wan"

    @property
    def N(self) -> int:
        return self.f * self.h * self.w

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def monarch_flops(self) -> float:
        """Algorithmic FLOPs of the forward pass (multiply-add = 2): the work the
        method needs, not what a given kernel schedule issues.

        Per (b, h): every iteration's R-step takes the logits of the aggregated
        queries against each key block and Ktil = R K (2 + 2 = 4*t*N*b2*d); the
        last one also forms Z = R V (2*t*N*b2*d more).  Every iteration's L-step
        takes the logits q.Ktil (2*N*b1*d) and then either re-aggregates the
        queries with L (iterations before the last) or forms Y = L Z (the last),
        2*N*b1*d either way.  Total (4T + 2)*t*N*b2*d + 4T*N*b1*d.
        """
        T, t, N = self.iters, self.tiles, self.N
        per_head = (4 * T + 2) * t * N * self.b2 * self.d + 4 * T * N * self.b1 * self.d
        return float(self.B * self.H * per_head)

    def monarch_flops_keytiles(self) -> float:
        """Algorithmic FLOPs of the forward pass with key-column tiles (the tiles
        split the key columns of every block; multiply-add = 2).

        Per (b, h): every iteration's R-step takes, for each block and column, the
        logits of the aggregated query against its key tile's columns only (all t
        tiles together: 2*N*b2*d) and Ktil = R K (2*N*b2*d); the last one also
        forms Z = R V (2*N*b2*d).  Every iteration's L-step takes the logits of
        each query against the t*b1 super-keys (2*t*N*b1*d) and then forms Y = L Z
        or re-aggregates the queries (2*t*N*b1*d).  Total
        (4T + 2)*N*b2*d + 4T*t*N*b1*d.
        """
        T, t, N = self.iters, self.tiles, self.N
        per_head = (4 * T + 2) * N * self.b2 * self.d + 4 * T * t * N * self.b1 * self.d
        return float(self.B * self.H * per_head)

    def backward_flops(self) -> float:
        """Algorithmic FLOPs of the backward pass of one iteration (multiply-add =
        2), without recomputing the forward's R-step.

        Per (b, h): the L-step side takes the logits again, dL = dY Z^T, dq = dB
        Ktil, dKtil = dB^T Q and dZ = L^T dY (5 x 2*N*b1*d); the R-step side
        takes its logits again, dR = dKtil k + dZ v (two products), dqbar = dA k,
        dk = dA qbar + R^T dKtil (two) and dv = R^T dZ (7 x 2*t*N*b2*d).
        """
        return float(self.B * self.H * (10 * self.N * self.b1 + 14 * self.tiles * self.N * self.b2)
                     * self.d)

    def dense_flops(self) -> float:
        """FLOPs of exact softmax attention on the same shape (4*N^2*d per head)."""
        return float(4 * self.B * self.H * self.N * self.N * self.d)

    def io_bytes(self) -> int:
        """Q, K, V read once and O written once, in the working dtype."""
        es = 2 if self.dtype == "bf16" else 4
        return 4 * self.B * self.H * self.N * self.d * es


WORKLOADS = {
    # tiny oracle case; b1 = 1 and b2 = 1 variants are derived in the tests
    "tiny": Workload("tiny", 1, 2, 32, 3, 8, 8, 24, 8, 1, 1, "f32", 0, "tiny"),
    # Wan-1.3B-shaped single chunk at 480p
    "480p_chunk": Workload("480p_chunk", 1, 12, 128, 3, 30, 52, 90, 52, 1, 1, "bf16", 1, "wan"),
    # Wan-1.3B full clip at 480p (tiles swept over 1, 2, 4, 8)
    "480p_full": Workload("480p_full", 1, 12, 128, 21, 30, 52, 630, 52, 1, 1, "bf16", 2, "wan"),
    # 720p clip: the headline throughput shape
    "720p": Workload("720p", 1, 12, 128, 21, 45, 80, 945, 80, 4, 1, "bf16", 3, "wan"),
    # Wan-14B-shaped stress case (iters swept over 1, 2, 5, 10)
    "14b": Workload("14b", 2, 40, 128, 21, 30, 52, 630, 52, 2, 1, "bf16", 4, "wan"),
}


# ----------------------------------------------------------------------------
# counter-based generator (synth_gen.c, built on first use with gcc + OpenMP)
# ----------------------------------------------------------------------------
_HERE = os.path.dirname(os.path.abspath(__file__))
_GEN_SRC = os.path.join(_HERE, "synth_gen.c")
_GEN_LIB = os.path.join(_HERE, "_build", "libsynth.so")
_gen = None


def build_generator(force: bool = False) -> str:
    if force or not os.path.exists(_GEN_LIB) or \
            os.path.getmtime(_GEN_LIB) < os.path.getmtime(_GEN_SRC):
        os.makedirs(os.path.dirname(_GEN_LIB), exist_ok=True)
        tmp = _GEN_LIB + ".tmp%d" % os.getpid()
        subprocess.run(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", _GEN_SRC,
                        "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _GEN_LIB)
    return _GEN_LIB


def _lib():
    global _gen
    if _gen is None:
        lib = ctypes.CDLL(build_generator())
        u64, i64 = ctypes.c_uint64, ctypes.c_int64
        dp = ctypes.POINTER(ctypes.c_double)
        lib.synth_mix64.argtypes = [u64]
        lib.synth_mix64.restype = u64
        lib.synth_uniform53.argtypes = [u64, i64, i64, dp]
        lib.synth_normals.argtypes = [u64, i64, dp]
        lib.synth_round_bf16.argtypes = [dp, i64, dp, ctypes.POINTER(ctypes.c_uint16)]
        _gen = lib
    return _gen


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def stream_key(seed: int, b: int, h: int, tensor: str, rank: int = 0) -> int:
    """Key of the stream for (seed, rank, b, h, tensor): a SplitMix64 mix of the fields."""
    x = seed & 0xFFFFFFFF
    for field in (rank, b, h, TENSOR_IDS[tensor]):
        x = _lib().synth_mix64((x + GAMMA * (field + 1)) & 0xFFFFFFFFFFFFFFFF)
    return x


def uniform53(key: int, start: int, count: int) -> np.ndarray:
    """Elements [start, start+count) of stream `key` as doubles in (0, 1]."""
    out = np.empty(count, dtype=np.float64)
    _lib().synth_uniform53(key, start, count, _dp(out))
    return out


def normals(key: int, count: int) -> np.ndarray:
    """`count` standard normals from stream `key` (Box-Muller on consecutive pairs)."""
    out = np.empty(count, dtype=np.float64)
    _lib().synth_normals(key, count, _dp(out))
    return out


# ----------------------------------------------------------------------------
# rounding to the working dtype
# ----------------------------------------------------------------------------
def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values once, to nearest even, to float32 or bfloat16; return float64."""
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype != "bf16":
        raise ValueError(dtype)
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    _lib().synth_round_bf16(_dp(x), x.size, _dp(out), None)
    return out


def to_device_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Pack already-rounded float64 values into the dtype's storage (float32 or bf16 bits as uint16)."""
    f = x.astype(np.float32)
    if dtype == "f32":
        return f
    return (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def from_device_bits(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 values of a float32 array or of bf16 bits stored as uint16."""
    if dtype == "f32":
        return a.astype(np.float64)
    return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# the recipe
# ----------------------------------------------------------------------------
def positional_code(f: int, h: int, w: int, d: int) -> np.ndarray:
    """Sinusoidal code over (frame, row, column): shape [f*h*w, d], float64."""
    g = (d // 3) & ~1
    sizes = (g, g, d - 2 * g)
    fi, hi, wi = np.meshgrid(np.arange(f), np.arange(h), np.arange(w), indexing="ij")
    pos = (fi.reshape(-1), hi.reshape(-1), wi.reshape(-1))
    cols = []
    for size, p in zip(sizes, pos):
        n = size // 2
        j = np.arange(n, dtype=np.float64)
        omega = 10000.0 ** (-j / max(n, 1))
        ang = p[:, None].astype(np.float64) * omega[None, :]
        blk = np.empty((p.shape[0], 2 * n), dtype=np.float64)
        blk[:, 0::2] = np.sin(ang)
        blk[:, 1::2] = np.cos(ang)
        if size > 2 * n:                   # odd group size: pad with a zero column
            blk = np.concatenate([blk, np.zeros((p.shape[0], size - 2 * n))], axis=1)
        cols.append(blk)
    return np.concatenate(cols, axis=1)


def planted_pairs(wl: Workload, b: int, h: int, rank: int = 0, npairs: int = 8):
    """The (query token, key token, unit direction) triples planted into one head."""
    key = stream_key(wl.seed, b, h, "pairs", rank)
    f, hh, ww, N = wl.f, wl.h, wl.w, wl.N
    pairs = []
    pos = 0
    while len(pairs) < npairs and pos < 1 << 20:
        u = uniform53(key, pos, 2)
        pos += 2
        i = min(int(u[0] * N), N - 1)
        j = min(int(u[1] * N), N - 1)
        fi, hi, wi = i // (hh * ww), (i // ww) % hh, i % ww
        fj, hj, wj = j // (hh * ww), (j // ww) % hh, j % ww
        if fi != fj and abs(hi - hj) > 2 and abs(wi - wj) > 2:
            pairs.append((i, j))
    dkey = stream_key(wl.seed, b, h, "pairs", rank + 7919)
    dirs = normals(dkey, npairs * wl.d).reshape(npairs, wl.d)
    dirs /= np.linalg.norm(dirs, axis=1, keepdims=True)
    return [(i, j, dirs[t]) for t, (i, j) in enumerate(pairs)]


def make_head(wl: Workload, b: int, h: int, rank: int = 0, pos_code: np.ndarray | None = None):
    """Q, K, V of one (b, h) as float64 [N, d] arrays, already rounded to wl.dtype."""
    N, d = wl.N, wl.d
    p = positional_code(wl.f, wl.h, wl.w, d) if pos_code is None else pos_code
    out = {}
    for name in ("q", "k", "v"):
        z = normals(stream_key(wl.seed, b, h, name, rank), N * d).reshape(N, d)
        if wl.kind == "tiny":
            x = z + p
        elif name == "v":
            x = z / math.sqrt(d)
        else:
            x = z + math.sqrt(6.0 / math.sqrt(d)) * p
        out[name] = x
    if wl.kind == "wan":
        beta = math.sqrt(4.0 * math.sqrt(d))
        for i, j, e in planted_pairs(wl, b, h, rank):
            out["q"][i] += beta * e
            out["k"][j] += beta * e
    return {name: round_to_dtype(x, wl.dtype) for name, x in out.items()}


def make_inputs(wl: Workload, rank: int = 0):
    """Q, K, V for all heads as float64 arrays [B, H, N, d] (rounded to wl.dtype)."""
    p = positional_code(wl.f, wl.h, wl.w, wl.d)
    shape = (wl.B, wl.H, wl.N, wl.d)
    q, k, v = (np.empty(shape) for _ in range(3))
    for b in range(wl.B):
        for h in range(wl.H):
            x = make_head(wl, b, h, rank, p)
            q[b, h], k[b, h], v[b, h] = x["q"], x["k"], x["v"]
    return q, k, v


def fill_device_bits(wl: Workload, q_out: np.ndarray, k_out: np.ndarray, v_out: np.ndarray,
                     rank: int = 0) -> None:
    """Write Q, K, V in storage format straight into caller arrays [B, H, N, d] (head by head)."""
    p = positional_code(wl.f, wl.h, wl.w, wl.d)
    for b in range(wl.B):
        for h in range(wl.H):
            x = make_head(wl, b, h, rank, p)
            q_out[b, h] = to_device_bits(x["q"], wl.dtype)
            k_out[b, h] = to_device_bits(x["k"], wl.dtype)
            v_out[b, h] = to_device_bits(x["v"], wl.dtype)
