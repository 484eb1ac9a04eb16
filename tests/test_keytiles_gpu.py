"""Key-column tiles (the tiles split the key columns v' of every block; each
query row's L runs over the b1*t (block, key tile) super-keys) on the GPU,
against the float64 oracle of that reading, element by element on seeded
inputs.  Tolerances as the other parity tests: relative Frobenius error
<= 1e-5 for float32 and <= 1e-2 for bfloat16 inputs."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import oracle  # noqa: E402
from structured_attention_video_b200 import _lib, synth  # noqa: E402
from structured_attention_video_b200.attention import (monarch_attention,  # noqa: E402
                                                       monarch_attention_tiled)

from helpers import TOL, device_inputs, from_torch, rel_fro, to_torch  # noqa: E402

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]


def run_keytiles(wl, q, k, v, layout="bhnd", **kw):
    args = dict(f=wl.f, h=wl.h, w=wl.w, b1=wl.b1, b2=wl.b2, tiles=wl.tiles, iters=wl.iters)
    args.update(kw)
    out = monarch_attention_tiled(q, k, v, axis="key_columns", layout=layout, **args)
    torch.cuda.synchronize()
    assert _lib.monarch_last_device_status(None) == 0
    return out


def dense_attention(q, k, v):
    s = q @ np.swapaxes(k, -1, -2) / np.sqrt(q.shape[-1])
    s -= s.max(-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(-1, keepdims=True)
    return p @ v


@pytest.fixture(scope="module")
def tiny64():
    return synth.make_inputs(TINY)


# (b1, b2, key tiles, iters): several and ragged key tiles (b2 = 8, 7, 24 and 16
# split into t uneven parts), one column per tile (exact attention), one tile
KEY_CASES = [(24, 8, 1, 1), (24, 8, 3, 1), (24, 8, 8, 1), (24, 8, 3, 2), (24, 8, 5, 3),
             (8, 24, 7, 1), (8, 24, 24, 2), (12, 16, 5, 2), (3, 64, 10, 1), (192, 1, 1, 1)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("b1,b2,tiles,iters", KEY_CASES)
def test_key_tiles_whole_output(tiny64, dtype, b1, b2, tiles, iters):
    q64, k64, v64 = (synth.round_to_dtype(x, dtype) for x in tiny64)
    ref = oracle.monarch_attn_keytiles(q64, k64, v64, b1, b2, tiles, iters)
    q, k, v = (to_torch(x, dtype) for x in (q64, k64, v64))
    got = from_torch(run_keytiles(TINY, q, k, v, b1=b1, b2=b2, tiles=tiles, iters=iters), dtype)
    assert np.isfinite(got).all()
    assert rel_fro(got, ref) <= TOL[dtype]


@pytest.mark.parametrize("d", [32, 64, 128])
def test_key_tiles_head_dims_and_odd_shapes(d):
    wl = TINY.replace(d=d, f=2, h=5, w=7, b1=10, b2=7, tiles=3, H=3)
    q64, k64, v64 = synth.make_inputs(wl)
    ref = oracle.monarch_attn_keytiles(q64, k64, v64, wl.b1, wl.b2, wl.tiles, 2)
    q, k, v = (to_torch(x, "f32") for x in (q64, k64, v64))
    got = from_torch(run_keytiles(wl, q, k, v, iters=2), "f32")
    assert rel_fro(got, ref) <= TOL["f32"]


def test_one_column_per_key_tile_is_exact_attention(tiny64):
    q64, k64, v64 = tiny64
    q, k, v = (to_torch(x, "f32") for x in tiny64)
    got = from_torch(run_keytiles(TINY, q, k, v, tiles=TINY.b2, iters=2), "f32")
    assert rel_fro(got, dense_attention(q64, k64, v64)) <= TOL["f32"]


def test_one_key_tile_is_the_query_tile_path_bit_for_bit(tiny64):
    """t = 1 is one tile on either axis: the generic kernels take the same
    arithmetic in the same order."""
    q, k, v = (to_torch(x, "f32") for x in tiny64)
    a = run_keytiles(TINY, q, k, v, tiles=1, iters=2)
    b = monarch_attention(q, k, v, f=TINY.f, h=TINY.h, w=TINY.w, b1=TINY.b1, b2=TINY.b2,
                          tiles=1, iters=2)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_key_tiles_bnhd_layout_matches_bhnd_bit_for_bit(dtype):
    wl = TINY.replace(B=2, H=3, d=64)
    q64, k64, v64 = (synth.round_to_dtype(x, dtype) for x in synth.make_inputs(wl))
    q, k, v = (to_torch(x, dtype) for x in (q64, k64, v64))
    ref = run_keytiles(wl, q, k, v, tiles=3, iters=2)
    qt, kt, vt = (x.transpose(1, 2).contiguous() for x in (q, k, v))
    out = run_keytiles(wl, qt, kt, vt, layout="bnhd", tiles=3, iters=2)
    assert torch.equal(out.transpose(1, 2), ref)
    want = oracle.monarch_attn_keytiles(q64, k64, v64, wl.b1, wl.b2, 3, 2)
    assert rel_fro(from_torch(ref, dtype), want) <= TOL[dtype]


def test_chunk_480p_key_tiles_whole_output():
    """The 480p chunk shape (B=1 H=12 d=128, N=4680, blocks (90, 52)) with four key
    tiles of 13 columns, bfloat16, every output row against the oracle."""
    wl = synth.WORKLOADS["480p_chunk"].replace(tiles=4)
    q, k, v = device_inputs(wl)
    assert _lib.monarch_attn_tiled_path(wl.B, wl.H, wl.f, wl.h, wl.w, wl.d, wl.b1, wl.b2, 4, 1,
                                        _lib.BF16, _lib.TILE_KEY_COLUMNS) == 1
    got = from_torch(run_keytiles(wl, q, k, v), wl.dtype)[0]
    q64, k64, v64 = synth.make_inputs(wl)
    ref = oracle.monarch_attn_keytiles(q64[0], k64[0], v64[0], wl.b1, wl.b2, 4, 1)
    assert np.isfinite(got).all()
    assert rel_fro(got, ref) <= TOL["bf16"]


def test_full_720p_key_tiles_sampled():
    """The 720p clip (B=1 H=12 d=128, N=75600, blocks (945, 80)) with four key
    tiles of 20 columns: sampled (head, column) problems, every query row of each,
    against the oracle; every output row is finite and a convex combination of
    value rows (inside the values' per-dimension range)."""
    wl = synth.WORKLOADS["720p"]
    q, k, v = device_inputs(wl)
    assert _lib.monarch_attn_tiled_path(wl.B, wl.H, wl.f, wl.h, wl.w, wl.d, wl.b1, wl.b2, 4, 1,
                                        _lib.BF16, _lib.TILE_KEY_COLUMNS) == 1
    out = run_keytiles(wl, q, k, v, tiles=4)
    rng = np.random.default_rng(3)
    probs = sorted({(0, 0), (wl.H - 1, wl.b2 - 1)} |
                   {(int(rng.integers(wl.H)), int(rng.integers(wl.b2))) for _ in range(22)})
    pos = synth.positional_code(wl.f, wl.h, wl.w, wl.d)
    got_rows, ref_rows = [], []
    for bh in sorted({p[0] for p in probs}):
        x = synth.make_head(wl, 0, bh, 0, pos)
        cols = [c for (hh, c) in probs if hh == bh]
        y = oracle.monarch_attn_keytiles(x["q"][None], x["k"][None], x["v"][None], wl.b1, wl.b2,
                                         4, 1, probs=[(0, c) for c in cols])[0]
        for c in cols:
            rows = np.arange(wl.b1) * wl.b2 + c
            got_rows.append(from_torch(out[0, bh, rows], wl.dtype))
            ref_rows.append(y[rows])
    assert rel_fro(np.concatenate(got_rows), np.concatenate(ref_rows)) <= TOL["bf16"]
    o = out.float()
    assert torch.isfinite(o).all()
    vf = v.float()
    lo, hi = vf.amin(dim=2, keepdim=True), vf.amax(dim=2, keepdim=True)
    tol = 1e-2 * (hi - lo)
    assert bool(((o >= lo - tol) & (o <= hi + tol)).all())


# bfloat16, d = 128 shapes on the tensor-core kernels: slabs that need padding
# rows (b1 = 24, 65, 129), several q̄ tiles (t*b2 > 128), one column per tile,
# ragged query pairs, two batches
TC_KEY_CASES = [(1, 3, 3, 8, 8, 24, 3), (2, 2, 5, 13, 8, 65, 8), (1, 2, 3, 43, 48, 129, 5),
                (1, 2, 3, 43, 48, 129, 7), (1, 3, 7, 16, 20, 112, 20)]


@pytest.mark.parametrize("B,H,f,h,w,b1,tiles", TC_KEY_CASES)
def test_key_tiles_tensor_core_whole_output(B, H, f, h, w, b1, tiles):
    b2 = f * h * w // b1
    wl = TINY.replace(B=B, H=H, d=128, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles, iters=1,
                      dtype="bf16")
    assert _lib.monarch_attn_tiled_path(B, H, f, h, w, 128, b1, b2, tiles, 1, _lib.BF16,
                                        _lib.TILE_KEY_COLUMNS) == 1
    q64, k64, v64 = (synth.round_to_dtype(x, "bf16") for x in synth.make_inputs(wl))
    q, k, v = (to_torch(x, "bf16") for x in (q64, k64, v64))
    got = from_torch(run_keytiles(wl, q, k, v), "bf16")
    ref = oracle.monarch_attn_keytiles(q64, k64, v64, b1, b2, tiles, 1)
    assert np.isfinite(got).all()
    assert rel_fro(got, ref) <= TOL["bf16"]


def test_chunk_480p_key_tiles_two_iterations_whole_output():
    """Later iterations with key-column tiles run on the generic kernels: the 480p
    chunk with four key tiles and two iterations, every output row against the
    oracle."""
    wl = synth.WORKLOADS["480p_chunk"].replace(tiles=4, iters=2)
    assert _lib.monarch_attn_tiled_path(wl.B, wl.H, wl.f, wl.h, wl.w, wl.d, wl.b1, wl.b2, 4, 2,
                                        _lib.BF16, _lib.TILE_KEY_COLUMNS) == 0
    q, k, v = device_inputs(wl)
    got = from_torch(run_keytiles(wl, q, k, v), wl.dtype)[0]
    q64, k64, v64 = synth.make_inputs(wl)
    ref = oracle.monarch_attn_keytiles(q64[0], k64[0], v64[0], wl.b1, wl.b2, 4, 2)
    assert np.isfinite(got).all()
    assert rel_fro(got, ref) <= TOL["bf16"]
