"""Backward pass on the GPU against the float64 oracle's backward, gradient by
gradient, on seeded inputs rounded to the dtype.  bfloat16 with d = 128 takes the
tensor-core kernels for the L-step side (the forward's tensor-core intermediates,
then dKtil, dZ, dH and dq by tcgen05 products); everything else, and the R-step
side, runs on the generic float32 kernels.

Tolerances as for the forward: relative Frobenius error <= 1e-5 for float32 and
<= 1e-2 for bfloat16 (the gradients are stored in bfloat16)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import oracle  # noqa: E402
from structured_attention_video_b200 import _lib, synth  # noqa: E402
from structured_attention_video_b200.attention import (kernel_path,  # noqa: E402
                                                       monarch_attention_backward)

from helpers import TOL, from_torch, rel_fro, to_torch  # noqa: E402

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]

CASES = [  # f, h, w, b1, b2, tiles, d
    (3, 8, 8, 24, 8, 1, 32),
    (3, 8, 8, 24, 8, 5, 64),      # five ragged tiles
    (3, 8, 8, 24, 8, 24, 32),     # one block row per tile
    (1, 1, 192, 1, 192, 1, 64),   # b1 = 1: one L block, 192 keys in six chunks
    (3, 8, 8, 192, 1, 7, 32),     # b2 = 1
    (2, 5, 7, 10, 7, 3, 128),     # odd sizes, d = 128
    (2, 50, 7, 100, 7, 2, 128),   # 100 keys per row: four chunks of the key blocks
]


def run_case(f, h, w, b1, b2, tiles, d, dtype, H=2, seed=0):
    wl = TINY.replace(H=H, d=d, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles)
    q64, k64, v64 = (synth.round_to_dtype(x, dtype) for x in synth.make_inputs(wl))
    rng = np.random.default_rng(seed)
    dy64 = synth.round_to_dtype(rng.standard_normal(q64.shape), dtype)
    ref = oracle.monarch_attn_bwd(q64, k64, v64, dy64, b1, b2, tiles)
    q, k, v, dy = (to_torch(x, dtype) for x in (q64, k64, v64, dy64))
    got = monarch_attention_backward(q, k, v, dy, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles)
    torch.cuda.synchronize()
    assert _lib.monarch_last_device_status(None) == 0
    return [from_torch(g, dtype) for g in got], ref


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("f,h,w,b1,b2,tiles,d", CASES)
def test_backward_matches_the_oracle(dtype, f, h, w, b1, b2, tiles, d):
    got, ref = run_case(f, h, w, b1, b2, tiles, d, dtype)
    for name, g, r in zip("qkv", got, ref):
        assert np.isfinite(g).all(), name
        assert rel_fro(g, r) <= TOL[dtype], name


def test_backward_480p_chunk():
    """The 480p chunk shape of the forward benchmarks (B=1, H=12, N=4680, d=128,
    blocks (90, 52)), bfloat16."""
    wl = synth.WORKLOADS["480p_chunk"]
    got, ref = run_case(wl.f, wl.h, wl.w, wl.b1, wl.b2, wl.tiles, wl.d, "bf16", H=wl.H)
    for name, g, r in zip("qkv", got, ref):
        assert rel_fro(g, r) <= TOL["bf16"], name


def test_backward_is_deterministic():
    wl = TINY.replace(H=2, d=64, f=3, h=8, w=8, b1=24, b2=8, tiles=5)
    q, k, v, dy = (to_torch(x, "f32") for x in
                   list(synth.make_inputs(wl)) + [np.ones((1, 2, 192, 64))])
    a = monarch_attention_backward(q, k, v, dy, f=3, h=8, w=8, b1=24, b2=8, tiles=5)
    b = monarch_attention_backward(q, k, v, dy, f=3, h=8, w=8, b1=24, b2=8, tiles=5)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_backward_refuses_more_than_one_iteration():
    q = torch.zeros(1, 1, 192, 32, device="cuda")
    with pytest.raises(_lib.MonarchError):
        monarch_attention_backward(q, q, q, q, f=3, h=8, w=8, b1=24, b2=8, tiles=1, iters=2)


# bfloat16, d = 128 shapes on the tensor-core L-step side: several 128-query tiles
# and 128-key blocks with ragged last ones, tiles of unequal length (the shorter
# tile has no second query tile), one block row (b1 = 1), two batches
TC_CASES = [  # B, H, f, h, w, b1, b2, tiles
    (1, 2, 3, 100, 4, 300, 4, 1),     # 300 queries and keys: 3 tiles and 3 key blocks (44 left)
    (1, 2, 1, 257, 8, 257, 8, 2),     # tiles of 128 and 129 rows
    (2, 1, 5, 13, 8, 65, 8, 3),       # two batches, 65 keys
    (1, 2, 1, 1, 128, 1, 128, 1),     # b1 = 1: one key per row
    (1, 2, 3, 43, 48, 129, 48, 5),    # 129 keys, five tiles of 25-26 rows
]


@pytest.mark.parametrize("B,H,f,h,w,b1,b2,tiles", TC_CASES)
def test_backward_tensor_core_lstep_side(B, H, f, h, w, b1, b2, tiles):
    wl = TINY.replace(B=B, H=H, d=128, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles, dtype="bf16")
    q64, k64, v64 = (synth.round_to_dtype(x, "bf16") for x in synth.make_inputs(wl))
    rng = np.random.default_rng(4)
    dy64 = synth.round_to_dtype(rng.standard_normal(q64.shape), "bf16")
    ref = oracle.monarch_attn_bwd(q64, k64, v64, dy64, b1, b2, tiles)
    q, k, v, dy = (to_torch(x, "bf16") for x in (q64, k64, v64, dy64))
    assert kernel_path(q, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles) == 1
    got = monarch_attention_backward(q, k, v, dy, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles)
    torch.cuda.synchronize()
    assert _lib.monarch_last_device_status(None) == 0
    for name, g, r in zip("qkv", got, ref):
        g = from_torch(g, "bf16")
        assert np.isfinite(g).all(), name
        assert rel_fro(g, r) <= TOL["bf16"], name


def test_backward_tensor_core_path_is_deterministic():
    wl = TINY.replace(H=2, d=128, f=1, h=257, w=8, b1=257, b2=8, tiles=2, dtype="bf16")
    q64, k64, v64 = (synth.round_to_dtype(x, "bf16") for x in synth.make_inputs(wl))
    dy64 = synth.round_to_dtype(np.random.default_rng(1).standard_normal(q64.shape), "bf16")
    q, k, v, dy = (to_torch(x, "bf16") for x in (q64, k64, v64, dy64))
    a = monarch_attention_backward(q, k, v, dy, f=1, h=257, w=8, b1=257, b2=8, tiles=2)
    b = monarch_attention_backward(q, k, v, dy, f=1, h=257, w=8, b1=257, b2=8, tiles=2)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
