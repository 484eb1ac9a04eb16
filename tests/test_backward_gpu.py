"""Backward pass on the GPU (generic float32 kernels) against the float64 oracle's
backward, gradient by gradient, on seeded inputs rounded to the dtype.

Tolerances as for the forward: relative Frobenius error <= 1e-5 for float32 and
<= 1e-2 for bfloat16 (the gradients are stored in bfloat16)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import oracle  # noqa: E402
from structured_attention_video_b200 import _lib, synth  # noqa: E402
from structured_attention_video_b200.attention import monarch_attention_backward  # noqa: E402

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
