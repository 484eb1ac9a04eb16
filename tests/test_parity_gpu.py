"""CUDA path against the float64 oracle, element by element on seeded inputs.

Tolerances: relative Frobenius error <= 1e-5 for float32 inputs and <= 1e-2 for
bfloat16 inputs (float32 accumulation); index maps bit-exact.  Small shapes
compare the whole output, and so does the 720p clip of the benchmark (every
head, tile and column, the oracle solving them one by one); the other full-size
shapes compare sampled (head, tile, column) problems plus properties that hold
at any size (every output row is a convex combination of value rows)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import oracle  # noqa: E402
from structured_attention_video_b200 import _lib, synth  # noqa: E402
from structured_attention_video_b200.attention import kernel_path, monarch_attention  # noqa: E402

from helpers import (TOL, device_inputs, from_torch, oracle_on_samples, rel_fro,  # noqa: E402
                     sample_problems, sampled_error, to_torch)

pytestmark = pytest.mark.gpu

TINY = synth.WORKLOADS["tiny"]


def dense_attention(q, k, v):
    s = q @ np.swapaxes(k, -1, -2) / np.sqrt(q.shape[-1])
    s -= s.max(-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(-1, keepdims=True)
    return p @ v


def run(wl, q, k, v, **kw):
    args = dict(f=wl.f, h=wl.h, w=wl.w, b1=wl.b1, b2=wl.b2, tiles=wl.tiles, iters=wl.iters)
    args.update(kw)
    out = monarch_attention(q, k, v, **args)
    torch.cuda.synchronize()
    assert _lib.monarch_last_device_status(None) == 0
    return out


@pytest.fixture(scope="module")
def tiny64():
    return synth.make_inputs(TINY)


# --------------------------------------------------------------------------
# whole-output parity on small shapes (several tiles, ragged tails)
# --------------------------------------------------------------------------
SMALL = [(24, 8, 1, 1), (24, 8, 5, 1), (24, 8, 24, 1), (24, 8, 5, 2), (24, 8, 3, 3),
         (1, 192, 1, 1), (192, 1, 1, 1), (192, 1, 7, 2), (3, 64, 2, 1), (8, 24, 3, 2),
         (12, 16, 5, 1)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("b1,b2,tiles,iters", SMALL)
def test_tiny_whole_output(tiny64, dtype, b1, b2, tiles, iters):
    q64, k64, v64 = (synth.round_to_dtype(x, dtype) for x in tiny64)
    ref = oracle.monarch_attn(q64, k64, v64, b1, b2, tiles, iters)
    q, k, v = (to_torch(x, dtype) for x in (q64, k64, v64))
    out = run(TINY, q, k, v, b1=b1, b2=b2, tiles=tiles, iters=iters)
    got = from_torch(out, dtype)
    assert np.isfinite(got).all()
    assert rel_fro(got, ref) <= TOL[dtype]


@pytest.mark.parametrize("d", [32, 64, 128])
def test_head_dims_and_odd_shapes_f32(d):
    wl = TINY.replace(d=d, f=2, h=5, w=7, b1=10, b2=7, tiles=3, H=3)
    q64, k64, v64 = synth.make_inputs(wl)
    ref = oracle.monarch_attn(q64, k64, v64, wl.b1, wl.b2, wl.tiles, 2)
    q, k, v = (to_torch(x, "f32") for x in (q64, k64, v64))
    got = from_torch(run(wl, q, k, v, iters=2), "f32")
    assert rel_fro(got, ref) <= TOL["f32"]


def test_single_token_is_identity_on_v():
    wl = TINY.replace(f=1, h=1, w=1, b1=1, b2=1, H=1)
    q64, k64, v64 = synth.make_inputs(wl)
    q, k, v = (to_torch(x, "f32") for x in (q64, k64, v64))
    got = from_torch(run(wl, q, k, v), "f32")
    assert np.array_equal(got, v64)


def test_zero_queries_give_mean_of_v(tiny64):
    _, k64, v64 = tiny64
    q = torch.zeros(to_torch(k64, "f32").shape, device="cuda")
    k, v = to_torch(k64, "f32"), to_torch(v64, "f32")
    got = from_torch(run(TINY, q, k, v, tiles=5, iters=2), "f32")
    assert np.abs(got - v64.mean(-2, keepdims=True)).max() < 1e-5


# tensor-core kernels at the edges of their dispatch range (bf16, d = 128, one
# iteration), whole output against the oracle
TC_EDGES = [
    # f, h, w, b1, b2, tiles
    (1, 64, 1, 64, 1, 2),        # b2 = 1: every R block is 1 x 1
    (1, 1, 128, 1, 128, 1),      # b1 = 1: a single L block (exact attention); b2 padded to 128
    (2, 3, 100, 6, 100, 2),      # b2 padded to 112, two 128-row qbar tiles
    (3, 4, 16, 12, 16, 12),      # one query row per tile (t = b1)
    (2, 100, 7, 200, 7, 3),      # b2 padded to 16; ragged last key chunk (200 = 128 + 72)
    (5, 60, 48, 300, 48, 5),     # 60 rows per tile: the second query tile of a pair is empty
    (10, 100, 16, 1000, 16, 1),  # 1000 query rows per tile: four pairs of query tiles
    (1, 65, 4, 65, 4, 2),        # 65 keys: a second 64-key half with one valid key
    (1, 129, 8, 129, 8, 3),      # 129 keys: the last 128-key chunk has a single half
    # packed R-step tiles (t*b2 <= 64: two or four blocks per 128-row tile), with a
    # head's last group of blocks only partly inside the head
    (1, 9, 16, 9, 16, 1),        # 16 rows: four blocks per tile, 9 blocks = 4 + 4 + 1
    (1, 7, 52, 7, 52, 1),        # 52 rows: two blocks per tile, 7 blocks = 2 + 2 + 2 + 1
    (3, 5, 20, 15, 20, 3),       # 60 rows (three tiles of 20): two blocks per tile, 15 blocks
]


@pytest.mark.parametrize("f,h,w,b1,b2,tiles", TC_EDGES)
def test_tensor_core_edge_shapes(f, h, w, b1, b2, tiles):
    wl = TINY.replace(H=2, d=128, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles, iters=1)
    q64, k64, v64 = (synth.round_to_dtype(x, "bf16") for x in synth.make_inputs(wl))
    q, k, v = (to_torch(x, "bf16") for x in (q64, k64, v64))
    assert kernel_path(q, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles) == 1
    ref = oracle.monarch_attn(q64, k64, v64, b1, b2, tiles, 1)
    got = from_torch(run(wl, q, k, v), "bf16")
    assert np.isfinite(got).all()
    assert rel_fro(got, ref) <= TOL["bf16"]


TC_ITER_EDGES = [
    # f, h, w, b1, b2, tiles, iters
    (2, 3, 100, 6, 100, 2, 2),      # b2 padded to 112, two aggregated-query tiles per block
    (5, 60, 48, 300, 48, 5, 3),     # 60 queries per tile, three alternating rounds
    (10, 100, 16, 1000, 16, 1, 2),  # 1000 queries per tile: 8 query chunks in the aggregation
    (1, 64, 1, 64, 1, 2, 2),        # b2 = 1
    (3, 4, 16, 12, 16, 12, 2),      # one query row per tile (t = b1)
    (2, 100, 7, 200, 7, 3, 4),      # ragged chunks of 128 on both sides
]


@pytest.mark.parametrize("f,h,w,b1,b2,tiles,iters", TC_ITER_EDGES)
def test_tensor_core_iterations_whole_output(f, h, w, b1, b2, tiles, iters):
    """iters > 1 on the tensor cores: the L-step's row statistics, the re-aggregated
    queries (S4) and the R-step on per-block queries, against the oracle."""
    wl = TINY.replace(H=2, d=128, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles, iters=iters)
    q64, k64, v64 = (synth.round_to_dtype(x, "bf16") for x in synth.make_inputs(wl))
    q, k, v = (to_torch(x, "bf16") for x in (q64, k64, v64))
    assert kernel_path(q, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles, iters=iters) == 1
    ref = oracle.monarch_attn(q64, k64, v64, b1, b2, tiles, iters)
    got = from_torch(run(wl, q, k, v), "bf16")
    assert np.isfinite(got).all()
    assert rel_fro(got, ref) <= TOL["bf16"]


def test_chunk_480p_whole_output():
    wl = synth.WORKLOADS["480p_chunk"]
    q, k, v = device_inputs(wl)
    out = run(wl, q, k, v)
    q64, k64, v64 = (from_torch(x, wl.dtype) for x in (q, k, v))
    ref = oracle.monarch_attn(q64, k64, v64, wl.b1, wl.b2, wl.tiles, wl.iters)
    assert rel_fro(from_torch(out, wl.dtype), ref) <= TOL[wl.dtype]


def test_chunk_480p_one_block_is_exact_attention():
    """b1 = 1: a single R block of N x N, i.e. softmax attention (checked on 2 heads)."""
    wl = synth.WORKLOADS["480p_chunk"].replace(H=2, b1=1, b2=4680)
    q, k, v = device_inputs(wl)
    out = from_torch(run(wl, q, k, v), wl.dtype)
    q64, k64, v64 = (from_torch(x, wl.dtype) for x in (q, k, v))
    assert rel_fro(out, dense_attention(q64, k64, v64)) <= TOL[wl.dtype]


# --------------------------------------------------------------------------
# full-size shapes: sampled problems and size-independent properties
# --------------------------------------------------------------------------
def convex_hull_check(out, v):
    """Every output row is a convex combination of value rows of its head."""
    o = out.float()
    vf = v.float()
    lo = vf.amin(dim=2, keepdim=True)
    hi = vf.amax(dim=2, keepdim=True)
    slack = 1e-2 * (hi - lo) + 1e-6
    assert torch.isfinite(o).all()
    assert bool(((o >= lo - slack) & (o <= hi + slack)).all())


@pytest.fixture(scope="module")
def inputs_480p():
    return device_inputs(synth.WORKLOADS["480p_full"])


@pytest.mark.parametrize("tiles", [1, 2, 4, 8])
def test_full_480p_tile_sweep(inputs_480p, tiles):
    wl = synth.WORKLOADS["480p_full"].replace(tiles=tiles)
    q, k, v = inputs_480p
    assert kernel_path(q, f=wl.f, h=wl.h, w=wl.w, b1=wl.b1, b2=wl.b2, tiles=tiles) == 1
    out = run(wl, q, k, v)
    convex_hull_check(out, v)
    probs = sample_problems(wl, 12, seed=tiles)
    assert sampled_error(wl, out, probs) <= TOL[wl.dtype]


@pytest.fixture(scope="module")
def inputs_720p():
    return device_inputs(synth.WORKLOADS["720p"])


def test_full_720p_headline(inputs_720p):
    wl = synth.WORKLOADS["720p"]
    q, k, v = inputs_720p
    assert kernel_path(q, f=wl.f, h=wl.h, w=wl.w, b1=wl.b1, b2=wl.b2, tiles=wl.tiles) == 1
    out = run(wl, q, k, v)
    convex_hull_check(out, v)
    probs = sample_problems(wl, 24, seed=720)
    assert sampled_error(wl, out, probs) <= TOL[wl.dtype]


def test_full_720p_whole_output(inputs_720p):
    """Every output element of the 720p clip against the oracle: all heads x tiles x
    columns, head by head (the oracle regenerates each head from the seeded
    generator); the error bound holds for the whole output and for every head."""
    wl = synth.WORKLOADS["720p"]
    q, k, v = inputs_720p
    out = run(wl, q, k, v)
    probs = [(bh, g, c) for bh in range(wl.B * wl.H) for g in range(wl.tiles)
             for c in range(wl.b2)]
    ref = oracle_on_samples(wl, probs)
    num = den = 0.0
    for bh in range(wl.B * wl.H):
        b, h = divmod(bh, wl.H)
        got = from_torch(out[b, h], wl.dtype)
        assert not np.isnan(ref[bh]).any()
        e2 = float(np.sum((got - ref[bh]) ** 2))
        r2 = float(np.sum(ref[bh] ** 2))
        assert np.sqrt(e2 / r2) <= TOL[wl.dtype], bh
        num += e2
        den += r2
    assert np.sqrt(num / den) <= TOL[wl.dtype]


def test_full_720p_deterministic(inputs_720p):
    wl = synth.WORKLOADS["720p"]
    q, k, v = inputs_720p
    a = run(wl, q, k, v)
    b = run(wl, q, k, v)
    assert torch.equal(a, b)


@pytest.fixture(scope="module")
def inputs_14b():
    return device_inputs(synth.WORKLOADS["14b"])


@pytest.mark.parametrize("iters", [1, 2, 5, 10])
def test_full_14b_iteration_sweep(inputs_14b, iters):
    wl = synth.WORKLOADS["14b"].replace(iters=iters)
    q, k, v = inputs_14b
    assert kernel_path(q, f=wl.f, h=wl.h, w=wl.w, b1=wl.b1, b2=wl.b2, tiles=wl.tiles,
                       iters=iters) == 1
    out = run(wl, q, k, v)
    convex_hull_check(out, v)
    probs = sample_problems(wl, 64, seed=iters)
    assert sampled_error(wl, out, probs) <= TOL[wl.dtype]


# --------------------------------------------------------------------------
# entry points and maps
# --------------------------------------------------------------------------
@pytest.mark.parametrize("f,h,w,b1,b2,tiles", [(3, 8, 8, 24, 8, 5), (3, 8, 8, 192, 1, 192),
                                                (21, 45, 80, 945, 80, 4),
                                                (21, 30, 52, 630, 52, 8)])
def test_device_index_maps_bit_exact(f, h, w, b1, b2, tiles):
    N = f * h * w
    maps = [torch.full((N,), -1, dtype=torch.int32, device="cuda") for _ in range(3)]
    tb = torch.full((tiles + 1,), -1, dtype=torch.int32, device="cuda")
    st = _lib.monarch_index_maps_device(f, h, w, b1, b2, tiles, *(m.data_ptr() for m in maps),
                                        tb.data_ptr(), None)
    assert st == 0
    torch.cuda.synchronize()
    ref = oracle.index_maps(f, h, w, b1, b2, tiles)
    for m, key in zip(maps, ("u_of_n", "v_of_n", "perm")):
        assert np.array_equal(m.cpu().numpy(), ref[key])
    assert np.array_equal(tb.cpu().numpy(), ref["tile_lo"])


def test_entry_points_agree(tiny64):
    """monarch_attn_fwd (library workspace), _ws and _host give identical bits."""
    wl = TINY.replace(tiles=5, iters=2)
    q64, k64, v64 = tiny64
    q, k, v = (to_torch(x, "f32") for x in (q64, k64, v64))
    ref = run(wl, q, k, v)
    shape = (wl.B, wl.H, wl.f, wl.h, wl.w, wl.d, wl.b1, wl.b2, wl.tiles, wl.iters)
    out = torch.empty_like(q)
    assert _lib.monarch_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 *shape, _lib.F32, None) == 0
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
    oh = torch.empty_like(qh).pin_memory()
    assert _lib.monarch_attn_fwd_host(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), oh.data_ptr(),
                                      *shape, _lib.F32, None) == 0
    torch.cuda.synchronize()
    assert torch.equal(oh, ref.cpu())


@pytest.mark.parametrize("name,dtype,kw,cuts", [
    ("480p_chunk", "bf16", dict(H=4, tiles=3), (0, 5, 7, 12)),     # tensor-core path
    ("tiny", "f32", dict(tiles=5, iters=2), (0, 3, 4, 10)),         # generic path, iters > 1
])
def test_unit_ranges_partition_the_output(name, dtype, kw, cuts):
    """Calls over a partition of the (head, tile) units give the full call's output
    bit for bit, and a call writes no row outside its units."""
    wl = synth.WORKLOADS[name].replace(dtype=dtype, **kw)
    q64, k64, v64 = (synth.round_to_dtype(x, dtype) for x in synth.make_inputs(wl))
    q, k, v = (to_torch(x, dtype) for x in (q64, k64, v64))
    dt = _lib.F32 if dtype == "f32" else _lib.BF16
    shape = (wl.B, wl.H, wl.f, wl.h, wl.w, wl.d, wl.b1, wl.b2, wl.tiles, wl.iters)
    need = _lib.monarch_attn_workspace_bytes(*shape, dt)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    full = run(wl, q, k, v)
    assert cuts[-1] == wl.B * wl.H * wl.tiles
    parts = torch.full_like(q, float("nan"))
    for b, e in zip(cuts, cuts[1:]):
        one = torch.full_like(q, float("nan"))
        for out in (parts, one):
            assert _lib.monarch_attn_fwd_units_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                  out.data_ptr(), *shape, dt, b, e,
                                                  ws.data_ptr(), need, None) == 0
        torch.cuda.synchronize()
        mine = torch.zeros(q.shape[:3], dtype=torch.bool)
        for unit in range(b, e):
            bh, g = divmod(unit, wl.tiles)
            rows = oracle.tile_rows(wl.b1, wl.tiles, g)[:, None] * wl.b2 + np.arange(wl.b2)
            mine[bh // wl.H, bh % wl.H, torch.as_tensor(rows.ravel())] = True
        written = ~torch.isnan(one.float()).any(dim=-1).cpu()
        assert torch.equal(written, mine)
    assert _lib.monarch_last_device_status(None) == 0
    assert torch.equal(parts, full)
    assert _lib.monarch_attn_fwd_units_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                          parts.data_ptr(), *shape, dt, 0, cuts[-1] + 1,
                                          ws.data_ptr(), need, None) == 2


def test_device_entry_points_reject_bad_buffers(tiny64):
    q = to_torch(tiny64[0], "f32")
    shape = (1, 2, 3, 8, 8, 32, 24, 8, 1, 1)
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    p = q.data_ptr()
    assert _lib.monarch_attn_fwd_ws(p + 4, p, p, p, *shape, 0, ws.data_ptr(), 1 << 20, None) == 3
    assert _lib.monarch_attn_fwd_ws(p, p, p, p, *shape, 0, ws.data_ptr(), 64, None) == 5
    assert _lib.monarch_last_device_status(None) == 0


def test_injected_stall_times_out_and_the_next_call_is_correct():
    """Fault injection on the host: with the stall hook on, each tensor-core kernel's
    MMA warp waits on a barrier that nothing completes.  The bounded wait must give
    up, so the status is MONARCH_ERR_TIMEOUT for certain; the kernels then take
    their abort path (the other roles stop, in-flight copies and MMAs drain, tensor
    memory is freed) and the following call on the same context is correct."""
    wl = synth.WORKLOADS["480p_chunk"].replace(H=4)
    q, k, v = device_inputs(wl)
    assert kernel_path(q, f=wl.f, h=wl.h, w=wl.w, b1=wl.b1, b2=wl.b2, tiles=wl.tiles) == 1
    old_limit = _lib.monarch_set_wait_limit(1 << 12)
    old_stall = _lib.monarch_debug_inject_stall(1)
    try:
        monarch_attention(q, k, v, f=wl.f, h=wl.h, w=wl.w, b1=wl.b1, b2=wl.b2, tiles=wl.tiles)
        torch.cuda.synchronize()
        assert _lib.monarch_last_device_status(None) == 7
    finally:
        _lib.monarch_debug_inject_stall(old_stall)
        _lib.monarch_set_wait_limit(old_limit)
    assert _lib.monarch_last_device_status(None) == 0   # the word was read and cleared
    out = run(wl, q, k, v)
    q64, k64, v64 = (from_torch(x, wl.dtype) for x in (q, k, v))
    ref = oracle.monarch_attn(q64, k64, v64, wl.b1, wl.b2, wl.tiles, wl.iters)
    assert rel_fro(from_torch(out, wl.dtype), ref) <= TOL[wl.dtype]


def test_tensor_core_path_survives_a_tiny_wait_limit():
    """Bounded waits: with a limit of a few polls the kernels give up (status
    MONARCH_ERR_TIMEOUT) or finish, but never hang, and the next call is correct."""
    wl = synth.WORKLOADS["480p_chunk"].replace(H=4)
    q, k, v = device_inputs(wl)
    assert kernel_path(q, f=wl.f, h=wl.h, w=wl.w, b1=wl.b1, b2=wl.b2, tiles=wl.tiles) == 1
    old = _lib.monarch_set_wait_limit(64)
    try:
        monarch_attention(q, k, v, f=wl.f, h=wl.h, w=wl.w, b1=wl.b1, b2=wl.b2, tiles=wl.tiles)
        torch.cuda.synchronize()
        assert _lib.monarch_last_device_status(None) in (0, 7)
    finally:
        _lib.monarch_set_wait_limit(old)
    out = run(wl, q, k, v)
    q64, k64, v64 = (from_torch(x, wl.dtype) for x in (q, k, v))
    ref = oracle.monarch_attn(q64, k64, v64, wl.b1, wl.b2, wl.tiles, wl.iters)
    assert rel_fro(from_torch(out, wl.dtype), ref) <= TOL[wl.dtype]


# --------------------------------------------------------------------------
# a chunk of frames against a key/value cache (N_q != N_k)
# --------------------------------------------------------------------------
KV_CASES = [
    # name, dtype, d, fq, fk, h, w, b2, tiles, iters, path
    ("tiny", "f32", 32, 1, 3, 8, 8, 8, 3, 2, 0),
    ("tiny", "bf16", 32, 2, 3, 8, 8, 8, 1, 1, 0),
    ("480p_chunk", "bf16", 128, 1, 3, 8, 32, 32, 2, 1, 1),
    ("480p_chunk", "bf16", 128, 2, 6, 30, 52, 52, 2, 2, 1),
    ("480p_chunk", "bf16", 128, 3, 2, 10, 16, 16, 4, 1, 1),      # fewer key frames than query frames
    ("480p_chunk", "bf16", 128, 1, 4, 64, 1, 1, 2, 1, 1),        # b2 = 1
]


@pytest.mark.parametrize("name,dtype,d,fq,fk,h,w,b2,tiles,iters,path", KV_CASES)
def test_chunk_against_kv_cache_whole_output(name, dtype, d, fq, fk, h, w, b2, tiles, iters, path):
    """Queries of the newest fq frames of a clip against keys and values of all fk frames."""
    wl = synth.WORKLOADS[name].replace(H=2, d=d, f=max(fq, fk), h=h, w=w, b1=max(fq, fk) * h * w // b2,
                                       b2=b2, tiles=1, iters=1, dtype=dtype)
    q64, k64, v64 = (synth.round_to_dtype(x, dtype) for x in synth.make_inputs(wl))
    nq, nk = fq * h * w, fk * h * w
    q64 = np.ascontiguousarray(q64[..., wl.N - nq:, :])   # the chunk: the newest frames
    k64 = np.ascontiguousarray(k64[..., wl.N - nk:, :])
    v64 = np.ascontiguousarray(v64[..., wl.N - nk:, :])
    b1, b1k = nq // b2, nk // b2
    ref = oracle.monarch_attn_kv(q64, k64, v64, b1, b1k, b2, tiles, iters)
    q, k, v = (to_torch(x, dtype) for x in (q64, k64, v64))
    dt = _lib.F32 if dtype == "f32" else _lib.BF16
    shape = (wl.B, wl.H, fq, fk, h, w, d, b1, b1k, b2, tiles, iters)
    assert _lib.monarch_attn_kv_path(*shape, dt) == path
    need = _lib.monarch_attn_kv_workspace_bytes(*shape, dt)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out = torch.full_like(q, float("nan"))
    assert _lib.monarch_attn_fwd_kv_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                       *shape, dt, ws.data_ptr(), need, None) == 0
    torch.cuda.synchronize()
    assert _lib.monarch_last_device_status(None) == 0
    got = from_torch(out, dtype)
    assert np.isfinite(got).all()
    assert rel_fro(got, ref) <= TOL[dtype]


# --------------------------------------------------------------------------
# [B, N, H, d] inputs: the kernels read the strided rows directly; the result is
# the [B, H, N, d] computation's, bit for bit (only the addresses differ)
# --------------------------------------------------------------------------
LAYOUT_CASES = [
    # f, h, w, b1, b2, tiles, iters, d, dtype, kernel path
    (2, 3, 100, 6, 100, 2, 1, 128, "bf16", 1),
    (5, 60, 48, 300, 48, 5, 2, 128, "bf16", 1),    # iters > 1: queries on both MMA sides
    (2, 100, 7, 200, 7, 3, 1, 128, "bf16", 1),
    (3, 8, 8, 24, 8, 5, 2, 64, "f32", 0),
    (3, 8, 8, 24, 8, 3, 1, 32, "bf16", 0),
]


@pytest.mark.parametrize("f,h,w,b1,b2,tiles,iters,d,dtype,path", LAYOUT_CASES)
def test_bnhd_layout_matches_bhnd_bit_for_bit(f, h, w, b1, b2, tiles, iters, d, dtype, path):
    from structured_attention_video_b200.attention import monarch_attention_bnhd
    wl = TINY.replace(B=2, H=3, d=d, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles, iters=iters)
    q64, k64, v64 = (synth.round_to_dtype(x, dtype) for x in synth.make_inputs(wl))
    q, k, v = (to_torch(x, dtype) for x in (q64, k64, v64))
    assert kernel_path(q, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles, iters=iters) == path
    ref = run(wl, q, k, v)
    qt, kt, vt = (x.transpose(1, 2).contiguous() for x in (q, k, v))
    out = monarch_attention_bnhd(qt, kt, vt, f=f, h=h, w=w, b1=b1, b2=b2, tiles=tiles,
                                 iters=iters)
    torch.cuda.synchronize()
    assert _lib.monarch_last_device_status(None) == 0
    assert torch.equal(out.transpose(1, 2), ref)
    want = oracle.monarch_attn(q64, k64, v64, b1, b2, tiles, iters)
    assert rel_fro(from_torch(ref, dtype), want) <= TOL[dtype]
