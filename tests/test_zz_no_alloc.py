"""monarch_attn_fwd_noalloc, the entry point for callers that may not allocate
device memory (a host framework that owns every device allocation, or a loop
that cannot afford cudaMalloc's implicit synchronisation).  Its scratch is a
static device array, so two calls in a row must each match the entry point
that takes a caller-owned workspace, with no state leaking from the first call
into the second.  Collected last: it runs alone or after every other test."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from structured_attention_video_b200 import _lib, synth  # noqa: E402

from helpers import TOL, from_torch, rel_fro, to_torch  # noqa: E402

pytestmark = pytest.mark.gpu


def shape_args(wl, **kw):
    d = dict(B=wl.B, H=wl.H, f=wl.f, h=wl.h, w=wl.w, d=wl.d, b1=wl.b1, b2=wl.b2,
             tiles=wl.tiles, iters=wl.iters)
    d.update(kw)
    return tuple(d[k] for k in ("B", "H", "f", "h", "w", "d", "b1", "b2", "tiles", "iters"))


def with_workspace(q, k, v, args, dt):
    need = _lib.monarch_attn_workspace_bytes(*args, dt)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    _lib.check(_lib.monarch_attn_fwd_ws(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                        *args, dt, ws.data_ptr(), need, None), "fwd_ws")
    return out


def no_alloc(q, k, v, args, dt):
    out = torch.full_like(q, float("nan"))
    _lib.check(_lib.monarch_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                             out.data_ptr(), *args, dt, None), "fwd_noalloc")
    return out


CASES = [("tiny", "f32", dict(tiles=5, iters=2)), ("tiny", "bf16", dict(tiles=3, iters=1)),
         ("480p_chunk", "bf16", dict())]


@pytest.mark.parametrize("name,dtype,kw", CASES)
def test_two_calls_in_a_row_match_the_workspace_entry_point(name, dtype, kw):
    wl = synth.WORKLOADS[name].replace(dtype=dtype, **kw)
    args = shape_args(wl)
    dt = _lib.F32 if dtype == "f32" else _lib.BF16
    runs = []
    for rank in (0, 1):            # two different inputs, one call each, back to back
        q64, k64, v64 = synth.make_inputs(wl, rank=rank)
        q, k, v = (to_torch(x, dtype) for x in (q64, k64, v64))
        runs.append((q, k, v, no_alloc(q, k, v, args, dt)))
    torch.cuda.synchronize()
    assert _lib.monarch_last_device_status(None) == 0
    for q, k, v, got in runs:
        ref = with_workspace(q, k, v, args, dt)
        torch.cuda.synchronize()
        a, b = from_torch(got, dtype), from_torch(ref, dtype)
        assert np.isfinite(a).all()
        assert rel_fro(a, b) <= TOL[dtype]
    assert not torch.equal(runs[0][3], runs[1][3])


class DefaultPoolWatch:
    """The current device's default CUDA memory pool through the driver API: the
    pool that stream-ordered allocations (cudaMallocAsync) draw from."""
    RESERVED_CURRENT, USED_CURRENT, USED_HIGH = 5, 7, 8

    def __init__(self):
        import ctypes
        self.ct = ctypes
        self.cu = ctypes.CDLL("libcuda.so.1")
        dev = ctypes.c_int()
        assert self.cu.cuDeviceGet(ctypes.byref(dev), torch.cuda.current_device()) == 0
        self.pool = ctypes.c_void_p()
        assert self.cu.cuDeviceGetDefaultMemPool(ctypes.byref(self.pool), dev) == 0

    def get(self, attr):
        v = self.ct.c_uint64()
        assert self.cu.cuMemPoolGetAttribute(self.pool, attr, self.ct.byref(v)) == 0
        return v.value

    def reset_high(self):
        zero = self.ct.c_uint64(0)
        assert self.cu.cuMemPoolSetAttribute(self.pool, self.USED_HIGH, self.ct.byref(zero)) == 0


def test_a_call_allocates_nothing():
    """The defining property: after a first call (which looks up the static array's
    address for this context), a call changes neither torch's allocator counters,
    nor the device's free memory, nor the default memory pool's usage, not even
    transiently (the pool's high-water mark stays at its current usage)."""
    wl = synth.WORKLOADS["480p_chunk"].replace(H=2)
    args = shape_args(wl)
    q64, k64, v64 = synth.make_inputs(wl)
    q, k, v = (to_torch(x, "bf16") for x in (q64, k64, v64))
    out = torch.empty_like(q)
    call = lambda: _lib.check(_lib.monarch_attn_fwd_noalloc(   # noqa: E731
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), *args, _lib.BF16, None),
        "fwd_noalloc")
    call()
    torch.cuda.synchronize()
    pool = DefaultPoolWatch()
    pool.reset_high()
    before = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved(),
              torch.cuda.mem_get_info()[0], pool.get(pool.USED_CURRENT),
              pool.get(pool.RESERVED_CURRENT))
    call()
    torch.cuda.synchronize()
    after = (torch.cuda.memory_allocated(), torch.cuda.memory_reserved(),
             torch.cuda.mem_get_info()[0], pool.get(pool.USED_CURRENT),
             pool.get(pool.RESERVED_CURRENT))
    assert after == before
    assert pool.get(pool.USED_HIGH) == pool.get(pool.USED_CURRENT)
    assert _lib.monarch_last_device_status(None) == 0


def test_rejects_problems_beyond_the_static_scratch():
    wl = synth.WORKLOADS["720p"]
    args = shape_args(wl)
    q = torch.zeros(16, dtype=torch.bfloat16, device="cuda")   # never read: rejected first
    st = _lib.monarch_attn_fwd_noalloc(q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(),
                                       *args, _lib.BF16, None)
    assert st == 8
    assert "scratch" in _lib.monarch_status_string(st)
