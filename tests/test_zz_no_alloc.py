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


def test_rejects_problems_beyond_the_static_scratch():
    wl = synth.WORKLOADS["720p"]
    args = shape_args(wl)
    q = torch.zeros(16, dtype=torch.bfloat16, device="cuda")   # never read: rejected first
    st = _lib.monarch_attn_fwd_noalloc(q.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(),
                                       *args, _lib.BF16, None)
    assert st == 8
    assert "scratch" in _lib.monarch_status_string(st)
