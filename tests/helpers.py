"""Shared helpers of the GPU tests: seeded inputs on host and device, oracle
comparisons on full outputs or on sampled (head, tile, column) problems."""
from __future__ import annotations

import numpy as np

from oracle import oracle
from structured_attention_video_b200 import synth

TOL = {"f32": 1e-5, "bf16": 1e-2}   # relative Frobenius error against the float64 oracle


def to_torch(x64: np.ndarray, dtype: str, device="cuda"):
    """float64 values already rounded to `dtype` -> a torch tensor of that dtype."""
    import torch
    bits = synth.to_device_bits(x64, dtype)
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(bits)).to(device)
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def from_torch(t, dtype: str) -> np.ndarray:
    import torch
    if dtype == "f32":
        return t.detach().cpu().numpy().astype(np.float64)
    bits = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return synth.from_device_bits(bits, dtype)


def device_inputs(wl: synth.Workload, rank: int = 0):
    """(q, k, v) torch tensors [B, H, N, d] on the GPU, generated head by head."""
    import torch
    shape = (wl.B, wl.H, wl.N, wl.d)
    np_dtype = np.float32 if wl.dtype == "f32" else np.uint16
    q, k, v = (np.empty(shape, np_dtype) for _ in range(3))
    synth.fill_device_bits(wl, q, k, v, rank)

    def up(a):
        if wl.dtype == "f32":
            return torch.from_numpy(a).cuda()
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return up(q), up(k), up(v)


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def sample_problems(wl: synth.Workload, count: int, seed: int = 0):
    """Deterministic (bh, g, c) problems: both ends of every index plus random ones."""
    rng = np.random.default_rng(seed)
    BH = wl.B * wl.H
    probs = {(0, 0, 0), (BH - 1, wl.tiles - 1, wl.b2 - 1), (0, wl.tiles - 1, 0),
             (BH - 1, 0, wl.b2 - 1)}
    while len(probs) < count:
        probs.add((int(rng.integers(BH)), int(rng.integers(wl.tiles)), int(rng.integers(wl.b2))))
    return sorted(probs)


def rows_of(wl: synth.Workload, g: int, c: int) -> np.ndarray:
    lo = (g * wl.b1) // wl.tiles
    hi = ((g + 1) * wl.b1) // wl.tiles
    return np.arange(lo, hi) * wl.b2 + c


def oracle_on_samples(wl: synth.Workload, probs, rank: int = 0, nthreads: int = 0):
    """Run the oracle on sampled problems; each head's inputs are regenerated on the
    host by the seeded generator (the same values the device received).
    Returns {bh: y [N, d]} with only the sampled rows filled."""
    heads = sorted({p[0] for p in probs})
    pos = synth.positional_code(wl.f, wl.h, wl.w, wl.d)
    out = {}
    for bh in heads:
        b, h = divmod(bh, wl.H)
        x = synth.make_head(wl, b, h, rank, pos)
        sub = [(0, g, c) for (hh, g, c) in probs if hh == bh]
        y = oracle.monarch_problems(x["q"][None], x["k"][None], x["v"][None], wl.b1, wl.b2,
                                    wl.tiles, wl.iters, sub, nthreads)
        out[bh] = y[0]
    return out


def sampled_error(wl: synth.Workload, out_dev, probs, rank: int = 0):
    ref = oracle_on_samples(wl, probs, rank)
    got_rows, ref_rows = [], []
    for bh, g, c in probs:
        b, h = divmod(bh, wl.H)
        rows = rows_of(wl, g, c)
        got_rows.append(from_torch(out_dev[b, h, rows], wl.dtype))
        ref_rows.append(ref[bh][rows])
    return rel_fro(np.concatenate(got_rows), np.concatenate(ref_rows))
