"""Pins of the oracle's backward pass (one iteration), against things other than
itself:

- central finite differences of the forward oracle, element by element on tiny
  shapes and along random directions on larger ones (the definition of the
  gradient);
- the closed-form backward of softmax attention, which the method reduces to
  when one Monarch factor is the whole matrix (b1 = 1: one L block; b2 = 1: every
  R block is 1 x 1), so dQ = s dS K, dK = s dS^T Q, dV = P^T dY with
  dS = P (dP - rowsum(P dP)), dP = dY V^T;
- planted errors in a copy of the backward's source, each of which the
  directional finite-difference pin must reject.

The pages give the finetuning that trains through the Monarch attention
(summary page, "Approach"; explainer page, "创新三：微调与高效内核") but no
backward; the oracle's backward is the chain rule of its forward map.
"""
import os
import subprocess

import numpy as np
import pytest

from oracle import oracle

SHAPES = [  # f, h, w, b1, b2, tiles
    (2, 3, 4, 6, 4, 1),
    (2, 3, 4, 6, 4, 2),      # two tiles of three block rows
    (2, 3, 4, 6, 4, 4),      # ragged tiles (1, 2, 1, 2 rows)
    (2, 3, 4, 6, 4, 6),      # one block row per tile
    (1, 1, 24, 1, 24, 1),    # b1 = 1: a single L block
    (2, 3, 4, 24, 1, 5),     # b2 = 1: 1 x 1 R blocks
]


def phi(dy, q, k, v, b1, b2, t, lib=None):
    return float(np.sum(dy * oracle.monarch_attn(q, k, v, b1, b2, t, 1, lib=lib)))


def inputs(N, d, BH=2, seed=0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((BH, N, d)) for _ in range(4)]


@pytest.mark.parametrize("f,h,w,b1,b2,t", SHAPES)
def test_backward_matches_central_differences(f, h, w, b1, b2, t):
    N, d = f * h * w, 4
    q, k, v, dy = inputs(N, d, seed=b1 * 10 + t)
    grads = oracle.monarch_attn_bwd(q, k, v, dy, b1, b2, t)
    eps = 1e-6
    for which, g in zip(range(3), grads):
        x = [q, k, v]
        fd = np.zeros_like(g)
        for idx in np.ndindex(g.shape):
            xp = [a.copy() for a in x]
            xm = [a.copy() for a in x]
            xp[which][idx] += eps
            xm[which][idx] -= eps
            fd[idx] = (phi(dy, *xp, b1, b2, t) - phi(dy, *xm, b1, b2, t)) / (2 * eps)
        assert np.abs(fd - g).max() <= 1e-6 * np.abs(fd).max(), which


def directional_error(q, k, v, dy, b1, b2, t, seed=1, lib=None):
    """|<grad, delta> - central difference along delta| / |<grad, delta>|, worst of
    three random directions (each moves q, k and v together)."""
    dq, dk, dv = oracle.monarch_attn_bwd(q, k, v, dy, b1, b2, t, lib=lib)
    rng = np.random.default_rng(seed)
    worst = 0.0
    for _ in range(3):
        e = [rng.standard_normal(q.shape) for _ in range(3)]
        lin = float(np.sum(dq * e[0]) + np.sum(dk * e[1]) + np.sum(dv * e[2]))
        h = 1e-5
        fp = phi(dy, q + h * e[0], k + h * e[1], v + h * e[2], b1, b2, t)
        fm = phi(dy, q - h * e[0], k - h * e[1], v - h * e[2], b1, b2, t)
        worst = max(worst, abs((fp - fm) / (2 * h) - lin) / abs(lin))
    return worst


@pytest.mark.parametrize("f,h,w,b1,b2,t,d", [(3, 8, 8, 24, 8, 5, 16), (3, 8, 8, 192, 1, 7, 8),
                                              (2, 5, 7, 10, 7, 3, 32)])
def test_backward_along_random_directions(f, h, w, b1, b2, t, d):
    q, k, v, dy = inputs(f * h * w, d, BH=1, seed=d)
    assert directional_error(q, k, v, dy, b1, b2, t) <= 1e-6


def attention_backward(q, k, v, dy):
    s = 1.0 / np.sqrt(q.shape[-1])
    a = s * q @ np.swapaxes(k, -1, -2)
    p = np.exp(a - a.max(-1, keepdims=True))
    p /= p.sum(-1, keepdims=True)
    dp = dy @ np.swapaxes(v, -1, -2)
    ds = p * (dp - np.sum(p * dp, -1, keepdims=True))
    return s * ds @ k, s * np.swapaxes(ds, -1, -2) @ q, np.swapaxes(p, -1, -2) @ dy


@pytest.mark.parametrize("b1,b2,t", [(1, 48, 1), (48, 1, 1), (48, 1, 48)])
def test_degenerate_blocks_give_the_attention_backward(b1, b2, t):
    q, k, v, dy = inputs(48, 8, seed=b1 + t)
    got = oracle.monarch_attn_bwd(q, k, v, dy, b1, b2, t)
    for g, r in zip(got, attention_backward(q, k, v, dy)):
        assert np.abs(g - r).max() <= 1e-12 * np.abs(r).max()


MUTANTS = {
    "entropy_gradient_dropped": (
        "- dH[up] * Rr[vp] * (Ar[vp] - ea);", ";"),
    "aggregation_not_averaged": (
        "+= dqbar[j] / nq;", "+= dqbar[j];"),
    "ktilde_path_of_keys_dropped": (
        "dkr[j] += s * da * qbar[j] + Rr[vp] * dKt[(size_t)up * d + j];",
        "dkr[j] += s * da * qbar[j];"),
    "softmax_backward_without_centering": (
        "dBr[up] = Lr[up] * (row[up] - ldl);", "dBr[up] = Lr[up] * row[up];"),
    "bias_gradient_dropped": (
        "dH[up] += dBr[up];", "dH[up] += 0.0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_backward_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, "mutation site not found: " + name
    mutated = os.path.join(tmp_path, "mutant.c")
    with open(mutated, "w") as fh:
        fh.write(src.replace(old, new))
    lib_path = os.path.join(tmp_path, "libmutant.so")
    subprocess.run(["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", mutated, "-o",
                    lib_path, "-lm"], check=True)
    q, k, v, dy = inputs(3 * 8 * 8, 16, BH=1, seed=5)
    assert directional_error(q, k, v, dy, 24, 8, 5, lib=lib_path) > 1e-3
