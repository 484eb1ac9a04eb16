"""Pins of the oracle's other reading of the tiles: the tiles split the key
columns v' of every block ("创新二：平铺Monarch参数化": each block is split into
tiles that are factorised independently; the pages do not say along which axis).

With key tile g' = [floor(g'*b2/t), floor((g'+1)*b2/t)) the Monarch matrix is
M[(u,v),(u',v')] = L_v[u,(u',g'(v'))] * R_{u',g'(v')}[v,v'].  Every check is
computed outside the oracle: textbook attention (t = b2, or b2 = 1), the Q = 0
mean, the matrix M assembled from the factors, and the variational objective of
softmax evaluated on it.  Planted errors in a copy of the oracle source must be
caught by the same checks.
"""
import os

import numpy as np
import pytest

from oracle import oracle
from structured_attention_video_b200 import synth

from test_oracle_pins import dense_attention, objective, rel

B1, B2 = 24, 8


@pytest.fixture(scope="module")
def tiny():
    q, k, v = synth.make_inputs(synth.WORKLOADS["tiny"])
    return q[0], k[0], v[0]          # [H, N, d]


def col_tiles(b2, tiles):
    lo = [(g * b2) // tiles for g in range(tiles + 1)]
    g_of = np.empty(b2, int)
    for g in range(tiles):
        g_of[lo[g]:lo[g + 1]] = g
    return g_of


def brute_force_m_keytiles(L, R, b1, b2, tiles):
    """M[(u,v),(u',v')] = L_v[u, g'(v')*b1 + u'] * R_{u',g'(v')}[v,v'] for one head."""
    N = b1 * b2
    g_of = col_tiles(b2, tiles)
    M = np.zeros((N, N))
    for u in range(b1):
        for v in range(b2):
            for up in range(b1):
                for vp in range(b2):
                    g = g_of[vp]
                    M[u * b2 + v, up * b2 + vp] = L[v, u, g * b1 + up] * R[up, g, v, vp]
    return M


def _random_simplex(rng, n):
    x = rng.exponential(size=n)
    return x / x.sum()


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------
@pytest.mark.parametrize("iters", [1, 2, 3])
def test_one_column_per_tile_is_exact_attention(tiny, iters):
    q, k, v = tiny
    y = oracle.monarch_attn_keytiles(q, k, v, B1, B2, B2, iters)
    assert rel(y, dense_attention(q, k, v)) < 1e-12


@pytest.mark.parametrize("b1,b2,tiles", [(192, 1, 1), (3, 64, 64), (12, 16, 16)])
def test_degenerate_shapes_are_exact_attention(tiny, b1, b2, tiles):
    q, k, v = tiny
    y = oracle.monarch_attn_keytiles(q, k, v, b1, b2, tiles, 1)
    assert rel(y, dense_attention(q, k, v)) < 1e-12


@pytest.mark.parametrize("tiles,iters", [(1, 1), (3, 1), (5, 2), (8, 2)])
def test_zero_queries_give_the_mean_of_v(tiny, tiles, iters):
    """Q = 0: R is uniform on each tile, H = log |T'_g'|, so L weighs super-key
    (u', g') by |T'_g'| / N and y is the mean of all values, whatever the tiles."""
    _, k, v = tiny
    y = oracle.monarch_attn_keytiles(np.zeros_like(k), k, v, B1, B2, tiles, iters)
    assert np.abs(y - v.mean(-2, keepdims=True)).max() < 1e-13


def test_one_tile_is_plain_monarch(tiny):
    """t = 1 is one tile on either axis: the two readings give the same map."""
    q, k, v = tiny
    y = oracle.monarch_attn_keytiles(q, k, v, B1, B2, 1, 2)
    assert rel(y, oracle.monarch_attn(q, k, v, B1, B2, 1, 2)) < 1e-13


# --------------------------------------------------------------------------
# the Monarch form and the variational objective
# --------------------------------------------------------------------------
@pytest.mark.parametrize("tiles,iters", [(1, 1), (3, 1), (4, 2)])
def test_brute_force_m_is_row_stochastic_and_reproduces_output(tiny, tiles, iters):
    q, k, v = tiny[0][1], tiny[1][1], tiny[2][1]
    y, L, R = oracle.monarch_attn_keytiles(q, k, v, B1, B2, tiles, iters, factors=True)
    M = brute_force_m_keytiles(L, R, B1, B2, tiles)
    assert M.min() >= 0.0
    assert np.abs(M.sum(1) - 1.0).max() < 1e-12
    assert rel(y, M @ v) < 1e-13
    # R rows live on their tile's columns only
    g_of = col_tiles(B2, tiles)
    for g in range(tiles):
        assert np.all(R[:, g][..., g_of != g] == 0.0)
        assert np.abs(R[:, g].sum(-1) - 1.0).max() < 1e-12


@pytest.mark.parametrize("tiles", [1, 3])
def test_objective_never_decreases_over_half_steps(tiny, tiles):
    q, k, v = tiny[0][0], tiny[1][0], tiny[2][0]
    prev = -np.inf
    for hs in range(1, 7):
        _, L, R = oracle.monarch_attn_keytiles(q, k, v, B1, B2, tiles, half_steps=hs,
                                               factors=True)
        F = objective(brute_force_m_keytiles(L, R, B1, B2, tiles), q, k)
        assert F >= prev - 1e-9, (hs, F, prev)
        prev = F


@pytest.mark.parametrize("tiles", [2, 3])
def test_each_half_step_is_a_maximiser(tiny, tiles):
    """No feasible perturbation of the factor just updated increases F: an R row
    moves inside its tile's simplex, an L row inside the super-key simplex."""
    q, k, v = tiny[0][1], tiny[1][1], tiny[2][1]
    rng = np.random.default_rng(11)
    lo = [(g * B2) // tiles for g in range(tiles + 1)]
    _, L, R = oracle.monarch_attn_keytiles(q, k, v, B1, B2, tiles, half_steps=3, factors=True)
    F0 = objective(brute_force_m_keytiles(L, R, B1, B2, tiles), q, k)
    for _ in range(15):
        up, g, vv = rng.integers(B1), rng.integers(tiles), rng.integers(B2)
        for eps in (1e-2, 0.3):
            R2 = R.copy()
            row = np.zeros(B2)
            row[lo[g]:lo[g + 1]] = _random_simplex(rng, lo[g + 1] - lo[g])
            R2[up, g, vv] = (1 - eps) * R[up, g, vv] + eps * row
            F = objective(brute_force_m_keytiles(L, R2, B1, B2, tiles), q, k)
            assert F <= F0 + 1e-10
    _, L, R = oracle.monarch_attn_keytiles(q, k, v, B1, B2, tiles, half_steps=4, factors=True)
    F0 = objective(brute_force_m_keytiles(L, R, B1, B2, tiles), q, k)
    for _ in range(15):
        vv, u = rng.integers(B2), rng.integers(B1)
        for eps in (1e-2, 0.3):
            L2 = L.copy()
            L2[vv, u] = (1 - eps) * L[vv, u] + eps * _random_simplex(rng, tiles * B1)
            F = objective(brute_force_m_keytiles(L2, R, B1, B2, tiles), q, k)
            assert F <= F0 + 1e-10


def test_error_vs_dense_reaches_zero_at_one_column_per_tile(tiny):
    """Nested key tilings t = 1, 2, 4, 8 (b2 = 8) on the seeded tiny inputs; the
    last is exact.  Monotone decrease is not a theorem: a violation is reported."""
    q, k, v = tiny
    yd = dense_attention(q, k, v)
    errs = [rel(oracle.monarch_attn_keytiles(q, k, v, B1, B2, t, 1), yd) for t in (1, 2, 4, 8)]
    assert all(b <= a + 1e-12 for a, b in zip(errs, errs[1:])), errs
    assert errs[-1] < 1e-12


# --------------------------------------------------------------------------
# the sampled-problem form agrees with the full pass; bad shapes are refused
# --------------------------------------------------------------------------
@pytest.mark.parametrize("tiles,iters", [(3, 1), (5, 2)])
def test_problem_subset_matches_full(tiny, tiles, iters):
    q, k, v = tiny
    full = oracle.monarch_attn_keytiles(q, k, v, B1, B2, tiles, iters)
    probs = [(0, 0), (1, 5), (1, 7)]
    y = oracle.monarch_attn_keytiles(q, k, v, B1, B2, tiles, iters, probs=probs)
    for bh, c in probs:
        rows = np.arange(B1) * B2 + c
        assert np.array_equal(y[bh, rows], full[bh, rows])
    assert np.isnan(y[0, 1]).all()


def test_keytiles_rejects_bad_shapes(tiny):
    q, k, v = tiny
    for b1, b2, t in [(24, 8, 0), (24, 8, 9), (25, 8, 1)]:
        with pytest.raises(ValueError):
            oracle.monarch_attn_keytiles(q, k, v, b1, b2, t, 1)
    with pytest.raises(ValueError):
        oracle.monarch_attn_keytiles(q, k, v, B1, B2, 2, 1, probs=[(0, 8)])


# --------------------------------------------------------------------------
# planted errors in the key-tile half-steps
# --------------------------------------------------------------------------
MUTANTS = {
    "tile_spans_whole_block": ("const int c1 = key_tile_first_col(g + 1, b2, tiles);",
                               "const int c1 = b2;"),
    "entropy_dropped": ("logit[j] = s * acc + H[j];", "logit[j] = s * acc;"),
    "superkeys_interleaved": ("const int j = g * b1k + up;", "const int j = up * tiles + g;"),
    "weights_of_next_superkey": ("double wgt = L[(size_t)u * nsk + j];",
                                 "double wgt = L[(size_t)u * nsk + (j + 1) % nsk];"),
    "half_the_query_rows": ("for (int u = 0; u < b1; u++) {\n                        double wgt",
                            "for (int u = 0; u < (b1 + 1) / 2; u++) {\n"
                            "                        double wgt"),
    "values_from_keys": ("z += r * v[((int64_t)up * b2 + vp) * d + jj];",
                         "z += r * k[((int64_t)up * b2 + vp) * d + jj];"),
}


def keytile_pins_pass(lib, q, k, v):
    yd = dense_attention(q, k, v)
    for iters in (1, 2):
        if rel(oracle.monarch_attn_keytiles(q, k, v, B1, B2, B2, iters, lib=lib), yd) > 1e-12:
            return False
    y0 = oracle.monarch_attn_keytiles(np.zeros_like(k), k, v, B1, B2, 3, 1, lib=lib)
    if np.abs(y0 - v.mean(-2, keepdims=True)).max() > 1e-13:
        return False
    qh, kh, vh = q[0], k[0], v[0]
    for t in (3,):
        y, L, R = oracle.monarch_attn_keytiles(qh, kh, vh, B1, B2, t, 1, factors=True, lib=lib)
        M = brute_force_m_keytiles(L, R, B1, B2, t)
        if M.min() < 0 or np.abs(M.sum(1) - 1).max() > 1e-12 or rel(y, M @ vh) > 1e-13:
            return False
        prev = -np.inf
        for hs in range(1, 5):
            _, L, R = oracle.monarch_attn_keytiles(qh, kh, vh, B1, B2, t, half_steps=hs,
                                                   factors=True, lib=lib)
            F = objective(brute_force_m_keytiles(L, R, B1, B2, t), qh, kh)
            if F < prev - 1e-9:
                return False
            prev = F
        # after the first R-step, no R row moved inside its tile's simplex gains
        rng = np.random.default_rng(5)
        lo = [(g * B2) // t for g in range(t + 1)]
        _, L, R = oracle.monarch_attn_keytiles(qh, kh, vh, B1, B2, t, half_steps=1,
                                               factors=True, lib=lib)
        F0 = objective(brute_force_m_keytiles(L, R, B1, B2, t), qh, kh)
        for _ in range(12):
            up, g, vv = rng.integers(B1), rng.integers(t), rng.integers(B2)
            R2 = R.copy()
            row = np.zeros(B2)
            row[lo[g]:lo[g + 1]] = _random_simplex(rng, lo[g + 1] - lo[g])
            R2[up, g, vv] = 0.99 * R[up, g, vv] + 0.01 * row
            if objective(brute_force_m_keytiles(L, R2, B1, B2, t), qh, kh) > F0 + 1e-10:
                return False
    return True


def test_unmutated_keytile_oracle_passes(tiny):
    assert keytile_pins_pass(None, *tiny)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_keytile_mutant_is_caught(tmp_path, tiny, name):
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, "mutation site not unique: " + name
    mutated = os.path.join(tmp_path, "mutant.c")
    with open(mutated, "w") as fh:
        fh.write(src.replace(old, new, 1))
    lib = oracle.build(force=True, src=mutated, out=os.path.join(tmp_path, "libmutant.so"))
    assert not keytile_pins_pass(lib, *tiny), "pins did not catch mutant " + name
