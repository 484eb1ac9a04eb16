"""Pins of the float64 CPU oracle against facts fixed outside the oracle.

Every check here is computed independently of oracle/monarch_oracle.c: textbook
softmax attention written with numpy, closed forms, the Monarch definition
M = P^T L P R assembled as explicit matrices, and the variational objective of
softmax evaluated on the brute-force matrix M.  Sources: the explainer page
"卡内基梅隆大学提出MonarchRT…", sections "Monarch矩阵" (a fixed permutation and two
block-diagonal factors; MonarchAttention's alternating optimisation of L and R
from Q and K, Fig. 3), "创新一：块对齐策略" (N = f*h*w, (b1, b2) = (f*h, w)) and
"创新二：平铺Monarch参数化" (tiles, error monotonically tunable, Fig. 2); the
abstract of "MonarchRT: Efficient Attention for Real-Time Video Generation".
"""
import numpy as np
import pytest

from oracle import oracle
from structured_attention_video_b200 import synth

TINY = synth.WORKLOADS["tiny"]


def dense_attention(q, k, v):
    """Textbook softmax(Q K^T / sqrt(d)) V in float64."""
    s = q @ np.swapaxes(k, -1, -2) / np.sqrt(q.shape[-1])
    s = s - s.max(-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(-1, keepdims=True)
    return p @ v


def rel(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.fixture(scope="module")
def tiny():
    q, k, v = synth.make_inputs(TINY)
    return q[0], k[0], v[0]          # [H, N, d]


def brute_force_m(L, R, b1, b2, tiles):
    """M[(u,v),(u',v')] = L_v[u,u'] * R_{u',g(u)}[v,v'] for one head, as an N x N matrix."""
    N = b1 * b2
    lo = [(g * b1) // tiles for g in range(tiles + 1)]
    g_of_u = np.empty(b1, int)
    for g in range(tiles):
        g_of_u[lo[g]:lo[g + 1]] = g
    M = np.zeros((N, N))
    for u in range(b1):
        for v in range(b2):
            row = u * b2 + v
            for up in range(b1):
                M[row, up * b2:(up + 1) * b2] = L[v, u, up] * R[up, g_of_u[u], v, :]
    return M


def objective(M, q, k):
    """Variational softmax objective: sum_i [ <M_i, s q_i K^T> + entropy(M_i) ]."""
    S = q @ k.T / np.sqrt(q.shape[-1])
    ent = -np.sum(np.where(M > 0, M * np.log(np.where(M > 0, M, 1.0)), 0.0))
    return float(np.sum(M * S) + ent)


# --------------------------------------------------------------------------
# index maps
# --------------------------------------------------------------------------
@pytest.mark.parametrize("f,h,w,b1,b2,tiles", [(3, 8, 8, 24, 8, 1), (3, 8, 8, 24, 8, 5),
                                                (3, 8, 8, 3, 64, 2), (21, 45, 80, 945, 80, 4)])
def test_index_maps_are_a_shuffle_and_partition(f, h, w, b1, b2, tiles):
    m = oracle.index_maps(f, h, w, b1, b2, tiles)
    N = f * h * w
    perm = m["perm"]
    # a bijection of [N]
    assert np.array_equal(np.sort(perm), np.arange(N))
    inv = np.empty(N, np.int64)
    inv[perm] = np.arange(N)
    assert np.array_equal(perm[inv], np.arange(N))
    # the perfect shuffle sends each block of b2 consecutive tokens to stride-b1 slots,
    # and its transpose sends consecutive runs of b1 back to stride b2
    n = np.arange(N)
    assert np.array_equal(m["u_of_n"] * b2 + m["v_of_n"], n)
    assert np.all((m["v_of_n"] >= 0) & (m["v_of_n"] < b2))
    runs = inv.reshape(b2, b1)
    assert np.all(np.diff(runs, axis=1) == b2)
    # tile partition covers [b1] with contiguous, non-empty tiles whose sizes differ by <= 1
    lo = m["tile_lo"]
    assert lo[0] == 0 and lo[-1] == b1 and np.all(np.diff(lo) >= 1)
    assert np.diff(lo).max() - np.diff(lo).min() <= 1
    for g in range(tiles):
        assert np.all(m["tile_of_u"][lo[g]:lo[g + 1]] == g)


def test_tile_partitions_golden():
    """Tile boundaries of the benchmark shapes: tests/golden/tile_partitions.txt."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tile_partitions.txt")
    seen = 0
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        b1, tiles, bounds = line.split(None, 2)
        want = [int(x) for x in bounds.split(",")]
        got = oracle.index_maps(1, 1, int(b1), int(b1), 1, int(tiles))["tile_lo"]
        assert got.tolist() == want
        seen += 1
    assert seen >= 6


def test_monarch_form_p_l_p_r(tiny):
    """Untiled M equals P^T L P R with explicit permutation and block-diagonal matrices."""
    q, k, v = tiny[0][0], tiny[1][0], tiny[2][0]
    b1, b2 = 24, 8
    N = b1 * b2
    y, L, R = oracle.monarch_attn(q, k, v, b1, b2, 1, 1, factors=True)
    perm = oracle.index_maps(3, 8, 8, b1, b2, 1)["perm"]
    P = np.zeros((N, N))
    P[perm, np.arange(N)] = 1.0                    # (P x)[P(n)] = x[n]
    Rbig = np.zeros((N, N))
    for up in range(b1):
        Rbig[up * b2:(up + 1) * b2, up * b2:(up + 1) * b2] = R[up, 0]
    Lbig = np.zeros((N, N))
    for vv in range(b2):
        Lbig[vv * b1:(vv + 1) * b1, vv * b1:(vv + 1) * b1] = L[vv]
    M = P.T @ Lbig @ P @ Rbig
    assert np.allclose(M, brute_force_m(L, R, b1, b2, 1), atol=1e-15)
    assert rel(y, M @ v) < 1e-13


# --------------------------------------------------------------------------
# degenerate shapes reduce to textbook softmax attention
# --------------------------------------------------------------------------
@pytest.mark.parametrize("b1,b2,tiles", [(1, 192, 1), (192, 1, 1), (192, 1, 7), (192, 1, 192),
                                         (24, 8, 24), (3, 64, 3), (8, 24, 8)])
def test_degenerate_blocks_are_exact_attention(tiny, b1, b2, tiles):
    q, k, v = tiny
    y = oracle.monarch_attn(q, k, v, b1, b2, tiles, 1)
    assert rel(y, dense_attention(q, k, v)) < 1e-12


@pytest.mark.parametrize("iters", [2, 5])
def test_degenerate_blocks_exact_at_any_iteration(tiny, iters):
    q, k, v = tiny
    for b1, b2, t in [(1, 192, 1), (192, 1, 3), (24, 8, 24)]:
        y = oracle.monarch_attn(q, k, v, b1, b2, t, iters)
        assert rel(y, dense_attention(q, k, v)) < 1e-12


# --------------------------------------------------------------------------
# closed forms and invariants
# --------------------------------------------------------------------------
@pytest.mark.parametrize("tiles,iters", [(1, 1), (5, 1), (3, 4)])
def test_zero_queries_give_the_mean_of_v(tiny, tiles, iters):
    _, k, v = tiny
    y = oracle.monarch_attn(np.zeros_like(k), k, v, 24, 8, tiles, iters)
    assert np.abs(y - v.mean(-2, keepdims=True)).max() < 1e-13


@pytest.mark.parametrize("tiles,iters", [(1, 1), (4, 1), (5, 2)])
def test_brute_force_m_is_row_stochastic_and_reproduces_output(tiny, tiles, iters):
    q, k, v = tiny[0][1], tiny[1][1], tiny[2][1]
    y, L, R = oracle.monarch_attn(q, k, v, 24, 8, tiles, iters, factors=True)
    M = brute_force_m(L, R, 24, 8, tiles)
    assert M.min() >= 0.0
    assert np.abs(M.sum(1) - 1.0).max() < 1e-12
    assert rel(y, M @ v) < 1e-13


@pytest.mark.parametrize("tiles", [1, 3])
def test_objective_never_decreases_over_half_steps(tiny, tiles):
    q, k, v = tiny[0][0], tiny[1][0], tiny[2][0]
    prev = -np.inf
    for hs in range(1, 9):
        _, L, R = oracle.monarch_attn(q, k, v, 24, 8, tiles, half_steps=hs, factors=True)
        F = objective(brute_force_m(L, R, 24, 8, tiles), q, k)
        assert F >= prev - 1e-9, (hs, F, prev)
        prev = F


def _random_simplex(rng, n):
    x = rng.exponential(size=n)
    return x / x.sum()


@pytest.mark.parametrize("tiles", [1, 4])
def test_each_half_step_is_a_maximiser(tiny, tiles):
    """No feasible perturbation of the factor just updated increases F."""
    q, k, v = tiny[0][1], tiny[1][1], tiny[2][1]
    rng = np.random.default_rng(7)
    b1, b2 = 24, 8
    # after an R-step (odd half-step count): R maximises F(L, .)
    _, L, R = oracle.monarch_attn(q, k, v, b1, b2, tiles, half_steps=3, factors=True)
    F0 = objective(brute_force_m(L, R, b1, b2, tiles), q, k)
    for _ in range(40):
        up, g, vv = rng.integers(b1), rng.integers(tiles), rng.integers(b2)
        for eps in (1e-2, 0.3):
            R2 = R.copy()
            R2[up, g, vv] = (1 - eps) * R[up, g, vv] + eps * _random_simplex(rng, b2)
            assert objective(brute_force_m(L, R2, b1, b2, tiles), q, k) <= F0 + 1e-10
    # after an L-step (even count): L maximises F(., R)
    _, L, R = oracle.monarch_attn(q, k, v, b1, b2, tiles, half_steps=4, factors=True)
    F0 = objective(brute_force_m(L, R, b1, b2, tiles), q, k)
    for _ in range(40):
        vv, u = rng.integers(b2), rng.integers(b1)
        for eps in (1e-2, 0.3):
            L2 = L.copy()
            L2[vv, u] = (1 - eps) * L[vv, u] + eps * _random_simplex(rng, b1)
            assert objective(brute_force_m(L2, R, b1, b2, tiles), q, k) <= F0 + 1e-10


# --------------------------------------------------------------------------
# behaviour the pages state
# --------------------------------------------------------------------------
def test_error_vs_dense_non_increasing_in_nested_tiles(tiny):
    """Tiled Monarch: nested tilings t = 1, 2, 4, 8 (b1 = 24) on the seeded tiny inputs.

    Not a theorem at one iteration; a violation here is reported, not tuned away."""
    q, k, v = tiny
    yd = dense_attention(q, k, v)
    errs = [rel(oracle.monarch_attn(q, k, v, 24, 8, t, 1), yd) for t in (1, 2, 4, 8, 24)]
    assert all(b <= a + 1e-12 for a, b in zip(errs, errs[1:])), errs
    assert errs[-1] < 1e-12


def test_more_iterations_do_not_hurt_on_tiny(tiny):
    q, k, v = tiny
    yd = dense_attention(q, k, v)
    errs = [rel(oracle.monarch_attn(q, k, v, 24, 8, 1, it), yd) for it in (1, 2, 5, 10)]
    assert errs[-1] <= errs[0]


# --------------------------------------------------------------------------
# the sampled-problem entry point agrees with the full pass
# --------------------------------------------------------------------------
@pytest.mark.parametrize("tiles,iters", [(1, 1), (5, 3)])
def test_problem_subset_matches_full(tiny, tiles, iters):
    q, k, v = tiny
    y = oracle.monarch_attn(q, k, v, 24, 8, tiles, iters)
    probs = [(0, 0, 3), (1, tiles - 1, 7), (1, tiles // 2, 0)]
    ys = oracle.monarch_problems(q, k, v, 24, 8, tiles, iters, probs)
    lo = oracle.index_maps(3, 8, 8, 24, 8, tiles)["tile_lo"]
    for bh, g, c in probs:
        rows = np.arange(lo[g], lo[g + 1]) * 8 + c
        assert np.array_equal(ys[bh, rows], y[bh, rows])


def test_oracle_rejects_bad_shapes(tiny):
    q, k, v = tiny
    with pytest.raises(ValueError):
        oracle.monarch_attn(q, k, v, 25, 8, 1)
    with pytest.raises(ValueError):
        oracle.monarch_attn(q, k, v, 24, 8, 25)


def test_golden_regression_rows():
    """Stored oracle values (tests/golden/make_golden.py) guard against unnoticed changes."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle_rows.txt")
    q, k, v = synth.make_inputs(TINY)
    cache = {}
    n = 0
    for line in open(path):
        line = line.split("#")[0].strip()
        if not line:
            continue
        b1, b2, tiles, iters, hh, row, col, val = line.split()
        key = (int(b1), int(b2), int(tiles), int(iters))
        if key not in cache:
            cache[key] = oracle.monarch_attn(q[0], k[0], v[0], *key)
        got = cache[key][int(hh), int(row), int(col)]
        assert abs(got - float(val)) <= 1e-12 * max(1.0, abs(float(val)))
        n += 1
    assert n > 0


# --------------------------------------------------------------------------
# queries of a chunk of frames against a key/value cache (N_q != N_k)
# --------------------------------------------------------------------------
@pytest.fixture(scope="module")
def chunk_and_cache():
    """Queries of the last frame of a 3-frame clip against keys and values of all three
    frames (the cache holds the two earlier ones): f_q = 1, f_k = 3, h = w = 8."""
    q, k, v = synth.make_inputs(TINY)          # [1, 2, 192, 32]: frames of 64 tokens
    return q[0][:, 128:], k[0], v[0]           # queries [2, 64, 32], keys/values [2, 192, 32]


def brute_force_m_kv(L, R, b1, b1k, b2, tiles):
    """M[(u,v),(u',v')] = L_v[u,u'] R_{u',g(u)}[v,v'] as a (b1*b2) x (b1k*b2) matrix."""
    lo = [(g * b1) // tiles for g in range(tiles + 1)]
    M = np.zeros((b1 * b2, b1k * b2))
    for g in range(tiles):
        for u in range(lo[g], lo[g + 1]):
            for v in range(b2):
                for up in range(b1k):
                    M[u * b2 + v, up * b2:(up + 1) * b2] = L[v, u, up] * R[up, g, v, :]
    return M


def test_kv_with_the_clip_itself_is_the_self_attention_oracle(tiny):
    q, k, v = tiny
    for b1, b2, t, it in [(24, 8, 3, 2), (8, 24, 2, 1)]:
        a = oracle.monarch_attn(q, k, v, b1, b2, t, it)
        b = oracle.monarch_attn_kv(q, k, v, b1, b1, b2, t, it)
        assert np.array_equal(a, b)


@pytest.mark.parametrize("iters", [1, 3])
def test_kv_single_token_blocks_are_exact_rectangular_attention(chunk_and_cache, iters):
    """b2 = 1: every R block is 1 x 1 and the L-step is softmax over all N_k keys."""
    q, k, v = chunk_and_cache
    y = oracle.monarch_attn_kv(q, k, v, 64, 192, 1, 1, iters)
    assert rel(y, dense_attention(q, k, v)) < 1e-12


@pytest.mark.parametrize("b1,b1k,b2", [(8, 24, 8), (1, 3, 64), (4, 12, 16)])
def test_kv_one_query_row_per_tile_is_exact_rectangular_attention(chunk_and_cache, b1, b1k, b2):
    """t = b1: each tile holds one query row, so R is that row's exact softmax within
    each key block and L weighs the blocks by their log-sum-exp."""
    q, k, v = chunk_and_cache
    y = oracle.monarch_attn_kv(q, k, v, b1, b1k, b2, b1, 1)
    assert rel(y, dense_attention(q, k, v)) < 1e-12


def test_kv_zero_queries_give_the_mean_of_all_values(chunk_and_cache):
    _, k, v = chunk_and_cache
    q = np.zeros((2, 64, 32))
    y = oracle.monarch_attn_kv(q, k, v, 8, 24, 8, 3, 2)
    assert np.abs(y - v.mean(-2, keepdims=True)).max() < 1e-12


@pytest.mark.parametrize("tiles,iters", [(1, 1), (3, 2)])
def test_kv_brute_force_m_is_row_stochastic_and_reproduces_y(chunk_and_cache, tiles, iters):
    q, k, v = chunk_and_cache
    b1, b1k, b2 = 8, 24, 8
    y, L, R = oracle.monarch_attn_kv(q, k, v, b1, b1k, b2, tiles, iters, factors=True)
    for h in range(q.shape[0]):
        M = brute_force_m_kv(L[h], R[h], b1, b1k, b2, tiles)
        assert (M >= 0).all()
        assert np.abs(M.sum(1) - 1).max() < 1e-12
        assert rel(M @ v[h], y[h]) < 1e-12
