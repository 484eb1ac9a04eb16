"""The pins catch plausible mistakes: each mutant is a copy of the oracle source
with one planted error, compiled on the CPU in a temporary folder; at least one
pin (textbook attention in degenerate shapes, the Q = 0 mean, the Monarch form,
row-stochasticity, objective ascent) must reject it."""
import os

import numpy as np
import pytest

from oracle import oracle
from structured_attention_video_b200 import synth

from test_oracle_pins import brute_force_m, dense_attention, objective, rel

MUTANTS = {
    "entropy_sign": ("logit[up] = s * acc + H[up];", "logit[up] = s * acc - H[up];"),
    "entropy_dropped": ("logit[up] = s * acc + H[up];", "logit[up] = s * acc;"),
    "no_weight_normalisation": ("qbar[j] = wsum > 0.0 ? qbar[j] / wsum : 0.0;",
                                "qbar[j] = wsum > 0.0 ? qbar[j] : 0.0;"),
    "missing_scale": ("const double s = 1.0 / sqrt((double)d);", "const double s = 1.0;"),
    "key_token_transposed": ("const double *kr = k + ((int64_t)up * b2 + vp) * d;",
                             "const double *kr = k + ((int64_t)vp * b1 + up) * d;"),
    "values_from_keys": ("z += r * v[((int64_t)up * b2 + vp) * d + j];",
                         "z += r * k[((int64_t)up * b2 + vp) * d + j];"),
    "output_from_ktilde": ("acc += L[(size_t)(u - u0) * b1k + up] * Z[(size_t)up * d + j];",
                           "acc += L[(size_t)(u - u0) * b1k + up] * Kt[(size_t)up * d + j];"),
    "query_column_swapped": ("const double *qr = q + ((int64_t)u * b2 + c) * d;\n"
                             "                double mx",
                             "const double *qr = q + ((int64_t)c * b1 + u) * d;\n"
                             "                double mx"),
    "lse_without_log_sum": ("double lse = mx + log(sum);\n                double ent",
                            "double lse = mx;\n                double ent"),
    "tile_end_short": ("u1 = tile_first_row(g + 1, b1, tiles);",
                       "u1 = tile_first_row(g + 1, b1, tiles) - (g + 1 < tiles);"),
}


def pins_pass(lib, q, k, v):
    """The subset of the pins that needs only the forward pass and the factors."""
    qh, kh, vh = q[0], k[0], v[0]
    yd = dense_attention(q, k, v)
    for b1, b2, t in [(1, 192, 1), (192, 1, 3), (24, 8, 24), (3, 64, 3)]:
        if rel(oracle.monarch_attn(q, k, v, b1, b2, t, 1, lib=lib), yd) > 1e-12:
            return False
    y0 = oracle.monarch_attn(np.zeros_like(k), k, v, 24, 8, 3, 1, lib=lib)
    if np.abs(y0 - v.mean(-2, keepdims=True)).max() > 1e-13:
        return False
    for t in (1, 4):
        y, L, R = oracle.monarch_attn(qh, kh, vh, 24, 8, t, 1, factors=True, lib=lib)
        M = brute_force_m(L, R, 24, 8, t)
        if M.min() < 0 or np.abs(M.sum(1) - 1).max() > 1e-12 or rel(y, M @ vh) > 1e-13:
            return False
        prev = -np.inf
        for hs in range(1, 5):
            _, L, R = oracle.monarch_attn(qh, kh, vh, 24, 8, t, half_steps=hs, factors=True,
                                          lib=lib)
            F = objective(brute_force_m(L, R, 24, 8, t), qh, kh)
            if F < prev - 1e-9:
                return False
            prev = F
    return True


@pytest.fixture(scope="module")
def tiny():
    q, k, v = synth.make_inputs(synth.WORKLOADS["tiny"])
    return q[0], k[0], v[0]


def test_unmutated_oracle_passes(tiny):
    assert pins_pass(None, *tiny)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, tiny, name):
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(old) >= 1, "mutation site not found: " + name
    mutated = os.path.join(tmp_path, "mutant.c")
    with open(mutated, "w") as fh:
        fh.write(src.replace(old, new, 1))
    lib = oracle.build(force=True, src=mutated, out=os.path.join(tmp_path, "libmutant.so"))
    assert not pins_pass(lib, *tiny), "pins did not catch mutant " + name
