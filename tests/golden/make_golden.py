"""Writes tests/golden/tiny_oracle_rows.txt from the float64 oracle alone.

Regression values: they pin nothing by themselves, but any change to the
oracle's arithmetic shows up against them and must then cite its reason.
Run:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import oracle  # noqa: E402
from structured_attention_video_b200 import synth  # noqa: E402

CASES = [(24, 8, 1, 1), (24, 8, 4, 1), (24, 8, 5, 3), (3, 64, 2, 1), (8, 24, 3, 2)]


def main():
    wl = synth.WORKLOADS["tiny"]
    q, k, v = synth.make_inputs(wl)
    rng = np.random.default_rng(2024)
    lines = ["# tiny workload (seed 0), float64 oracle outputs: b1 b2 tiles iters head row col value"]
    for case in CASES:
        y = oracle.monarch_attn(q[0], k[0], v[0], *case)
        for _ in range(6):
            hh, row, col = rng.integers(wl.H), rng.integers(wl.N), rng.integers(wl.d)
            lines.append("%d %d %d %d %d %d %d %.17e" % (case + (hh, row, col, y[hh, row, col])))
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle_rows.txt")
    with open(path, "w") as fh:
        fh.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
