"""Writes the oracle's regression fixtures in this folder (calls only ``oracle/``).

The pages print no worked example with input and output values, so every stored value here
comes from the fp64 oracle, on small integer inputs that are stored beside the results (the
fixture does not depend on a random generator's stability).  ``tests/test_golden_cpu.py``
recomputes each fixture with the oracle: any change to the oracle's arithmetic shows up there
and has to be justified by the passage of the pages it follows.

Usage: python tests/golden/make_golden.py
"""

from __future__ import annotations

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as orc  # noqa: E402

CITATION = ("MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다 — section 무엇과 다른가 "
            "(anchor step: dense attention, query groups, KV tokens by exact probabilities, "
            "R = O_full - O_sparse) and section 어떻게 쓰나 (tile-aligned equal-size groups by "
            "median-split PDDP, token-level KV selection, two-pass exact selection)")

CASES = [
    # name, N, d, C, k, seed
    ("anchor_n16_d4_c4_k5", 16, 4, 4, 5, 3),
    ("anchor_n24_d8_c4_k7", 24, 8, 4, 7, 5),
]


def fixture(name, N, d, C, k, seed):
    rng = np.random.default_rng(seed)
    q, kk, v = (rng.integers(-3, 4, size=(N, d)).astype(np.float64) for _ in range(3))
    scale = orc.default_scale(d)
    res = orc.anchor(q, kk, v, C, k, scale)
    return {
        "name": name,
        "citation": CITATION,
        "written_by": "tests/golden/make_golden.py (oracle only)",
        "N": N, "d": d, "C": C, "k": k, "scale": scale,
        "Q": q.astype(int).tolist(), "K": kk.astype(int).tolist(), "V": v.astype(int).tolist(),
        "perm": [int(x) for x in res["perm"]],
        "idx": [[int(x) for x in row] for row in res["idx"]],
        "lse": [float(x) for x in res["lse"]],
        "O_full": [[float(x) for x in row] for row in res["O_full"]],
        "O_sparse": [[float(x) for x in row] for row in res["O_sparse"]],
    }


def main():
    for case in CASES:
        f = fixture(*case)
        with open(os.path.join(HERE, f["name"] + ".json"), "w") as fh:
            json.dump(f, fh, indent=1)
            fh.write("\n")


if __name__ == "__main__":
    main()
