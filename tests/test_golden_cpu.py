"""Oracle regression fixtures in tests/golden (written by tests/golden/make_golden.py, which
calls only the oracle).  Each fixture is recomputed by the oracle (groups and indices equal,
floats to 1e-12), and its stored floats are re-derived from their definitions in plain Python
(math.exp over lists: no NumPy, no oracle), so a stored value never rests on the oracle alone.
"""

import glob
import json
import math
import os

import numpy as np
import pytest

import oracle as orc

HERE = os.path.dirname(os.path.abspath(__file__))
FIXTURES = sorted(glob.glob(os.path.join(HERE, "golden", "*.json")))


def load(path):
    with open(path) as fh:
        return json.load(fh)


def test_fixtures_present():
    assert FIXTURES, "no golden fixtures"


@pytest.mark.parametrize("path", FIXTURES, ids=[os.path.basename(p) for p in FIXTURES])
def test_oracle_reproduces_fixture(path):
    f = load(path)
    q, k, v = (np.array(f[n], dtype=np.float64) for n in ("Q", "K", "V"))
    res = orc.anchor(q, k, v, f["C"], f["k"], f["scale"])
    assert res["perm"].tolist() == f["perm"]
    assert res["idx"].tolist() == f["idx"]
    np.testing.assert_allclose(res["lse"], f["lse"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["O_full"], f["O_full"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(res["O_sparse"], f["O_sparse"], rtol=0, atol=1e-12)


def _softmax_rows(q_row, keys, vals, scale):
    logits = [scale * sum(a * b for a, b in zip(q_row, kr)) for kr in keys]
    m = max(logits)
    w = [math.exp(x - m) for x in logits]
    z = sum(w)
    out = [sum(wj * vr[c] for wj, vr in zip(w, vals)) / z for c in range(len(vals[0]))]
    return out, m + math.log(z)


@pytest.mark.parametrize("path", FIXTURES, ids=[os.path.basename(p) for p in FIXTURES])
def test_fixture_floats_from_definitions(path):
    f = load(path)
    Q, K, V, C = f["Q"], f["K"], f["V"], f["C"]
    N = len(Q)
    # groups: an equal-size partition, each leaf listed in ascending query order
    assert sorted(f["perm"]) == list(range(N))
    for g in range(N // C):
        leaf = f["perm"][g * C:(g + 1) * C]
        assert leaf == sorted(leaf)
    for row in f["idx"]:
        assert row == sorted(set(row)) and len(row) == f["k"] and 0 <= row[0] and row[-1] < N
    for i in range(N):
        o, lse = _softmax_rows(Q[i], K, V, f["scale"])
        assert abs(lse - f["lse"][i]) < 1e-12
        assert max(abs(a - b) for a, b in zip(o, f["O_full"][i])) < 1e-12
    for g, cols in enumerate(f["idx"]):
        for i in f["perm"][g * C:(g + 1) * C]:
            o, _ = _softmax_rows(Q[i], [K[j] for j in cols], [V[j] for j in cols], f["scale"])
            assert max(abs(a - b) for a, b in zip(o, f["O_sparse"][i])) < 1e-12


@pytest.mark.parametrize("path", FIXTURES, ids=[os.path.basename(p) for p in FIXTURES])
def test_fixture_indices_are_the_largest_group_probabilities(path):
    # each group's k keys carry the largest summed exact probabilities (ties to the lower key),
    # checked against plain-Python probabilities from the stored LSE
    f = load(path)
    Q, K, C, kk, scale = f["Q"], f["K"], f["C"], f["k"], f["scale"]
    for g, cols in enumerate(f["idx"]):
        rows = f["perm"][g * C:(g + 1) * C]
        score = [sum(math.exp(scale * sum(a * b for a, b in zip(Q[i], K[j])) - f["lse"][i]) for i in rows)
                 for j in range(len(K))]
        chosen = sorted(range(len(K)), key=lambda j: (-score[j], j))[:kk]
        assert sorted(chosen) == cols
