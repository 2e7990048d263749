"""Pins for the fp64 oracle against facts the pages and the mathematics fix (CPU only).

Each test checks one function of ``oracle.mcs_oracle`` against something other than itself:
a closed form, an invariant the method guarantees, an independent library routine, or brute
force on a tiny input.  A plausible mistake in the oracle (a dropped term, a wrong sign or
index, an uncentered PDDP, a wrong split rank, a wrong tie rule) fails at least one of them.
"""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle as orc


def rng(seed):
    return np.random.default_rng(seed)


def bf16_round(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).double().numpy()


# ---------------------------------------------------------------- dense attention
def test_dense_matches_torch_sdpa():
    r = rng(0)
    q, k, v = (r.standard_normal((300, 32)) for _ in range(3))
    scale = 0.3
    o, lse = orc.dense(q, k, v, scale, block=128)
    tq, tk, tv = (torch.from_numpy(x)[None, None] for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale)[0, 0].numpy()
    ref_lse = torch.logsumexp(torch.from_numpy(scale * q @ k.T), dim=1).numpy()
    assert np.abs(o - ref).max() < 1e-12
    assert np.abs(lse - ref_lse).max() < 1e-12


def test_dense_identical_keys_closed_form():
    # all keys equal: attention is uniform, O_i = mean_j v_j, LSE_i = log N + scale q_i.k
    r = rng(1)
    N, d = 200, 16
    q = r.standard_normal((N, d))
    k = np.tile(r.standard_normal(d), (N, 1))
    v = r.standard_normal((N, 8))
    scale = 0.25
    o, lse = orc.dense(q, k, v, scale)
    assert np.abs(o - v.mean(axis=0)).max() < 1e-12
    assert np.abs(lse - (math.log(N) + scale * q @ k[0])).max() < 1e-12


def test_dense_one_hot_keys_closed_form():
    # q = t e_0, keys e_0 and 0: two-way softmax with a logistic weight
    q = np.array([[2.0, 0.0], [-1.0, 0.0]])
    k = np.array([[1.0, 0.0], [0.0, 0.0]])
    v = np.array([[1.0], [0.0]])
    o, lse = orc.dense(q, k, v, 1.0)
    for i, t in enumerate((2.0, -1.0)):
        assert abs(o[i, 0] - 1 / (1 + math.exp(-t))) < 1e-15
        assert abs(lse[i] - math.log(math.exp(t) + 1)) < 1e-15


# ---------------------------------------------------------------- sparse attention
def _random_metadata(r, N, C, kk):
    perm = r.permutation(N)
    G = N // C
    for g in range(G):
        perm[g * C:(g + 1) * C] = np.sort(perm[g * C:(g + 1) * C])
    idx = np.stack([np.sort(r.choice(N, kk, replace=False)) for _ in range(G)])
    return perm, idx


def test_sparse_equals_masked_dense_sdpa():
    # second formulation: dense attention with -inf on unselected keys (torch routine)
    r = rng(2)
    N, d, C, kk = 128, 16, 16, 20
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    perm, idx = _random_metadata(r, N, C, kk)
    scale = 1 / 4
    o = orc.sparse(q, k, v, perm, idx, C, scale)
    mask = torch.zeros(N, N, dtype=torch.bool)
    for g in range(N // C):
        rows = torch.from_numpy(perm[g * C:(g + 1) * C])
        mask[rows[:, None], torch.from_numpy(idx[g])[None, :]] = True
    t = [torch.from_numpy(x)[None, None] for x in (q, k, v)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t, attn_mask=mask, scale=scale)[0, 0]
    assert np.abs(o - ref.numpy()).max() < 1e-12


def test_sparse_full_density_is_dense_and_residual_zero():
    r = rng(3)
    N, d, C = 96, 8, 32
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    res = orc.anchor(q, k, v, C, N, 0.5)
    assert np.array_equal(res["idx"], np.tile(np.arange(N), (N // C, 1)))
    assert np.abs(res["O_sparse"] - res["O_full"]).max() < 1e-12
    assert np.abs(res["R"]).max() < 1e-12


def test_anchor_identity_and_reuse_on_anchor_inputs():
    r = rng(4)
    N, d, C, kk = 128, 16, 32, 24
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    res = orc.anchor(q, k, v, C, kk, 0.25)
    assert np.abs(res["O_sparse"] + res["R"] - res["O_full"]).max() < 1e-12
    o_hat = orc.reuse(q, k, v, res["perm"], res["idx"], res["R"], C, 0.25)
    assert np.abs(o_hat - res["O_full"]).max() < 1e-12
    # and R is not trivially zero at this density
    assert np.abs(res["R"]).max() > 1e-3


# ---------------------------------------------------------------- selection (pass 2 + top-k)
def test_group_scores_sum_to_group_size():
    # each query's exact probabilities sum to 1, so a group's scores sum to C
    r = rng(5)
    N, d, C = 160, 16, 32
    q, k = r.standard_normal((N, d)), r.standard_normal((N, d))
    perm = r.permutation(N)
    _, lse = orc.dense(q, k, np.zeros((N, 1)), 0.7)
    s = orc.group_scores(q, k, perm, C, lse, 0.7)
    assert np.abs(s.sum(axis=1) - C).max() < 1e-11
    assert (s > 0).all()


def test_group_scores_match_torch_softmax_column_sums():
    r = rng(6)
    N, d, C = 64, 8, 16
    q, k = r.standard_normal((N, d)), r.standard_normal((N, d))
    perm = r.permutation(N)
    _, lse = orc.dense(q, k, np.zeros((N, 1)), 0.5)
    s = orc.group_scores(q, k, perm, C, lse, 0.5)
    P = torch.softmax(torch.from_numpy(0.5 * q @ k.T), dim=1).numpy()
    for g in range(N // C):
        assert np.abs(s[g] - P[perm[g * C:(g + 1) * C]].sum(axis=0)).max() < 1e-13


def test_topk_matches_brute_force_with_ties():
    r = rng(7)
    for trial in range(40):
        n = int(r.integers(1, 24))
        kk = int(r.integers(1, n + 1))
        scores = r.integers(0, 4, size=(3, n)).astype(float)  # many exact ties
        got = orc.select_topk(scores, kk)
        for g in range(3):
            brute = sorted(range(n), key=lambda j: (-scores[g, j], j))[:kk]
            assert list(got[g]) == sorted(brute)


def test_topk_uniform_and_full():
    s = np.full((2, 10), 0.1)
    assert np.array_equal(orc.select_topk(s, 4), np.tile(np.arange(4), (2, 1)))
    s = rng(8).random((2, 10))
    assert np.array_equal(orc.select_topk(s, 10), np.tile(np.arange(10), (2, 1)))


def test_selection_picks_largest_probability_keys_exhaustively():
    # brute force over all k-subsets on a tiny head: the chosen set maximises captured mass
    r = rng(9)
    N, d, C, kk = 8, 4, 4, 3
    q, k = r.standard_normal((N, d)), r.standard_normal((N, d))
    perm = np.arange(N)
    _, lse = orc.dense(q, k, np.zeros((N, 1)), 1.0)
    s = orc.group_scores(q, k, perm, C, lse, 1.0)
    idx = orc.select_topk(s, kk)
    for g in range(N // C):
        best = max(itertools.combinations(range(N), kk), key=lambda S: sum(s[g, j] for j in S))
        assert tuple(idx[g]) == tuple(sorted(best))


# ---------------------------------------------------------------- PDDP grouping
def _check_partition(perm, N, C):
    assert sorted(perm.tolist()) == list(range(N))
    for g in range(N // C):
        grp = perm[g * C:(g + 1) * C]
        assert np.all(np.diff(grp) > 0)


@pytest.mark.parametrize("N,C", [(64, 8), (96, 8), (252 * 4, 4), (1024, 64)])
def test_pddp_partition_invariants(N, C):
    q = bf16_round(rng(10).standard_normal((N, 16)))
    perm = orc.pddp_groups(q, C)
    _check_partition(perm, N, C)


def test_pddp_collinear_is_rank_blocks():
    # q_i = t_i u + c with distinct t: every split is a sort by t, so groups are rank blocks
    r = rng(11)
    N, C, d = 96, 8, 6
    t = r.permutation(N).astype(float) - 40
    u = np.array([3.0, -1, 2, 0, 1, -2])  # largest component positive: v = +u/|u|
    c = np.array([1.0, 2, -3, 4, 0, 5])
    q = t[:, None] * u[None, :] + c[None, :]
    perm = orc.pddp_groups(q, C)
    ranks = np.argsort(t, kind="stable")
    for g in range(N // C):
        assert np.array_equal(perm[g * C:(g + 1) * C], np.sort(ranks[g * C:(g + 1) * C]))


def test_pddp_sign_rule_orders_children():
    # collinear along u whose largest-magnitude component is negative: v = -u/|u|, so the
    # left child gets the largest t
    N, C = 32, 8
    t = np.arange(N, dtype=float)
    u = np.array([1.0, -4.0, 2.0])
    q = t[:, None] * u[None, :]
    perm = orc.pddp_groups(q, C)
    assert np.array_equal(perm[:C], np.arange(N - C, N))


def test_pddp_centering_matters():
    # large offset along e0, spread along e1: the centered principal direction is e1
    r = rng(12)
    N = 64
    q = np.zeros((N, 3))
    q[:, 0] = 100.0 + 0.01 * r.standard_normal(N)
    q[:, 1] = np.linspace(-5, 5, N)
    q[:, 2] = 0.01 * r.standard_normal(N)
    left, right, v, _ = orc.split_node(q, np.arange(N), 2, 32)
    assert abs(abs(v[1]) - 1) < 1e-6 and v[1] > 0
    assert np.array_equal(left, np.arange(32)) and np.array_equal(right, np.arange(32, 64))


def test_pddp_split_rank_is_floor_half():
    # m = 3: the left child gets floor(3/2) * C queries.  A far cluster of C points on the low
    # side becomes leaf 0; the 2C points spread along y split by y into leaves 1 and 2.
    r = rng(13)
    C = 16
    far = np.column_stack([-100 + 0.01 * r.standard_normal(C), 0.01 * r.standard_normal(C)])
    y = r.permutation(2 * C).astype(float) * 3 - 48
    near = np.column_stack([0.01 * r.standard_normal(2 * C), y])
    q = np.vstack([near, far])  # far cluster has the highest ids
    perm = orc.pddp_groups(q, C)
    far_ids = np.arange(2 * C, 3 * C)
    assert np.array_equal(perm[:C], far_ids)
    lo = np.sort(np.argsort(y)[:C])
    hi = np.sort(np.argsort(y)[C:])
    rest = [perm[C:2 * C], perm[2 * C:]]
    assert any(np.array_equal(rest[0], a) and np.array_equal(rest[1], b) for a, b in ((lo, hi), (hi, lo)))


def test_pddp_two_clusters_root_split():
    r = rng(14)
    N, C, d = 128, 8, 8
    centers = np.zeros((2, d))
    centers[0, 2], centers[1, 2] = -20, 20
    lab = r.permutation(np.repeat([0, 1], N // 2))
    q = centers[lab] + r.standard_normal((N, d))
    perm = orc.pddp_groups(q, C)
    first = set(perm[: N // 2].tolist())
    assert first in (set(np.flatnonzero(lab == 0).tolist()), set(np.flatnonzero(lab == 1).tolist()))


def test_power_iteration_matches_eigh_with_large_gap():
    r = rng(15)
    N, d = 400, 12
    scales = np.array([10.0] + [1.0] * (d - 1))
    q = r.standard_normal((N, d)) * scales
    Q, _ = np.linalg.qr(r.standard_normal((d, d)))
    x = q @ Q.T
    xc = x - x.mean(axis=0)
    v = orc.principal_direction(xc)
    w, U = np.linalg.eigh(xc.T @ xc)
    assert w[-1] / w[-2] > 10
    top = U[:, -1] * np.sign(U[np.argmax(np.abs(U[:, -1])), -1])
    assert np.abs(v - top).max() < 1e-9


def test_pddp_identical_queries_split_by_index():
    # X_c = 0: v is kept, every projection is 0 and ties go to the lower index
    q = np.ones((24, 4))
    perm = orc.pddp_groups(q, 4)
    assert np.array_equal(perm, np.arange(24))


def test_pddp_projection_split_is_a_median_cut():
    # every split sends the floor(m/2)*C smallest projections left (checked directly)
    r = rng(16)
    N, C = 80, 8
    q = r.standard_normal((N, 5))
    members = np.arange(N)
    left, right, v, p = orc.split_node(q, members, 10, C)
    assert len(left) == 5 * C
    assert p[left].max() <= p[right].min()
