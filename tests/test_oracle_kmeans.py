"""Pins of the oracle's k-means grouping (the grouping-cost baseline set against Fast PDDP,
"MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다", section 전제와 한계): results fixed
by hand, by construction, or by the defining property of each step."""

import numpy as np

import oracle as orc


def test_hand_worked_example():
    # d = 1, C = 2: block means 5 and 6; one Lloyd step sends 0 and 1 to the first centroid and
    # 10 and 11 to the second (means 0.5 and 10.5); the first cluster then takes 0 and 1
    q = np.array([[0.0], [10.0], [1.0], [11.0]])
    assert np.array_equal(orc.kmeans_groups(q, 2, iters=1), [0, 2, 1, 3])
    # with no Lloyd step the first centroid (5) takes distance 16 (query 2) and then the tie at
    # 25 between queries 0 and 1 goes to the lower index
    assert np.array_equal(orc.kmeans_groups(q, 2, iters=0), [0, 2, 1, 3])
    # both block means are 3: queries 2 and 3 (squared distance 4 each, ties to the lower
    # index) go to the first cluster, 0 and 1 (distance 9) to the second
    q2 = np.array([[6.0], [0.0], [5.0], [1.0]])
    assert np.array_equal(orc.kmeans_groups(q2, 2, iters=0), [2, 3, 0, 1])


def test_partition_invariants():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((32 * 12, 16))
    perm = orc.kmeans_groups(q, 32, iters=3)
    assert np.array_equal(np.sort(perm), np.arange(q.shape[0]))
    groups = perm.reshape(12, 32)
    assert np.all(np.diff(groups, axis=1) > 0)


def test_separated_clusters_are_recovered():
    # two tight clusters of exactly C points at +-10 e_1, interleaved so that each contiguous
    # block (the initial centroids) holds a 70/30 mix: one Lloyd step separates them
    C, d = 40, 8
    rng = np.random.default_rng(5)
    a = 10.0 * np.eye(d)[0] + 0.01 * rng.standard_normal((C, d))
    b = -10.0 * np.eye(d)[0] + 0.01 * rng.standard_normal((C, d))
    rows = [a[i] for i in range(28)] + [b[i] for i in range(12)] + [a[i] for i in range(28, C)] + \
           [b[i] for i in range(12, C)]
    q = np.stack(rows)
    which = np.array([0] * 28 + [1] * 12 + [0] * 12 + [1] * 28)
    perm = orc.kmeans_groups(q, C, iters=2)
    g0, g1 = perm[:C], perm[C:]
    assert set(which[g0]) == {0} and set(which[g1]) == {1}


def test_equal_clusters_in_block_order_are_the_blocks():
    # identical points per block, blocks far apart: the block means are the clusters' exact
    # positions and every step keeps them
    C, G, d = 16, 5, 4
    centers = 100.0 * np.arange(G)[:, None] * np.ones(d)
    q = np.repeat(centers, C, axis=0)
    for it in (0, 1, 4):
        assert np.array_equal(orc.kmeans_groups(q, C, iters=it), np.arange(G * C))


def test_balanced_assignment_property():
    # each group g holds C queries no farther from its final centroid than any query that no
    # earlier group took (ties to the lower index); checked with the centroids the definition
    # gives after the Lloyd steps, recomputed here from the output's own membership rule
    rng = np.random.default_rng(11)
    C, G, d = 8, 6, 3
    q = np.round(rng.standard_normal((C * G, d)) * 4) / 4  # quarter steps: ties happen
    perm = orc.kmeans_groups(q, C, iters=0)
    cent = np.stack([q[g * C:(g + 1) * C].mean(axis=0) for g in range(G)])  # iters = 0: block means
    dist = ((q[:, None, :] - cent[None, :, :]) ** 2).sum(axis=2)
    taken = np.zeros(C * G, dtype=bool)
    for g in range(G):
        mem = perm[g * C:(g + 1) * C]
        rest = np.nonzero(~taken)[0]
        rest = rest[~np.isin(rest, mem)]
        worst_in = max((dist[i, g], i) for i in mem)
        best_out = min(((dist[i, g], i) for i in rest), default=(np.inf, 0))
        assert worst_in < best_out, f"group {g}"
        taken[mem] = True
