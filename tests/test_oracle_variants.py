"""Pins for the oracle's selection variants (CPU only): block oracle, vanilla BSA and the
per-query oracle of the controlled comparison ("MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를
좁힌다", section 어떻게 동작하나).  Each is checked against something other than itself: a
reduction to another formulation, brute force, a library routine, or the kept-mass ordering
that the definitions imply (a finer selection space can only keep more exact probability)."""

import itertools

import numpy as np
import torch

import oracle as orc


def data(seed, N=64, d=8):
    r = np.random.default_rng(seed)
    q, k, v = (r.standard_normal((N, d)) for _ in range(3))
    return q, k, v


def test_block_oracle_with_unit_blocks_is_the_token_oracle():
    q, k, _ = data(0)
    scale = 0.35
    _, lse = orc.dense(q, k, np.zeros((64, 1)), scale)
    perm = np.arange(64)
    tok = orc.select_topk(orc.group_scores(q, k, perm, 16, lse, scale), 10)
    blk, _ = orc.block_oracle_select(q, k, perm, 16, 1, 10, lse, scale)
    assert np.array_equal(tok, blk)


def test_block_oracle_is_the_best_block_set_by_brute_force():
    q, k, _ = data(1, N=48)
    scale = 0.5
    _, lse = orc.dense(q, k, np.zeros((48, 1)), scale)
    perm = np.random.default_rng(2).permutation(48)
    C, BK, kb = 12, 8, 2
    idx, bs = orc.block_oracle_select(q, k, perm, C, BK, kb, lse, scale)
    for g in range(48 // C):
        rows = perm[g * C:(g + 1) * C]
        P = np.exp(scale * q[rows] @ k.T - lse[rows][:, None])
        best = max(itertools.combinations(range(48 // BK), kb),
                   key=lambda c: (sum(P[:, b * BK:(b + 1) * BK].sum() for b in c), [-x for x in c]))
        assert np.array_equal(idx[g], np.concatenate([np.arange(b * BK, (b + 1) * BK) for b in best]))
        np.testing.assert_allclose(bs[g], P.reshape(C, -1, BK).sum(axis=(0, 2)), rtol=1e-12)


def test_bsa_with_single_queries_and_unit_blocks_is_the_logit_topk():
    q, k, _ = data(3)
    idx, bs = orc.bsa_select(q, k, np.arange(64), 1, 1, 7)
    for i in range(64):
        L = k @ q[i]
        assert np.array_equal(idx[i], np.sort(np.argsort(-L, kind="stable")[:7]))
        np.testing.assert_allclose(bs[i], L, rtol=1e-12)


def test_bsa_pools_by_means():
    q, k, _ = data(4)
    idx, bs = orc.bsa_select(q, k, np.arange(64), 16, 8, 3)
    qbar = q[:16].mean(axis=0)
    kbar = k[8:16].mean(axis=0)
    np.testing.assert_allclose(bs[0, 1], qbar @ kbar, rtol=1e-12)


def test_perquery_full_is_dense_sdpa():
    q, k, v = data(5)
    out = orc.perquery(q, k, v, 64, 0.4)
    ref = torch.nn.functional.scaled_dot_product_attention(*(torch.tensor(x)[None, None] for x in (q, k, v)),
                                                           scale=0.4)[0, 0].numpy()
    np.testing.assert_allclose(out, ref, atol=1e-12)


def test_perquery_is_the_token_oracle_with_single_query_groups():
    q, k, v = data(6)
    scale = 0.3
    _, lse = orc.dense(q, k, np.zeros((64, 1)), scale)
    perm = np.arange(64)
    idx = orc.select_topk(orc.group_scores(q, k, perm, 1, lse, scale), 9)
    np.testing.assert_allclose(orc.perquery(q, k, v, 9, scale), orc.sparse(q, k, v, perm, idx, 1, scale), atol=1e-12)


def test_kept_mass_orders_the_variants():
    # per-query >= token >= block oracle >= BSA at equal density, by the definitions
    for seed in range(4):
        q, k, _ = data(10 + seed, N=128, d=16)
        scale = 0.25
        _, lse = orc.dense(q, k, np.zeros((128, 1)), scale)
        perm = np.arange(128)
        C, BK, kb = 16, 8, 4
        kk = kb * BK
        tok = orc.select_topk(orc.group_scores(q, k, perm, C, lse, scale), kk)
        blk, _ = orc.block_oracle_select(q, k, perm, C, BK, kb, lse, scale)
        bsa, _ = orc.bsa_select(q, k, perm, C, BK, kb)
        pq = orc.select_topk(orc.group_scores(q, k, perm, 1, lse, scale), kk)
        m = [orc.kept_mass(q, k, perm, pq, 1, lse, scale), orc.kept_mass(q, k, perm, tok, C, lse, scale),
             orc.kept_mass(q, k, perm, blk, C, lse, scale), orc.kept_mass(q, k, perm, bsa, C, lse, scale)]
        assert m[0] >= m[1] - 1e-12 and m[1] >= m[2] - 1e-12 and m[2] >= m[3] - 1e-12, m
        assert 0.0 < m[3] and m[0] <= 1.0 + 1e-12
