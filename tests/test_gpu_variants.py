"""Selection variants of the controlled oracle comparison against the fp64 oracle
("MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다", section 어떻게 동작하나): block oracle
and vanilla BSA block selections (exact outside a certified rounding band, emitted as whole
ascending blocks), the per-query oracle's outputs (bf16 tolerances), and the kept-mass ordering
per-query >= token >= block oracle >= BSA on the GPU's own selections."""

import math

import numpy as np
import pytest
import torch

import oracle as orc
from free_sparse_attention_reuse_b200 import api, workload
from helpers import MAX_ABS_TOL, REL_FROB_TOL, assert_close, check_selection

pytestmark = pytest.mark.gpu

CASES = [  # (H, d, grid, C, BK, kb)
    (2, 64, (4, 16, 16), 64, 64, 4),
    (2, 128, (2, 16, 32), 128, 128, 3),
]


def setup(H, d, grid, C, seed):
    wl = workload.custom(f"var{seed}", 1, H, d, grid, C, index=50 + seed)
    Q, K, V = workload.Generator(wl).current()
    return wl, Q, K, V


def head(t, h):
    return t[0, h].double().numpy()


def blocks_of(idx_row, BK):
    b = idx_row.reshape(-1, BK)
    assert np.all(b == b[:, :1] + np.arange(BK)), "not whole blocks"
    assert np.all(b[:, 0] % BK == 0)
    return b[:, 0] // BK


def band(bs, kb, rel, absolute=0.0):
    taus = np.sort(bs, axis=1)[:, ::-1][:, kb - 1]
    eps = 2 * (np.abs(taus) * rel + absolute)
    return taus, eps


@pytest.mark.parametrize("case", range(len(CASES)))
def test_block_oracle_and_bsa(case):
    H, d, grid, C, BK, kb = CASES[case]
    wl, Q, K, V = setup(H, d, grid, C, case)
    N = wl.N
    scale = 1.0 / math.sqrt(d)
    Qd, Kd = Q.cuda(), K.cuda()
    perm = api.group(Qd, C)
    _, lse = api.dense_attn(Qd, Kd, Kd, want_out=False)
    io = api.select_blocks(Qd, Kd, perm, C, BK, kb, "oracle", lse=lse)
    ib = api.select_blocks(Qd, Kd, perm, C, BK, kb, "bsa")
    api.sync_status()
    P, IO, IB = perm.cpu().numpy()[0], io.cpu().numpy()[0], ib.cpu().numpy()[0]
    assert IO.shape == (H, N // C, kb * BK) and IB.shape == IO.shape
    swaps = 0
    for h in range(H):
        q, k = head(Q, h), head(K, h)
        _, lse64 = orc.dense(q, k, np.zeros((N, 1)), scale)
        _, bs_o = orc.block_oracle_select(q, k, P[h], C, BK, kb, lse64, scale)
        dot_abs = (np.abs(q) @ np.abs(k).T).max() * scale
        rel = 2 * d * 2.0 ** -24 * dot_abs + 2.0 ** -20 + (C + 4) * 2.0 ** -22 + BK * 2.0 ** -23
        taus, eps = band(bs_o, kb, rel)
        swaps += check_selection(np.stack([blocks_of(r, BK) for r in IO[h]]), bs_o, taus, eps, kb)
        _, bs_b = orc.bsa_select(q, k, P[h], C, BK, kb)
        G = N // C
        qbar = np.stack([q[P[h][g * C:(g + 1) * C]].mean(axis=0) for g in range(G)])
        kbar = k.reshape(N // BK, BK, d).mean(axis=1)
        absb = (np.abs(qbar) @ np.abs(kbar).T).max(axis=1)
        taus, _ = band(bs_b, kb, 0.0)
        eps = 2 * (C + BK + d + 4) * 2.0 ** -24 * absb
        swaps += check_selection(np.stack([blocks_of(r, BK) for r in IB[h]]), bs_b, taus, eps, kb)
    print(f"case {case}: swaps inside the band: {swaps}")


@pytest.mark.parametrize("H,d,grid,k", [(2, 64, (4, 16, 16), 256), (1, 128, (2, 16, 16), 100)])
def test_perquery_attention(H, d, grid, k):
    wl, Q, K, V = setup(H, d, grid, 64, 7)
    out = api.perquery_attn(Q.cuda(), K.cuda(), V.cuda(), k)
    api.sync_status()
    scale = 1.0 / math.sqrt(d)
    ref = np.stack([orc.perquery(head(Q, h), head(K, h), head(V, h), k, scale) for h in range(H)])[None]
    assert_close(out, ref, "per-query oracle")


def test_perquery_full_density_is_dense():
    wl, Q, K, V = setup(2, 64, (4, 16, 16), 64, 8)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    a = api.perquery_attn(Qd, Kd, Vd, wl.N)
    b, _ = api.dense_attn(Qd, Kd, Vd, want_lse=False)
    api.sync_status()
    d = (a.float() - b.float()).abs().max().item()
    assert d <= MAX_ABS_TOL, d


def test_kept_mass_ordering_on_gpu_selections():
    H, d, grid, C, BK, kb = 2, 64, (4, 16, 16), 64, 64, 4
    wl, Q, K, V = setup(H, d, grid, C, 9)
    N, k = wl.N, kb * BK
    Qd, Kd = Q.cuda(), K.cuda()
    ident = torch.arange(N, dtype=torch.int32, device="cuda").repeat(1, H, 1).contiguous()
    _, lse = api.dense_attn(Qd, Kd, Kd, want_out=False)
    tok = api.select(Qd, Kd, ident, C, k, lse=lse).cpu().numpy()[0]
    blk = api.select_blocks(Qd, Kd, ident, C, BK, kb, "oracle", lse=lse).cpu().numpy()[0]
    bsa = api.select_blocks(Qd, Kd, ident, C, BK, kb, "bsa").cpu().numpy()[0]
    api.sync_status()
    scale = 1.0 / math.sqrt(d)
    for h in range(H):
        q, kk = head(Q, h), head(K, h)
        _, lse64 = orc.dense(q, kk, np.zeros((N, 1)), scale)
        perm = np.arange(N)
        pq = orc.select_topk(orc.group_scores(q, kk, perm, 1, lse64, scale), k)
        m = [orc.kept_mass(q, kk, perm, pq, 1, lse64, scale), orc.kept_mass(q, kk, perm, tok[h], C, lse64, scale),
             orc.kept_mass(q, kk, perm, blk[h], C, lse64, scale), orc.kept_mass(q, kk, perm, bsa[h], C, lse64, scale)]
        tol = 1e-5  # selections inside the rounding band may differ by a near-tie
        assert m[0] >= m[1] - tol and m[1] >= m[2] - tol and m[2] >= m[3] - tol, m


def test_block_selection_edge_cases():
    # kb = N/BK takes every block (the whole key range); kb = 1 one block; both methods
    H, d, grid, C, BK = 2, 64, (4, 16, 16), 64, 64
    wl, Q, K, V = setup(H, d, grid, C, 11)
    N = wl.N
    Qd, Kd = Q.cuda(), K.cuda()
    perm = api.group(Qd, C)
    for method in ("oracle", "bsa"):
        full = api.select_blocks(Qd, Kd, perm, C, BK, N // BK, method)
        one = api.select_blocks(Qd, Kd, perm, C, BK, 1, method)
        api.sync_status()
        assert torch.equal(full, torch.arange(N, dtype=torch.int32, device="cuda").expand_as(full))
        o = one.cpu().numpy()
        assert np.all(o % BK == np.arange(BK)) and np.all(np.diff(o, axis=-1) == 1)


def test_variant_arguments_are_rejected():
    wl, Q, K, V = setup(2, 64, (4, 16, 16), 64, 12)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    perm = api.group(Qd, 64)
    for BK, kb in ((32, 4), (64, 0), (64, 17), (96, 2)):  # BK < 64, kb out of range, N % BK != 0
        with pytest.raises(api._lib.MCSError):
            api.select_blocks(Qd, Kd, perm, 64, BK, kb, "oracle")
    with pytest.raises(api._lib.MCSError):
        api.perquery_attn(Qd, Kd, Vd, 0)
    api.sync_status()


def test_perquery_single_key_is_the_argmax_value():
    wl, Q, K, V = setup(1, 64, (2, 16, 16), 64, 13)
    out = api.perquery_attn(Q.cuda(), K.cuda(), V.cuda(), 1)
    api.sync_status()
    q, k, v = head(Q, 0), head(K, 0), head(V, 0)
    j = np.argmax(q @ k.T, axis=1)  # ties to the lower key, as the selection rule
    ref = v[j][None, None]
    assert_close(out, ref, "per-query k=1")
