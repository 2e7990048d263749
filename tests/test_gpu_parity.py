"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200).

Bars: perm bit-exact; idx bit-exact on lattice inputs and exact outside a certified rounding
band elsewhere; bf16 outputs within max-abs 2e-2 and relative Frobenius 1e-2.
"""

import math

import numpy as np
import pytest
import torch

import oracle as orc
from free_sparse_attention_reuse_b200 import api, workload
from helpers import (assert_close, check_selection, oracle_anchor, scale_of, selection_band, to64)

pytestmark = pytest.mark.gpu

DEV = "cuda"


def dev(*ts):
    return [t.to(DEV).contiguous() for t in ts]


def small(name, H, d, grid, C, index=20):
    return workload.custom(name, 1, H, d, grid, C, index=index)


# ---------------------------------------------------------------- dense attention
@pytest.mark.parametrize("H,d,N", [(2, 64, 1024), (2, 128, 1000), (1, 128, 130), (3, 64, 77)])
def test_dense_matches_oracle(H, d, N):
    g = torch.Generator().manual_seed(N + d)
    Q, K, V = (torch.randn(1, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    Qd, Kd, Vd = dev(Q, K, V)
    O, lse = api.dense_attn(Qd, Kd, Vd)
    api.sync_status()
    q, k, v = to64(Q), to64(K), to64(V)
    for h in range(H):
        o_ref, lse_ref = orc.dense(q[0, h], k[0, h], v[0, h], scale_of(d))
        assert_close(O[0, h], o_ref, f"dense head {h}")
        assert np.abs(to64(lse[0, h]) - lse_ref).max() < 2e-3


def test_dense_lse_only_matches_full():
    Q, K, V = dev(*workload.make_qkv(workload.WORKLOADS["tiny"]))
    _, lse_a = api.dense_attn(Q, K, V)
    _, lse_b = api.dense_attn(Q, K, V, want_out=False)
    api.sync_status()
    assert torch.equal(lse_a, lse_b)


# ---------------------------------------------------------------- grouping
@pytest.mark.parametrize("H,d,grid,C", [
    (2, 64, (4, 16, 16), 64),     # the Tiny shape: G = 16
    (2, 128, (3, 8, 16), 128),    # G = 3 (odd split at the root)
    (1, 128, (12, 8, 16), 128),   # G = 12
    (1, 64, (31, 8, 8), 64),      # G = 31
])
def test_group_bit_exact(H, d, grid, C):
    wl = small("g", H, d, grid, C)
    Q, _, _ = workload.make_qkv(wl)
    perm = api.group(dev(Q)[0], C)
    api.sync_status()
    q = to64(Q)
    for h in range(H):
        ref = orc.pddp_groups(q[0, h], C)
        got = perm[0, h].cpu().numpy()
        assert np.array_equal(got, ref), f"head {h}: {np.count_nonzero(got != ref)} positions differ"


def test_group_identical_queries_index_order():
    Q = torch.ones(1, 1, 512, 64, dtype=torch.bfloat16)
    perm = api.group(dev(Q)[0], 64)
    api.sync_status()
    assert np.array_equal(perm[0, 0].cpu().numpy(), np.arange(512))


# ---------------------------------------------------------------- selection
def test_select_lattice_bit_exact():
    # queries replicated within each group: the score order is the order of exact logits
    C, G, d, k = 64, 8, 64, 100
    N = C * G
    g = torch.Generator().manual_seed(7)
    base = torch.randint(-2, 3, (1, 1, G, d), generator=g)
    Q = base.repeat_interleave(C, dim=2).to(torch.bfloat16)
    K = torch.randint(-2, 3, (1, 1, N, d), generator=g).to(torch.bfloat16)
    perm = torch.arange(N, dtype=torch.int32).reshape(1, 1, N)
    Qd, Kd, pd = dev(Q, K, perm)
    idx = api.select(Qd, Kd, pd, C, k)
    api.sync_status()
    q, kk = to64(Q)[0, 0], to64(K)[0, 0]
    _, lse = orc.dense(q, kk, np.zeros((N, 1)), 1 / 8)
    ref = orc.select_topk(orc.group_scores(q, kk, perm[0, 0].numpy(), C, lse, 1 / 8), k)
    assert np.array_equal(idx[0, 0].cpu().numpy(), ref)


@pytest.mark.parametrize("d,C,k", [(64, 64, 256), (128, 128, 200), (128, 64, 1)])
def test_select_certified(d, C, k):
    wl = small("s", 2, d, (4, 16, 16), C)
    Q, K, _ = workload.make_qkv(wl)
    q, kk = to64(Q), to64(K)
    perm = np.stack([orc.pddp_groups(q[0, h], C) for h in range(2)])[None].astype(np.int32)
    Qd, Kd, pd = dev(Q, K, torch.from_numpy(perm))
    idx = api.select(Qd, Kd, pd, C, k).cpu().numpy()
    api.sync_status()
    total = 0
    for h in range(2):
        _, lse = orc.dense(q[0, h], kk[0, h], np.zeros((q.shape[2], 1)), scale_of(d))
        scores, taus, eps = selection_band(q[0, h], kk[0, h], perm[0, h], C, k, lse, scale_of(d))
        total += check_selection(idx[0, h], scores, taus, eps, k)
    print(f"selection swaps inside the band: {total}")


# ---------------------------------------------------------------- sparse attention
@pytest.mark.parametrize("d,C,k", [(64, 64, 256), (128, 128, 200), (128, 64, 1), (64, 128, 1024)])
def test_sparse_and_residual_match_oracle(d, C, k):
    wl = small("p", 2, d, (4, 16, 16), C)
    gen = workload.Generator(wl)
    Q, K, V = gen.current()
    res = oracle_anchor(Q, K, V, C, k)
    perm = torch.from_numpy(res["perm"].astype(np.int32))
    idx = torch.from_numpy(res["idx"].astype(np.int32))
    Qd, Kd, Vd, pd, id_ = dev(Q, K, V, perm, idx)
    O_full = torch.from_numpy(res["O_full"]).to(torch.bfloat16).to(DEV)
    # residual on the anchor's own inputs
    R = api.residual(Qd, Kd, Vd, pd, C, id_, O_full)
    api.sync_status()
    ref_R = to64(O_full.cpu()) - res["O_sparse"]
    assert_close(R, ref_R, "residual", norm_ref=res["O_full"])
    # reuse step on perturbed inputs with the oracle's residual
    Q2, K2, V2 = gen.advance()
    Rb = torch.from_numpy(res["R"]).to(torch.bfloat16)
    out = api.sparse_attn(*dev(Q2, K2, V2), pd, C, id_, R=dev(Rb)[0])
    api.sync_status()
    q2, k2, v2 = to64(Q2), to64(K2), to64(V2)
    ref = np.stack([orc.reuse(q2[0, h], k2[0, h], v2[0, h], res["perm"][0, h], res["idx"][0, h], res["R"][0, h],
                              C, scale_of(d)) for h in range(2)])[None]
    assert_close(out, ref, "reuse")
    # no residual: pure sparse attention
    out0 = api.sparse_attn(*dev(Q2, K2, V2), pd, C, id_)
    api.sync_status()
    assert_close(out0, ref - res["R"], "sparse")


def test_sparse_full_density_equals_dense():
    wl = small("f", 2, 128, (2, 8, 16), 128)
    Q, K, V = dev(*workload.make_qkv(wl))
    N = Q.shape[2]
    perm = torch.arange(N, dtype=torch.int32, device=DEV).repeat(1, 2, 1)
    idx = torch.arange(N, dtype=torch.int32, device=DEV).repeat(1, 2, N // 128, 1)
    out = api.sparse_attn(Q, K, V, perm, 128, idx)
    O, _ = api.dense_attn(Q, K, V)
    api.sync_status()
    assert (out.float() - O.float()).abs().max().item() < 2e-2


# ---------------------------------------------------------------- the whole anchor + reuse
def test_anchor_tiny_end_to_end():
    wl = workload.WORKLOADS["tiny"]
    gen = workload.Generator(wl)
    Q, K, V = gen.current()
    C, k = wl.C, wl.k(0.25)
    res = oracle_anchor(Q, K, V, C, k)
    Qd, Kd, Vd = dev(Q, K, V)
    O_full, perm, idx, R = api.anchor(Qd, Kd, Vd, C, k)
    api.sync_status()
    assert np.array_equal(perm.cpu().numpy(), res["perm"])
    assert_close(O_full, res["O_full"], "O_full")
    q, kk = to64(Q), to64(K)
    for h in range(wl.H):
        scores, taus, eps = selection_band(q[0, h], kk[0, h], res["perm"][0, h], C, k, res["lse"][0, h],
                                           scale_of(wl.d))
        swaps = check_selection(idx[0, h].cpu().numpy(), scores, taus, eps, k)
        assert swaps == 0
    # the KV indices of the Tiny configuration are the oracle's, bit for bit
    assert np.array_equal(idx.cpu().numpy(), res["idx"])
    # reuse on the anchor's own inputs reproduces the dense output
    again = api.sparse_attn(Qd, Kd, Vd, perm, C, idx, R=R)
    api.sync_status()
    assert_close(again, res["O_full"], "anchor replay")
    # three reuse steps against the oracle fed the GPU's metadata
    for _ in range(3):
        Q2, K2, V2 = gen.advance()
        out = api.sparse_attn(*dev(Q2, K2, V2), perm, C, idx, R=R)
        api.sync_status()
        q2, k2, v2 = to64(Q2), to64(K2), to64(V2)
        Rg = to64(R)
        ref = np.stack([orc.reuse(q2[0, h], k2[0, h], v2[0, h], perm[0, h].cpu().numpy(), idx[0, h].cpu().numpy(),
                                  Rg[0, h], C, scale_of(wl.d)) for h in range(wl.H)])[None]
        assert_close(out, ref, "reuse step")


@pytest.mark.parametrize("d,C,k", [(64, 64, 21), (128, 128, 77)])
def test_anchor_single_group(d, C, k):
    # N = C: one group per head, so the PDDP tree has no level and the group is the identity;
    # the selection ranks every key of the head for that one group
    N, H = C, 2
    g = torch.Generator().manual_seed(C + k)
    Q, K, V = (torch.randn(1, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    res = oracle_anchor(Q, K, V, C, k)
    Qd, Kd, Vd = dev(Q, K, V)
    O_full, perm, idx, R = api.anchor(Qd, Kd, Vd, C, k)
    api.sync_status()
    assert np.array_equal(perm.cpu().numpy(), np.tile(np.arange(N), (1, H, 1)))
    assert np.array_equal(perm.cpu().numpy(), res["perm"])
    assert_close(O_full, res["O_full"], "O_full")
    q, kk = to64(Q), to64(K)
    for h in range(H):
        scores, taus, eps = selection_band(q[0, h], kk[0, h], res["perm"][0, h], C, k, res["lse"][0, h], scale_of(d))
        check_selection(idx[0, h].cpu().numpy(), scores, taus, eps, k)
    again = api.sparse_attn(Qd, Kd, Vd, perm, C, idx, R=R)
    api.sync_status()
    assert_close(again, res["O_full"], "anchor replay")


def test_outputs_are_deterministic():
    wl = workload.WORKLOADS["tiny"]
    Q, K, V = dev(*workload.make_qkv(wl))
    a = api.anchor(Q, K, V, wl.C, 256)
    b = api.anchor(Q, K, V, wl.C, 256)
    api.sync_status()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


# ---------------------------------------------------------------- ABI errors
def test_abi_rejects_bad_arguments():
    from free_sparse_attention_reuse_b200 import MCSError
    Q = torch.zeros(1, 1, 1000, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(MCSError) as e:
        api.group(Q, 64)  # N % C != 0
    assert e.value.status in (2,)
    Q = torch.zeros(1, 1, 1024, 96, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(MCSError):
        api.dense_attn(Q, Q, Q)  # d = 96
    Q = torch.zeros(1, 1, 1024, 64, dtype=torch.bfloat16, device=DEV)
    perm = torch.arange(1024, dtype=torch.int32, device=DEV).reshape(1, 1, 1024)
    idx = torch.zeros(1, 1, 16, 4, dtype=torch.int32, device=DEV)
    with pytest.raises(MCSError):
        api.sparse_attn(Q, Q, Q, perm, 64, idx[..., :0].contiguous())  # k = 0


def test_bad_index_is_reported_not_faulted():
    from free_sparse_attention_reuse_b200 import MCSError
    N = 1024
    Q = torch.zeros(1, 1, N, 64, dtype=torch.bfloat16, device=DEV)
    perm = torch.arange(N, dtype=torch.int32, device=DEV).reshape(1, 1, N)
    idx = torch.zeros(1, 1, N // 64, 8, dtype=torch.int32, device=DEV)
    idx[0, 0, 3, 5] = N + 7  # out of range: the kernel skips it and raises the status word
    api.sparse_attn(Q, Q, Q, perm, 64, idx)
    with pytest.raises(MCSError) as e:
        api.sync_status()
    assert e.value.status == 6
    api.sync_status()  # cleared


@pytest.mark.parametrize("d", [64, 128])
def test_growing_logits_force_rescales(d):
    # keys whose logits grow steeply with the key index: every later stage of each softmax
    # stream raises its running maximum by far more than 2^8, so O is rescaled in TMEM at
    # almost every stage (and the stage-ordered waits before each rescale are exercised)
    N, C, k = 2048, 128, 1536
    g = torch.Generator().manual_seed(7)
    q = torch.randn(1, 1, N, d, generator=g)
    base = torch.randn(1, 1, N, d, generator=g)
    u = torch.nn.functional.normalize(torch.ones(d), dim=0)
    ramp = torch.linspace(0.0, 60.0 * math.sqrt(d), N)[None, None, :, None]
    Q = (q * 0.1 + u).to(torch.bfloat16)
    K = (base * 0.1 + ramp * u).to(torch.bfloat16)
    V = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    perm = torch.arange(N, dtype=torch.int32)[None, None]
    idx = torch.arange(N - k, N, dtype=torch.int32).repeat(N // C, 1)[None, None].contiguous()
    Qd, Kd, Vd, pd, idd = dev(Q, K, V, perm, idx)
    out = api.sparse_attn(Qd, Kd, Vd, pd, C, idd)
    api.sync_status()
    q64, k64, v64 = to64(Q)[0, 0], to64(K)[0, 0], to64(V)[0, 0]
    ref = orc.sparse(q64, k64, v64, np.arange(N), idx[0, 0].numpy(), C, scale_of(d))[None, None]
    assert_close(out, ref, "sparse with rescales")
    Of, _ = api.dense_attn(Qd, Kd, Vd)
    api.sync_status()
    ref_d, _ = orc.dense(q64, k64, v64, scale_of(d))
    assert_close(Of, ref_d[None, None], "dense with rescales")


def _octave_keys(d, N, targets, seed):
    """Q rows a_i * 1 (a_i in [0.97, 1]) and K rows c_j * 1, so that the base-2 logit of query i
    and key j is a_i * t_j, with t_j = targets.get(j, small jitter); V random."""
    g = torch.Generator().manual_seed(seed)
    t = -2.0 * torch.rand(N, generator=g, dtype=torch.float64)
    for j, v in targets.items():
        t[j] = v
    c = t / (math.sqrt(d) * math.log2(math.e))
    K = (c[:, None] * torch.ones(N, d, dtype=torch.float64))[None, None].to(torch.bfloat16)
    a = 1.0 - 0.03 * (torch.arange(N, dtype=torch.float64) % 8) / 8
    Q = (a[:, None] * torch.ones(N, d, dtype=torch.float64))[None, None].to(torch.bfloat16)
    V = torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16)
    return Q, K, V


# stage j holds keys [128 j, 128 j + 128); even stages belong to softmax stream A, odd to B
_JUMPS = {
    # a key whose P passes 2^64 against the running reference, in a later chunk of the stage
    # than a key of comparable weight: the stored chunk is rescaled, then both keys matter
    "octaves": {256 + 5: 63.0, 256 + 40: 66.0, 384 + 70: 63.5, 384 + 100: 66.5},
    # P that overflows fp32 against the reference (a jump of ~130 octaves), then keys near it
    "overflow": {256 + 40: 66.0, 512 + 40: 196.0, 512 + 120: 195.0, 768 + 3: 194.5, 640 + 90: 195.5},
    # the same in the last chunk of a stage (after the first part of P has gone to the tensor
    # core), in both streams, one of them an overflow
    "late": {512 + 20: 63.0, 512 + 110: 66.0, 640 + 10: 62.0, 640 + 100: 196.0},
    # whole stages whose P sums pass 2^16: the reference moves at the stream's next stage
    **{"deferred": {j: v for s, v in ((2, 12.0), (3, 13.0), (4, 12.0), (5, 13.0))
                    for j in range(128 * s, 128 * s + 128)}},
}


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("case", sorted(_JUMPS))
def test_logit_jumps_raise_reference(case, d):
    # logits that jump far above everything before them inside a later stage of either softmax
    # stream; checks dense (with LSE) and sparse outputs against the oracle
    N, C, k = 2048, 128, 1536
    Q, K, V = _octave_keys(d, N, _JUMPS[case], seed=11 + d)
    perm = torch.arange(N, dtype=torch.int32)[None, None]
    idx = torch.arange(k, dtype=torch.int32).repeat(N // C, 1)[None, None].contiguous()
    Qd, Kd, Vd, pd, idd = dev(Q, K, V, perm, idx)
    q64, k64, v64 = to64(Q)[0, 0], to64(K)[0, 0], to64(V)[0, 0]
    Of, lse = api.dense_attn(Qd, Kd, Vd)
    api.sync_status()
    ref_d, lse_ref = orc.dense(q64, k64, v64, scale_of(d))
    assert_close(Of, ref_d[None, None], f"dense, {case}")
    assert np.abs(to64(lse[0, 0]) - lse_ref).max() < 2e-3
    out = api.sparse_attn(Qd, Kd, Vd, pd, C, idd)
    api.sync_status()
    ref = orc.sparse(q64, k64, v64, np.arange(N), idx[0, 0].numpy(), C, scale_of(d))[None, None]
    assert_close(out, ref, f"sparse, {case}")
