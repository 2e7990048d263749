"""The k-means grouping-cost baseline on the GPU against the fp64 oracle: equal-size groups,
bit-exact (the same fp64 arithmetic in the same order), through the C ABI."""

import numpy as np
import pytest
import torch

import oracle as orc
from free_sparse_attention_reuse_b200 import MCSError, api, workload
from helpers import to64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,d,grid,C,iters", [
    (2, 64, (4, 16, 16), 64, 0),
    (2, 64, (4, 16, 16), 64, 10),    # the Tiny shape
    (1, 128, (3, 8, 16), 128, 4),    # G = 3
    (2, 128, (12, 8, 16), 128, 6),   # G = 12
    (1, 64, (31, 8, 8), 64, 3),      # G = 31
])
def test_kmeans_groups_bit_exact(H, d, grid, C, iters):
    wl = workload.custom("km", 1, H, d, grid, C, index=61)
    Q, _, _ = workload.make_qkv(wl)
    perm = api.group_kmeans(Q.cuda(), C, iters)
    api.sync_status()
    q = to64(Q)
    for h in range(H):
        ref = orc.kmeans_groups(q[0, h], C, iters)
        got = perm[0, h].cpu().numpy()
        assert np.array_equal(got, ref), f"head {h}: {np.count_nonzero(got != ref)} positions differ"


def test_kmeans_identical_queries():
    Q = torch.ones(1, 1, 512, 64, dtype=torch.bfloat16, device="cuda")
    perm = api.group_kmeans(Q, 64, 3)
    api.sync_status()
    assert np.array_equal(perm[0, 0].cpu().numpy(), np.arange(512))


def test_kmeans_rejects_bad_arguments():
    Q = torch.zeros(1, 1, 1000, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(MCSError):
        api.group_kmeans(Q, 64, 3)  # N % C != 0
    Q = torch.zeros(1, 1, 1024, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(MCSError):
        api.group_kmeans(Q, 64, -1)
