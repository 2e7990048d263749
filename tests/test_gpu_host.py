"""Reuse step from host memory (mcs_sparse_attn_host) against the device-resident call: the
same kernels on the same data, so outputs must be bit-identical, for every chunking of the
heads (one head per chunk, ragged last chunk, one chunk), with and without R, from pinned and
pageable host memory, on the default and on a side stream."""

import pytest
import torch

from free_sparse_attention_reuse_b200 import MCSError, api, workload

pytestmark = pytest.mark.gpu


def _case(B, H, d, grid, C, k):
    wl = workload.custom("host", B, H, d, grid, C, index=31)
    Q, K, V = workload.make_qkv(wl)
    dQ, dK, dV = (t.cuda() for t in (Q, K, V))
    _, perm, idx, R = api.anchor(dQ, dK, dV, C, k)
    return (Q, K, V), (dQ, dK, dV), perm, idx, R


@pytest.mark.parametrize("hc", [1, 2, 4, 6, 9])
@pytest.mark.parametrize("with_r", [True, False])
def test_host_matches_device(hc, with_r):
    (Q, K, V), (dQ, dK, dV), perm, idx, R = _case(2, 3, 64, (2, 16, 16), 64, 200)  # B*H = 6, N = 512
    R = R if with_r else None
    ref = api.sparse_attn(dQ, dK, dV, perm, 64, idx, R=R)
    hQ, hK, hV = (t.pin_memory() for t in (Q, K, V))
    out = api.sparse_attn_host(hQ, hK, hV, perm, 64, idx, R=R, heads_per_chunk=hc)
    torch.cuda.current_stream().synchronize()
    api.sync_status()
    assert torch.equal(out, ref.cpu())


def test_host_pageable_side_stream_and_reuse_of_buffers():
    (Q, K, V), (dQ, dK, dV), perm, idx, R = _case(1, 5, 128, (2, 16, 16), 128, 300)  # N = 512, d = 128
    ref = api.sparse_attn(dQ, dK, dV, perm, 128, idx, R=R).cpu()
    staging = api.host_staging(tuple(Q.shape), 2)
    out = torch.empty(Q.shape, dtype=torch.bfloat16)  # pageable
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        # first a call on other inputs, then the real one into the same output and staging:
        # the second must see none of the first
        api.sparse_attn_host(V, K, Q, perm, 128, idx, R=R, out=out, heads_per_chunk=2, staging=staging)
        api.sparse_attn_host(Q, K, V, perm, 128, idx, R=R, out=out, heads_per_chunk=2, staging=staging)
    side.synchronize()
    api.sync_status()
    assert torch.equal(out, ref)


def test_host_argument_errors():
    (Q, K, V), _, perm, idx, R = _case(1, 2, 64, (2, 8, 8), 64, 64)
    with pytest.raises(MCSError, match="INVALID_ARG"):
        api.sparse_attn_host(Q, K, V, perm, 64, idx, heads_per_chunk=0, staging=torch.empty(256, dtype=torch.uint8,
                                                                                              device="cuda"))
    small = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(MCSError, match="WORKSPACE"):
        api.sparse_attn_host(Q, K, V, perm, 64, idx, heads_per_chunk=1, staging=small)
