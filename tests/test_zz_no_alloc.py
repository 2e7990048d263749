"""The allocation-free selection entry point (mcs_select_noalloc) against mcs_select.

mcs_select_noalloc exists for callers that cannot allocate device memory (an engine that owns
all memory through its own pool, a loop that must never allocate), so it keeps its score
scratch in a fixed array inside the library instead of a caller workspace.  Its results must
equal those of mcs_select, which runs the same kernel with a workspace: the indices are
integers, so the comparison is exact.  Two calls in a row, with different shapes, check that
what the shared array holds from one call does not leak into the next.

This file is collected last on purpose, and passes both alone and after the other tests.
"""

import ctypes

import numpy as np
import pytest
import torch

from free_sparse_attention_reuse_b200 import _lib, api, workload

pytestmark = pytest.mark.gpu


def _case(H, d, grid, C, k, index):
    wl = workload.custom("noalloc", 1, H, d, grid, C, index=index)
    Q, K, _ = (t.cuda() for t in workload.make_qkv(wl))
    N = Q.shape[2]
    # groups: contiguous blocks (any partition is valid input to the selection)
    perm = torch.arange(N, dtype=torch.int32, device="cuda").repeat(1, H, 1).contiguous()
    _, lse = api.dense_attn(Q, K, K, want_out=False)
    return Q, K, perm, lse, C, k


def _noalloc_via_abi(Q, K, perm, lse, C, k):
    lib = _lib.load()
    B, H, N, d = Q.shape
    idx = torch.full((B, H, N // C, k), -1, dtype=torch.int32, device="cuda")
    st = lib.mcs_select_noalloc(_lib.Shape(B, H, N, d, 0.0), _lib.ptr(Q), _lib.ptr(K), _lib.ptr(perm), C, k,
                                _lib.ptr(lse), _lib.ptr(idx), _lib.stream_ptr())
    assert st == 0, lib.mcs_status_string(st)
    return idx


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [
        _case(2, 128, (4, 16, 16), 128, 300, 41),  # N = 1024
        _case(3, 64, (8, 16, 16), 64, 517, 42),    # N = 2048, different shape and k
    ]
    for Q, K, perm, lse, C, k in cases:
        got = _noalloc_via_abi(Q, K, perm, lse, C, k)
        ref = api.select(Q, K, perm, C, k, lse=lse)
        api.sync_status()
        assert np.array_equal(got.cpu().numpy(), ref.cpu().numpy())


def test_noalloc_rejects_problems_beyond_its_fixed_scratch():
    lib = _lib.load()
    small = torch.zeros(16, dtype=torch.int32, device="cuda")
    too_big_n = (2 << 20) + 64  # two half-score rows of round_up(N, 64) exceed the 4 Mi floats
    st = lib.mcs_select_noalloc(_lib.Shape(1, 1, too_big_n, 64, 0.0), _lib.ptr(small), _lib.ptr(small),
                                _lib.ptr(small), 64, 8, _lib.ptr(small), _lib.ptr(small), _lib.stream_ptr())
    assert st == 8  # MCS_ERR_WORKSPACE, returned before anything is launched
    st = lib.mcs_select_noalloc(_lib.Shape(1, 1, 1024, 64, 0.0), _lib.ptr(small), _lib.ptr(small),
                                _lib.ptr(small), 64, 8, ctypes.c_void_p(None), _lib.ptr(small), _lib.stream_ptr())
    assert st == 1  # lse is required
    api.sync_status()
