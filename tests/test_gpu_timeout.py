"""The failure path of the attention kernels on the GPU, made to run without a fault: every
launch first waits for a flag in device memory that nothing sets, within a short bound, so
the wait runs out.  The kernel then abandons its work, lets what it already issued land,
frees its tensor memory and returns; mcs_sync_status reports MCS_ERR_TIMEOUT and the context
stays usable, so the very next calls on the same stream give the oracle's results."""

import ctypes

import numpy as np
import pytest
import torch

from free_sparse_attention_reuse_b200 import MCSError, _lib, api, workload
from helpers import assert_close, oracle_anchor

pytestmark = pytest.mark.gpu

TIMEOUT = 7  # MCS_ERR_TIMEOUT
LIMIT_NS = 20_000_000  # 20 ms: far above the normal waits of these small launches


def _hold(flag):
    return ctypes.c_void_p(flag.data_ptr()) if flag is not None else None


@pytest.mark.parametrize("d", [64, 128])
def test_wait_that_runs_out_is_reported_and_the_next_call_is_correct(d):
    wl = workload.custom("timeout", 1, 2, d, (4, 16, 16), 64, index=51)
    C, k = wl.C, 200
    Q, K, V = workload.make_qkv(wl)
    res = oracle_anchor(Q, K, V, C, k)
    Qd, Kd, Vd = (t.cuda() for t in (Q, K, V))
    perm = torch.from_numpy(res["perm"].astype(np.int32)).cuda()
    idx = torch.from_numpy(res["idx"].astype(np.int32)).cuda()
    R = torch.from_numpy(res["R"]).to(torch.bfloat16).cuda()
    lib = _lib.load()
    api.sync_status()
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")  # never set
    prev = lib.mcs_set_attn_wait_limit(LIMIT_NS, _hold(flag))
    try:
        # sparse (cp.async gathers in flight), dense (TMA loads in flight) and residual mode
        api.sparse_attn(Qd, Kd, Vd, perm, C, idx, R=R)
        with pytest.raises(MCSError) as e:
            api.sync_status()
        assert e.value.status == TIMEOUT
        api.dense_attn(Qd, Kd, Vd)
        with pytest.raises(MCSError) as e:
            api.sync_status()
        assert e.value.status == TIMEOUT
        api.residual(Qd, Kd, Vd, perm, C, idx, torch.zeros_like(Qd))
        with pytest.raises(MCSError) as e:
            api.sync_status()
        assert e.value.status == TIMEOUT
    finally:
        lib.mcs_set_attn_wait_limit(0, None)
    assert prev == 2_000_000_000
    # the same calls on the same stream, with the hook reset, are correct
    out = api.sparse_attn(Qd, Kd, Vd, perm, C, idx, R=R)
    O, lse = api.dense_attn(Qd, Kd, Vd)
    Rg = api.residual(Qd, Kd, Vd, perm, C, idx, O)
    api.sync_status()
    assert_close(out, res["O_sparse"] + res["R"], "reuse after a timeout")
    assert_close(O, res["O_full"], "dense after a timeout")
    assert np.abs(lse.cpu().double().numpy() - res["lse"]).max() < 2e-3
    assert_close(Rg, res["R"], "residual after a timeout", norm_ref=res["O_full"])
    # and a flag that is set lets the launch through
    flag.fill_(1)
    lib.mcs_set_attn_wait_limit(LIMIT_NS, _hold(flag))
    try:
        out2 = api.sparse_attn(Qd, Kd, Vd, perm, C, idx, R=R)
        api.sync_status()
    finally:
        lib.mcs_set_attn_wait_limit(0, None)
    assert torch.equal(out2, out)
