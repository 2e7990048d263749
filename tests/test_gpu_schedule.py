"""The anchor/reuse schedule (host side, row a9) driving the C ABI on the Tiny shape for 50
denoising steps: dense warm-up for steps 0-3, anchors at 4, 14, 24, 34, 44, reuse otherwise
("MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다", section 무엇과 다른가: the anchor is
the last step of the dense warm-up or of a refresh interval)."""

import math

import numpy as np
import pytest

import oracle as orc
from free_sparse_attention_reuse_b200 import api, workload
from helpers import assert_close

pytestmark = pytest.mark.gpu


def test_schedule_50_steps_tiny():
    wl = workload.WORKLOADS["tiny"]
    C, k = wl.C, wl.k(0.25)
    sched = api.Schedule(C, k, warmup=5, period=10)
    kinds = [sched.kind(t) for t in range(50)]
    assert kinds[:4] == ["dense"] * 4
    assert [t for t in range(50) if kinds[t] == "anchor"] == [4, 14, 24, 34, 44]
    assert kinds.count("reuse") == 41
    gen = workload.Generator(wl)
    scale = 1.0 / math.sqrt(wl.d)
    qkv = gen.current()
    for t in range(50):
        if t > 0:
            qkv = gen.advance()
        out = sched(t, *(x.cuda() for x in qkv))
        api.sync_status()
        if t not in (0, 4, 5, 13, 14, 15, 49):
            continue
        q, kk, v = (x.double().numpy()[0] for x in qkv)
        for h in range(wl.H):
            if kinds[t] in ("dense", "anchor"):
                ref, _ = orc.dense(q[h], kk[h], v[h], scale)
            else:
                m = sched.meta
                ref = orc.reuse(q[h], kk[h], v[h], m.perm[0, h].cpu().numpy(), m.idx[0, h].cpu().numpy(),
                                m.R[0, h].cpu().double().numpy(), C, scale)
            assert_close(out[0, h], ref, f"step {t} ({kinds[t]}) head {h}")
    m = sched.meta
    assert m.perm.shape == (1, wl.H, wl.N) and m.idx.shape == (1, wl.H, wl.G, k)
