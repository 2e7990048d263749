"""The multi-layer metadata cache planner (no device): every reuse reads the latest anchor
version of its own layer, loads happen exactly when the slot holds something else, and two
consecutive metadata-using invocations never share a slot (so a load can overlap compute)."""

import itertools

import pytest

from free_sparse_attention_reuse_b200.cache import plan, schedule_kind


def simulate(acts, layers, slots):
    """Replay the actions on a model of the slots and of the host copies; return the number of
    loads.  Fails on any read of stale or foreign metadata."""
    slot = [None] * slots                  # (layer, version) in each slot
    host = [None] * layers                 # version of each layer's host copy
    latest = [-1] * layers
    loads = 0
    prev_slot = None
    for a in acts:
        if a.kind == "dense":
            continue
        assert 0 <= a.slot < slots
        assert a.slot != prev_slot, "consecutive invocations share a slot"
        prev_slot = a.slot
        if a.kind == "anchor":
            latest[a.layer] += 1
            assert a.version == latest[a.layer]
            slot[a.slot] = (a.layer, a.version)
            assert a.writeback
            host[a.layer] = a.version
        else:
            if a.load:
                loads += 1
                assert host[a.layer] == latest[a.layer], "loading a stale host copy"
                assert slot[a.slot] != (a.layer, latest[a.layer]), "needless load"
                slot[a.slot] = (a.layer, host[a.layer])
            assert slot[a.slot] == (a.layer, latest[a.layer]), "reuse reads stale metadata"
            assert a.version == latest[a.layer]
    return loads


@pytest.mark.parametrize("layers,slots,warmup,period", [(3, 2, 2, 4), (4, 2, 5, 10), (5, 3, 3, 5), (2, 2, 1, 3)])
def test_plan_is_consistent(layers, slots, warmup, period):
    steps = 23
    acts = plan(steps, layers, lambda t: schedule_kind(t, warmup, period), slots)
    assert [(a.step, a.layer) for a in acts] == list(itertools.product(range(steps), range(layers)))
    loads = simulate(acts, layers, slots)
    reuse = sum(a.kind == "reuse" for a in acts)
    if layers > slots:
        assert loads > 0
    assert loads <= reuse


def test_plan_every_reuse_loads_when_layers_exceed_slots():
    # round-robin over 2 slots with 3 layers: a layer never finds itself in its slot again
    acts = plan(12, 3, lambda t: schedule_kind(t, 2, 4), 2)
    assert all(a.load for a in acts if a.kind == "reuse")


def test_plan_rejects_reuse_before_anchor_and_single_slot():
    with pytest.raises(ValueError):
        plan(3, 2, lambda t: "reuse", 2)
    with pytest.raises(ValueError):
        plan(3, 2, lambda t: schedule_kind(t), 1)


def test_schedule_kind_matches_the_reading():
    kinds = [schedule_kind(t, 5, 10) for t in range(50)]
    assert kinds[:4] == ["dense"] * 4
    assert [t for t, k in enumerate(kinds) if k == "anchor"] == [4, 14, 24, 34, 44]
    assert kinds.count("reuse") == 41


def test_plan_consistent_for_arbitrary_step_kinds():
    # any sequence of step kinds whose first metadata step is an anchor, any layer and slot count
    from hypothesis import given, settings
    from hypothesis import strategies as st

    kinds = st.lists(st.sampled_from(["dense", "anchor", "reuse"]), min_size=1, max_size=30).filter(
        lambda ks: next((k for k in ks if k != "dense"), "anchor") == "anchor")

    @settings(max_examples=300, deadline=None)
    @given(kinds, st.integers(1, 6), st.integers(2, 7))
    def check(ks, layers, slots):
        acts = plan(len(ks), layers, lambda t: ks[t], slots)
        assert [(a.step, a.layer) for a in acts] == list(itertools.product(range(len(ks)), range(layers)))
        loads = simulate(acts, layers, slots)
        assert loads <= sum(a.kind == "reuse" for a in acts)

    check()
