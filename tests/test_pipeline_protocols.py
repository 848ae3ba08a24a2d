"""The mbarrier protocols of the six pipelined kernels, model-checked on the CPU.

``tests/pipeline_model.py`` restates each kernel's roles (TMA producer, MMA
issuer, eight math warps) with their waits, arrivals, commits and buffer
accesses, and runs them under random interleavings with TMA loads and MMAs
completing at random times. The kernels' protocols must finish every schedule
with no deadlock, no phase aliasing, no overwrite of a buffer an unfinished
operation still reads, and no read of anything but the expected tile, over item
lists with one-tile items, long items and mixes of both. Each planted mistake
(a release moved too early, a wait left out) must be caught.
"""
import random

import pytest

import pipeline_model as pm

ITEM_LISTS = {
    "forward": [[1], [3], [1, 1, 1, 1], [2, 5, 1, 3], [6, 1, 2]],
    "backward_dkv": [[1], [4], [1, 1, 1, 1, 1], [3, 1, 5, 2]],
    "backward_dq": [[1], [4], [1, 1, 1, 1, 1, 1], [3, 1, 5, 2, 1]],
    "forward_x3": [[1], [3], [1, 1, 1, 1], [2, 5, 1, 3], [6, 1, 2]],
    "backward_dkv_x3": [[1], [4], [1, 1, 1, 1, 1], [3, 1, 5, 2]],
    "backward_dq_x3": [[1], [4], [1, 1, 1, 1, 1, 1], [3, 1, 5, 2, 1]],
}
SEEDS = 30


@pytest.mark.parametrize("kernel", sorted(ITEM_LISTS))
def test_protocol_holds_under_random_schedules(kernel):
    for items in ITEM_LISTS[kernel]:
        for seed in range(SEEDS):
            pm.check(kernel, items, seed)


@pytest.mark.parametrize("kernel,mutation", pm.MUTATIONS, ids=[m for _, m in pm.MUTATIONS])
def test_planted_protocol_mistake_is_caught(kernel, mutation):
    for items in ITEM_LISTS[kernel]:
        for seed in range(200):
            try:
                pm.check(kernel, items, seed, mutation)
            except pm.ProtocolError:
                return
    pytest.fail(f"{mutation}: no schedule showed the mistake")


def test_barrier_model_follows_the_parity_rule():
    b = pm.Barrier("b", 2)
    assert not b.passes(0)
    b.arrive()
    assert not b.passes(0)
    b.expect_tx(1)                       # second arrival, but a load is still in flight
    assert not b.passes(0)
    b.complete_tx(1)
    assert b.passes(0) and not b.passes(1)
    b.arrive(2)
    with pytest.raises(pm.ProtocolError):
        b.passes(0)                      # two phases ahead: the parity test would alias
    with pytest.raises(pm.ProtocolError):
        b.arrive(3)                      # more arrivals than the count


def test_deadlock_is_reported():
    sim = pm.Sim(random.Random(0))
    sim.bar("never")

    def waiter():
        yield ("wait", "never", 0)

    sim.role("w", waiter())
    with pytest.raises(pm.ProtocolError, match="deadlock"):
        sim.run()


@pytest.mark.parametrize("kernel", sorted(ITEM_LISTS))
def test_kernels_rely_on_in_order_mma_issue(kernel):
    """Every kernel issues an MMA into a TMEM region right behind the MMA that
    reads it (the forwards' next QK behind the PV that reads P; dP^T behind dK;
    S^T behind dV; S or dP behind dQ), relying on tcgen05.mma operations of one
    thread being performed in issue order. Without that rule the same schedules
    must fail, and only on that overlap."""
    flagged = 0
    for seed in range(20):
        sim = pm.Sim(random.Random(seed))
        pm.KERNELS[kernel](sim, [3], None)
        sim.mma_in_order = False
        try:
            sim.run()
        except pm.ProtocolError as e:
            assert "while an unfinished operation reads it" in str(e)
            flagged += 1
    assert flagged > 0
