"""The decode kernel's staging protocol, model-checked on the CPU.

``flint_attn_decode`` (csrc/decode.cu) stages each warp's 16-key steps of K and
V into two shared-memory buffers with ``cp.async``: every loop iteration
commits one copy group (empty past the last step) and waits until at most one
group is pending, so the group of the step about to be computed has landed.
Each warp's first step is issued before the CTA's prologue math, except the
step that holds slot p (the new token's key and value), which the owning CTA
writes first. This module restates that schedule per warp and runs it with
copy groups completing at random times. The protocol must never compute a step
from a buffer that holds another step or an unfinished copy, never overwrite a
buffer a step still reads, and never stage slot p before the append. Planted
mistakes must each be caught.
"""
import random

import pytest

STEP, WARPS, STAGES = 16, 4, 2


class StagingError(AssertionError):
    pass


def run_cta(k0, k1, p, owner, seed, mutation=None):
    """One CTA: keys [k0, k1) of a pair whose new token sits in slot p (the owner's
    range ends at p + 1). Returns the steps each warp computed."""
    rng = random.Random(seed)
    nsteps = (k1 - k0 + STEP - 1) // STEP
    slot_p_written = False
    bufs = {(w, b): None for w in range(WARPS) for b in range(STAGES)}   # (step, done?)
    groups = {w: [] for w in range(WARPS)}        # per warp: FIFO of groups (lists of copies)
    pending = {w: [] for w in range(WARPS)}       # copies issued but not yet in a group
    computed = {w: [] for w in range(WARPS)}

    def holds_p(step):
        kb = k0 + step * STEP
        return kb <= p < min(kb + STEP, k1)

    def issue(w, step, b):
        if bufs[(w, b)] is not None and bufs[(w, b)][2]:
            raise StagingError(f"warp {w} refills buffer {b} while step "
                               f"{bufs[(w, b)][0]} still reads it")
        if owner and holds_p(step) and not slot_p_written:
            raise StagingError(f"warp {w} stages slot p (step {step}) before the append")
        copy = {"step": step, "buf": b, "done": False}
        bufs[(w, b)] = [step, copy, False]
        pending[w].append(copy)

    def commit(w):
        groups[w].append(pending[w])
        pending[w] = []

    def land_some():
        for w in range(WARPS):
            for g in groups[w]:
                for c in g:
                    if not c["done"] and rng.random() < 0.4:
                        c["done"] = True

    def wait_group(w, n):
        # cp.async.wait_group n: the oldest groups complete in order until at most
        # n are pending (here, landing the copies the wait needs)
        while sum(1 for g in groups[w] if any(not c["done"] for c in g)) > n:
            land_some()
        # groups complete in commit order: everything older than the last n done
        done_upto = len(groups[w]) - n
        for g in groups[w][:max(done_upto, 0)]:
            for c in g:
                c["done"] = True

    # ---- early staging, before the prologue math and the append
    first_early = {}
    for w in range(WARPS):
        early = w < nsteps and not (owner and p < k0 + (w + 1) * STEP)
        if mutation == "early_even_with_slot_p":
            early = w < nsteps
        first_early[w] = early
        if early:
            issue(w, w, 0)
    land_some()
    # ---- prologue: the owner appends slot p; a block barrier follows
    if owner:
        slot_p_written = True
    # ---- the prefill group and the step loop, warp by warp (warps are independent)
    for w in range(WARPS):
        if w < nsteps and not first_early[w]:
            issue(w, w, 0)
        commit(w)
        it, step = 0, w
        while step < nsteps:
            b = it % STAGES
            ahead = step + WARPS * (STAGES - 1)
            nb = (it + 1) % STAGES if mutation != "ahead_into_current_buffer" else b
            if ahead < nsteps:
                issue(w, ahead, nb)
            commit(w)
            wait_group(w, 2 if mutation == "wait_one_group_too_few" else STAGES - 1)
            cell = bufs[(w, b)]
            if cell is None or cell[0] != step:
                raise StagingError(f"warp {w} computes step {step} from buffer {b} holding "
                                   f"{None if cell is None else cell[0]}")
            if not cell[1]["done"]:
                raise StagingError(f"warp {w} computes step {step} before its copy landed")
            cell[2] = True                     # reading (ldmatrix) the buffer
            land_some()
            computed[w].append(step)
            cell[2] = False                    # __syncwarp: the buffer is free again
            step += WARPS
            it += 1
        wait_group(w, 0)
    return computed


CASES = [
    # k0, k1, p, owner
    (0, 1, 0, True),            # a single key: slot p is in warp 0's first step
    (0, 40, 39, True),          # three steps, slot p in warp 2's first step
    (100, 164, 163, True),      # four steps, slot p in warp 3's first step
    (100, 200, 199, True),      # seven steps: slot p in warp 2's second step
    (0, 1376, 1375, True),      # the serving shape's chunk, owning CTA
    (0, 1376, 5000, False),     # the same chunk, not owning slot p
    (16, 33, 32, True),         # ragged: 17 keys, slot p alone in the second step
]


@pytest.mark.parametrize("k0,k1,p,owner", CASES)
def test_staging_protocol_holds(k0, k1, p, owner):
    nsteps = (k1 - k0 + STEP - 1) // STEP
    for seed in range(40):
        computed = run_cta(k0, k1, p, owner, seed)
        assert sorted(s for w in computed for s in computed[w]) == list(range(nsteps))


@pytest.mark.parametrize("mutation", ["early_even_with_slot_p", "wait_one_group_too_few",
                                      "ahead_into_current_buffer"])
def test_planted_staging_mistake_is_caught(mutation):
    for k0, k1, p, owner in CASES:
        for seed in range(40):
            try:
                run_cta(k0, k1, p, owner, seed, mutation)
            except StagingError:
                return
    pytest.fail(f"{mutation}: no schedule showed the mistake")
