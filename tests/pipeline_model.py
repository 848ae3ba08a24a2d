"""Model checker for the mbarrier protocols of the pipelined attention kernels.

TEST INFRASTRUCTURE. The forward kernel (csrc/attn_fwd_sm100.cu), the two
backward kernels (csrc/attn_bwd_sm100.cu: dK/dV key-major, dQ query-major) and
their FP32-input counterparts (csrc/attn_x3_sm100.cu) coordinate a TMA producer
thread, an MMA issuing thread and four or eight math warps
through shared-memory mbarriers. This module restates, role by role, the waits,
arrivals, commits and buffer accesses of each kernel's normal path (the abort
and drain paths are left out) and runs them under random interleavings:

* an mbarrier completes a phase when its arrival count and its outstanding
  transaction units both reach zero; a wait names the phase it needs, and the
  check is the hardware's parity test, so a waiter two phases behind or ahead
  of the barrier (phase aliasing) is reported instead of passing or hanging;
* TMA loads complete in any order and complete transaction units on their
  barrier; MMAs from the one issuing thread complete in issue order, and a
  commit arrives on its barrier once every MMA issued before it has completed;
* every shared-memory tile and every TMEM column chunk of each 32-lane quarter
  is a cell with a content tag: a TMA load or an MMA writes its cells over the
  whole interval from issue to completion, an MMA reads its operands over that
  interval, and a math warp's tcgen05.ld / st is instantaneous.

Violations: a deadlock (no role can move and nothing is in flight); a write
into a cell that an unfinished operation reads or writes (except an MMA
accumulating into the accumulator that earlier MMAs of the same chain write);
a read of a cell while a write to it is in flight, or whose content is not the
tile the reader expects; phase aliasing; arrivals past a barrier's count.
MMAs from the one issuing thread are performed in issue order, so a model may
declare (``Sim.mma_in_order``) that an MMA overwrites cells an earlier,
unfinished MMA reads: every kernel issues an MMA into a TMEM region right
behind the MMA that reads it (the forwards' next QK behind the PV that reads P;
dP^T behind dK and, in the FP32-input kernel, S^T behind dV; S or dP behind
dQ). Any other overlap is flagged.

``MUTATIONS`` plants known mistakes in the restated protocols, so that tests can
show the checker finds them.
"""
from __future__ import annotations

import random
from collections import deque

K_SLOTS = 5          # K/V ring of the forward and dQ kernels
ITEM_SLOTS = 4       # item-index ring of the backward kernels
Q_STAGES_DKV = 3     # Q stages of the dK/dV kernel (dO has 2)
MATH_WARPS = 8


class ProtocolError(AssertionError):
    pass


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.completed = count, 0, 0

    def arrive(self, n=1):
        if self.pending - n < 0:
            raise ProtocolError(f"{self.name}: arrivals past the count in phase {self.completed}")
        self.pending -= n
        self._complete()

    def expect_tx(self, units):
        self.tx += units
        self.arrive(1)

    def complete_tx(self, units):
        self.tx -= units
        if self.tx < 0:
            raise ProtocolError(f"{self.name}: more transaction units than expected")
        self._complete()

    def _complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def passes(self, k):
        """The hardware parity test for 'phase k has completed'."""
        c = self.completed
        if c == k:
            return False
        if c == k + 1:
            return True
        raise ProtocolError(f"{self.name}: wait for phase {k} while {c} phases have completed "
                            "(parity aliasing)")


class Cell:
    __slots__ = ("name", "tag", "next_tag", "readers", "writers")

    def __init__(self, name):
        self.name, self.tag, self.next_tag = name, None, None
        self.readers, self.writers = set(), set()


class Op:
    _ids = 0

    def __init__(self, kind, reads=(), writes=(), tag=None, bar=None, accumulate=False):
        Op._ids += 1
        self.id = Op._ids
        self.kind, self.reads, self.writes = kind, list(reads), list(writes)
        self.tag, self.bar, self.accumulate = tag, bar, accumulate


class Sim:
    def __init__(self, rng):
        self.rng = rng
        self.bars, self.cells = {}, {}
        self.roles = {}            # name -> [generator, blocked (bar, k) or None]
        self.tma = []              # in-flight TMA loads
        self.mma = deque()         # issued MMAs and commit markers, in issue order
        self.mma_in_order = False  # an MMA may overwrite what earlier MMAs still read
        self.steps = 0

    # -- setup
    def bar(self, name, count=1):
        self.bars[name] = Barrier(name, count)

    def cell(self, name):
        c = self.cells.get(name)
        if c is None:
            c = self.cells[name] = Cell(name)
        return c

    def role(self, name, gen):
        self.roles[name] = [gen, None]

    # -- actions
    def _read_ok(self, names, tag, who):
        for n in names:
            c = self.cell(n)
            if c.writers:
                raise ProtocolError(f"{who} reads {n} while a write to it is in flight")
            if c.tag != tag:
                raise ProtocolError(f"{who} reads {n}: holds {c.tag}, expected {tag}")

    def _write_begin(self, names, tag, op, who, accumulate=False):
        for n in names:
            c = self.cell(n)
            in_order = (self.mma_in_order and op.kind == "mma"
                        and all(r.kind == "mma" for r in c.readers))
            if c.readers and not in_order:
                raise ProtocolError(f"{who} writes {n} while an unfinished operation reads it")
            if c.writers:
                chain = accumulate and c.next_tag == tag and all(
                    w.kind == "mma" for w in c.writers)
                if not chain:
                    raise ProtocolError(f"{who} writes {n} while another write is in flight")
            elif accumulate and c.tag != tag:
                raise ProtocolError(f"{who} accumulates into {n}: holds {c.tag}, expected {tag}")
            c.writers.add(op)
            c.next_tag = tag

    def _write_end(self, names, tag, op):
        for n in names:
            c = self.cell(n)
            c.writers.discard(op)
            c.tag = tag

    def _do(self, who, act):
        kind = act[0]
        if kind == "wait":
            return not self.bars[act[1]].passes(act[2])
        if kind == "arrive":
            self.bars[act[1]].arrive(act[2] if len(act) > 2 else 1)
        elif kind == "expect_tx":
            self.bars[act[1]].expect_tx(act[2])
        elif kind == "tma":                       # ("tma", cells, tag, bar)
            op = Op("tma", writes=act[1], tag=act[2], bar=act[3])
            self._write_begin(act[1], act[2], op, who)
            self.tma.append(op)
        elif kind == "mma":                       # ("mma", [(cells, tag)...], cells, tag, acc)
            op = Op("mma", reads=act[1], writes=act[2], tag=act[3], accumulate=act[4])
            for names, tag in act[1]:
                self._read_ok(names, tag, who)
            for names, _ in act[1]:
                for n in names:
                    self.cell(n).readers.add(op)
            self._write_begin(act[2], act[3], op, who, accumulate=act[4])
            self.mma.append(op)
        elif kind == "commit":
            self.mma.append(Op("commit", bar=act[1]))
        elif kind == "read":                      # ("read", cells, tag)
            self._read_ok(act[1], act[2], who)
        elif kind == "write":                     # ("write", cells, tag)
            op = Op("sync")
            self._write_begin(act[1], act[2], op, who)
            self._write_end(act[1], act[2], op)
        else:
            raise ValueError(kind)
        return False

    def _step_role(self, name):
        st = self.roles[name]
        gen, blocked = st
        if blocked is not None:
            if not self.bars[blocked[0]].passes(blocked[1]):
                return
            st[1] = None
        try:
            act = next(gen)
        except StopIteration:
            del self.roles[name]
            return
        if self._do(name, act):
            st[1] = (act[1], act[2])

    def _complete_tma(self, op):
        self.tma.remove(op)
        self._write_end(op.writes, op.tag, op)
        self.bars[op.bar].complete_tx(1)

    def _complete_mma_head(self):
        op = self.mma.popleft()
        if op.kind == "commit":
            self.bars[op.bar].arrive(1)
            return
        for names, _ in op.reads:
            for n in names:
                self.cell(n).readers.discard(op)
        self._write_end(op.writes, op.tag, op)

    def run(self, max_steps=2_000_000):
        # per-run bias: how eagerly each engine makes progress
        w_role = self.rng.uniform(0.2, 1.0)
        w_tma = self.rng.uniform(0.05, 1.0)
        w_mma = self.rng.uniform(0.05, 1.0)
        while self.roles or self.tma or self.mma:
            self.steps += 1
            if self.steps > max_steps:
                raise ProtocolError("no end after max_steps (livelock?)")
            ready = [n for n, (_, b) in self.roles.items()
                     if b is None or self.bars[b[0]].passes(b[1])]
            choices = [("role", n, w_role) for n in ready]
            choices += [("tma", op, w_tma) for op in self.tma]
            if self.mma:
                choices.append(("mma", None, w_mma))
            if not choices:
                blocked = {n: b for n, (_, b) in self.roles.items()}
                raise ProtocolError(f"deadlock: {blocked}")
            total = sum(c[2] for c in choices)
            x = self.rng.uniform(0, total)
            for kind, arg, w in choices:
                x -= w
                if x <= 0:
                    break
            if kind == "role":
                self._step_role(arg)
            elif kind == "tma":
                self._complete_tma(arg)
            else:
                self._complete_mma_head()


# ============================================================================
# Cells
# ============================================================================

def tmem(region, chunks, quarters=range(4)):
    """TMEM cells: column chunks of 16 columns of a region, per 32-lane quarter."""
    return [f"tmem:{region}:{c}:{q}" for c in chunks for q in quarters]


ALL_CHUNKS = range(8)          # 128 columns = 8 chunks of 16


def _ring_push(k, idx_tag):
    """Item ring, fetching thread: publish the k-th item index."""
    s = k % ITEM_SLOTS
    if k >= ITEM_SLOTS:
        yield ("wait", f"ring_empty{s}", k // ITEM_SLOTS - 1)
    yield ("write", [f"ring{s}"], idx_tag)
    yield ("arrive", f"ring_full{s}")


def _ring_pop(k, idx_tag):
    """Item ring, one consuming warp: read the k-th index, free the slot."""
    s = k % ITEM_SLOTS
    yield ("wait", f"ring_full{s}", k // ITEM_SLOTS)
    yield ("read", [f"ring{s}"], idx_tag)
    yield ("arrive", f"ring_empty{s}")


def _ring_bars(sim, consumers=MATH_WARPS + 1):
    for s in range(ITEM_SLOTS):
        sim.bar(f"ring_full{s}", 1)
        sim.bar(f"ring_empty{s}", consumers)


# ============================================================================
# Forward (attn_fwd_sm100_kernel): items are query-tile pairs, taken through the
# item ring like the backward kernels'
# ============================================================================

def forward(sim, items, mut=None):
    """items: key tiles per item (>= 1). Tiles i = 0, 1 of the pair."""
    sim.mma_in_order = True
    sim.bar("q_full"), sim.bar("q_empty")
    for s in range(K_SLOTS):
        sim.bar(f"kv_full{s}"), sim.bar(f"kv_empty{s}")
    for i in range(2):
        sim.bar(f"s_full{i}"), sim.bar(f"p_half{i}", 4), sim.bar(f"p_full{i}", 4)
        sim.bar(f"o_full{i}"), sim.bar(f"o_empty{i}", 4)
    _ring_bars(sim)
    seq = list(items) + [None]

    def kv_tag(load):
        return ("V" if load & 1 else "K", load // 2)

    def producer():
        kv_load = 0
        for item, nt in enumerate(seq):
            yield from _ring_push(item, ("idx", item))
            if nt is None:
                return
            if item > 0:
                yield ("wait", "q_empty", item - 1)
            yield ("expect_tx", "q_full", 2)
            for i in range(2):
                yield ("tma", [f"smem:Q{i}"], ("Q", item, i), "q_full")
            for j in range(2 * nt):
                s = kv_load % K_SLOTS
                if kv_load >= K_SLOTS:
                    yield ("wait", f"kv_empty{s}", kv_load // K_SLOTS - 1)
                yield ("expect_tx", f"kv_full{s}", 1)
                yield ("tma", [f"smem:kv{s}"], kv_tag(kv_load), f"kv_full{s}")
                kv_load += 1

    def mma():
        kv_load, pc = 0, [0, 0]

        def qk(i, item, slot, g):
            return ("mma", [([f"smem:Q{i}"], ("Q", item, i)), ([f"smem:kv{slot}"], ("K", g))],
                    tmem(f"S{i}", ALL_CHUNKS), ("S", i, g), False)

        for item, nt in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nt is None:
                return
            g0 = kv_load // 2
            yield ("wait", "q_full", item)
            s = kv_load % K_SLOTS
            yield ("wait", f"kv_full{s}", kv_load // K_SLOTS)
            for i in range(2):
                yield qk(i, item, s, g0)
                yield ("commit", f"s_full{i}")
            yield ("commit", f"kv_empty{s}")
            if nt == 1:
                yield ("commit", "q_empty")
            for n in range(nt):
                lv = kv_load + 2 * n + 1
                lk = lv + 1
                s, s2 = lv % K_SLOTS, lk % K_SLOTS
                has_next = n + 1 < nt
                g = g0 + n
                yield ("wait", f"kv_full{s}", lv // K_SLOTS)
                for i in range(2):
                    yield ("wait", f"p_half{i}", pc[i])
                    if n == 0 and item > 0:
                        yield ("wait", f"o_empty{i}", item - 1)
                    o = tmem(f"O{i}", ALL_CHUNKS)
                    yield ("mma", [(tmem(f"S{i}", [0, 1, 2]), ("P", i, g)),
                                   ([f"smem:kv{s}"], ("V", g))], o, ("O", i, item), n > 0)
                    if mut == "fwd_o_full_before_last_pv" and not has_next:
                        yield ("commit", f"o_full{i}")
                    yield ("wait", f"p_full{i}", pc[i])
                    pc[i] += 1
                    if mut == "fwd_qk_before_pv" and has_next:
                        # the next QK overtakes the PV that still has to read P
                        if i == 0:
                            yield ("wait", f"kv_full{s2}", lk // K_SLOTS)
                        yield qk(i, item, s2, g + 1)
                    yield ("mma", [(tmem(f"S{i}", [3]), ("P", i, g)),
                                   ([f"smem:kv{s}"], ("V", g))], o, ("O", i, item), True)
                    if not has_next and mut != "fwd_o_full_before_last_pv":
                        yield ("commit", f"o_full{i}")
                    if i == 1:
                        yield ("commit", f"kv_empty{s}")
                    if has_next:
                        if i == 0 and mut != "fwd_qk_before_pv":
                            yield ("wait", f"kv_full{s2}", lk // K_SLOTS)
                        if mut == "fwd_q_empty_before_last_qk" and i == 1 and n + 2 == nt:
                            yield ("commit", "q_empty")
                        if mut != "fwd_qk_before_pv":
                            yield qk(i, item, s2, g + 1)
                        yield ("commit", f"s_full{i}")
                        if i == 1:
                            yield ("commit", f"kv_empty{s2}")
                            if n + 2 == nt and mut != "fwd_q_empty_before_last_qk":
                                yield ("commit", "q_empty")
            kv_load += 2 * nt

    def softmax(i, q):
        s_count, kv_load = 0, 0
        quarter = [q]
        for item, nt in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nt is None:
                return
            g0 = kv_load // 2
            for n in range(nt):
                g = g0 + n
                yield ("wait", f"s_full{i}", s_count)
                s_count += 1
                yield ("read", tmem(f"S{i}", ALL_CHUNKS, quarter), ("S", i, g))
                yield ("write", tmem(f"S{i}", [0], quarter), ("P", i, g))
                if n > 0 and sim.rng.random() < 0.5:          # lazy rescale of O
                    o = tmem(f"O{i}", ALL_CHUNKS, quarter)
                    yield ("read", o, ("O", i, item))
                    yield ("write", o, ("O", i, item))
                if mut == "fwd_p_half_early":
                    yield ("arrive", f"p_half{i}")
                yield ("write", tmem(f"S{i}", [1, 2], quarter), ("P", i, g))
                if mut != "fwd_p_half_early":
                    yield ("arrive", f"p_half{i}")
                yield ("write", tmem(f"S{i}", [3], quarter), ("P", i, g))
                yield ("arrive", f"p_full{i}")
            yield ("wait", f"o_full{i}", item)
            yield ("read", tmem(f"O{i}", ALL_CHUNKS, quarter), ("O", i, item))
            yield ("arrive", f"o_empty{i}")
            kv_load += 2 * nt

    sim.role("tma", producer())
    sim.role("mma", mma())
    for w in range(MATH_WARPS):
        sim.role(f"softmax{w}", softmax(w >> 2, w & 3))


# ============================================================================
# dK/dV (attn_bwd_dkv_kernel): items are key tiles, each over nq query tiles
# ============================================================================

def backward_dkv(sim, items, mut=None):
    sim.bar("kv_full"), sim.bar("kv_empty")
    for s in range(Q_STAGES_DKV):
        sim.bar(f"q_full{s}"), sim.bar(f"q_empty{s}")
    for s in range(2):
        sim.bar(f"do_full{s}", 2), sim.bar(f"do_empty{s}")
    sim.mma_in_order = True
    sim.bar("s_full"), sim.bar("dp_full"), sim.bar("acc_full")
    for b in ("p_full", "ds_full", "dp_free", "acc_empty"):
        sim.bar(b, MATH_WARPS)
    _ring_bars(sim)
    seq = list(items) + [None]

    def region(t):
        return "R" + str(t & 1)

    def producer():
        qd = 0
        for item, nq in enumerate(seq):
            yield from _ring_push(item, ("idx", item))
            if nq is None:
                return
            if item > 0:
                yield ("wait", "kv_empty", item - 1)
            yield ("expect_tx", "kv_full", 2)
            yield ("tma", ["smem:K"], ("K", item), "kv_full")
            yield ("tma", ["smem:V"], ("V", item), "kv_full")
            for m in range(nq):
                sq, s = qd % Q_STAGES_DKV, qd & 1
                if qd >= Q_STAGES_DKV:
                    yield ("wait", f"q_empty{sq}", qd // Q_STAGES_DKV - 1)
                yield ("expect_tx", f"q_full{sq}", 1)
                yield ("tma", [f"smem:Q{sq}"], ("Q", qd), f"q_full{sq}")
                if qd >= 2:
                    yield ("wait", f"do_empty{s}", qd // 2 - 1)
                yield ("expect_tx", f"do_full{s}", 1)
                yield ("tma", [f"smem:dO{s}"], ("dO", qd), f"do_full{s}")
                yield ("write", [f"smem:stats{s}"], ("st", qd))
                yield ("arrive", f"do_full{s}")
                qd += 1

    def mma():
        t, p_cnt, ds_cnt, dpf_cnt = 0, 0, 0, 0

        def issue_s(tt, item):
            yield ("mma", [(["smem:K"], ("K", item)),
                           ([f"smem:Q{tt % Q_STAGES_DKV}"], ("Q", tt))],
                   tmem(region(tt), ALL_CHUNKS), ("ST", tt), False)
            yield ("commit", "s_full")

        def issue_dp(tt, item):
            yield ("mma", [(["smem:V"], ("V", item)), ([f"smem:dO{tt & 1}"], ("dO", tt))],
                   tmem(region(tt + 1), ALL_CHUNKS), ("dPT", tt), False)
            yield ("commit", "dp_full")

        for item, nq in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nq is None:
                return
            yield ("wait", "kv_full", item)
            yield ("wait", f"q_full{t % Q_STAGES_DKV}", t // Q_STAGES_DKV)
            yield from issue_s(t, item)
            yield ("wait", f"do_full{t & 1}", t >> 1)
            yield from issue_dp(t, item)
            for m in range(nq):
                X = region(t)
                has_next = m + 1 < nq
                yield ("wait", "p_full", p_cnt)
                p_cnt += 1
                if m == 0 and item > 0:
                    yield ("wait", "acc_empty", item - 1)
                # dV += P^T dO: P^T in X chunks 0-1 (warpgroup 0) and 4-5 (warpgroup 1)
                yield ("mma", [(tmem(X, [0, 1, 4, 5]), ("PT", t)),
                               ([f"smem:dO{t & 1}"], ("dO", t))],
                       tmem("dV", ALL_CHUNKS), ("dV", item), m > 0)
                if has_next:
                    if mut != "dkv_s_without_dp_free":
                        yield ("wait", "dp_free", dpf_cnt)
                    yield ("wait", f"q_full{(t + 1) % Q_STAGES_DKV}", (t + 1) // Q_STAGES_DKV)
                    yield from issue_s(t + 1, item)
                dpf_cnt += 1
                if mut == "dkv_do_empty_before_ds":
                    yield ("commit", f"do_empty{t & 1}")
                yield ("wait", "ds_full", ds_cnt)
                ds_cnt += 1
                if mut != "dkv_do_empty_before_ds":
                    yield ("commit", f"do_empty{t & 1}")
                # dK += dS^T Q: dS^T in X chunks 2-3 and 6-7
                yield ("mma", [(tmem(X, [2, 3, 6, 7]), ("dST", t)),
                               ([f"smem:Q{t % Q_STAGES_DKV}"], ("Q", t))],
                       tmem("dK", ALL_CHUNKS), ("dK", item), m > 0)
                yield ("commit", f"q_empty{t % Q_STAGES_DKV}")
                if has_next:
                    yield ("wait", f"do_full{(t + 1) & 1}", (t + 1) >> 1)
                    yield from issue_dp(t + 1, item)
                t += 1
            yield ("commit", "kv_empty")
            yield ("commit", "acc_full")

    def math(wg, q):
        quarter = [q]
        mine = [4 * wg, 4 * wg + 1, 4 * wg + 2, 4 * wg + 3]      # columns [64wg, 64wg+64)
        t, s_cnt, dp_cnt = 0, 0, 0
        for item, nq in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nq is None:
                return
            for m in range(nq):
                X, Y = region(t), region(t + 1)
                yield ("wait", f"do_full{t & 1}", t >> 1)
                yield ("wait", "s_full", s_cnt)
                s_cnt += 1
                yield ("read", tmem(X, mine, quarter), ("ST", t))
                yield ("read", [f"smem:stats{t & 1}"], ("st", t))
                yield ("write", tmem(X, mine[:2], quarter), ("PT", t))
                yield ("arrive", "p_full")
                yield ("wait", "dp_full", dp_cnt)
                dp_cnt += 1
                yield ("read", tmem(Y, mine, quarter), ("dPT", t))
                yield ("arrive", "dp_free")
                yield ("read", [f"smem:stats{t & 1}"], ("st", t))
                yield ("write", tmem(X, mine[2:], quarter), ("dST", t))
                yield ("arrive", "ds_full")
                t += 1
            yield ("wait", "acc_full", item)
            yield ("read", tmem("dV", mine, quarter), ("dV", item))
            yield ("read", tmem("dK", mine, quarter), ("dK", item))
            yield ("arrive", "acc_empty")

    sim.role("tma", producer())
    sim.role("mma", mma())
    for w in range(MATH_WARPS):
        sim.role(f"math{w}", math(w >> 2, w & 3))


# ============================================================================
# dQ (attn_bwd_dq_kernel): items are query tiles, each over ntiles key tiles
# ============================================================================

def backward_dq(sim, items, mut=None):
    sim.mma_in_order = True
    sim.bar("qd_full"), sim.bar("qd_empty")
    for s in range(K_SLOTS):
        sim.bar(f"kv_full{s}"), sim.bar(f"kv_empty{s}")
    for b in range(2):
        sim.bar(f"s_full{b}")
    sim.bar("dp_full"), sim.bar("acc_full")
    sim.bar("ds_full", MATH_WARPS), sim.bar("acc_empty", MATH_WARPS)
    _ring_bars(sim)
    seq = list(items) + [None]

    def kv_tag(load):
        return ("V" if load & 1 else "K", load // 2)

    def producer():
        kv_load = 0
        for item, nt in enumerate(seq):
            yield from _ring_push(item, ("idx", item))
            if nt is None:
                return
            if item > 0:
                yield ("wait", "qd_empty", item - 1)
            yield ("expect_tx", "qd_full", 2)
            yield ("tma", ["smem:Q"], ("Q", item), "qd_full")
            yield ("tma", ["smem:dO"], ("dO", item), "qd_full")
            for j in range(2 * nt):
                s = kv_load % K_SLOTS
                if kv_load >= K_SLOTS:
                    yield ("wait", f"kv_empty{s}", kv_load // K_SLOTS - 1)
                yield ("expect_tx", f"kv_full{s}", 1)
                yield ("tma", [f"smem:kv{s}"], kv_tag(kv_load), f"kv_full{s}")
                kv_load += 1

    def mma():
        t, ds_cnt = 0, 0

        def issue_s(tt, item):
            b, lk = tt & 1, 2 * tt
            st = lk % K_SLOTS
            yield ("wait", f"kv_full{st}", lk // K_SLOTS)
            yield ("mma", [(["smem:Q"], ("Q", item)), ([f"smem:kv{st}"], ("K", tt))],
                   tmem(f"S{b}", ALL_CHUNKS), ("S", tt), False)
            yield ("commit", f"s_full{b}")

        for item, nt in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nt is None:
                return
            yield ("wait", "qd_full", item)
            yield from issue_s(t, item)
            for n in range(nt):
                sk, lv = (2 * t) % K_SLOTS, 2 * t + 1
                sv = lv % K_SLOTS
                yield ("wait", f"kv_full{sv}", lv // K_SLOTS)
                if mut == "dq_qd_empty_before_last_dp" and n + 1 == nt:
                    yield ("commit", "qd_empty")
                yield ("mma", [(["smem:dO"], ("dO", item)), ([f"smem:kv{sv}"], ("V", t))],
                       tmem("dP", ALL_CHUNKS), ("dP", t), False)
                yield ("commit", "dp_full")
                yield ("commit", f"kv_empty{sv}")
                if n + 1 == nt and mut != "dq_qd_empty_before_last_dp":
                    yield ("commit", "qd_empty")
                if mut == "dq_k_released_after_dp":
                    yield ("commit", f"kv_empty{sk}")
                if n + 1 < nt:
                    yield from issue_s(t + 1, item)
                if mut != "dq_dq_without_ds_full":
                    yield ("wait", "ds_full", ds_cnt)
                ds_cnt += 1
                if n == 0 and item > 0:
                    yield ("wait", "acc_empty", item - 1)
                b = t & 1
                # dQ += dS K: dS in S-buffer chunks 0-1 (warpgroup 0) and 4-5 (warpgroup 1)
                yield ("mma", [(tmem(f"S{b}", [0, 1, 4, 5]), ("dS", t)),
                               ([f"smem:kv{sk}"], ("K", t))],
                       tmem("dQ", ALL_CHUNKS), ("dQ", item), n > 0)
                if mut != "dq_k_released_after_dp":
                    yield ("commit", f"kv_empty{sk}")
                t += 1
            yield ("commit", "acc_full")

    def math(wg, q):
        quarter = [q]
        mine = [4 * wg, 4 * wg + 1, 4 * wg + 2, 4 * wg + 3]      # keys [64wg, 64wg+64)
        t = 0
        for item, nt in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nt is None:
                return
            for n in range(nt):
                b = t & 1
                yield ("wait", f"s_full{b}", t >> 1)
                yield ("read", tmem(f"S{b}", mine, quarter), ("S", t))
                yield ("wait", "dp_full", t)
                yield ("read", tmem("dP", mine, quarter), ("dP", t))
                yield ("write", tmem(f"S{b}", mine[:2], quarter), ("dS", t))
                yield ("arrive", "ds_full")
                t += 1
            yield ("wait", "acc_full", item)
            yield ("read", tmem("dQ", mine, quarter), ("dQ", item))
            yield ("arrive", "acc_empty")

    sim.role("tma", producer())
    sim.role("mma", mma())
    for w in range(MATH_WARPS):
        sim.role(f"math{w}", math(w >> 2, w & 3))


# ============================================================================
# FP32 inputs on the tensor cores (csrc/attn_x3_sm100.cu): every operand has a hi
# and a lo part. An MMA below stands for the group of MMAs (three per product)
# that the kernel issues between two barrier operations.
# ============================================================================

X3_KV_SLOTS_FWD = 5
X3_KV_SLOTS_DQ = 12
X3_DRAIN_TILES = 2   # the dK/dV kernel drains every 16 tiles; 2 exercises more drains
PARTS = ("Kh", "Kl", "Vh", "Vl")


def forward_x3(sim, items, mut=None):
    """attn_fwd_x3_kernel: one query tile per item, two S buffers, 4 softmax warps."""
    sim.mma_in_order = True
    sim.bar("q_full"), sim.bar("q_empty")
    for s in range(X3_KV_SLOTS_FWD):
        sim.bar(f"kv_full{s}"), sim.bar(f"kv_empty{s}")
    for b in range(2):
        sim.bar(f"s_full{b}"), sim.bar(f"p_half{b}", 4), sim.bar(f"p_full{b}", 4)
        sim.bar(f"pv_done{b}")
    sim.bar("o_full"), sim.bar("o_empty", 4)
    _ring_bars(sim, 5)
    seq = list(items) + [None]
    NS = X3_KV_SLOTS_FWD

    def producer():
        kv_load = 0
        for item, nt in enumerate(seq):
            yield from _ring_push(item, ("idx", item))
            if nt is None:
                return
            if item > 0:
                yield ("wait", "q_empty", item - 1)
            yield ("expect_tx", "q_full", 2)
            yield ("tma", ["smem:Qh"], ("Qh", item), "q_full")
            yield ("tma", ["smem:Ql"], ("Ql", item), "q_full")
            # K one key tile ahead of V: K(0), then K(n+1), V(n), ..., V(nt-1)
            order = [("K", 0)]
            for n in range(nt):
                if n + 1 < nt:
                    order.append(("K", n + 1))
                order.append(("V", n))
            for kind, n in order:
                for part in ("h", "l"):
                    s = kv_load % NS
                    if kv_load >= NS:
                        yield ("wait", f"kv_empty{s}", kv_load // NS - 1)
                    yield ("expect_tx", f"kv_full{s}", 1)
                    yield ("tma", [f"smem:kv{s}"], (kind + part, item, n), f"kv_full{s}")
                    kv_load += 1

    def mma():
        t, kv_base = 0, 0

        def pos_k(n):
            return 0 if n == 0 else 4 * n - 2

        def pos_v(n, nt):
            return 4 * n + 4 if n + 1 < nt else 4 * n + 2

        def slot_read(pos, tag):
            return ([f"smem:kv{pos % NS}"], tag)

        def issue_qk(n, tt, item, last):
            b, pos = tt & 1, kv_base + pos_k(n)
            yield ("wait", f"kv_full{pos % NS}", pos // NS)
            yield ("wait", f"kv_full{(pos + 1) % NS}", (pos + 1) // NS)
            yield ("mma", [(["smem:Qh"], ("Qh", item)), (["smem:Ql"], ("Ql", item)),
                           slot_read(pos, ("Kh", item, n)), slot_read(pos + 1, ("Kl", item, n))],
                   tmem(f"S{b}", ALL_CHUNKS), ("S", tt), False)
            yield ("commit", f"s_full{b}")
            yield ("commit", f"kv_empty{pos % NS}")
            yield ("commit", f"kv_empty{(pos + 1) % NS}")
            if last:
                yield ("commit", "q_empty")

        for item, nt in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nt is None:
                return
            yield ("wait", "q_full", item)
            yield from issue_qk(0, t, item, nt == 1)
            if nt > 1:
                yield from issue_qk(1, t + 1, item, nt == 2)
            for n in range(nt):
                tt = t + n
                b = tt & 1
                pos = kv_base + pos_v(n, nt)
                vh, vl = slot_read(pos, ("Vh", item, n)), slot_read(pos + 1, ("Vl", item, n))
                yield ("wait", f"kv_full{pos % NS}", pos // NS)
                yield ("wait", f"kv_full{(pos + 1) % NS}", (pos + 1) // NS)
                yield ("wait", f"p_half{b}", tt >> 1)
                if n == 0 and item > 0:
                    yield ("wait", "o_empty", item - 1)
                o = tmem("O", ALL_CHUNKS)
                # keys 0-63: P' hi in chunks 0-1, lo in chunks 2-3 of the S buffer
                yield ("mma", [(tmem(f"S{b}", [0, 1, 2, 3]), ("P", tt)), vh, vl], o,
                       ("O", item), n > 0)
                if mut == "x3f_qk_before_pv" and n + 2 < nt:
                    # the QK into this S buffer overtakes the PV that still reads P
                    yield from issue_qk(n + 2, tt + 2, item, n + 3 == nt)
                if mut != "x3f_pv_without_p_full":
                    yield ("wait", f"p_full{b}", tt >> 1)
                yield ("mma", [(tmem(f"S{b}", [4, 5, 6, 7]), ("P", tt)), vh, vl], o,
                       ("O", item), True)
                yield ("commit", f"pv_done{b}")
                yield ("commit", f"kv_empty{pos % NS}")
                yield ("commit", f"kv_empty{(pos + 1) % NS}")
                if n + 1 == nt:
                    yield ("commit", "o_full")
                if n + 2 < nt and mut != "x3f_qk_before_pv":
                    yield from issue_qk(n + 2, tt + 2, item, n + 3 == nt)
            kv_base += 4 * nt
            t += nt

    def softmax(q):
        quarter = [q]
        t = 0
        for item, nt in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nt is None:
                return
            for n in range(nt):
                tt = t + n
                b = tt & 1
                yield ("wait", f"s_full{b}", tt >> 1)
                yield ("read", tmem(f"S{b}", ALL_CHUNKS, quarter), ("S", tt))
                yield ("write", tmem(f"S{b}", [0, 2], quarter), ("P", tt))    # keys 0-31
                if n > 0 and sim.rng.random() < 0.5:       # lazy rescale of O
                    if mut != "x3f_rescale_without_pv_done":
                        yield ("wait", f"pv_done{(tt - 1) & 1}", (tt - 1) >> 1)
                    o = tmem("O", ALL_CHUNKS, quarter)
                    yield ("read", o, ("O", item))
                    yield ("write", o, ("O", item))
                yield ("write", tmem(f"S{b}", [1, 3], quarter), ("P", tt))    # keys 32-63
                yield ("arrive", f"p_half{b}")
                yield ("write", tmem(f"S{b}", [4, 6, 5, 7], quarter), ("P", tt))
                yield ("arrive", f"p_full{b}")
            t += nt
            yield ("wait", "o_full", item)
            yield ("read", tmem("O", ALL_CHUNKS, quarter), ("O", item))
            yield ("arrive", "o_empty")

    sim.role("tma", producer())
    sim.role("mma", mma())
    for w in range(4):
        sim.role(f"softmax{w}", softmax(w))


def backward_dkv_x3(sim, items, mut=None):
    """attn_bwd_dkv_x3_kernel: V's parts in TMEM, 64-row query tiles, drains of dV/dK."""
    sim.mma_in_order = True
    sim.bar("kv_full"), sim.bar("kv_empty")
    for s in range(Q_STAGES_DKV):
        sim.bar(f"q_full{s}"), sim.bar(f"q_empty{s}")
    for s in range(2):
        sim.bar(f"do_full{s}", 2), sim.bar(f"do_empty{s}")
    for b in ("s_full", "dp_full", "acc_full"):
        sim.bar(b)
    for b in ("v_full", "p_full", "ds_full", "acc_empty"):
        sim.bar(b, MATH_WARPS)
    _ring_bars(sim)
    seq = list(items) + [None]
    QS = Q_STAGES_DKV

    def producer():
        qd = 0
        for item, nq in enumerate(seq):
            yield from _ring_push(item, ("idx", item))
            if nq is None:
                return
            if item > 0:
                yield ("wait", "kv_empty", item - 1)
            yield ("expect_tx", "kv_full", 2)
            yield ("tma", ["smem:Kh"], ("Kh", item), "kv_full")
            yield ("tma", ["smem:Kl"], ("Kl", item), "kv_full")
            for m in range(nq):
                sq, s = qd % QS, qd & 1
                if qd >= QS:
                    yield ("wait", f"q_empty{sq}", qd // QS - 1)
                yield ("expect_tx", f"q_full{sq}", 2)
                yield ("tma", [f"smem:Q{sq}h"], ("Qh", qd), f"q_full{sq}")
                yield ("tma", [f"smem:Q{sq}l"], ("Ql", qd), f"q_full{sq}")
                if qd >= 2:
                    yield ("wait", f"do_empty{s}", qd // 2 - 1)
                yield ("expect_tx", f"do_full{s}", 2)
                yield ("tma", [f"smem:dO{s}h"], ("dOh", qd), f"do_full{s}")
                yield ("tma", [f"smem:dO{s}l"], ("dOl", qd), f"do_full{s}")
                yield ("write", [f"smem:stats{s}"], ("st", qd))
                yield ("arrive", f"do_full{s}")
                qd += 1

    def q_read(tt):
        return [([f"smem:Q{tt % QS}h"], ("Qh", tt)), ([f"smem:Q{tt % QS}l"], ("Ql", tt))]

    def do_read(tt):
        return [([f"smem:dO{tt & 1}h"], ("dOh", tt)), ([f"smem:dO{tt & 1}l"], ("dOl", tt))]

    X, Y = tmem("X", range(4)), tmem("Y", range(4))

    def mma():
        t, p_cnt, ds_cnt, drains = 0, 0, 0, 0

        def issue_s(tt, item):
            yield ("mma", [(["smem:Kh"], ("Kh", item)), (["smem:Kl"], ("Kl", item))] + q_read(tt),
                   X, ("ST", tt), False)
            yield ("commit", "s_full")

        def issue_dp(tt, item):
            yield ("mma", [(tmem("V", ALL_CHUNKS), ("V", item))] + do_read(tt),
                   Y, ("dPT", tt), False)
            yield ("commit", "dp_full")

        for item, nq in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nq is None:
                return
            yield ("wait", "kv_full", item)
            yield ("wait", f"q_full{t % QS}", t // QS)
            yield from issue_s(t, item)
            yield ("wait", "v_full", item)
            yield ("wait", f"do_full{t & 1}", t >> 1)
            yield from issue_dp(t, item)
            for m in range(nq):
                has_next = m + 1 < nq
                c_first = m % X3_DRAIN_TILES == 0
                c_last = (m + 1) % X3_DRAIN_TILES == 0 or not has_next
                yield ("wait", "p_full", p_cnt)
                p_cnt += 1
                # implied by p_full (a math warp arrives on it only after its own drain),
                # kept as in the kernel
                if c_first and drains > 0:
                    yield ("wait", "acc_empty", drains - 1)
                if mut == "x3k_s_before_dv" and has_next:
                    # S^T(t+1) into X ahead of the dV(t) that reads P^T(t) there
                    yield ("wait", f"q_full{(t + 1) % QS}", (t + 1) // QS)
                    yield from issue_s(t + 1, item)
                yield ("mma", [(X, ("PT", t))] + do_read(t), tmem("dV", ALL_CHUNKS),
                       ("dV", drains), not c_first)
                if has_next and mut != "x3k_s_before_dv":
                    yield ("wait", f"q_full{(t + 1) % QS}", (t + 1) // QS)
                    yield from issue_s(t + 1, item)
                yield ("wait", "ds_full", ds_cnt)
                ds_cnt += 1
                yield ("commit", f"do_empty{t & 1}")
                yield ("mma", [(Y, ("dST", t))] + q_read(t), tmem("dK", ALL_CHUNKS),
                       ("dK", drains), not c_first)
                yield ("commit", f"q_empty{t % QS}")
                if c_last:
                    yield ("commit", "acc_full")
                    drains += 1
                if has_next:
                    yield ("wait", f"do_full{(t + 1) & 1}", (t + 1) >> 1)
                    yield from issue_dp(t + 1, item)
                t += 1
            yield ("commit", "kv_empty")

    def math(wg, q):
        quarter = [q]
        mine = [2 * wg, 2 * wg + 1]                # query columns [32wg, 32wg+32)
        chans = [4 * wg + c for c in range(4)]     # channels [64wg, 64wg+64)
        t, drains = 0, 0
        early_v = False
        for item, nq in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nq is None:
                return
            if not early_v:
                # V's parts: warpgroup 0 the hi part (chunks 0-3), 1 the lo part (4-7)
                yield ("write", tmem("V", chans, quarter), ("V", item))
                yield ("arrive", "v_full")
            early_v = False
            for m in range(nq):
                has_next = m + 1 < nq
                yield ("wait", f"do_full{t & 1}", t >> 1)
                yield ("wait", "s_full", t)
                yield ("read", tmem("X", mine, quarter), ("ST", t))
                yield ("read", [f"smem:stats{t & 1}"], ("st", t))
                yield ("write", tmem("X", mine, quarter), ("PT", t))
                yield ("arrive", "p_full")
                if mut == "x3k_v_before_last_dp" and not has_next and seq[item + 1]:
                    # planted: the next item's V while this item's last dP^T may still run
                    yield ("write", tmem("V", chans, quarter), ("V", item + 1))
                    yield ("arrive", "v_full")
                    early_v = True
                yield ("wait", "dp_full", t)
                yield ("read", tmem("Y", mine, quarter), ("dPT", t))
                yield ("read", [f"smem:stats{t & 1}"], ("st", t))
                yield ("write", tmem("Y", mine, quarter), ("dST", t))
                yield ("arrive", "ds_full")
                if (m + 1) % X3_DRAIN_TILES == 0 or not has_next:
                    yield ("wait", "acc_full", drains)
                    yield ("read", tmem("dV", chans, quarter), ("dV", drains))
                    yield ("read", tmem("dK", chans, quarter), ("dK", drains))
                    yield ("arrive", "acc_empty")
                    drains += 1
                t += 1

    sim.role("tma", producer())
    sim.role("mma", mma())
    for w in range(MATH_WARPS):
        sim.role(f"math{w}", math(w >> 2, w & 3))


def backward_dq_x3(sim, items, mut=None):
    """attn_bwd_dq_x3_kernel: Q's and dO's parts in TMEM, 64-key tiles, rotating regions."""
    sim.mma_in_order = True
    NS = X3_KV_SLOTS_DQ
    for s in range(NS):
        sim.bar(f"kv_full{s}"), sim.bar(f"kv_empty{s}")
    for b in ("s_full", "dp_full", "acc_full"):
        sim.bar(b)
    for b in ("qd_full", "dp_free", "ds_full", "acc_empty"):
        sim.bar(b, MATH_WARPS)
    _ring_bars(sim)
    seq = list(items) + [None]

    def region(tt):
        return "R" + str(tt & 1)

    def producer():
        kv_load = 0
        for item, nt in enumerate(seq):
            yield from _ring_push(item, ("idx", item))
            if nt is None:
                return
            for j in range(4 * nt):
                s = kv_load % NS
                if kv_load >= NS:
                    yield ("wait", f"kv_empty{s}", kv_load // NS - 1)
                yield ("expect_tx", f"kv_full{s}", 1)
                yield ("tma", [f"smem:kv{s}"], (PARTS[j & 3], kv_load // 4), f"kv_full{s}")
                kv_load += 1

    def mma():
        t, kv_base, dpf_cnt, ds_cnt = 0, 0, 0, 0

        def slot_read(pos):
            return ([f"smem:kv{pos % NS}"], (PARTS[pos & 3], pos // 4))

        def issue_s(n, tt, item):
            pos = kv_base + 4 * n
            yield ("wait", f"kv_full{pos % NS}", pos // NS)
            yield ("wait", f"kv_full{(pos + 1) % NS}", (pos + 1) // NS)
            yield ("mma", [(tmem("QD", range(8)), ("Q", item)), slot_read(pos),
                           slot_read(pos + 1)], tmem(region(tt), range(4)), ("S", tt), False)
            yield ("commit", "s_full")

        def issue_dp(n, tt, item):
            pos = kv_base + 4 * n + 2
            yield ("wait", f"kv_full{pos % NS}", pos // NS)
            yield ("wait", f"kv_full{(pos + 1) % NS}", (pos + 1) // NS)
            yield ("mma", [(tmem("QD", range(8, 16)), ("dO", item)), slot_read(pos),
                           slot_read(pos + 1)], tmem(region(tt + 1), range(4)), ("dP", tt),
                   False)
            yield ("commit", "dp_full")
            yield ("commit", f"kv_empty{pos % NS}")
            yield ("commit", f"kv_empty{(pos + 1) % NS}")

        for item, nt in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nt is None:
                return
            yield ("wait", "qd_full", item)
            if t > 0:
                yield ("wait", "dp_free", dpf_cnt - 1)
            yield from issue_s(0, t, item)
            yield from issue_dp(0, t, item)
            for n in range(nt):
                tt = t + n
                has_next = n + 1 < nt
                if has_next:
                    if mut != "x3d_s_without_dp_free":
                        yield ("wait", "dp_free", dpf_cnt)
                    yield from issue_s(n + 1, tt + 1, item)
                dpf_cnt += 1
                yield ("wait", "ds_full", ds_cnt)
                ds_cnt += 1
                if n == 0 and item > 0:
                    yield ("wait", "acc_empty", item - 1)
                pos = kv_base + 4 * n
                if mut == "x3d_dp_before_dq" and has_next:
                    # dP(t+1) into R(t) ahead of the dQ(t) that reads dS(t) there
                    yield from issue_dp(n + 1, tt + 1, item)
                yield ("mma", [(tmem(region(tt), range(4)), ("dS", tt)), slot_read(pos),
                               slot_read(pos + 1)], tmem("dQ", ALL_CHUNKS), ("dQ", item), n > 0)
                yield ("commit", f"kv_empty{pos % NS}")
                yield ("commit", f"kv_empty{(pos + 1) % NS}")
                if has_next and mut != "x3d_dp_before_dq":
                    yield from issue_dp(n + 1, tt + 1, item)
            yield ("commit", "acc_full")
            kv_base += 4 * nt
            t += nt

    def math(wg, q):
        quarter = [q]
        mine = [2 * wg, 2 * wg + 1]                # keys [32wg, 32wg+32) of a tile
        t = 0
        for item, nt in enumerate(seq):
            yield from _ring_pop(item, ("idx", item))
            if nt is None:
                return
            # Q's parts (warpgroup 0, chunks 0-7) or dO's (warpgroup 1, chunks 8-15)
            yield ("write", tmem("QD", range(8 * wg, 8 * wg + 8), quarter),
                   ("dO" if wg else "Q", item))
            yield ("arrive", "qd_full")
            for n in range(nt):
                X, Y = region(t), region(t + 1)
                yield ("wait", "s_full", t)
                yield ("read", tmem(X, mine, quarter), ("S", t))
                yield ("wait", "dp_full", t)
                yield ("read", tmem(Y, mine, quarter), ("dP", t))
                yield ("arrive", "dp_free")
                yield ("write", tmem(X, mine, quarter), ("dS", t))
                yield ("arrive", "ds_full")
                t += 1
            if mut != "x3d_epilogue_without_acc_full":
                yield ("wait", "acc_full", item)
            yield ("read", tmem("dQ", [4 * wg + c for c in range(4)], quarter), ("dQ", item))
            yield ("arrive", "acc_empty")

    sim.role("tma", producer())
    sim.role("mma", mma())
    for w in range(MATH_WARPS):
        sim.role(f"math{w}", math(w >> 2, w & 3))


KERNELS = {"forward": forward, "backward_dkv": backward_dkv, "backward_dq": backward_dq,
           "forward_x3": forward_x3, "backward_dkv_x3": backward_dkv_x3,
           "backward_dq_x3": backward_dq_x3}

# planted mistakes: (kernel, mutation)
MUTATIONS = [
    ("forward", "fwd_q_empty_before_last_qk"),
    ("forward", "fwd_p_half_early"),
    ("forward", "fwd_o_full_before_last_pv"),
    ("forward", "fwd_qk_before_pv"),
    ("backward_dkv", "dkv_s_without_dp_free"),
    ("backward_dkv", "dkv_do_empty_before_ds"),
    ("backward_dq", "dq_dq_without_ds_full"),
    ("backward_dq", "dq_qd_empty_before_last_dp"),
    ("backward_dq", "dq_k_released_after_dp"),
    ("forward_x3", "x3f_pv_without_p_full"),
    ("forward_x3", "x3f_qk_before_pv"),
    ("forward_x3", "x3f_rescale_without_pv_done"),
    ("backward_dkv_x3", "x3k_s_before_dv"),
    ("backward_dkv_x3", "x3k_v_before_last_dp"),
    ("backward_dq_x3", "x3d_s_without_dp_free"),
    ("backward_dq_x3", "x3d_dp_before_dq"),
    ("backward_dq_x3", "x3d_epilogue_without_acc_full"),
]


def check(kernel, items, seed, mut=None):
    """One random schedule of `kernel` over `items`; raises ProtocolError on a violation."""
    sim = Sim(random.Random(seed))
    KERNELS[kernel](sim, items, mut)
    sim.run()
    for b in sim.bars.values():
        if b.pending != b.count or b.tx != 0:
            raise ProtocolError(f"{b.name}: a phase left half complete at the end")
    return sim.steps
