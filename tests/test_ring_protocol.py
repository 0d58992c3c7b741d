"""CPU model of the shared-memory pipeline protocol of the TMA decode kernels.

The kernels stream 16-token K/V sub-tiles through a ring of `stages` shared-
memory slots. A producer warp issues the loads of positions g = 0, 1, 2, ...
(slot g % stages, round g // stages), up to `stages` lanes at a time; after a
wait on the slot's EMPTY barrier for the previous round, it arms the slot's
FULL barrier with the byte count and starts the load. Consumer warp w takes
positions w, w + warps, ... of each work item, waits on FULL with the round's
parity, reads the slot and arrives on EMPTY; all consumer warps meet at a
barrier between work items. mbarrier waits test a phase PARITY, so a waiter
that is two phases early sees the wrong phase as complete.

This model runs random interleavings of that protocol and checks that no
consumer reads a slot before its load landed, no load overwrites a slot that
was not consumed, nothing deadlocks, and every position is consumed. It pins
the rule the kernels enforce with a static_assert: the stage count must be a
multiple of the consumer-warp count (with other counts the model finds early
reads, the failure that made a 6-stage, 4-warp build fault on the GPU).
"""
import random

import pytest


class Barrier:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.phase = 0
        self.tx = 0

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        self._advance()

    def complete_tx(self, n):
        self.tx -= n
        self._advance()

    def _advance(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def test_parity(self, parity):
        """mbarrier.try_wait.parity: true iff the phase with this parity completed,
        i.e. the current phase's parity differs."""
        return (self.phase & 1) != parity


def simulate(stages, warps, items, seed, max_steps=2_000_000):
    rnd = random.Random(seed)
    full = [Barrier(1) for _ in range(stages)]
    empty = [Barrier(1) for _ in range(stages)]
    slot = [None] * stages
    inflight = []
    producer = []
    g = 0
    for n_sub in items:
        for base in range(0, n_sub, 32):
            cnt = min(32, n_sub - base)
            for k0 in range(0, cnt, stages):
                producer.append([g + base + l for l in range(k0, min(k0 + stages, cnt))])
        g += n_sub
    total = g
    programs = []
    for w in range(warps):
        ops, g = [], 0
        for n_sub in items:
            ops += [("sub", g + i) for i in range(w, n_sub, warps)]
            ops.append(("barrier", None))
            g += n_sub
        programs.append(ops)
    pc = [0] * warps
    at_barrier = [False] * warps
    arrived = 0
    pi, pending = 0, None
    consumed = set()
    for _ in range(max_steps):
        progress = False
        if inflight and rnd.random() < 0.5:
            st, pos = inflight.pop(rnd.randrange(len(inflight)))
            slot[st] = pos
            full[st].complete_tx(1)
            progress = True
        if pi < len(producer) and rnd.random() < 0.5:
            if pending is None:
                pending = list(producer[pi])
            for pos in list(pending):
                st, rd = pos % stages, pos // stages
                if empty[st].test_parity((rd & 1) ^ 1):
                    if slot[st] is not None and slot[st] not in consumed:
                        return f"slot {st} overwritten before position {slot[st]} was read"
                    full[st].arrive(tx=1)
                    inflight.append((st, pos))
                    pending.remove(pos)
                    progress = True
            if not pending:
                pending = None
                pi += 1
        w = rnd.randrange(warps)
        if pc[w] < len(programs[w]):
            op, pos = programs[w][pc[w]]
            if op == "sub":
                st, rd = pos % stages, pos // stages
                if full[st].test_parity(rd & 1):
                    if slot[st] != pos:
                        return f"position {pos} read from slot {st} holding {slot[st]}"
                    consumed.add(pos)
                    empty[st].arrive()
                    pc[w] += 1
                    progress = True
            elif not at_barrier[w]:
                at_barrier[w] = True
                arrived += 1
                if arrived == warps:
                    arrived = 0
                    at_barrier = [False] * warps
                    pc = [x + 1 for x in pc]
                progress = True
        if pi >= len(producer) and all(pc[x] >= len(programs[x]) for x in range(warps)) \
                and not inflight:
            return "ok" if len(consumed) == total else "positions lost"
        if not progress and not inflight:
            lanes = (pending if pending is not None else producer[pi]) if pi < len(producer) else []
            can = any(empty[p % stages].test_parity(((p // stages) & 1) ^ 1) for p in lanes)
            for x in range(warps):
                if pc[x] < len(programs[x]):
                    op, pos = programs[x][pc[x]]
                    can |= (full[pos % stages].test_parity((pos // stages) & 1) if op == "sub"
                            else not at_barrier[x])
            if not can:
                return "deadlock"
    return "did not finish"


def kernel_stages(stage_bytes, ring_bytes=65536, warps=4):
    """The kernels' stage count: what fits, rounded down to a multiple of the warps."""
    fit = ring_bytes // stage_bytes
    return warps if fit < warps else (fit // warps) * warps


def _items(seed):
    r = random.Random(seed)
    return [r.choice([32, 32, 7, 1, 45, 64, 3, 16]) for _ in range(r.randint(1, 5))]


@pytest.mark.parametrize("stage_bytes", [4096, 8192, 16384])   # bf16 d64, bf16 d128 / f32 d64, f32 d128
def test_shipped_configurations_are_safe(stage_bytes):
    stages = kernel_stages(stage_bytes)
    assert stages % 4 == 0
    for seed in range(60):
        assert simulate(stages, 4, _items(seed), seed) == "ok"


@pytest.mark.parametrize("stages,warps", [(4, 4), (8, 4), (12, 4), (6, 6), (16, 8)])
def test_multiples_are_safe(stages, warps):
    for seed in range(40):
        assert simulate(stages, warps, _items(seed), seed) == "ok"


@pytest.mark.parametrize("stages,warps", [(6, 4), (12, 8), (10, 4)])
def test_non_multiples_break(stages, warps):
    results = [simulate(stages, warps, _items(seed), seed) for seed in range(40)]
    assert any(r != "ok" for r in results)


def test_rounding_rule():
    assert kernel_stages(8192, 49152) == 4          # 6 fit: rounded down to 4
    assert kernel_stages(8192, 65536) == 8
    assert kernel_stages(16384, 65536) == 4
    assert kernel_stages(16384, 32768) == 4         # never fewer than the warps


# ---------------------------------------------------------------------------
# The grouped kernel's ring: every consumer warp reads EVERY position (each
# position is a unit some of the group's sequences use), the EMPTY barrier
# counts all consumer warps, and there is no barrier between work items. A
# warp can then never be more than one phase ahead of a slot, whatever the
# stage count, because the producer cannot refill a slot that this warp has
# not released.
# ---------------------------------------------------------------------------
def simulate_broadcast(stages, warps, batches, seed, max_steps=2_000_000):
    rnd = random.Random(seed)
    full = [Barrier(1) for _ in range(stages)]
    empty = [Barrier(warps) for _ in range(stages)]
    slot = [None] * stages
    reads = [0] * stages              # warps that read the slot's current position
    inflight = []
    producer = []
    g = 0
    for units in batches:             # units issued by one batch, sub-rounds of `stages`
        for k0 in range(0, units, stages):
            producer.append([g + u for u in range(k0, min(k0 + stages, units))])
        g += units
    total = g
    pc = [0] * warps
    pi, pending = 0, None
    for _ in range(max_steps):
        progress = False
        if inflight and rnd.random() < 0.5:
            st, pos = inflight.pop(rnd.randrange(len(inflight)))
            slot[st] = pos
            reads[st] = 0
            full[st].complete_tx(1)
            progress = True
        if pi < len(producer) and rnd.random() < 0.5:
            if pending is None:
                pending = list(producer[pi])
            for pos in list(pending):
                st, rd = pos % stages, pos // stages
                if empty[st].test_parity((rd & 1) ^ 1):
                    if slot[st] is not None and reads[st] != warps:
                        return f"slot {st} overwritten before all warps read position {slot[st]}"
                    full[st].arrive(tx=1)
                    inflight.append((st, pos))
                    pending.remove(pos)
                    progress = True
            if not pending:
                pending = None
                pi += 1
        w = rnd.randrange(warps)
        if pc[w] < total:
            pos = pc[w]
            st, rd = pos % stages, pos // stages
            if full[st].test_parity(rd & 1):
                if slot[st] != pos:
                    return f"warp {w}: position {pos} read from slot {st} holding {slot[st]}"
                reads[st] += 1
                empty[st].arrive()
                pc[w] += 1
                progress = True
        if pi >= len(producer) and all(x >= total for x in pc) and not inflight:
            return "ok"
        if not progress and not inflight:
            lanes = (pending if pending is not None else producer[pi]) if pi < len(producer) else []
            can = any(empty[p % stages].test_parity(((p // stages) & 1) ^ 1) for p in lanes)
            can |= any(pc[x] < total and full[pc[x] % stages].test_parity((pc[x] // stages) & 1)
                       for x in range(warps))
            if not can:
                return "deadlock"
    return "did not finish"


def _batches(seed):
    r = random.Random(seed)
    return [r.choice([1, 3, 32, 40, 64, 7, 128]) for _ in range(r.randint(1, 6))]


@pytest.mark.parametrize("stages,warps", [(6, 2), (6, 4), (5, 3), (12, 1), (3, 4), (7, 8)])
def test_broadcast_ring_is_safe_for_any_stage_count(stages, warps):
    for seed in range(40):
        assert simulate_broadcast(stages, warps, _batches(seed), seed) == "ok"


def test_broadcast_ring_needs_every_warp_to_release():
    """With an EMPTY count below the number of readers the producer refills a
    slot that a warp has not read: the model must catch it."""
    def broken(stages, warps, batches, seed):
        orig = Barrier.__init__

        def init(self, count):
            orig(self, 1 if count == warps else count)
        Barrier.__init__ = init
        try:
            return simulate_broadcast(stages, warps, batches, seed)
        finally:
            Barrier.__init__ = orig
    results = [broken(6, 2, _batches(seed), seed) for seed in range(40)]
    assert any(r != "ok" for r in results)
