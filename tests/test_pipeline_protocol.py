"""Model check of the decode kernel's shared-memory pipeline protocol (CPU).

The persistent decode kernel runs one producer warp and NW consumer warps over
a ring of STAGES shared-memory stages, synchronised by mbarriers:

* ``empty[s]`` (NW arrivals): the consumers are done with stage s;
* ``full[s]`` (1 arrival + the bytes of the stage's page copies);
* ``qbar[s]`` (1 arrival + the bytes of the item's q copy): only an item's
  first stage uses it; the producer arrives after writing the item id (and
  the rope table) into the stage's slots, so the consumers learn the item
  and build their q fragments while the pages are still in flight.  The
  end-of-work sentinel (item -1) also arrives on qbar;
* ``merge`` (all consumer threads): the item-end merge of the warps' rows.

Each warp writes its merge rows into its page slots of the item's last
stage, keeps that stage until the merged row is stored, then releases it; or,
where the rows do not fit there, into one separate region that a second
merge-barrier round protects.

This file restates that protocol as a small simulation (the mbarrier
semantics: a phase completes when its pending arrivals and transaction bytes
both reach zero; a waiter waits for the completion of one phase, named by
its parity) and runs it under many random interleavings of the warps and of
the asynchronous copies landing.  It checks that every read sees the data of
its own item and stage, that no barrier ever runs two phases ahead of a
waiter (the parity could then alias), and that every run terminates.  It is
a model of the protocol, not of the CUDA source: the GPU parity tests check
the kernel itself.
"""
from __future__ import annotations

import random

import pytest


class MBarrier:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phase = 0  # completed phases

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self):
        assert self.pending > 0
        self.pending -= 1
        self._maybe_complete()

    def expect_tx(self, n):
        self.tx += n

    def complete_tx(self, n):
        assert self.tx >= n
        self.tx -= n
        self._maybe_complete()

    def done(self, phase):
        """Has phase ``phase`` completed?  A parity wait can only tell phases
        apart while the barrier is at most one phase past the waiter."""
        assert self.phase <= phase + 1, "barrier ran two phases ahead of a waiter"
        return self.phase > phase


class Machine:
    def __init__(self, stages, nw, separate_merge):
        self.S = stages
        self.NW = nw
        self.separate = separate_merge
        self.full = [MBarrier(1) for _ in range(stages)]
        self.empty = [MBarrier(nw) for _ in range(stages)]
        self.qbar = [MBarrier(1) for _ in range(stages)]
        self.merge = MBarrier(nw)
        self.pages = [None] * stages            # (item, stage index) of the landed pages
        self.q = [None] * stages                # item whose q landed
        self.item_id = [None] * stages          # written by the producer
        self.rope = [None] * stages             # rope table tag
        self.rows = [[None] * nw for _ in range(stages)]   # merge rows in the page slots
        self.sep_rows = [None] * nw             # the separate merge region
        self.inflight = []                      # copies issued and not landed
        self.merged = []                        # (warp, item) of every merge read


def producer(m, items):
    uses = [0] * m.S
    stage = 0
    for item, nst in enumerate(items):
        for si in range(nst):
            # wait for the consumers to release the stage's previous use
            e = uses[stage]
            yield lambda s=stage, e=e: e == 0 or m.empty[s].done(e - 1)
            first = si == 0
            m.full[stage].expect_tx(1)
            m.inflight.append(("pages", stage, (item, si)))
            if first:
                m.qbar[stage].expect_tx(1)
                m.inflight.append(("q", stage, item))
            yield lambda: True
            m.item_id[stage] = item
            m.rope[stage] = item
            yield lambda: True
            if first:
                m.qbar[stage].arrive()
            m.full[stage].arrive()
            uses[stage] += 1
            stage = (stage + 1) % m.S
            yield lambda: True
    e = uses[stage]
    yield lambda s=stage, e=e: e == 0 or m.empty[s].done(e - 1)
    m.item_id[stage] = -1
    m.qbar[stage].arrive()


def consumer(m, w, items, second_sync=True):
    qexp = [0] * m.S
    fexp = [0] * m.S
    mexp = 0
    stage = 0
    while True:
        e = qexp[stage]
        yield lambda s=stage, e=e: m.qbar[s].done(e)
        qexp[stage] += 1
        item = m.item_id[stage]
        if item == -1:
            return
        # q fragments and the rope table, before any page of the item landed
        assert m.q[stage] == item, "q read before it landed or after it was replaced"
        assert m.rope[stage] == item
        yield lambda: True
        nst = items[item]
        last = stage
        for si in range(nst):
            e = fexp[stage]
            yield lambda s=stage, e=e: m.full[s].done(e)
            fexp[stage] += 1
            assert m.pages[stage] == (item, si), "page read before it landed or after reuse"
            yield lambda: True
            last = stage
            if si + 1 < nst or m.separate:
                m.empty[stage].arrive()
            stage = (stage + 1) % m.S
            yield lambda: True
        # item end: rows, merge barrier, merged read, release
        if m.separate:
            m.sep_rows[w] = item
        else:
            m.rows[last][w] = item
        m.merge.arrive()
        e = mexp
        yield lambda e=e: m.merge.done(e)
        mexp += 1
        rows = m.sep_rows if m.separate else m.rows[last]
        assert all(r == item for r in rows), "merge rows overwritten before they were read"
        m.merged.append((w, item))
        yield lambda: True
        if m.separate and second_sync:
            # nobody writes the next item's rows before every warp read these
            m.merge.arrive()
            e = mexp
            yield lambda e=e: m.merge.done(e)
            mexp += 1
        elif not m.separate:
            m.empty[last].arrive()
        yield lambda: True


def land(m, copy):
    kind, stage, tag = copy
    if kind == "pages":
        m.pages[stage] = tag
        m.rows[stage] = [None] * m.NW   # the new pages overwrite the merge rows
        m.full[stage].complete_tx(1)
    else:
        m.q[stage] = tag
        m.qbar[stage].complete_tx(1)


def run(seed, stages, nw, separate, items, make_producer=producer, second_sync=True):
    rng = random.Random(seed)
    m = Machine(stages, nw, separate)
    procs = {"p": make_producer(m, items)}
    for w in range(nw):
        procs[w] = consumer(m, w, items, second_sync)
    waits = {k: next(g) for k, g in procs.items()}
    steps = 0
    while waits:
        steps += 1
        assert steps < 100000
        ready = [k for k, cond in waits.items() if cond()]
        choices = [("proc", k) for k in ready] + [("land", i) for i in range(len(m.inflight))]
        assert choices, "deadlock: every warp waits and no copy is in flight"
        kind, k = rng.choice(choices)
        if kind == "land":
            land(m, m.inflight.pop(k))
            continue
        try:
            waits[k] = next(procs[k])
        except StopIteration:
            del waits[k]
    assert not m.inflight
    assert sorted(m.merged) == sorted((w, i) for w in range(nw) for i in range(len(items)))


@pytest.mark.parametrize("stages", [1, 2, 3, 4])
@pytest.mark.parametrize("nw", [1, 2, 4])
@pytest.mark.parametrize("separate", [False, True])
def test_random_interleavings_keep_every_read_on_its_own_data(stages, nw, separate):
    rng = random.Random(1000 * stages + 10 * nw + separate)
    for trial in range(150):
        items = [rng.randint(1, 5) for _ in range(rng.randint(0, 6))]
        run(rng.randrange(1 << 30), stages, nw, separate, items)


def _early_publish(m, items):
    """A broken producer: it arrives on qbar before writing the item id."""
    uses = [0] * m.S
    stage = 0
    for item, nst in enumerate(items):
        for si in range(nst):
            e = uses[stage]
            yield lambda s=stage, e=e: e == 0 or m.empty[s].done(e - 1)
            first = si == 0
            m.full[stage].expect_tx(1)
            m.inflight.append(("pages", stage, (item, si)))
            if first:
                m.qbar[stage].expect_tx(1)
                m.inflight.append(("q", stage, item))
                m.qbar[stage].arrive()
            yield lambda: True
            m.item_id[stage] = item
            m.rope[stage] = item
            m.full[stage].arrive()
            uses[stage] += 1
            stage = (stage + 1) % m.S
            yield lambda: True
    e = uses[stage]
    yield lambda s=stage, e=e: e == 0 or m.empty[s].done(e - 1)
    m.item_id[stage] = -1
    m.qbar[stage].arrive()


def _failures(n, **kw):
    rng = random.Random(7)
    failures = 0
    for _ in range(n):
        try:
            run(rng.randrange(1 << 30), **kw)
        except (AssertionError, TypeError):
            failures += 1
    return failures


def test_the_model_catches_an_early_publish():
    """Control: arriving on qbar before the item id is written lets a
    consumer read a stale id under some interleaving."""
    assert _failures(300, stages=2, nw=2, separate=False, items=[2, 1, 3, 1],
                     make_producer=_early_publish) > 0


def test_the_model_catches_a_reused_merge_region():
    """Control: with one separate merge region and no second merge-barrier
    round, a fast warp writes the next item's rows over rows another warp
    has not read yet."""
    assert _failures(300, stages=3, nw=4, separate=True, items=[1, 1, 2, 1, 1],
                     second_sync=False) > 0
