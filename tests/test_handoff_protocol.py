"""Model check of the backward kernels' per-tile hand-off through named barriers.

In the key-owner kernel, and in the query-owner kernel where its resident Q
rows are in shared memory, each tile passes between the 16 gradient warps and
the MMA warp through two hardware named barriers: "student logits read" (the
MMA warp waits on it before it issues the student logits of tile t+2 into the
same logit buffer) and "dS written" (it waits on it before the gradient MMA
of tile t), each kind on four ids used in turn (tile t on id t mod 4).  The
gradient warps only arrive (bar.arrive); the MMA warp waits (bar.sync).  A named barrier has no timeout, so the protocol
must leave no schedule in which a participant waits for ever, including the
schedules in which a bounded mbarrier wait gives up part-way (then the warp
keeps taking part in the named barriers, with bar.sync, without doing the
work).

This test runs that protocol as a model: one MMA actor and G gradient actors
take their steps in random orders, and every bounded wait may give up at any
moment (a superset of what the 2 s budget allows).  It checks that

- no schedule deadlocks (every actor finishes);
- every phase of a named barrier is completed by arrivals for one and the
  same tile (a gradient warp never runs ahead into a phase the MMA warp has
  not passed);
- with no wait giving up, every tile's logits are committed and every tile is
  processed.

The model follows the kernels' steps: the MMA actor commits the logits of
tiles 0 and 1 up front (each after a stage wait that may give up); in iteration t it waits on "student logits read" of t
(when t+2 exists), issues the student logits of t+2 (a wait for the key or
query stage, which may give up), waits on "dS written" of t, then issues the
gradient MMA of t and the teacher logits of t+2 and commits tile t+2.  A
gradient actor waits for tile t's logits (a bounded mbarrier wait), arrives on
"student logits read" of t when t+2 exists, then on "dS written" of t.
"""
import random

import pytest

DS, SS = 1, 5          # first ids of the "dS written" and "student logits read" barriers
NIDS = 4               # ids of each kind, used in turn by tile index (t mod 4)


class NamedBarrier:
    """A CTA named barrier: `count` arrivals complete a phase and release its waiters."""

    def __init__(self, count):
        self.count = count
        self.arrived = []           # tiles of the arrivals in the current phase
        self.waiters = []           # actors blocked in bar.sync on the current phase
        self.phases = 0

    def arrive(self, tile):
        self.arrived.append(tile)
        if len(self.arrived) == self.count:
            assert len(set(self.arrived)) == 1, f"phase mixes tiles {self.arrived}"
            released = self.waiters
            self.arrived, self.waiters = [], []
            self.phases += 1
            return released
        return None


class Model:
    def __init__(self, n_tiles, n_grad, p_fail, rng, nids=NIDS):
        self.n = n_tiles
        self.rng = rng
        self.p_fail = p_fail
        self.nids = nids
        self.bars = {base + k: NamedBarrier(n_grad + 1) for base in (DS, SS) for k in range(nids)}
        self.committed = set()       # tiles whose logits the MMA actor has committed
        self.processed = [0] * n_tiles
        self.abort = False
        self.actors = [self.mma()] + [self.grad() for _ in range(n_grad)]
        self.state = {a: ("run", None) for a in self.actors}   # run | sync | wait
        self.result = {}

    # ---- steps an actor yields: ("arrive", id, t) ("sync", id, t) ("wait", t) ("try",) ("commit", t)
    def mma(self):
        n = self.n
        ok = True
        for t in range(min(2, n)):                # the first two tiles, each after its stage wait
            ok = yield ("try",)
            if not ok:
                break
            yield ("commit", t)
        for t in range(n):
            nxt = t + 2 < n
            if nxt:
                yield ("sync", SS + t % self.nids, t)
                if ok:
                    ok = yield ("try",)           # stage wait before the student logits of t+2
            yield ("sync", DS + t % self.nids, t)
            if ok and nxt:
                yield ("commit", t + 2)

    def grad(self):
        n = self.n
        ok = True
        for t in range(n):
            ssid = SS + t % self.nids if t + 2 < n else None
            if ok:
                ok = yield ("wait", t)
            if not ok:
                if ssid is not None:
                    yield ("sync", ssid, t)
                yield ("sync", DS + t % self.nids, t)
                continue
            self.processed[t] += 1
            if ssid is not None:
                yield ("arrive", ssid, t)
            yield ("arrive", DS + t % self.nids, t)

    # ---- scheduler
    def _advance(self, actor, value):
        try:
            req = actor.send(value)
        except StopIteration:
            self.state[actor] = ("done", None)
            return
        kind = req[0]
        if kind == "arrive":
            released = self.bars[req[1]].arrive(req[2])
            self._release(released)
            self.state[actor] = ("run", None)
        elif kind == "sync":
            bar = self.bars[req[1]]
            bar.waiters.append(actor)
            self.state[actor] = ("sync", req[1])
            self._release(bar.arrive(req[2]))
        elif kind == "wait":
            self.state[actor] = ("wait", req[1])
        elif kind == "try":
            fail = self.rng.random() < self.p_fail
            if fail:
                self.abort = True
            self.state[actor] = ("run", not fail)
        elif kind == "commit":
            self.committed.add(req[1])
            self.state[actor] = ("run", None)

    def _release(self, actors):
        for a in actors or []:
            self.state[a] = ("run", None)

    def run(self, max_steps=100000):
        for a in self.actors:
            self._advance(a, None)
        for _ in range(max_steps):
            live = [a for a in self.actors if self.state[a][0] != "done"]
            if not live:
                return True
            movable = []
            for a in live:
                kind, arg = self.state[a]
                if kind == "run":
                    movable.append(a)
                elif kind == "wait":
                    movable.append(a)          # a bounded wait can always end (success or give-up)
            if not movable:
                raise AssertionError("deadlock: " + ", ".join(str(self.state[a]) for a in live))
            a = self.rng.choice(movable)
            kind, arg = self.state[a]
            if kind == "run":
                self._advance(a, arg)
            else:                               # a bounded mbarrier wait on tile `arg`
                if arg in self.committed:
                    self._advance(a, True)
                elif self.abort or self.rng.random() < self.p_fail:
                    self.abort = True          # gave up (or saw another role give up)
                    self._advance(a, False)
                # else: keeps polling
        raise AssertionError("no progress within the step limit")


@pytest.mark.parametrize("n_grad", [1, 2, 3])
def test_no_schedule_deadlocks_or_mixes_tiles(n_grad):
    rng = random.Random(1234 + n_grad)
    for trial in range(1500):
        n = rng.choice([1, 2, 3, 4, 5, 6, 9])
        p_fail = rng.choice([0.0, 0.0, 0.01, 0.05, 0.2, 0.6])
        m = Model(n, n_grad, p_fail, rng)
        assert m.run(), (trial, n, p_fail)
        # every named barrier completed exactly as many phases as the MMA actor waited on it
        waited = {DS + k: sum(1 for t in range(n) if t % NIDS == k) for k in range(NIDS)}
        waited.update({SS + k: sum(1 for t in range(n) if t + 2 < n and t % NIDS == k) for k in range(NIDS)})
        for i, bar in m.bars.items():
            assert bar.phases == waited[i] and not bar.arrived and not bar.waiters, (trial, i)


@pytest.mark.parametrize("n", [1, 2, 3, 8, 17])
def test_without_give_ups_every_tile_is_processed(n):
    rng = random.Random(n)
    for _ in range(200):
        m = Model(n, 3, 0.0, rng)
        assert m.run()
        assert m.committed == set(range(n))
        assert m.processed == [3] * n
        assert not m.abort


def test_one_id_per_logit_buffer_is_not_enough():
    # With two ids of each kind (one per logit buffer) a gradient warp whose
    # wait gave up (another role had given up first) reaches tile t+2 while
    # its own arrival for tile t, on the same id, still waits for the MMA warp:
    # the phase then completes with tiles t and t+2, and the MMA warp's later
    # wait on it can never complete.  Normal arrivals run at most two tiles
    # ahead of the MMA warp (a tile's logits are committed only after the MMA
    # warp has passed tile t-2), so three ids would do; four are used.
    rng = random.Random(7)
    failures = 0
    for _ in range(1500):
        m = Model(rng.choice([3, 4, 5, 6, 9]), rng.choice([1, 2, 3]), rng.choice([0.05, 0.2, 0.6]), rng, nids=2)
        try:
            m.run()
        except AssertionError:
            failures += 1
    assert failures > 0


@pytest.mark.parametrize("nids", [3, 4])
def test_three_ids_suffice(nids):
    rng = random.Random(99 + nids)
    for _ in range(1500):
        m = Model(rng.choice([1, 2, 3, 4, 5, 6, 9]), rng.choice([1, 2, 3]), rng.choice([0.0, 0.05, 0.2, 0.6]), rng,
                  nids=nids)
        assert m.run()


def test_a_gradient_warp_that_only_arrived_after_giving_up_would_deadlock():
    # The reason the give-up path uses bar.sync: with bar.arrive there, a warp
    # that gave up races through the remaining tiles, a phase collects the
    # arrivals of two different tiles and the MMA warp waits for ever.
    class ArriveOnGiveUp(Model):
        def grad(self):
            n = self.n
            ok = True
            for t in range(n):
                ssid = SS + t % self.nids if t + 2 < n else None
                if ok:
                    ok = yield ("wait", t)
                if not ok:
                    if ssid is not None:
                        yield ("arrive", ssid, t)
                    yield ("arrive", DS + t % self.nids, t)
                    continue
                if ssid is not None:
                    yield ("arrive", ssid, t)
                yield ("arrive", DS + t % self.nids, t)

    rng = random.Random(7)
    failures = 0
    for _ in range(400):
        m = ArriveOnGiveUp(9, 2, 0.3, rng)
        try:
            m.run()
        except AssertionError:
            failures += 1
    assert failures > 0
