"""Event model of the encoder's shared-memory stage ring (host only).

The encoder CTA has one producer and 23 consumer warps.  The producer fills
4 stages with units of 16 warp items.  Warp w takes items w, w + 23, ...,
so it has no item in some units.  mbarrier waits test a phase parity, which
tells only two phases of a barrier apart.  This model replays the ring with
random copy latencies, so copies can land out of order.  It checks that with
two full barriers per stage (unit u on barrier u mod 8, as the kernel does)
no wait ever returns before its own unit has landed, no barrier phase gets
an extra arrival, every warp finishes, and every item reads its own unit.
It also checks that the same model catches the failure of one full barrier
per stage, so a model too coarse to see aliasing would fail here.
"""
import heapq
import random

import pytest

STAGES, ITEMS, WARPS = 4, 16, 23


class Barrier:
    """Phase counter with an arrival count and a transaction count."""

    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0
        self.over_arrivals = 0

    def _complete_if_done(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self, tx=0):
        if self.pending <= 0:
            self.over_arrivals += 1
        self.tx += tx
        self.pending -= 1
        self._complete_if_done()

    def complete_tx(self, n):
        self.tx -= n
        self._complete_if_done()

    def parity_passed(self, parity):
        """try_wait.parity: true once the phase of that parity is not the current one."""
        return (self.phase & 1) != parity


def replay(units, seed, full_per_stage, work, latency, jitter, gap):
    rng = random.Random(seed)
    n_full = full_per_stage * STAGES
    full = [Barrier(1) for _ in range(n_full)]
    empty = [Barrier(ITEMS) for _ in range(STAGES)]
    holds = [None] * STAGES            # unit whose bytes a stage holds
    landed_halves = {}
    out = dict(early=0, wrong_unit=0)
    events, seq = [], [0]

    def at(t, *what):
        heapq.heappush(events, (t, seq[0], what))
        seq[0] += 1

    # warp w's items: units of items w, w + 23, ...
    plans = []
    for w in range(WARPS):
        plans.append([i // ITEMS for i in range(w, units * ITEMS, WARPS)])
    pc = [0] * WARPS
    issued = [0]

    def producer(t):
        u = issued[0]
        if u >= units:
            return
        s = u % STAGES
        if not empty[s].parity_passed(((u // STAGES) & 1) ^ 1):
            at(t + 0.05, "producer")
            return
        full[u % n_full].arrive(tx=2)          # K and V copies
        issued[0] += 1
        for half in range(2):
            at(t + latency + rng.expovariate(1.0 / jitter), "landed", u, half)
        at(t + gap, "producer")

    def consumer(w, t):
        if pc[w] >= len(plans[w]):
            return
        u = plans[w][pc[w]]
        f = full[u % n_full]
        if not f.parity_passed((u // n_full) & 1):
            at(t + 0.05, "consumer", w)
            return
        if f.phase <= u // n_full:             # passed before unit u's own phase completed
            out["early"] += 1
        if holds[u % STAGES] != u:
            out["wrong_unit"] += 1
        at(t + rng.expovariate(1.0 / work), "released", w, u % STAGES)

    at(0.0, "producer")
    for w in range(WARPS):
        at(0.0, "consumer", w)
    deadline = 5.0 * units + 100.0
    while events:
        t, _, what = heapq.heappop(events)
        if t > deadline:
            out["deadlock"] = True
            break
        kind = what[0]
        if kind == "producer":
            producer(t)
        elif kind == "consumer":
            consumer(what[1], t)
        elif kind == "landed":
            u = what[1]
            landed_halves[u] = landed_halves.get(u, 0) + 1
            if landed_halves[u] == 2:
                holds[u % STAGES] = u
            full[u % n_full].complete_tx(1)
        else:                                  # released
            w, s = what[1], what[2]
            empty[s].arrive()
            pc[w] += 1
            at(t, "consumer", w)
    out["over_arrivals"] = sum(b.over_arrivals for b in full + empty)
    out["finished"] = all(pc[w] == len(plans[w]) for w in range(WARPS))
    out["deadlock"] = out.get("deadlock", False)
    return out


# (consumer work, copy latency, latency jitter, producer issue gap), arbitrary time units;
# fast consumers and widely spread copy latencies make out-of-order landings common
TIMINGS = [(0.05, 0.5, 1.0, 0.1), (0.05, 1.5, 3.0, 0.4), (0.2, 0.5, 3.0, 0.8), (0.5, 1.5, 1.0, 0.1)]


@pytest.mark.parametrize("timing", TIMINGS)
def test_two_full_barriers_per_stage_keep_every_wait_exact(timing):
    for seed in range(4):
        r = replay(120, seed, 2, *timing)
        assert r == dict(early=0, wrong_unit=0, over_arrivals=0, finished=True, deadlock=False), (seed, r)


def test_one_full_barrier_per_stage_is_caught_by_the_model():
    early = sum(replay(120, seed, 1, *timing)["early"] for timing in TIMINGS for seed in range(4))
    assert early > 0
