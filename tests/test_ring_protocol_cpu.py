"""A host model of the CUDA-core kernel's ring protocol over pages that tiles
straddle (attn_simt.cu, producer and consumers), run under random
interleavings.

The model takes the kernel's barrier operations one for one:
- stage tags, set by the producer once a stage is free;
- the empty barrier of every stage, released by the consumer of its tile (or
  by the producer for a skipped slot);
- the quad barriers, armed by copies that land at arbitrary later times and
  closed by one producer arrival;
- the consumers' parity waits, with the hardware's rule that a parity wait
  returns once the phase before the current one has that parity.

Tiles go round-robin to the consumer warps, by their CTA tile index.  A
segment's first tile starts a quad; the slots after its last tile, up to the
next quad, are skipped.

Every run must finish without a deadlock, and every consumer must read its
tile's own data, landed.  The test also checks that the order the first build
used, closing a segment's last quad before the skipped slots' waits, fails
under the same model.
"""
import random

import pytest


class Barrier:
    """mbarrier: arrivals expected per phase, a transaction count, and the
    number of completed phases."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.completed = 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count

    def arrive(self):
        self.pending -= 1
        self._maybe_complete()

    def expect_tx(self, n):
        self.tx += n

    def complete_tx(self, n):
        self.tx -= n
        self._maybe_complete()

    def parity_done(self, parity):
        # the phase before the current one has parity `parity`
        return (self.completed & 1) != parity


def simulate(n_stage, n_cw, seg_tiles, seed, close_first=False):
    """Returns None on success, else a description of the failure."""
    rng = random.Random(seed)
    full = [Barrier(1) for _ in range(n_stage)]
    empty = [Barrier(1) for _ in range(n_stage)]
    tag = [-1] * n_stage
    data = [None] * n_stage          # (tile, landed) of each stage's rows
    in_flight = []                   # copies: (stage, tile, barrier)
    # tiles: CTA index of every tile, per segment (a segment starts a quad)
    tiles, T = [], 0
    for n in seg_tiles:
        tiles.append(list(range(T, T + n)))
        T += n
        T = (T + 3) & ~3
    errors = []

    def producer():
        T = 0
        for seg in tiles:
            quad = -1
            for Tt in seg:
                s = Tt % n_stage
                if Tt >> 2 != quad:
                    if quad >= 0:
                        full[(quad * 4 + 3) % n_stage].arrive()
                    quad = Tt >> 2
                yield lambda s=s, Tt=Tt: empty[s].parity_done(((Tt // n_stage) & 1) ^ 1)
                tag[s] = Tt
                data[s] = (Tt, False)
                bar = full[(quad * 4 + 3) % n_stage]
                bar.expect_tx(1)
                in_flight.append((s, Tt, bar))
                T = Tt + 1
            skipped = list(range(T, (T + 3) & ~3))
            if close_first:
                full[(quad * 4 + 3) % n_stage].arrive()
                for Ts in skipped:
                    s = Ts % n_stage
                    yield lambda s=s, Ts=Ts: empty[s].parity_done(((Ts // n_stage) & 1) ^ 1)
                    empty[s].arrive()
            else:
                for Ts in skipped:
                    s = Ts % n_stage
                    yield lambda s=s, Ts=Ts: empty[s].parity_done(((Ts // n_stage) & 1) ^ 1)
                full[(quad * 4 + 3) % n_stage].arrive()
                for Ts in skipped:
                    empty[Ts % n_stage].arrive()
            T = (T + 3) & ~3

    def consumer(w):
        for seg in tiles:
            for Tt in seg:
                if Tt % n_cw != w:
                    continue
                s = Tt % n_stage
                yield lambda s=s, Tt=Tt: tag[s] == Tt
                yield lambda s=s, Tt=Tt: full[s | 3].parity_done((Tt // n_stage) & 1)
                if data[s] != (Tt, True):
                    errors.append(f"warp {w} read tile {Tt}: stage {s} holds {data[s]}")
                    return
                empty[s].arrive()

    agents = [producer()] + [consumer(w) for w in range(n_cw)]
    waits = [None] * len(agents)
    live = list(range(len(agents)))
    for i in live:
        waits[i] = next(agents[i], None)
    live = [i for i in live if waits[i] is not None]
    steps = 0
    while (live or in_flight) and not errors:
        steps += 1
        if steps > 200000:
            return "no progress bound reached"
        ready = [i for i in live if waits[i]()]
        choices = ready + (["land"] if in_flight else [])
        if not choices:
            return "deadlock: " + ", ".join(str(i) for i in live)
        c = rng.choice(choices)
        if c == "land":
            s, Tt, bar = in_flight.pop(rng.randrange(len(in_flight)))
            if data[s] == (Tt, False):
                data[s] = (Tt, True)
            bar.complete_tx(1)
            continue
        waits[c] = next(agents[c], None)
        if waits[c] is None:
            live.remove(c)
    return errors[0] if errors else None


def random_segments(rng, n):
    # short segments (1 to 6 tiles) with some longer ones
    return [rng.choice([1, 1, 2, 3, 4, 5, 6, 9, 13]) for _ in range(n)]


@pytest.mark.parametrize("n_stage,n_cw", [(12, 7), (12, 8), (8, 7)])
def test_quad_protocol_holds_under_random_interleavings(n_stage, n_cw):
    rng = random.Random(1000 + n_stage * 10 + n_cw)
    for trial in range(150):
        segs = random_segments(rng, rng.randrange(1, 25))
        res = simulate(n_stage, n_cw, segs, seed=trial)
        assert res is None, (segs, trial, res)


def test_closing_a_quad_before_the_skipped_waits_fails():
    """The first build's order: some interleaving deadlocks or reads stale data."""
    rng = random.Random(77)
    failures = 0
    for trial in range(400):
        segs = random_segments(rng, rng.randrange(2, 25))
        if simulate(8, 7, segs, seed=trial, close_first=True) is not None:
            failures += 1
    assert failures > 0
