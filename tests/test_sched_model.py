"""A step-by-step model of the grouped GEMM's run-time tile hand-out, run under random
interleavings of the CTA pairs and random early stops (a wait that ran out).

The kernel's leader producer draws tickets from a per-mode counter with atomicAdd: one
before its loop, then the next tile's ticket when a tile starts, published a few K blocks
later (a ticket at or past the tile count publishes "no more tiles").  A pair that stopped
early keeps drawing until it holds a ticket past the end.  The pair that draws ticket
tiles + pairs - 1 resets the counter.  The model checks what the reset relies on, for every
schedule: each pair draws exactly one ticket at or past the tile count; the reset happens
once, after the last draw of the launch, so the counter ends at 0; without early stops every
tile is processed exactly once, and with them no tile is processed twice.

Passage: dots.llm1 Technical Report, §3.2 "Efficient implementation of Grouped GEMM" (tiles
of aligned expert segments are scheduled like those of a plain GEMM).
"""
import random

import pytest


class Launch:
    def __init__(self, tiles, pairs):
        self.tiles, self.pairs = tiles, pairs
        self.counter = 0
        self.draws = 0
        self.resets = 0
        self.draws_at_reset = None
        self.processed = []

    def draw(self):
        t = self.counter
        self.counter += 1
        self.draws += 1
        return t

    def ticket_done(self, t):
        if t == self.tiles + self.pairs - 1:
            self.counter = 0
            self.resets += 1
            self.draws_at_reset = self.draws


def writer(launch, stop_after, stop_in_k_loop):
    """The leader producer's ticket logic as a generator: one yield per atomic step.
    stop_after: the number of tiles after which this pair's waits run out (None: never).
    stop_in_k_loop: the wait that runs out is a stage wait inside the K loop, after which
    the drawn ticket is still published; otherwise it is the wait for other ranks' rows,
    before the K loop, which leaves the drawn ticket unpublished."""
    state = {"cur": -1, "nxt": -1, "last": False, "past_end": 0}

    def publish(tk):
        state["cur"] = tk
        if tk >= launch.tiles:
            state["past_end"] += 1
            launch.ticket_done(tk)
            state["last"] = True
            state["cur"] = -1

    publish(launch.draw())
    yield
    done = 0
    aborted = False
    while True:
        tile = state["cur"]
        if tile < 0:
            break
        state["nxt"] = launch.draw()
        yield
        if stop_after is not None and done >= stop_after:
            aborted = True
            if stop_in_k_loop:  # the K loop broke; the tile's publish step still runs
                tk, state["nxt"] = state["nxt"], -1
                publish(tk)
                yield
            break
        launch.processed.append(tile)
        done += 1
        tk, state["nxt"] = state["nxt"], -1
        publish(tk)
        yield
    if not state["last"]:
        tk = state["nxt"] if state["nxt"] >= 0 else launch.draw()
        yield
        while tk < launch.tiles:
            tk = launch.draw()
            yield
        state["past_end"] += 1
        launch.ticket_done(tk)
    return state["past_end"], aborted


def run(tiles, pairs, seed, stop_prob):
    rng = random.Random(seed)
    launch = Launch(tiles, pairs)
    stops = [rng.randrange(0, 4) if rng.random() < stop_prob else None for _ in range(pairs)]
    gens = [writer(launch, s, rng.random() < 0.5) for s in stops]
    results = [None] * pairs
    live = list(range(pairs))
    while live:
        p = rng.choice(live)
        try:
            next(gens[p])
        except StopIteration as fin:
            results[p] = fin.value
            live.remove(p)
    return launch, results, stops


@pytest.mark.parametrize("tiles,pairs", [(0, 3), (1, 4), (7, 3), (40, 6), (300, 74)])
@pytest.mark.parametrize("stop_prob", [0.0, 0.3])
def test_every_pair_draws_one_ticket_past_the_end_and_the_counter_resets(tiles, pairs, stop_prob):
    for seed in range(25):
        launch, results, stops = run(tiles, pairs, seed, stop_prob)
        assert all(r[0] == 1 for r in results), (seed, results)
        assert launch.resets == 1, seed
        assert launch.draws_at_reset == launch.draws, seed  # no draw after the reset
        assert launch.counter == 0, seed
        assert len(set(launch.processed)) == len(launch.processed), seed  # never twice
        assert all(0 <= t < tiles for t in launch.processed), seed
        if not any(r[1] for r in results):
            assert sorted(launch.processed) == list(range(tiles)), seed
