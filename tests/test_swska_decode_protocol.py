"""A randomized model of the stage ring of the SW-SKA decode kernel (csrc/swska_decode_warp.cu),
checked on the CPU.

A producer warp copies stages of 8 window slots into a ring of `stages` buffers (stage st in
buffer st mod stages). Each of the CTA's HG head warps reads every stage in order, and a buffer
is refilled once all HG of them have arrived on its empty barrier. The model uses mbarrier parity
semantics and copies that land at random times. It checks that every head reads every stage
once, in order, from a buffer that holds it.

The negative control is a variant that was tried and dropped. There, each head's stages were
shared round-robin among WS warps over the same ring. A fast warp could then wait on a buffer
whose previous stage, another warp's, was not yet loaded: a parity wait two phases ahead passes
at once. The model catches it.
"""
import random

import pytest

from .barrier_model import Bar, simulate


def run(HG, stages, nst, seed, ws=1):
    """ws > 1: the dropped variant, ws warps per head sharing the ring round-robin."""
    full = [Bar(1) for _ in range(stages)]
    empty = [Bar(HG) for _ in range(stages)]
    ring = [None] * stages
    seen = {}
    copies = []

    def producer():
        for st in range(nst):
            b = st % stages
            if st >= stages:
                yield ("wait", empty[b], ((st // stages) - 1) & 1)
            full[b].expect_tx(1)
            copies.append((b, st))
            yield ("step",)

    def consumer(h, w):
        seen[(h, w)] = []
        for st in range(w, nst, ws):
            b = st % stages
            yield ("wait", full[b], (st // stages) & 1)
            assert ring[b] == st, f"head {h} warp {w} read stage {ring[b]} for {st}"
            seen[(h, w)].append(st)
            yield ("step",)
            empty[b].arrive()

    def land(copy):
        b, st = copy
        ring[b] = st
        full[b].complete_tx(1)

    actors = {"producer": producer()}
    for h in range(HG):
        for w in range(ws):
            actors[f"head {h} warp {w}"] = consumer(h, w)
    simulate(seed, actors, [], copies, lambda op: None, land)
    for (h, w), got in seen.items():
        assert got == list(range(w, nst, ws))


@pytest.mark.parametrize("HG,stages", [(16, 3), (8, 4), (4, 8), (1, 16)])
def test_single_consumer_ring_holds(HG, stages):
    for seed in range(60):
        run(HG, stages, random.Random(seed).choice([0, 1, 2, 5, 17, 33, 64]), seed)


def test_model_catches_the_shared_round_robin_variant():
    caught = 0
    for seed in range(100):
        try:
            run(4, 6, 40, seed, ws=4)
        except AssertionError:
            caught += 1
    assert caught >= 50, f"caught in {caught} of 100 runs"
