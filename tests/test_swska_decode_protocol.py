"""A randomized model of the stage rings of the SW-SKA decode kernel (csrc/swska_decode_warp.cu),
checked on the CPU.

A producer warp copies stages of 8 window slots into C rings of D buffers: stage st goes to ring
st mod C, buffer (st / C) mod D of it. It sends the stages C at a time (one warp instruction
carries the copies of a batch, one stage per ring), once each of those buffers has been released.
Each head has C head warps; warp c of a head reads the stages c, c + C, ... of ring c in order,
and a buffer is refilled once the HG head warps that read it (one per head) have arrived on its
empty barrier. With C = 1 this is the single ring of the large-batch launches. The model uses
mbarrier parity semantics and copies that land at random times. It checks that every head warp
reads each of its stages once, in order, from a buffer that holds it.

Two negative controls. A producer that skips the wait for a buffer's release is caught. And the
variant that was tried and dropped: each head's stages shared round-robin among several warps
over ONE ring. A fast warp could then wait on a buffer whose previous stage, another warp's, was
not yet loaded: a parity wait two phases ahead passes at once. The model catches it.
"""
import random

import pytest

from .barrier_model import Bar, simulate


def run(HG, stages, nst, seed, ws=1, C=1, skip_wait=False):
    """C rings of `stages` buffers, C head warps per head (the kernel's layout). ws > 1: the
    dropped variant, ws warps per head sharing one ring round-robin (C must be 1). skip_wait:
    the planted mistake, a batch issued without waiting for its buffers' release."""
    full = [Bar(1) for _ in range(C * stages)]
    empty = [Bar(HG) for _ in range(C * stages)]
    ring = [None] * (C * stages)
    seen = {}
    copies = []

    def buf(st):
        return (st % C) * stages + (st // C) % stages

    def producer():
        for st0 in range(0, nst, C):
            u = st0 // C
            nb = min(C, nst - st0)
            if u >= stages and not skip_wait:
                for st in range(st0, st0 + nb):
                    yield ("wait", empty[buf(st)], ((u // stages) - 1) & 1)
            for st in range(st0, st0 + nb):
                full[buf(st)].expect_tx(1)
                copies.append((buf(st), st))
            yield ("step",)

    def consumer(h, w):
        seen[(h, w)] = []
        for st in range(w, nst, max(ws, C)):
            b = buf(st)
            yield ("wait", full[b], ((st // C) // stages) & 1)
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
        for w in range(max(ws, C)):
            actors[f"head {h} warp {w}"] = consumer(h, w)
    simulate(seed, actors, [], copies, lambda op: None, land)
    for (h, w), got in seen.items():
        assert got == list(range(w, nst, max(ws, C)))


@pytest.mark.parametrize("HG,stages,C", [(16, 3, 1), (8, 4, 1), (4, 8, 1), (1, 16, 1), (1, 2, 8), (2, 4, 4),
                                         (4, 2, 2), (1, 4, 4)])
def test_rings_hold(HG, stages, C):
    for seed in range(60):
        run(HG, stages, random.Random(seed).choice([0, 1, 2, 5, 17, 33, 64]), seed, C=C)


def test_model_catches_a_batch_that_skips_the_release_wait():
    caught = 0
    for seed in range(100):
        try:
            run(1, 2, 40, seed, C=8, skip_wait=True)
        except AssertionError:
            caught += 1
    assert caught >= 50, f"caught in {caught} of 100 runs"


def test_model_catches_the_shared_round_robin_variant():
    caught = 0
    for seed in range(100):
        try:
            run(4, 6, 40, seed, ws=4)
        except AssertionError:
            caught += 1
    assert caught >= 50, f"caught in {caught} of 100 runs"
