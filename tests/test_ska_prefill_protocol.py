"""A randomized model of the hand-off protocol of the persistent tensor-core SW-SKA prefill
(csrc/swska_prefill_tc.cu), checked on the CPU.

The kernel's roles meet only at mbarriers:
- the TMA producer loads Q per item, then the K, V0, V1 tiles of every key tile into a
  four-slot ring;
- the MMA issuer issues S_h = Q_h K^T and O_h += P_h V_h;
- two softmax warpgroups (one per head of the pair) turn S_h into P_h, handing it over in two
  halves of 64 keys, and write each item's output rows once the item's last P V is done.

The model runs these roles as coroutines under a random scheduler. The barriers follow mbarrier
semantics, including the parity wait that cannot tell a phase from the one two phases back.
MMAs execute in issue order, with a commit arriving once everything issued before it has
executed, and TMA copies land at random times. Every read is checked against the data it must
see:
- each MMA reads the Q, K, V and P tiles of its own (item, key tile);
- O is reset only after the previous item's output rows were read, and is accumulated in order;
- no ring slot or Q buffer is overwritten before all of its readers ran;
- the epilogue sees the complete O of its item.

Three planted protocol mistakes must each be caught.
"""
import random

import pytest

from .barrier_model import Bar, simulate

NSLOT = 4


def run(items, seed, mistake=None):
    """items: key tiles per work item of one CTA, in order. Raises AssertionError on a
    protocol violation or a deadlock."""
    full = [Bar(1) for _ in range(NSLOT)]
    empty = [Bar(1) for _ in range(NSLOT)]
    qfull, qempty = Bar(1), Bar(1)
    sfull = [Bar(1), Bar(1)]
    phalf = [Bar(128), Bar(128)]
    pfull = [Bar(128), Bar(128)]
    odone = [Bar(1), Bar(1)]
    slot, slot_reads = [None] * NSLOT, [0] * NSLOT
    st = {"q": None, "q_reads": 0}
    S, S_reading = [None, None], [False, False]
    P = [[None, None], [None, None]]
    O = [None, None]
    epilogue_done = [set(), set()]
    pipe, copies = [], []

    def producer():
        nq = L = 0
        for it, n_it in enumerate(items):
            if nq > 0 and mistake != "q_loaded_without_qempty":
                yield ("wait", qempty, (nq - 1) & 1)
            qfull.expect_tx(2)
            copies.append(("q", None, it, qfull, 2))
            nq += 1
            for l in range(3 * n_it):
                s, use = L % NSLOT, L // NSLOT
                if use > 0:
                    yield ("wait", empty[s], (use - 1) & 1)
                j, which = divmod(l, 3)
                tile = ("K", it, j) if which == 0 else ("V", which - 1, it, j)
                full[s].expect_tx(1)
                copies.append(("slot", s, tile, full[s], 1))
                L += 1
                yield ("step",)

    def issuer():
        Lb = tb = 0
        for it, n_it in enumerate(items):
            yield ("wait", qfull, it & 1)
            yield ("wait", full[Lb % NSLOT], (Lb // NSLOT) & 1)
            pipe.extend([("S", 0, it, 0, Lb % NSLOT), ("C", sfull[0]), ("S", 1, it, 0, Lb % NSLOT),
                         ("C", sfull[1]), ("C", empty[Lb % NSLOT])])
            if n_it == 1:
                pipe.append(("C", qempty))
            for j in range(n_it):
                more, Lj, tj = j + 1 < n_it, Lb + 3 * j, tb + j
                for h in (0, 1):
                    Lv = Lj + 1 + h
                    yield ("wait", full[Lv % NSLOT], (Lv // NSLOT) & 1)
                    yield ("wait", phalf[h], tj & 1)
                    pipe.append(("PV", h, it, j, 0, Lv % NSLOT))
                    yield ("wait", pfull[h], tj & 1)
                    pipe.extend([("PV", h, it, j, 1, Lv % NSLOT), ("C", empty[Lv % NSLOT])])
                    if not more:
                        pipe.append(("C", odone[h]))
                        continue
                    Lk = Lj + 3
                    if h == 0:
                        yield ("wait", full[Lk % NSLOT], (Lk // NSLOT) & 1)
                    pipe.extend([("S", h, it, j + 1, Lk % NSLOT), ("C", sfull[h])])
                    if h == 1:
                        pipe.append(("C", empty[Lk % NSLOT]))
                        if j + 2 == n_it:
                            pipe.append(("C", qempty))
            Lb += 3 * n_it
            tb += n_it

    def softmax(h):
        tb = 0
        for it, n_it in enumerate(items):
            for j in range(n_it):
                parity = (j if mistake == "tile_parity_per_item" else tb + j) & 1
                yield ("wait", sfull[h], parity)
                assert S[h] == (it, j), f"softmax {h} read S {S[h]}, expected {(it, j)}"
                S_reading[h] = True
                yield ("step",)
                S_reading[h] = False
                P[h][0] = (it, j)
                phalf[h].arrive(128)
                yield ("step",)
                P[h][1] = (it, j)
                pfull[h].arrive(128)
            if mistake == "next_item_before_epilogue":
                tb += n_it
                continue
            yield ("wait", odone[h], it & 1)
            assert O[h] == (it, 2 * n_it), f"epilogue {h} of item {it} saw O {O[h]}"
            yield ("step",)
            epilogue_done[h].add(it)
            tb += n_it

    def execute(op):
        if op[0] == "C":
            op[1].arrive()
            return
        if op[0] == "S":
            _, h, it, j, s = op
            assert st["q"] == it and slot[s] == ("K", it, j), f"S{h}{(it, j)} read Q {st['q']}, {slot[s]}"
            assert not S_reading[h], "S overwritten while the softmax reads it"
            S[h], P[h] = (it, j), [None, None]
            slot_reads[s] += 1
            st["q_reads"] += 1
            return
        _, h, it, j, half, s = op
        assert P[h][half] == (it, j), f"PV{h}{(it, j, half)} read P {P[h][half]}"
        assert slot[s] == ("V", h, it, j), f"PV{h}{(it, j)} read {slot[s]}"
        if j == 0 and half == 0:
            assert it == 0 or (it - 1) in epilogue_done[h], "O reset before the last epilogue read it"
            O[h] = (it, 1)
        else:
            assert O[h] == (it, 2 * j + half), f"PV{h}{(it, j, half)} accumulates onto {O[h]}"
            O[h] = (it, 2 * j + half + 1)
        slot_reads[s] += 1

    def land(copy):
        kind, s, tile, bar, nbytes = copy
        if kind == "q":
            prev = items[tile - 1] if tile > 0 else 0
            assert st["q_reads"] == 2 * prev, "Q overwritten before its score MMAs ran"
            st["q"], st["q_reads"] = tile, 0
        else:
            assert slot[s] is None or slot_reads[s] == 2, f"slot {s} overwritten: {slot[s]}"
            slot[s], slot_reads[s] = tile, 0
        bar.complete_tx(nbytes)

    actors = {"producer": producer(), "issuer": issuer(), "softmax0": softmax(0), "softmax1": softmax(1)}
    simulate(seed, actors, [pipe], copies, execute, land)
    if mistake != "next_item_before_epilogue":
        assert all(len(epilogue_done[h]) == len(items) for h in (0, 1))


def _items(seed, at_least=1):
    rnd = random.Random(seed)
    return [rnd.choice([1, 1, 2, 3, 5, 33]) for _ in range(rnd.randint(at_least, 6))]


def test_protocol_holds_over_random_item_sequences():
    for seed in range(400):
        run(_items(seed), seed)


@pytest.mark.parametrize("mistake", ["q_loaded_without_qempty", "tile_parity_per_item",
                                     "next_item_before_epilogue"])
def test_model_catches_planted_protocol_mistakes(mistake):
    caught = 0
    for seed in range(100):
        try:
            run(_items(seed, at_least=2), seed, mistake)
        except AssertionError:
            caught += 1
    assert caught >= 50, f"{mistake}: caught in {caught} of 100 runs"
