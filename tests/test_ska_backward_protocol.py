"""Randomized models of the hand-off protocols of the tensor-core SW-SKA backward
(csrc/swska_backward_tc.cu), checked on the CPU: the key-tile kernel (ska_bwd_dkdv_kernel) here,
the query-tile kernel (ska_bwd_dq_kernel) further down.

One CTA owns a key tile and walks U = HG x n_q (head, query tile) units:
- the producer loads K once, the V tile of each head, and each unit's Q, dO and row
  statistics into a two-slot ring;
- the issuing warp computes S^T = K Q^T, dP^T = V dO^T, dV += P^T dO and dK += dS^T Q;
- two softmax warpgroups (one per half of the unit's queries) read S^T, write P^T over the first
  half of their dP^T columns (after reading it), then dS^T over the second half, and store each
  head's dV rows when the head's last unit is done.

The model runs these roles as coroutines under a random scheduler, with mbarrier parity
semantics, MMAs executing in issue order with commits, and copies landing at random times.
Every read is checked against the data it must see:
- each MMA reads the right K, V, Q, dO, P^T and dS^T;
- S^T and dP^T are overwritten only after both warpgroups have finished with them;
- dV is reset only after the previous head's rows were stored;
- dK accumulates every unit once;
- statistics and ring slots are reloaded only after their last reader.

Three planted protocol mistakes must each be caught. The model also shows that the issuer's
wait on dvfree before a head's first dV product is implied by its wait on pwritten: each
warpgroup stores the previous head's dV rows before it hands over the next P^T, so dropping
that wait breaks nothing (checked below).
"""
import random

import pytest

from .barrier_model import Bar, simulate


def run(HG, n_q, seed, mistake=None):
    U = HG * n_q
    kfull, vfull, vempty = Bar(1), Bar(1), Bar(1)
    full, empty = [Bar(1), Bar(1)], [Bar(1), Bar(1)]
    sfull, pfull, dvdone, done = Bar(1), Bar(1), Bar(1), Bar(1)
    sread, pwritten, dsready, dvfree = Bar(256), Bar(256), Bar(256), Bar(256)
    m = {"K": None, "V": None, "slot": [None, None], "slot_readers": [set(), set()],
         "S": None, "S_readers": set(), "dP": None, "P": [None, None], "dS": [None, None],
         "dP_readers": set(), "dV": None, "dV_stored": set(), "dK": 0}
    pipe, copies = [], []

    def producer():
        kfull.expect_tx(1)
        copies.append(("K", None, 0, kfull))
        for u in range(U):
            hi = u // n_q
            if u % n_q == 0:
                if hi > 0:
                    yield ("wait", vempty, (hi - 1) & 1)
                vfull.expect_tx(1)
                copies.append(("V", None, hi, vfull))
            s, use = u % 2, u // 2
            if use > 0 and mistake != "slot_reloaded_early":
                yield ("wait", empty[s], (use - 1) & 1)
            full[s].expect_tx(1)
            copies.append(("unit", s, u, full[s]))
            yield ("step",)

    def issuer():
        yield ("wait", kfull, 0)
        yield ("wait", vfull, 0)
        yield ("wait", full[0], 0)
        pipe.extend([("ST", 0), ("C", sfull), ("DPT", 0), ("C", pfull)])
        if n_q == 1:
            pipe.append(("C", vempty))
        for u in range(U):
            hi, first, last = u // n_q, u % n_q == 0, u % n_q == n_q - 1
            if u + 1 < U:
                if mistake != "next_s_before_sread":
                    yield ("wait", sread, u & 1)
                yield ("wait", full[(u + 1) % 2], ((u + 1) // 2) & 1)
                pipe.extend([("ST", u + 1), ("C", sfull)])
            yield ("wait", pwritten, u & 1)
            if first and hi > 0 and mistake != "dv_reset_without_dvfree":
                yield ("wait", dvfree, (hi - 1) & 1)
            pipe.append(("DV", u, first))
            if last:
                pipe.append(("C", dvdone))
            if mistake == "dpt_before_dsready" and u + 1 < U and (u + 1) % n_q != 0:
                pipe.extend([("DPT", u + 1), ("C", pfull)])
            yield ("wait", dsready, u & 1)
            pipe.extend([("DK", u), ("C", empty[u % 2])])
            if u + 1 < U and not (mistake == "dpt_before_dsready" and (u + 1) % n_q != 0):
                if (u + 1) % n_q == 0:
                    yield ("wait", vfull, ((u + 1) // n_q) & 1)
                pipe.extend([("DPT", u + 1), ("C", pfull)])
                if (u + 1) % n_q == n_q - 1:
                    pipe.append(("C", vempty))
        pipe.append(("C", done))

    def softmax(w):
        for u in range(U):
            hi = u // n_q
            yield ("wait", sfull, u & 1)
            assert m["S"] == u, f"half {w} read S^T of unit {m['S']} for {u}"
            assert m["slot"][u % 2] == u, "row statistics of another unit"
            m["S_readers"].add(w)
            sread.arrive(128)
            yield ("step",)
            yield ("wait", pfull, u & 1)
            assert m["dP"] == u, f"half {w} read dP^T of unit {m['dP']} for {u}"
            m["P"][w] = u          # over the first half of this warpgroup's dP^T columns
            pwritten.arrive(128)
            yield ("step",)
            assert m["dP"] == u, "dP^T overwritten before its second half was read"
            assert m["slot"][u % 2] == u, "row statistics reloaded before dS^T was formed"
            m["dS"][w] = u
            m["dP_readers"].add(w)
            dsready.arrive(128)
            if u % n_q == n_q - 1:
                yield ("wait", dvdone, hi & 1)
                assert m["dV"] == (hi, n_q), f"half {w} stored dV {m['dV']} for head {hi}"
                yield ("step",)
                m["dV_stored"].add((hi, w))
                dvfree.arrive(128)
        yield ("wait", done, 0)
        assert m["dK"] == U, f"dK holds {m['dK']} of {U} units"

    def execute(op):
        kind = op[0]
        if kind == "C":
            op[1].arrive()
        elif kind == "ST":
            u = op[1]
            assert m["K"] == 0 and m["slot"][u % 2] == u
            assert m["S"] is None or m["S_readers"] == {0, 1}, "S^T overwritten while being read"
            m["S"], m["S_readers"] = u, set()
            m["slot_readers"][u % 2].add("ST")
        elif kind == "DPT":
            u = op[1]
            assert m["V"] == u // n_q and m["slot"][u % 2] == u
            assert m["dP"] is None or m["dP_readers"] == {0, 1}, "dP^T overwritten while in use"
            assert m["dP"] is None or m["dS"] == [m["dP"], m["dP"]], "dP^T overwritten before dK read dS^T"
            m["dP"], m["dP_readers"] = u, set()
            m["slot_readers"][u % 2].add("DPT")
        elif kind == "DV":
            u, first = op[1], op[2]
            hi = u // n_q
            assert m["P"] == [u, u] and m["slot"][u % 2] == u, f"dV({u}) read P^T {m['P']}"
            if first:
                assert hi == 0 or {(hi - 1, 0), (hi - 1, 1)} <= m["dV_stored"], \
                    "dV reset before the previous head's rows were stored"
                m["dV"] = (hi, 1)
            else:
                assert m["dV"] == (hi, u % n_q), f"dV({u}) accumulates onto {m['dV']}"
                m["dV"] = (hi, u % n_q + 1)
            m["slot_readers"][u % 2].add("DV")
        elif kind == "DK":
            u = op[1]
            assert m["dS"] == [u, u] and m["slot"][u % 2] == u, f"dK({u}) read dS^T {m['dS']}"
            assert m["dK"] == u
            m["dK"] += 1
            m["slot_readers"][u % 2].add("DK")

    def land(copy):
        kind, s, what, bar = copy
        if kind == "K":
            m["K"] = what
        elif kind == "V":
            m["V"] = what
        else:
            prev = m["slot"][s]
            assert prev is None or m["slot_readers"][s] == {"ST", "DPT", "DV", "DK"}, \
                f"slot {s} reloaded while unit {prev} is in use"
            m["slot"][s], m["slot_readers"][s] = what, set()
        bar.complete_tx(1)

    actors = {"producer": producer(), "issuer": issuer(), "half0": softmax(0), "half1": softmax(1)}
    simulate(seed, actors, [pipe], copies, execute, land)


def _shape(seed):
    rnd = random.Random(seed)
    return rnd.choice([1, 2, 3, 16]), rnd.choice([1, 2, 3, 5, 33])


def test_protocol_holds_over_random_shapes():
    for seed in range(300):
        HG, n_q = _shape(seed)
        run(HG, n_q, seed)


def test_dvfree_wait_is_implied_by_the_pwritten_hand_off():
    for seed in range(100):
        HG, n_q = _shape(seed)
        run(max(HG, 2), max(n_q, 2), seed, "dv_reset_without_dvfree")


@pytest.mark.parametrize("mistake", ["next_s_before_sread", "dpt_before_dsready", "slot_reloaded_early"])
def test_model_catches_planted_protocol_mistakes(mistake):
    caught = 0
    for seed in range(100):
        HG, n_q = _shape(seed)
        try:
            run(max(HG, 2), max(n_q, 2), seed, mistake)
        except AssertionError:
            caught += 1
    assert caught >= 50, f"{mistake}: caught in {caught} of 100 runs"


# ---- launch 2: query tiles (ska_bwd_dq_kernel) -------------------------------------------------
# One CTA owns a query tile and walks its n key tiles: K(u) through a three-slot ring, V(u)
# through a two-slot ring; S(u) = Q K(u)^T into TMEM buffer u mod 2, dP(u) = dO V(u)^T into one
# region; the two softmax warpgroups (one per half of the keys) form P from S, then
# dS = P (dP - D) over the first columns of the same S buffer; dQ += dS(u) K(u). The issue
# order S(0) dP(0) S(1) | dQ(0) dP(1) S(2) | dQ(1) dP(2) S(3) | ... puts S(u+2) into the buffer
# dQ(u) reads, which the in-order pipe allows.


def run_dq(n, seed, mistake=None):
    KS, VS = 3, 2
    kfull, kempty = [Bar(1) for _ in range(KS)], [Bar(1) for _ in range(KS)]
    vfull, vempty = [Bar(1) for _ in range(VS)], [Bar(1) for _ in range(VS)]
    qfull, pfull, done = Bar(1), Bar(1), Bar(1)
    sfull, dsready = [Bar(1), Bar(1)], Bar(256)
    m = {"q": False, "k": [None] * KS, "k_readers": [set() for _ in range(KS)],
         "v": [None] * VS, "v_readers": [set() for _ in range(VS)],
         "S": [None, None], "dS": [set(), set()], "dP": None, "dP_readers": set(), "dQ": 0}
    pipe, copies = [], []

    def producer():
        qfull.expect_tx(1)
        copies.append(("q", None, None, qfull))
        for u in range(n):
            if u >= KS and mistake != "k_slot_reloaded_early":
                yield ("wait", kempty[u % KS], (u // KS - 1) & 1)
            kfull[u % KS].expect_tx(1)
            copies.append(("k", u % KS, u, kfull[u % KS]))
            if u >= VS:
                yield ("wait", vempty[u % VS], (u // VS - 1) & 1)
            vfull[u % VS].expect_tx(1)
            copies.append(("v", u % VS, u, vfull[u % VS]))
            yield ("step",)

    def issuer():
        yield ("wait", qfull, 0)
        yield ("wait", kfull[0], 0)
        pipe.extend([("S", 0), ("C", sfull[0])])
        yield ("wait", vfull[0], 0)
        pipe.extend([("DP", 0), ("C", pfull), ("C", vempty[0])])
        if n > 1:
            yield ("wait", kfull[1], 0)
            pipe.extend([("S", 1), ("C", sfull[1])])
        for u in range(n):
            if mistake == "s_before_dsready" and u + 2 < n:
                yield ("wait", kfull[(u + 2) % KS], ((u + 2) // KS) & 1)
                pipe.extend([("S", u + 2), ("C", sfull[(u + 2) & 1])])
            yield ("wait", dsready, u & 1)
            pipe.extend([("DQ", u), ("C", kempty[u % KS])])
            if u + 1 < n:
                yield ("wait", vfull[(u + 1) % VS], ((u + 1) // VS) & 1)
                pipe.extend([("DP", u + 1), ("C", pfull), ("C", vempty[(u + 1) % VS])])
            if u + 2 < n and mistake != "s_before_dsready":
                yield ("wait", kfull[(u + 2) % KS], ((u + 2) // KS) & 1)
                pipe.extend([("S", u + 2), ("C", sfull[(u + 2) & 1])])
        pipe.append(("C", done))

    def softmax(w):
        for u in range(n):
            yield ("wait", sfull[u & 1], (u >> 1) & 1)
            assert m["S"][u & 1] == u, f"half {w} read S {m['S'][u & 1]} for {u}"
            yield ("step",)
            assert m["S"][u & 1] == u, "S overwritten while being read"
            yield ("wait", pfull, u & 1)
            assert m["dP"] == u, f"half {w} read dP {m['dP']} for {u}"
            m["dS"][u & 1].add(w)
            m["dP_readers"].add(w)
            dsready.arrive(128)
        yield ("wait", done, 0)
        assert m["dQ"] == n

    def execute(op):
        kind = op[0]
        if kind == "C":
            op[1].arrive()
        elif kind == "S":
            u = op[1]
            assert m["q"] and m["k"][u % KS] == u
            b = u & 1
            assert m["S"][b] is None or m["dQ"] > m["S"][b], "S buffer overwritten before dQ read its dS"
            m["S"][b], m["dS"][b] = u, set()
            m["k_readers"][u % KS].add("S")
        elif kind == "DP":
            u = op[1]
            assert m["v"][u % VS] == u
            assert m["dP"] is None or m["dP_readers"] == {0, 1}, "dP overwritten while in use"
            m["dP"], m["dP_readers"] = u, set()
            m["v_readers"][u % VS].add("DP")
        else:
            u = op[1]
            assert m["S"][u & 1] == u and m["dS"][u & 1] == {0, 1}, f"dQ({u}) read an unfinished dS"
            assert m["k"][u % KS] == u and m["dQ"] == u
            m["dQ"] += 1
            m["k_readers"][u % KS].add("DQ")

    def land(copy):
        kind, s, u, bar = copy
        if kind == "q":
            m["q"] = True
        elif kind == "k":
            assert m["k"][s] is None or m["k_readers"][s] == {"S", "DQ"}, f"K slot {s} reloaded early"
            m["k"][s], m["k_readers"][s] = u, set()
        else:
            assert m["v"][s] is None or m["v_readers"][s] == {"DP"}, f"V slot {s} reloaded early"
            m["v"][s], m["v_readers"][s] = u, set()
        bar.complete_tx(1)

    actors = {"producer": producer(), "issuer": issuer(), "half0": softmax(0), "half1": softmax(1)}
    simulate(seed, actors, [pipe], copies, execute, land)


def test_query_tile_protocol_holds():
    for seed in range(300):
        run_dq(random.Random(seed).choice([1, 2, 3, 4, 7, 33]), seed)


@pytest.mark.parametrize("mistake", ["s_before_dsready", "k_slot_reloaded_early"])
def test_query_tile_model_catches_planted_mistakes(mistake):
    caught = 0
    for seed in range(100):
        try:
            run_dq(random.Random(seed).choice([4, 7, 33]), seed, mistake)
        except AssertionError:
            caught += 1
    assert caught >= 50, f"{mistake}: caught in {caught} of 100 runs"
