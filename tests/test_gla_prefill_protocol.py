"""A randomized model of the hand-off protocol of the tensor-core recurrence prefill
(csrc/gla_prefill_tc.cu, gla_chunk_kernel), checked on the CPU.

One CTA walks the chunks of a segment through two stages (chunk n in stage n mod 2). In the
output pass (pass C):
- the producer loads q, k, v, g of chunk n (after the stage's previous MMAs are done: empty);
- the operand warps build the chunk's operands in the stage (q~, k~, k^, the fp32 readout
  operand), publish the route and rescale flags, and arrive on ops. On the exact route they
  store the scores A into TMEM buffer n mod 2 themselves. When the chunk rescales R^T, they wait
  for the chunk's readout (barRO), rescale R^T in place and arrive on rdone;
- the state warps first load S_in into R^T (rinit); then per chunk they wait for the scores
  (aready), form P into the stage (pready), and write the previous chunk's output rows from
  O^T buffer (n-1) mod 2 once its MMAs are done (barO);
- the issuer waits for ops, issues A (commit aready; on the exact route it arrives on aready
  itself), waits for pready, issues the readout O^T = R^T q~^T and O^T += V^T P^T, on a rescale
  chunk commits barRO and waits for rdone, then issues R^T += V^T k^ and commits barO and empty.
All MMAs come from the one issuing warp and run in order. (The issuer's wait on rinit is implied
by its wait on pready for chunk 0, which the state warps give only after loading S_in; it is
kept as a guard.) The O^T accumulator is double-buffered: the state warps write chunk n-1's rows
after forming chunk n's P, so the readout of chunk n must not reuse chunk n-1's buffer. Every
read is checked against the chunk it must see: the scores, P and the operands of their own
chunk; the readout reads R^T after exactly n updates and before this chunk's rescale; each TMEM
buffer and stage is overwritten only after its last reader.

Pass A (segment contributions only) keeps the producer, the operand warps (which rescale R^T
before arriving on ops, after the previous chunk's MMAs) and the issuer (R^T += V^T k^ per
chunk); the state warps wait on a barrier committed once after the last chunk (fin) and store
the segment's state. Planted protocol mistakes must each be caught.
"""
import random

import pytest

from .barrier_model import Bar, simulate


def run_pass_c(routes, rescales, seed, mistake=None):
    """routes: per chunk, True for the fast route (scores on the tensor cores);
    rescales: per chunk, True when the chunk rescales R^T."""
    N = len(routes)
    full, empty = [Bar(1), Bar(1)], [Bar(1), Bar(1)]
    ops, aready, pready, barO = [Bar(1), Bar(1)], [Bar(1), Bar(1)], [Bar(1), Bar(1)], [Bar(1), Bar(1)]
    barRO, rdone, rinit, fin = Bar(1), Bar(1), Bar(1), Bar(1)
    m = {"stage": [None, None], "operands": [None, None], "P": [None, None],
         "readers": [set(), set()], "flag": [None, None],
         "A": [None, None], "A_read": [None, None], "O": [None, None], "O_read": [None, None],
         "R": None, "rescaled": set(), "read_out": set()}
    pipe, copies = [], []

    def producer():
        for n in range(N):
            st = n & 1
            if n >= 2 and mistake != "stage_reloaded_early":
                yield ("wait", empty[st], ((n >> 1) - 1) & 1)
            full[st].expect_tx(1)
            copies.append((st, n, full[st]))
            yield ("step",)

    def operands():
        nresc = 0
        for n in range(N):
            st = n & 1
            yield ("wait", full[st], (n >> 1) & 1)
            assert m["stage"][st] == n, f"operands of chunk {n} built from chunk {m['stage'][st]}"
            yield ("step",)
            m["operands"][st] = n
            m["flag"][st] = n
            m["readers"][st].add("ops")
            if not routes[n]:  # exact route: the scores stored into TMEM by these warps
                assert m["A"][st] is None or m["A_read"][st] == m["A"][st], "A overwritten before P was formed"
                m["A"][st] = n
            ops[st].arrive()
            if rescales[n]:
                if mistake != "rescale_without_barRO":
                    yield ("wait", barRO, nresc & 1)
                nresc += 1
                assert n in m["read_out"], f"R^T rescaled for chunk {n} before its readout"
                assert m["R"] == n, f"R^T rescaled for chunk {n} after {m['R']} updates"
                yield ("step",)
                m["rescaled"].add(n)
                rdone.arrive()

    def issuer():
        nresc = 0
        yield ("wait", rinit, 0)
        for n in range(N):
            st = n & 1
            yield ("wait", ops[st], (n >> 1) & 1)
            assert m["flag"][st] == n, "route flag of another chunk"
            if routes[n]:
                pipe.extend([("A", n, st), ("C", aready[st])])
            else:
                aready[st].arrive()
            yield ("wait", pready[st], (n >> 1) & 1)
            ob = 0 if mistake == "single_output_buffer" else st
            pipe.extend([("RO", n, ob), ("PV", n, ob)])
            if rescales[n]:
                pipe.append(("C", barRO))
                if mistake != "update_without_rdone":
                    yield ("wait", rdone, nresc & 1)
                nresc += 1
            pipe.extend([("U", n, st), ("C", barO[st]), ("C", empty[st])])
            if n == N - 1:
                pipe.append(("C", fin))

    def state():
        yield ("step",)
        m["R"] = 0  # S_in loaded into R^T
        rinit.arrive()

        def epilogue(k):
            ob = 0 if mistake == "single_output_buffer" else k & 1
            if mistake != "epilogue_without_barO":
                yield ("wait", barO[k & 1], (k >> 1) & 1)
            assert m["O"][ob] == k, f"output rows of chunk {k} read from O^T of chunk {m['O'][ob]}"
            yield ("step",)
            m["O_read"][ob] = k

        for n in range(N):
            st = n & 1
            if mistake != "p_without_aready":
                yield ("wait", aready[st], (n >> 1) & 1)
            assert m["A"][st] == n, f"P of chunk {n} formed from the scores of chunk {m['A'][st]}"
            m["A_read"][st] = n
            yield ("step",)
            m["P"][st] = n
            m["readers"][st].add("P")
            pready[st].arrive()
            if n > 0:
                yield from epilogue(n - 1)
        yield from epilogue(N - 1)
        assert m["R"] == N

    def execute(op):
        if op[0] == "C":
            op[1].arrive()
            return
        kind, n, st = op
        if kind in ("RO", "PV"):  # st names the O^T buffer; the stage is n mod 2
            ob, st = st, n & 1
        if kind == "A":
            assert m["operands"][st] == n, f"A({n}) read operands of chunk {m['operands'][st]}"
            assert m["A"][st] is None or m["A_read"][st] == m["A"][st], "A overwritten before P was formed"
            m["A"] = m["A"][:st] + [n] + m["A"][st + 1:]
            m["readers"][st].add("A")
        elif kind == "RO":
            assert m["R"] == n, f"readout of chunk {n} read R^T after {m['R']} updates"
            assert n not in m["rescaled"], "readout read R^T after this chunk's rescale"
            assert m["operands"][st] == n, "readout operand of another chunk"
            assert m["O"][ob] is None or m["O_read"][ob] == m["O"][ob], "O^T overwritten before its rows were written"
            m["O"][ob] = ("partial", n)
            m["read_out"].add(n)
            m["readers"][st].add("RO")
        elif kind == "PV":
            assert m["P"][st] == n and m["stage"][st] == n, f"P V of chunk {n} read P / V of another chunk"
            assert m["O"][ob] == ("partial", n)
            m["O"][ob] = n
            m["readers"][st].add("PV")
        else:
            assert m["R"] == n, "state update out of order"
            assert not rescales[n] or n in m["rescaled"], f"R^T updated for chunk {n} before its rescale"
            assert m["operands"][st] == n and m["stage"][st] == n
            m["R"] = n + 1
            m["readers"][st].add("U")

    def land(copy):
        st, n, bar = copy
        if m["stage"][st] is not None:
            prev = m["stage"][st]
            need = {"ops", "P", "RO", "PV", "U"} | ({"A"} if routes[prev] else set())
            assert m["readers"][st] >= need, f"stage {st} reloaded while chunk {prev} is in use"
        m["stage"][st], m["readers"][st] = n, set()
        m["operands"][st] = m["P"][st] = None
        bar.complete_tx(1)

    actors = {"producer": producer(), "operands": operands(), "issuer": issuer(), "state": state()}
    simulate(seed, actors, [pipe], copies, execute, land)


def _chunks(seed, n_min=1):
    rnd = random.Random(seed)
    n = rnd.randint(n_min, 12)
    return [rnd.random() < 0.8 for _ in range(n)], [rnd.random() < 0.3 for _ in range(n)]


def test_pass_c_protocol_holds_over_random_routes_and_rescales():
    for seed in range(400):
        routes, rescales = _chunks(seed)
        run_pass_c(routes, rescales, seed)


@pytest.mark.parametrize("mistake", ["stage_reloaded_early", "p_without_aready", "single_output_buffer",
                                     "rescale_without_barRO", "update_without_rdone",
                                     "epilogue_without_barO"])
def test_pass_c_model_catches_planted_protocol_mistakes(mistake):
    caught = 0
    for seed in range(200):
        routes, rescales = _chunks(seed, n_min=4)
        if mistake in ("rescale_without_barRO", "update_without_rdone"):
            rescales[1] = rescales[2] = True
        try:
            run_pass_c(routes, rescales, seed, mistake)
        except AssertionError:
            caught += 1
    assert caught >= 20, f"{mistake}: caught in {caught} of 200 runs"


def run_pass_a(rescales, seed, mistake=None):
    """Pass A: R^T += V^T k^ per chunk, no scores, P or outputs. The operand warps rescale R^T in
    place (a read-modify-write in TMEM) before arriving on ops, once the previous chunk's update
    is done; the state warps store the segment's state after the barrier committed once after
    the last chunk."""
    N = len(rescales)
    full, empty, ops, barO = [Bar(1), Bar(1)], [Bar(1), Bar(1)], [Bar(1), Bar(1)], [Bar(1), Bar(1)]
    fin = Bar(1)
    m = {"stage": [None, None], "operands": [None, None], "readers": [set(), set()],
         "R": 0, "rescaled": set()}
    pipe, copies = [], []

    def producer():
        for n in range(N):
            st = n & 1
            if n >= 2:
                yield ("wait", empty[st], ((n >> 1) - 1) & 1)
            full[st].expect_tx(1)
            copies.append((st, n, full[st]))
            yield ("step",)

    def operands():
        for n in range(N):
            st = n & 1
            yield ("wait", full[st], (n >> 1) & 1)
            assert m["stage"][st] == n
            yield ("step",)
            m["operands"][st] = n
            m["readers"][st].add("ops")
            if rescales[n] and n > 0:
                if mistake != "rescale_without_barO":
                    yield ("wait", barO[(n - 1) & 1], ((n - 1) >> 1) & 1)
                assert m["R"] == n, f"R^T rescaled for chunk {n} while {n - m['R']} updates are pending"
                yield ("step",)
                assert m["R"] == n, "R^T updated during its in-place rescale"
                m["rescaled"].add(n)
            ops[st].arrive()

    def issuer():
        for n in range(N):
            st = n & 1
            yield ("wait", ops[st], (n >> 1) & 1)
            pipe.extend([("U", n, st), ("C", barO[st]), ("C", empty[st])])
            if n == N - 1:
                pipe.append(("C", fin))

    def state():
        if mistake == "state_waits_last_barO":  # a parity wait on a barrier that has run on
            yield ("wait", barO[(N - 1) & 1], ((N - 1) >> 1) & 1)
        else:
            yield ("wait", fin, 0)
        assert m["R"] == N, f"segment state stored after {m['R']} of {N} updates"

    def execute(op):
        if op[0] == "C":
            op[1].arrive()
            return
        _, n, st = op
        assert m["operands"][st] == n and m["R"] == n
        assert not rescales[n] or n == 0 or n in m["rescaled"], "R^T updated before its rescale"
        m["R"] = n + 1
        m["readers"][st].add("U")

    def land(copy):
        st, n, bar = copy
        if m["stage"][st] is not None:
            assert m["readers"][st] >= {"ops", "U"}, f"stage {st} reloaded while in use"
        m["stage"][st], m["readers"][st], m["operands"][st] = n, set(), None
        bar.complete_tx(1)

    simulate(seed, {"producer": producer(), "operands": operands(), "issuer": issuer(), "state": state()},
             [pipe], copies, execute, land)


def test_pass_a_protocol_holds():
    for seed in range(300):
        rnd = random.Random(seed)
        run_pass_a([rnd.random() < 0.3 for _ in range(rnd.randint(1, 12))], seed)


@pytest.mark.parametrize("mistake", ["rescale_without_barO", "state_waits_last_barO"])
def test_pass_a_model_catches_planted_mistakes(mistake):
    """The second waits on the last chunk's phase of barO from the start: the barrier runs
    through a phase per two chunks meanwhile, and a parity wait passes at the first earlier
    phase of the same parity, so the segment's state would be read before its last updates.
    The kernel waits on a barrier committed once, after the last chunk, instead."""
    caught = 0
    for seed in range(300):
        rnd = random.Random(seed)
        rescales = [rnd.random() < 0.5 for _ in range(rnd.randint(5, 12))]
        try:
            run_pass_a(rescales, seed, mistake)
        except AssertionError:
            caught += 1
    assert caught >= 15, f"{mistake}: caught in {caught} of 300 runs"
