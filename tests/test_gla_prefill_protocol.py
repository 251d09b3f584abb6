"""A randomized model of the hand-off protocol of the tensor-core recurrence prefill
(csrc/gla_prefill_tc.cu, gla_chunk_kernel in its output pass), checked on the CPU.

One CTA walks the chunks of a segment through two 80 KB stages (chunk n in stage n mod 2):
- the producer loads q, k, v, g of chunk n;
- warpgroup 0 turns them into the operands in place (q~ over q, k^ over k, k~ over g) and
  publishes the chunk's decay factors. On the fast route its warp 0 issues A = q~ k~^T into TMEM
  buffer n mod 2 (commit barA); on the exact route warpgroup 0 stores A itself. It then arrives
  on ops;
- warpgroup 1 forms P = mask(A) into the stage and writes the previous chunk's output rows
  (after barO). It copies the state R to bf16 in one shared buffer, and its warp 4 issues
  R += k^^T V and O = P V + q~ R_bf16 (commits barO and the stage's empty).

The two issuing warps' MMAs run in order within each warp but in no order across them. Every
read is checked against the chunk it must see:
- every MMA reads its own chunk's operands, P and state copy;
- A, O, R and the bf16 copy are each overwritten only after their last reader;
- a stage is reloaded only after all its readers, the A product included.

Three planted protocol mistakes must each be caught.
"""
import random

import pytest

from .barrier_model import Bar, simulate


def run(routes, seed, mistake=None):
    """routes: per chunk, True for the fast route (A on the tensor cores)."""
    N = len(routes)
    full, empty = [Bar(1), Bar(1)], [Bar(1), Bar(1)]
    ops, barA = [Bar(1), Bar(1)], [Bar(1), Bar(1)]
    barO = Bar(1)
    m = {"stage": [None, None], "operands": [None, None], "P": [None, None],
         "readers": [set(), set()], "abuf": [None, None],
         "A": [None, None], "A_read": [None, None],
         "R": 0, "R_bf16": None, "R_bf16_read": None, "O": None, "O_read": None}
    pipe0, pipe4, copies = [], [], []

    def producer():
        for n in range(N):
            st = n & 1
            if n >= 2 and mistake != "stage_reloaded_early":
                yield ("wait", empty[st], ((n >> 1) - 1) & 1)
            full[st].expect_tx(1)
            copies.append((st, n, full[st]))
            yield ("step",)

    def operands():  # warpgroup 0 (warp 0 issues A)
        for n in range(N):
            st = n & 1
            yield ("wait", full[st], (n >> 1) & 1)
            assert m["stage"][st] == n, f"operands of chunk {n} built from chunk {m['stage'][st]}"
            yield ("step",)
            m["abuf"][st] = n
            m["operands"][st] = n
            m["readers"][st].add("wg0")
            if routes[n]:
                pipe0.extend([("A", n, st), ("C", barA[st])])
            else:  # exact route: A stored into TMEM by this warpgroup
                assert m["A"][st] is None or m["A_read"][st] == m["A"][st], "A overwritten before P was formed"
                m["A"][st] = n
            ops[st].arrive()

    def state():  # warpgroup 1 (warp 4 issues R and O)
        nA = [0, 0]
        for n in range(N):
            st = n & 1
            yield ("wait", ops[st], (n >> 1) & 1)
            assert m["abuf"][st] == n, "decay factors of another chunk"
            if routes[n] and mistake != "p_without_barA":
                yield ("wait", barA[st], nA[st] & 1)
                nA[st] += 1
            assert m["A"][st] == n, f"P of chunk {n} formed from A of chunk {m['A'][st]}"
            m["A_read"][st] = n
            m["P"][st] = n
            yield ("step",)
            if n > 0:
                if mistake != "state_copy_without_barO":
                    yield ("wait", barO, (n - 1) & 1)
                assert m["O"] == n - 1, f"output rows of chunk {n - 1} read from O of {m['O']}"
                m["O_read"] = n - 1
            assert m["R"] == n, f"state copy for chunk {n} taken from R after {m['R']} updates"
            assert m["R_bf16"] is None or m["R_bf16_read"] == m["R_bf16"], "state copy overwritten in use"
            m["R_bf16"] = n
            yield ("step",)
            pipe4.extend([("R", n, st), ("O", n, st), ("C", barO), ("C", empty[st])])
        yield ("wait", barO, (N - 1) & 1)
        assert m["O"] == N - 1 and m["R"] == N

    def execute(op):
        if op[0] == "C":
            op[1].arrive()
            return
        kind, n, st = op
        if kind == "A":
            assert m["operands"][st] == n, f"A({n}) read operands of chunk {m['operands'][st]}"
            assert m["A"][st] is None or m["A_read"][st] == m["A"][st], "A overwritten before P was formed"
            m["A"][st] = n
            m["readers"][st].add("A")
        elif kind == "R":
            assert m["operands"][st] == n and m["stage"][st] == n
            assert m["R"] == n and m["R_bf16"] == n, "R updated before its bf16 copy was taken"
            m["R"] = n + 1
            m["readers"][st].add("R")
        else:
            assert m["P"][st] == n and m["operands"][st] == n, f"O({n}) read P / operands of another chunk"
            assert m["R_bf16"] == n, f"O({n}) read the state copy of chunk {m['R_bf16']}"
            assert m["O"] is None or m["O_read"] == m["O"], "O overwritten before its rows were written"
            m["O"], m["R_bf16_read"] = n, n
            m["readers"][st].add("O")

    def land(copy):
        st, n, bar = copy
        if m["stage"][st] is not None:
            prev = m["stage"][st]
            need = {"wg0", "R", "O"} | ({"A"} if routes[prev] else set())
            assert m["readers"][st] >= need, f"stage {st} reloaded while chunk {prev} is in use"
        m["stage"][st], m["readers"][st] = n, set()
        m["operands"][st] = m["P"][st] = None
        bar.complete_tx(1)

    actors = {"producer": producer(), "operands": operands(), "state": state()}
    simulate(seed, actors, [pipe0, pipe4], copies, execute, land)


def _routes(seed, n_min=1):
    rnd = random.Random(seed)
    return [rnd.random() < 0.8 for _ in range(rnd.randint(n_min, 12))]


def test_protocol_holds_over_random_chunk_routes():
    for seed in range(400):
        run(_routes(seed), seed)


@pytest.mark.parametrize("mistake", ["stage_reloaded_early", "p_without_barA", "state_copy_without_barO"])
def test_model_catches_planted_protocol_mistakes(mistake):
    caught = 0
    for seed in range(100):
        try:
            run(_routes(seed, n_min=4), seed, mistake)
        except AssertionError:
            caught += 1
    assert caught >= 50, f"{mistake}: caught in {caught} of 100 runs"


def run_pass_a(rescales, seed, mistake=None):
    """Pass A (the segment's state contribution only): no A, P or O; warp 4 issues R += k^^T V
    per chunk. Warpgroup 1 waits for the previous chunk's MMAs only when R is rescaled in place
    (a read-modify-write of R in TMEM by its threads), which must not overlap an R update."""
    N = len(rescales)
    full, empty, ops = [Bar(1), Bar(1)], [Bar(1), Bar(1)], [Bar(1), Bar(1)]
    barO = Bar(1)
    m = {"stage": [None, None], "operands": [None, None], "readers": [set(), set()],
         "R": 0, "R_rescaled": set()}
    pipe4, copies = [], []

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
            m["readers"][st].add("wg0")
            ops[st].arrive()

    def state():
        for n in range(N):
            st = n & 1
            yield ("wait", ops[st], (n >> 1) & 1)
            # the previous chunk's MMAs are awaited before a rescale, and before the last chunk
            # (so that the final wait below cannot alias an earlier phase)
            last = n == N - 1 and mistake != "no_wait_before_last_chunk"
            if (rescales[n] or last) and n > 0 and mistake != "rescale_without_barO":
                yield ("wait", barO, (n - 1) & 1)
            if rescales[n] and n > 0:
                assert m["R"] == n, f"R rescaled for chunk {n} while {n - m['R']} updates are pending"
                yield ("step",)
                assert m["R"] == n, "R updated during its in-place rescale"
                m["R_rescaled"].add(n)
            pipe4.extend([("R", n, st), ("C", barO), ("C", empty[st])])
        yield ("wait", barO, (N - 1) & 1)
        assert m["R"] == N

    def execute(op):
        if op[0] == "C":
            op[1].arrive()
            return
        _, n, st = op
        assert m["operands"][st] == n and m["R"] == n
        assert not rescales[n] or n == 0 or n in m["R_rescaled"], "R updated before its rescale"
        m["R"] = n + 1
        m["readers"][st].add("R")

    def land(copy):
        st, n, bar = copy
        if m["stage"][st] is not None:
            assert m["readers"][st] >= {"wg0", "R"}, f"stage {st} reloaded while in use"
        m["stage"][st], m["readers"][st], m["operands"][st] = n, set(), None
        bar.complete_tx(1)

    simulate(seed, {"producer": producer(), "operands": operands(), "state": state()},
             [pipe4], copies, execute, land)


def test_pass_a_protocol_holds():
    for seed in range(300):
        rnd = random.Random(seed)
        run_pass_a([rnd.random() < 0.3 for _ in range(rnd.randint(1, 12))], seed)


@pytest.mark.parametrize("mistake", ["rescale_without_barO", "no_wait_before_last_chunk"])
def test_pass_a_model_catches_planted_mistakes(mistake):
    """The second is the pass's earlier form: without the wait before the last chunk, the final
    wait for phase N-1 could pass while phase N-2 was still pending (a parity wait two phases
    ahead), and the segment's state would be read before its last updates."""
    caught = 0
    for seed in range(300):
        rnd = random.Random(seed)
        rescales = [rnd.random() < 0.5 for _ in range(rnd.randint(4, 12))]
        if mistake == "no_wait_before_last_chunk":
            rescales[-1] = False
        try:
            run_pass_a(rescales, seed, mistake)
        except AssertionError:
            caught += 1
    assert caught >= 15, f"{mistake}: caught in {caught} of 300 runs"
