"""Randomized model of the hand-off protocol of the recurrence backward's gradient kernel
(gla_bwd_grad_kernel in csrc/gla_backward_tc.cu), checked on the CPU.

One CTA owns one chunk of one (b, h) and reuses every shared-memory region once its operand is
spent, so the order of the roles decides whether a value is read before it is overwritten:
- the producer (warp 0) brings q, k, v, dO, g, S_in and E with one transaction-counted barrier;
- the two operand warpgroups (WG1: tokens 0-31, WG2: tokens 32-63 of the scaling; in the
  epilogue WG1 owns dq and the query sums of dg, WG2 dk and the key sums) turn q into q~ and k
  into k~ (beside it) and k^ (over it), then hand over to the issuer;
- the issuer (warp 1) runs A2, QK, X1^T, X4^T, waits for the masks, then X2^T, X3^T and dv^T;
- warps 12-15 form rho from S_in and E, then the masks M(A2), M(QK) from TMEM, then dv;
- in the epilogue dq is staged over v, dk over dO, T1 over S_in, T2 over E, dg over q~ | k~ and
  dv over k^, and TMA stores read the staged tiles.

Each region carries a label for what it holds and the set of readers its content still owes.
A write asserts that every owed reader is done; a read asserts the label it expects. The
product route (the one every chunk with gates above 2^-8 takes) is modelled; the exact route
shares its barriers. Four planted mistakes must each be caught.

The model also shows that the masks hand-off alone orders warps 12-15's reads of S_in and E
(for rho) before T1 and T2 overwrite them: those warps read them before they write the masks,
and the epilogue starts after the last MMAs, which wait for the masks. Barrier 3 is kept for
the visibility of rho itself, which that chain, running through the tensor core's commit, does
not promise in the memory model.
"""
import pytest

from .barrier_model import Bar, simulate

MMA_G1 = ["A2", "QK", "X1", "X4"]
MMA_G2 = ["X2", "X3", "DV"]
# what each MMA reads (shared memory) and writes (TMEM)
MMA_READS = {
    "A2": ["DO", "V"], "QK": ["Q0", "Q1", "KT0", "KT1"], "X1": ["SIN", "DO"], "X4": ["E", "V"],
    "X2": ["KT0", "KT1", "A2M"], "X3": ["Q0", "Q1", "A2M"], "DV": ["DO", "QKM", "E", "K0", "K1"],
}
OPERAND = {"Q0": "q~", "Q1": "q~", "KT0": "k~", "KT1": "k~", "K0": "k^", "K1": "k^", "V": "v",
           "DO": "do", "SIN": "sin", "E": "e", "A2M": "a2m", "QKM": "qkm"}
# the readers each content owes before its region may be overwritten
OWED = {
    "q": {"op"}, "k": {"op"},
    "q~": {"QK", "X3", "epi1"}, "k~": {"QK", "X2", "epi2"}, "k^": {"DV"},
    "v": {"A2", "X4"}, "do": {"A2", "X1", "DV"}, "sin": {"X1", "rho"}, "e": {"X4", "DV", "rho"},
    "a2m": {"X2", "X3"}, "qkm": {"DV"},
    "T1": {"dg1", "dg2"}, "T2": {"fwd2"}, "T2f": {"dg1", "dg2"},
    "dq": {"st_dq"}, "dk": {"st_dk"}, "dg": {"st_dg"}, "dv": {"st_dv"},
}


def run(seed, mistake=None):
    full, ops, mma1, masks, mma2, drain = Bar(1), Bar(2), Bar(1), Bar(1), Bar(1), Bar(1)
    b1 = Bar(2)      # named barrier 1: the two operand warpgroups
    b3 = Bar(3)      # named barrier 3: the operand warpgroups wait, warps 12-15 only arrive
    stored = Bar(1)  # the issuing thread's bulk stores have read shared memory
    dv_stored = Bar(1)
    end = Bar(5)     # the closing __syncthreads
    smem = {r: ("none", set()) for r in
            ["Q0", "Q1", "KT0", "KT1", "K0", "K1", "V", "DO", "G", "SIN", "E", "A2M", "QKM"]}
    tmem = {}
    misc = {"rho": False, "abuf": False}
    pipe, copies = [], []

    def write(region, label):
        old, owed = smem[region]
        assert not owed, f"{region} overwritten with {label} while {old} still owes {sorted(owed)}"
        smem[region] = (label, set(OWED.get(label, ())))

    def read(region, label, who):
        cur, owed = smem[region]
        assert cur == label, f"{who} read {region} holding {cur}, expected {label}"
        owed.discard(who)

    def bar_sync(bar):
        parity = bar.phase & 1
        bar.arrive()
        return ("wait", bar, parity)

    def execute(op):
        if op[0] == "C":
            op[1].arrive()
            return
        name = op[1]
        for r in MMA_READS[name]:
            read(r, OPERAND[r], name)
        if name in ("X2", "X3"):
            assert tmem.get("A2") == "done", "mask of A2 formed before A2"
        tmem[name] = "done"

    def land(copy):
        kind = copy[0]
        if kind == "load":
            for r, label in (("Q0", "q"), ("Q1", "q"), ("K0", "k"), ("K1", "k"), ("V", "v"),
                             ("DO", "do"), ("G", "g"), ("SIN", "sin"), ("E", "e")):
                smem[r] = (label, set(OWED.get(label, ())))
            full.complete_tx(1)
        else:                     # a bulk store reading its staged tile(s)
            for r, label in copy[1]:
                read(r, label, copy[2])
            if copy[3] is not None:
                copy[3].arrive()

    def producer():
        full.expect_tx(1)
        copies.append(("load",))
        yield ("wait", full, 0)
        yield bar_sync(end)
        yield ("wait", end, 0)

    def issuer():
        yield ("wait", ops, 0)
        pipe.extend([("M", n) for n in MMA_G1] + [("C", mma1)])
        yield ("wait", masks, 0)
        pipe.extend([("M", n) for n in MMA_G2] + [("C", mma2)])
        pipe.append(("C", drain))
        yield ("wait", drain, 0)
        yield bar_sync(end)
        yield ("wait", end, 0)

    def operand(h):
        # scaling: gate products (a scan across both warpgroups), then q~, k~, k^ of this half
        yield ("wait", full, 0)
        read("G", "g", "op")
        yield bar_sync(b1)
        read(f"Q{h}", "q", "op")
        read(f"K{h}", "k", "op")
        write(f"KT{h}", "k~")
        write(f"K{h}", "k^")
        write(f"Q{h}", "q~")
        if h == 0:
            misc["abuf"] = True
        ops.arrive()
        yield ("step",)
        if mistake != "epilogue_before_mma2":
            yield ("wait", mma2, 0)
        yield bar_sync(b1)
        yield bar_sync(b3)
        assert misc["abuf"], "chunk decay read before it was written"
        # reverse sweep over the tokens
        if h == 0:
            assert tmem.get("X1") == "done" and tmem.get("X2") == "done" or mistake, "X1/X2 not ready"
            read("Q0", "q~", "epi1")
            read("Q1", "q~", "epi1")
            read("G", "g", "epi1")
            write("V", "dq")
            yield ("step",)
            write("SIN", "T1")
        else:
            assert tmem.get("X3") == "done" and tmem.get("X4") == "done" or mistake, "X3/X4 not ready"
            read("KT0", "k~", "epi2")
            read("KT1", "k~", "epi2")
            read("G", "g", "epi2")
            write("DO", "dk")
            yield ("step",)
            write("E", "T2")
            yield ("step",)
            # forward sweep of the key sums: k~ and X4 again, T2 updated in place
            read("KT0", "k~", "fwd2")
            read("KT1", "k~", "fwd2")
            read("E", "T2", "fwd2")
            write("E", "T2f")
        if h == 0 and mistake == "dg_before_key_sums":
            b1.arrive()         # arrives without waiting for WG2's sweeps
        else:
            yield bar_sync(b1)
        # dg: T1 + T2 (+ a rho) over this warpgroup's rows, staged over q~ (rows 0-31) or k~
        assert misc["rho"] or mistake, "rho read before warps 12-15 wrote it"
        read("SIN", "T1", f"dg{h + 1}")
        read("E", "T2f", f"dg{h + 1}")
        read("G", "g", f"dg{h + 1}")
        yield ("step",)
        if h == 0:
            write("Q0", "dg")
            write("Q1", "dg")
        else:
            write("KT0", "dg")
            write("KT1", "dg")
        if not (h == 0 and mistake == "stores_before_sync"):
            yield bar_sync(b1)
        if h == 0:
            copies.append(("store", [("V", "dq")], "st_dq", None))
            copies.append(("store", [("DO", "dk")], "st_dk", None))
            copies.append(("store", [("Q0", "dg"), ("Q1", "dg"), ("KT0", "dg"), ("KT1", "dg")],
                           "st_dg", stored))
            yield ("wait", stored, 0)
            if mistake == "stores_before_sync":
                yield bar_sync(b1)
        yield bar_sync(end)
        yield ("wait", end, 0)

    def warps12():
        yield ("wait", full, 0)
        read("SIN", "sin", "rho")
        read("E", "e", "rho")
        misc["rho"] = True
        b3.arrive()
        yield ("step",)
        if mistake != "masks_before_mma1":
            yield ("wait", mma1, 0)
        assert tmem.get("A2") == "done" and tmem.get("QK") == "done", "masks formed before A2 / QK"
        write("A2M", "a2m")
        write("QKM", "qkm")
        masks.arrive()
        yield ("wait", mma2, 0)
        assert tmem.get("DV") == "done", "dv read before its MMAs"
        write("K0", "dv")
        write("K1", "dv")
        copies.append(("store", [("K0", "dv"), ("K1", "dv")], "st_dv", dv_stored))
        yield ("wait", dv_stored, 0)
        yield bar_sync(end)
        yield ("wait", end, 0)

    actors = {"producer": producer(), "issuer": issuer(), "wg1": operand(0), "wg2": operand(1),
              "w12": warps12()}
    simulate(seed, actors, [pipe], copies, execute, land)
    for r in ("Q0", "Q1", "KT0", "KT1", "K0", "K1", "V", "DO"):
        assert not smem[r][1], f"{r} still owes {sorted(smem[r][1])} at the end"


@pytest.mark.parametrize("seed", range(300))
def test_gradient_kernel_protocol_holds(seed):
    run(seed)


@pytest.mark.parametrize("mistake", ["dg_before_key_sums", "masks_before_mma1", "stores_before_sync",
                                     "epilogue_before_mma2"])
def test_planted_mistakes_are_caught(mistake):
    caught = 0
    for seed in range(300):
        try:
            run(seed, mistake)
        except AssertionError:
            caught += 1
    assert caught > 0, f"{mistake} never caught in 300 schedules"


# ------------------------------------------------------------------------------------------------
# The contributions kernel (gla_bwd_contrib_kernel): each warp moves its 32 TMEM rows of U or U'
# out in four 32 x 32 fp32 tiles through two shared-memory buffers laid over the spent operand
# tiles. Before it writes a buffer the third time or later, the lane that issues the stores waits
# until all but its most recent bulk store have read shared memory (wait_group.read 1); before
# the CTA leaves, until all have (wait_group.read 0).
# ------------------------------------------------------------------------------------------------
def run_contrib(seed, mistake=None, warps=8, tiles=4):
    mma = Bar(1)
    tile_read = [[Bar(1) for _ in range(tiles)] for _ in range(warps)]
    end = Bar(warps + 1)
    operands = {"read_by_mma": False}
    buf = {}         # (warp, buffer) -> (tile staged there, read by its store yet)
    out = set()
    pipe, copies = [], []

    def execute(op):
        if op[0] == "C":
            op[1].arrive()
        else:
            operands["read_by_mma"] = True

    def land(copy):
        w, t, b = copy
        staged, _ = buf[(w, b)]
        assert staged == t, f"warp {w}: store of tile {t} read buffer {b} holding tile {staged}"
        buf[(w, b)] = (t, True)
        out.add((w, t))
        tile_read[w][t].arrive()

    def issuer():
        pipe.extend([("M", "U"), ("M", "U2"), ("C", mma)])
        yield ("step",)
        parity = end.phase & 1
        end.arrive()
        yield ("wait", end, parity)

    def warp(w):
        yield ("wait", mma, 0)
        for t in range(tiles):
            b = t % 2
            if t >= 2 and mistake != "no_read_wait":
                # wait_group.read 1: every store but the newest has read shared memory
                for u in range(t - 1):
                    yield ("wait", tile_read[w][u], 0)
            assert operands["read_by_mma"], "staging written over operands the MMAs still read"
            if (w, b) in buf:
                assert buf[(w, b)][1], f"warp {w}: buffer {b} rewritten before its store read it"
            buf[(w, b)] = (t, False)
            yield ("step",)
            copies.append((w, t, b))
        for u in range(tiles):  # wait_group.read 0 before the CTA leaves
            yield ("wait", tile_read[w][u], 0)
        assert all(buf[(w, b)][1] for b in range(2)), "CTA left before its stores read"
        parity = end.phase & 1
        end.arrive()
        yield ("wait", end, parity)

    actors = {"issuer": issuer()}
    actors.update({f"w{w}": warp(w) for w in range(warps)})
    simulate(seed, actors, [pipe], copies, execute, land)
    assert out == {(w, t) for w in range(warps) for t in range(tiles)}, "a tile was never stored"


@pytest.mark.parametrize("seed", range(200))
def test_contributions_staging_protocol_holds(seed):
    run_contrib(seed)


def test_contributions_staging_mistake_is_caught():
    # with no wait before a buffer's reuse, some schedule rewrites it before its store read it
    caught = 0
    for seed in range(200):
        try:
            run_contrib(seed, "no_read_wait")
        except AssertionError:
            caught += 1
    assert caught > 0
