"""Building blocks for the CPU models of the tensor-core kernels' hand-off protocols.

- `Bar` follows mbarrier semantics. A phase completes when its arrival count is reached and the
  transaction bytes it expects have landed. A parity wait succeeds unless the current phase has
  that parity, so a waiter two phases ahead passes at once, as on the GPU.
- `simulate` runs the kernel's roles as coroutines under a random scheduler, beside in-order MMA
  pipes, one per issuing warp (a commit arrives once everything its warp issued before it has
  executed), and copies that land at random times.
"""
import random


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, "more arrivals than the barrier's count"
        self._complete()

    def expect_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._complete()

    def _complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        return (self.phase & 1) != parity


def simulate(seed, actors, pipes, copies, execute, land, max_steps=2_000_000):
    """actors: name (a string) -> generator yielding ("wait", bar, parity) or ("step",).
    pipes: one list of issued ops per issuing warp, each executed in order by execute(op), with
    no order between pipes. copies: pending copies, each landed by land(copy) in random order.
    Raises AssertionError on a deadlock or no progress."""
    rnd = random.Random(seed)
    waiting = dict.fromkeys(actors)
    finished = set()
    for _ in range(max_steps):
        ready = [a for a in actors if a not in finished
                 and (waiting[a] is None or waiting[a][0].passed(waiting[a][1]))]
        ready += [("pipe", i) for i, p in enumerate(pipes) if p] + ["copy"] * bool(copies)
        if not ready:
            assert len(finished) == len(actors), f"deadlock, waiting: {waiting}"
            return
        a = rnd.choice(ready)
        if isinstance(a, tuple):
            execute(pipes[a[1]].pop(0))
        elif a == "copy":
            land(copies.pop(rnd.randrange(len(copies))))
        else:
            waiting[a] = None
            try:
                r = next(actors[a])
                if r[0] == "wait":
                    waiting[a] = (r[1], r[2])
            except StopIteration:
                finished.add(a)
    raise AssertionError("no progress")
