"""Randomised model checker for the kernels' barrier protocols (test infrastructure).

mbarrier model: `count` expected arrivals per phase, a transaction count; a phase completes
when all arrivals are in and the transaction count is back to 0.  wait(bar, parity) passes
when the barrier's current phase parity differs from `parity` (the hardware's rule, so a
waiter two phases behind is fooled exactly as on the GPU).

Roles are generators yielding actions:
  ("wait", bar, parity)             block until the parity test passes
  ("arrive", bar)                   plain arrive
  ("expect", bar, nbytes)           arrive.expect_tx
  ("tma", slot_key, tag, bar, nbytes)   async copy: at completion writes tag to slot, complete_tx
  ("mma", reads, writes)            async tensor op of this thread: at execution checks every
                                    (key, expected tag) in reads, then sets writes {key: tag}
  ("commit", bar)                   async marker: arrives once this thread's earlier ops ran
  ("read", reads) / ("write", writes)  synchronous register-side access (element-wise warps)
Async ops of one thread execute in issue order; different threads interleave freely.
"""
import random


class Hazard(Exception):
    pass


class Deadlock(Exception):
    pass


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.phase = name, count, count, 0, 0

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self):
        if self.pending <= 0:
            raise Hazard(f"over-arrival on {self.name}")
        self.pending -= 1
        self._check()

    def expect(self, n):
        self.tx += n
        self.arrive()

    def complete_tx(self, n):
        self.tx -= n
        if self.tx < 0:
            raise Hazard(f"tx underflow on {self.name}")
        self._check()

    def passes(self, parity):
        return (self.phase & 1) != parity


def run(roles, bars, seed, max_steps=2_000_000, async_bias=0.5):
    """roles: {name: generator}.  Explores one random schedule; raises Hazard/Deadlock."""
    rng = random.Random(seed)
    state = {}          # resource key -> tag
    queues = {n: [] for n in roles}   # per thread: pending async ops (in order)
    tma_pending = []    # async copies (any order)
    blocked = {n: None for n in roles}
    gens = dict(roles)
    done = set()

    def step_role(n):
        g = gens[n]
        while True:
            act = blocked[n]
            if act is None:
                try:
                    act = next(g)
                except StopIteration:
                    done.add(n)
                    return True
            kind = act[0]
            if kind == "wait":
                if not act[1].passes(act[2]):
                    blocked[n] = act
                    return False
                blocked[n] = None
                return True  # one wait per scheduling step
            blocked[n] = None
            if kind == "arrive":
                act[1].arrive()
            elif kind == "expect":
                act[1].expect(act[2])
            elif kind == "tma":
                tma_pending.append(act)
            elif kind in ("mma", "commit"):
                queues[n].append(act)
            elif kind == "read":
                for key, tag in act[1]:
                    if state.get(key) != tag:
                        raise Hazard(f"{n} read {key}: have {state.get(key)}, want {tag}")
            elif kind == "write":
                state.update(act[1])
            else:
                raise ValueError(kind)

    for _ in range(max_steps):
        runnable = [n for n in roles if n not in done and (blocked[n] is None or blocked[n][1].passes(blocked[n][2]))]
        asyncs = [("q", n) for n in roles if queues[n]] + [("t", i) for i in range(len(tma_pending))]
        if not runnable and not asyncs:
            if len(done) == len(roles):
                return state
            raise Deadlock({n: (blocked[n][1].name, blocked[n][2], blocked[n][1].phase) for n in roles
                            if n not in done and blocked[n] is not None})
        if asyncs and (not runnable or rng.random() < async_bias):
            kind, x = rng.choice(asyncs)
            if kind == "t":
                _, key, tag, bar, nbytes = tma_pending.pop(x)
                state[key] = tag
                bar.complete_tx(nbytes)
            else:
                act = queues[x].pop(0)
                if act[0] == "mma":
                    for key, tag in act[1]:
                        if state.get(key) != tag:
                            raise Hazard(f"{x} mma read {key}: have {state.get(key)}, want {tag}")
                    state.update(act[2])
                else:
                    act[1].arrive()
        else:
            step_role(rng.choice(runnable))
    raise Deadlock("step limit")
