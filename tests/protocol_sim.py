"""Random-schedule runner for models of the kernels' mbarrier protocols.

A model is a set of actors (Python generators, one step per `yield`) standing
for the kernel's warps, plus asynchronous completions (TMA copies landing,
tcgen05.commit arrivals) that fire at random later times; the commits of one
issuing thread fire in issue order, as the tensor pipe completes one thread's
MMAs in order. `Bar` counts arrivals per phase like an mbarrier; `ready` is a
parity wait that also fails the model if the waiter is more than one phase
behind (where a parity wait would misread the barrier).
"""

import random


class ProtocolError(Exception):
    pass


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.phase += 1


class Model:
    def __init__(self, seed):
        self.rng = random.Random(seed)
        self.bars = {}
        self.events = []  # ("commit", bar name, MMAs issued so far) or ("call", fn)
        self.n_mma = 0
        self.done = 0  # MMAs [0, done) have completed

    def bar(self, name, count=1):
        self.bars[name] = Bar(count)

    def ready(self, name, k):
        b = self.bars[name]
        if b.phase not in (k, k + 1):
            raise ProtocolError(f"{name}: waiting for phase {k} while at {b.phase}")
        return b.phase > k

    def wait(self, name, k):
        while not self.ready(name, k):
            yield

    def mma(self):
        self.n_mma += 1
        return self.n_mma - 1  # id; complete once self.done > id

    def commit(self, name):
        self.events.append(("commit", name, self.n_mma))

    def later(self, fn):
        self.events.append(("call", fn))

    def run(self, actors, max_steps=400000):
        actors = dict(actors)
        for _ in range(max_steps):
            if not actors and not self.events:
                return
            names = list(actors) + (["event"] if self.events else [])
            pick = self.rng.choice(names)
            if pick == "event":
                ev = self.rng.choice(self.events)
                if ev[0] == "commit":
                    ev = next(e for e in self.events if e[0] == "commit")
                self.events.remove(ev)
                if ev[0] == "commit":
                    self.done = max(self.done, ev[2])
                    self.bars[ev[1]].arrive()
                else:
                    ev[1]()
                continue
            try:
                next(actors[pick])
            except StopIteration:
                del actors[pick]
        raise ProtocolError("no progress: deadlock")
