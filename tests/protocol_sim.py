"""A small interleaving simulator for the kernels' mbarrier protocols (CPU).

Warp roles are generators.  A role yields a wait (the barrier and the phase
it wants) and, between waits, acts on barriers directly:

* ``arrive(name)``: a thread arrival, immediate;
* ``commit(name)``: a ``tcgen05.commit``, which arrives once the MMAs issued
  before it complete.  Commits complete in issue order, at times the
  simulator picks;
* ``load(name)``: a TMA copy whose bytes complete the barrier's phase, at a
  time the simulator picks, in any order relative to other copies.

Each move, the simulator picks at random among the roles whose wait is
satisfied, the oldest pending commit and any pending copy.  A "full" wait on
phase k passes once phase k has completed; an "empty" wait on phase k passes
once phase k - 1 has (the first pass is free).  The hardware only compares
parities, so two properties are checked: no deadlock, and no aliasing (a
passing wait sees exactly its phase completed, never two more).
"""
import collections
import random


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.done = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier's count"
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


class Sim:
    def __init__(self, seed):
        self.bars = {}
        self.rng = random.Random(seed)
        self.commits = collections.deque()
        self.loads = []

    def bar(self, name, count):
        self.bars[name] = Barrier(count)

    def arrive(self, name):
        self.bars[name].arrive()

    def commit(self, name):
        self.commits.append(name)

    def load(self, name):
        self.loads.append(name)

    @staticmethod
    def full(name, k):
        return (name, k, False)

    @staticmethod
    def empty(name, k):
        return (name, k, True)

    def _passes(self, role, wait):
        name, k, is_empty = wait
        bar = self.bars[name]
        if (bar.done & 1) == ((k & 1) ^ int(is_empty)):
            return False
        want = k if is_empty else k + 1
        assert bar.done == want, (f"{role} waited on {name} phase {k} ({'empty' if is_empty else 'full'}) "
                                  f"and passed with {bar.done} phases completed")
        return True

    def run(self, roles):
        """Run the roles to the end; return None, or the stuck roles' waits."""
        waits = {r: None for r in roles}
        alive = set(roles)
        while alive or self.commits or self.loads:
            moves = [r for r in sorted(alive) if waits[r] is None or self._passes(r, waits[r])]
            if self.commits:
                moves.append("<tensor core>")
            moves += [("<copy>", i) for i in range(len(self.loads))]
            if not moves:
                return {r: waits[r] for r in alive}
            m = self.rng.choice(moves)
            if m == "<tensor core>":
                self.arrive(self.commits.popleft())
            elif isinstance(m, tuple):
                self.arrive(self.loads.pop(m[1]))
            else:
                try:
                    waits[m] = next(roles[m])
                except StopIteration:
                    alive.discard(m)
                    waits[m] = None
        return None
