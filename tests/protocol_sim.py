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

Bounded waits: a role receives the outcome of each wait (``ok = yield w``),
True when it passed.  ``run(..., give_up=(role, n))`` makes that role's n-th
wait run out of time: it receives False and the CTA's abort word is set, after
which every role blocked on an abortable wait also receives False.  A wait
given as ``(name, k, is_empty, False)`` ignores the abort word (the waits by
which a role lets its own copies and MMAs land before it exits).  After a
run, ``in_flight_at_exit`` counts the commits and copies still pending when
the last role ended: it must be 0, or the CTA would exit with asynchronous
work still writing into its shared or tensor memory.
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
        self.aborted = False
        self.in_flight_at_exit = None
        self.pending_at_exit = None

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

    @staticmethod
    def drain(name, k):
        """A full wait that ignores the abort word."""
        return (name, k, False, False)

    def _passes(self, role, wait):
        name, k, is_empty = wait[:3]
        bar = self.bars[name]
        if (bar.done & 1) == ((k & 1) ^ int(is_empty)):
            return False
        want = k if is_empty else k + 1
        assert bar.done == want, (f"{role} waited on {name} phase {k} ({'empty' if is_empty else 'full'}) "
                                  f"and passed with {bar.done} phases completed")
        return True

    def run(self, roles, give_up=None):
        """Run the roles to the end; return None, or the stuck roles' waits.
        give_up: (role, n) makes that role's n-th wait (0-based) run out."""
        waits = {r: None for r in roles}
        started = set()
        n_waits = {r: 0 for r in roles}
        alive = set(roles)
        while alive or self.commits or self.loads:
            moves = []
            for r in sorted(alive):
                w = waits[r]
                if r not in started:
                    moves.append((r, None))
                elif give_up is not None and r == give_up[0] and n_waits[r] == give_up[1] + 1 \
                        and not self.aborted and w is not None and (len(w) < 4 or w[3]):
                    moves.append((r, "timeout"))
                elif self._passes(r, w):
                    moves.append((r, True))
                elif self.aborted and (len(w) < 4 or w[3]):
                    moves.append((r, False))
            if self.commits:
                moves.append("<tensor core>")
            moves += [("<copy>", i) for i in range(len(self.loads))]
            if not moves:
                return {r: waits[r] for r in alive}
            m = self.rng.choice(moves)
            if m == "<tensor core>":
                self.arrive(self.commits.popleft())
            elif m[0] == "<copy>":
                self.arrive(self.loads.pop(m[1]))
            else:
                r, outcome = m
                if outcome == "timeout":
                    self.aborted = True
                    outcome = False
                try:
                    if r in started:
                        waits[r] = roles[r].send(outcome)
                    else:
                        started.add(r)
                        waits[r] = next(roles[r])
                    n_waits[r] += 1
                except StopIteration:
                    alive.discard(r)
                    waits[r] = None
                    if not alive:
                        self.in_flight_at_exit = len(self.commits) + len(self.loads)
                        self.pending_at_exit = (list(self.commits), list(self.loads))
        return None
