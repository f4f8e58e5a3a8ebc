"""A model of the backward kernel's mbarrier protocol, run under random
interleavings of its warp roles (CPU only).

Each role of the backward kernel (TMA producer, MMA issuer, P warps, dS warps,
dQ drain) is modelled as a generator that waits on and arrives at the same
barriers, with the same counts and phase arithmetic, as
``tiled_attention_25_b200/csrc/bwd_sm100.cu``; a group of warps that arrive
together is one arrival here.  A wait names the phase it wants: a "full"
wait on phase k succeeds once k has completed, an "empty" wait on phase k
succeeds once k - 1 has (the first pass is free).  The hardware only compares
parities, so the checks are:

* no deadlock: some role can always move until all have finished;
* no aliasing: when a wait succeeds, the barrier has completed exactly the
  phase the waiter wants, never two more (a parity test cannot tell those
  apart, and the waiter would run on another step's data).

Unit lengths include units without steps, the case whose accumulator
hand-over needed its own ordering.
"""
import random

import pytest

STAGES = 3  # Q / dO stages


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.done = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier's count"
        if self.pending == 0:
            self.done += 1
            self.pending = self.count


def full(name, k):
    return ("wait", name, k, False)


def empty(name, k):
    return ("wait", name, k, True)


def ready(bar, k, is_empty):
    """The hardware's parity test: phase parity (k & 1) ^ is_empty has completed."""
    parity = (k & 1) ^ int(is_empty)
    return (bar.done & 1) != parity


def simulate(units, seed, drain_share=True, empty_unit_waits=True):
    """Run the roles to completion; return None, or the stuck roles' waits.
    The two switches remove a step of the protocol, to show the model notices."""
    B = {}

    def bar(name, count):
        B[name] = Barrier(count)

    for b in range(2):
        bar(f"list_full{b}", 1)      # TMA warp
        bar(f"list_empty{b}", 4)     # MMA, P, dS, drain each release the list
        bar(f"s_full{b}", 1)         # MMA commit
        bar(f"p_ready{b}", 1)        # P warps
        bar(f"ds_ready{b}", 2)       # dS warps + drain warps
        bar(f"ds_empty{b}", 1)       # drain
    bar("kv_full", 1)
    bar("kv_empty", 1)
    for s in range(STAGES):
        bar(f"q_full{s}", 1)
        bar(f"q_empty{s}", 1)
    bar("dp_full", 1)
    bar("dp_empty", 1)
    bar("dq_full", 1)
    bar("acc_full", 1)
    bar("acc_empty", 2)              # P warps + dS warps after the epilogue

    def tma():
        step = 0
        for u, n in enumerate(units):
            b = u & 1
            yield empty(f"list_empty{b}", u >> 1)
            B[f"list_full{b}"].arrive()
            yield empty("kv_empty", u)
            B["kv_full"].arrive()
            for _ in range(n):
                s = step % STAGES
                yield empty(f"q_empty{s}", step // STAGES)
                B[f"q_full{s}"].arrive()
                step += 1

    def mma():
        step = 0
        for u, n in enumerate(units):
            b = u & 1
            yield full(f"list_full{b}", u >> 1)
            yield full("kv_full", u)
            if n > 0:  # S^T(0) and dP^T(0) of the unit
                yield full(f"q_full{step % STAGES}", step // STAGES)
                B[f"s_full{step & 1}"].arrive()
                B["dp_full"].arrive()
            for k in range(n):
                nxt = k + 1 < n
                s, sb = step % STAGES, step & 1
                if nxt:  # S^T(j+1)
                    yield full(f"q_full{(step + 1) % STAGES}", (step + 1) // STAGES)
                    B[f"s_full{(step + 1) & 1}"].arrive()
                yield full(f"p_ready{sb}", step >> 1)  # dV(j)
                if k == 0:
                    yield empty("acc_empty", u)
                if nxt:  # dP^T(j+1)
                    yield full("dp_empty", step)
                    B["dp_full"].arrive()
                yield full(f"ds_ready{sb}", step >> 1)  # dK(j), dQ^T(j)
                B["dq_full"].arrive()
                B[f"q_empty{s}"].arrive()
                step += 1
            if n == 0 and empty_unit_waits:
                yield empty("acc_empty", u)
            B["kv_empty"].arrive()
            B["acc_full"].arrive()
            B[f"list_empty{b}"].arrive()

    def p_warps():
        step = 0
        for u, n in enumerate(units):
            b = u & 1
            yield full(f"list_full{b}", u >> 1)
            for _ in range(n):
                s, sb = step % STAGES, step & 1
                yield full(f"q_full{s}", step // STAGES)
                yield full(f"s_full{sb}", step >> 1)
                B[f"p_ready{sb}"].arrive()
                step += 1
            yield full("acc_full", u)
            B["acc_empty"].arrive()
            B[f"list_empty{b}"].arrive()

    def ds_warps():
        step = 0
        for u, n in enumerate(units):
            b = u & 1
            yield full(f"list_full{b}", u >> 1)
            for _ in range(n):
                s, sb = step % STAGES, step & 1
                yield full(f"q_full{s}", step // STAGES)
                yield full(f"p_ready{sb}", step >> 1)
                yield full("dp_full", step)
                B["dp_empty"].arrive()
                yield empty(f"ds_empty{sb}", step >> 1)
                B[f"ds_ready{sb}"].arrive()
                step += 1
            yield full("acc_full", u)
            B["acc_empty"].arrive()
            B[f"list_empty{b}"].arrive()

    def drain():
        step = 0
        if drain_share:
            B["ds_ready0"].arrive()  # its share of step 0, given up front
        for u, n in enumerate(units):
            b = u & 1
            yield full(f"list_full{b}", u >> 1)
            for _ in range(n):
                yield full("dq_full", step)
                # dQ^T(j) read: the share of step j+1, then the dS buffer of step j
                B[f"ds_ready{(step + 1) & 1}"].arrive()
                B[f"ds_empty{step & 1}"].arrive()
                step += 1
            B[f"list_empty{b}"].arrive()

    roles = {"tma": tma(), "mma": mma(), "p": p_warps(), "ds": ds_warps(), "drain": drain()}
    pending = {r: None for r in roles}
    alive = set(roles)
    rng = random.Random(seed)
    while alive:
        order = sorted(alive)
        rng.shuffle(order)
        moved = False
        for r in order:
            w = pending[r]
            if w is not None:
                _, name, k, is_empty = w
                if not ready(B[name], k, is_empty):
                    continue
                want = k if is_empty else k + 1
                assert B[name].done == want, (
                    f"{r} waited on {name} phase {k} ({'empty' if is_empty else 'full'}) "
                    f"and passed with {B[name].done} phases completed")
            try:
                pending[r] = next(roles[r])
            except StopIteration:
                alive.discard(r)
                pending[r] = None
            moved = True
            break
        if not moved:
            return {r: pending[r] for r in alive}
    return None


UNIT_PATTERNS = [[10], [4], [1], [2], [3], [10, 10], [3, 5, 1, 2], [0, 4], [7, 0, 2], [0, 0, 3],
                 [1, 1, 1, 1], [5, 0, 0, 5], [0], [0, 0], [2, 0, 1, 0, 3, 0]]


@pytest.mark.parametrize("units", UNIT_PATTERNS, ids=lambda u: "-".join(map(str, u)))
def test_backward_protocol_never_deadlocks_or_aliases(units):
    for seed in range(200):
        stuck = simulate(units, seed)
        assert stuck is None, f"deadlock with units {units}, seed {seed}: {stuck}"


def test_the_model_detects_a_missing_up_front_share():
    # without the drain's share of step 0, ds_ready never completes its first phase
    assert simulate([3], 0, drain_share=False) is not None


def test_the_model_detects_an_empty_unit_handing_over_early():
    # a unit without steps that announces its accumulators without waiting for the
    # previous unit's epilogue runs the acc_full phases ahead of their readers
    failures = 0
    for seed in range(200):
        try:
            failures += simulate([2, 0, 0, 3], seed, empty_unit_waits=False) is not None
        except AssertionError:
            failures += 1
    assert failures > 0
