"""A model of the backward kernel's mbarrier protocol, run under random
interleavings of its warp roles (CPU only).

Each role of the backward kernel (TMA producer, MMA issuer, P warps, dS warps,
dQ drain) is modelled as a generator that waits on and arrives at the same
barriers, with the same counts and phase arithmetic, as
``tiled_attention_25_b200/csrc/bwd_sm100.cu``; a group of warps that arrive
together is one arrival here.  MMA commits and TMA copies complete later, at
times the simulator picks (``protocol_sim``).  The checks: no deadlock, and
no aliasing (a passing wait sees exactly the phase it wants).

Unit lengths include units without steps, the case whose accumulator
hand-over needed its own ordering.
"""
import pytest

from protocol_sim import Sim

STAGES = 3  # Q / dO stages


def simulate(units, seed, drain_share=True, empty_unit_waits=True, clc=False):
    """Run the roles to completion; return None, or the stuck roles' waits.
    The two switches remove a step of the protocol, to show the model notices."""
    sim = Sim(seed)
    full, empty = sim.full, sim.empty
    for b in range(2):
        sim.bar(f"list_full{b}", 1)      # TMA warp
        sim.bar(f"list_empty{b}", 4)     # MMA, P, dS, drain each release the list
        sim.bar(f"s_full{b}", 1)         # MMA commit
        sim.bar(f"p_ready{b}", 1)        # P warps
        sim.bar(f"ds_ready{b}", 2)       # dS warps + drain warps
        sim.bar(f"ds_empty{b}", 1)       # drain
    sim.bar("kv_full", 1)
    sim.bar("kv_empty", 1)
    for s in range(STAGES):
        sim.bar(f"q_full{s}", 1)
        sim.bar(f"q_empty{s}", 1)
    sim.bar("dp_full", 1)
    sim.bar("dp_empty", 1)
    sim.bar("dq_full", 1)
    sim.bar("acc_full", 1)
    sim.bar("acc_empty", 2)              # P warps + dS warps after the epilogue
    sim.bar("clc_bar", 1)                # the cancel request's response (cluster launch control)
    walk = list(units) + [None]          # None: the published end of the walk

    def tma():
        step = 0
        for u, n in enumerate(walk):
            b = u & 1
            yield empty(f"list_empty{b}", u >> 1)
            sim.arrive(f"list_full{b}")
            if n is None:
                break
            if clc:
                sim.load("clc_bar")       # ask for the next unit; answered later
            yield empty("kv_empty", u)
            sim.load("kv_full")           # K and V, one expected byte count
            for _ in range(n):
                s = step % STAGES
                yield empty(f"q_empty{s}", step // STAGES)
                sim.load(f"q_full{s}")    # Q, dO and the row statistics
                step += 1
            if clc:
                yield full("clc_bar", u)  # the answer: the next unit, or the end

    def mma():
        step = 0
        for u, n in enumerate(walk):
            b = u & 1
            yield full(f"list_full{b}", u >> 1)
            if n is None:
                break
            yield full("kv_full", u)
            if n > 0:  # S^T(0) and dP^T(0) of the unit
                yield full(f"q_full{step % STAGES}", step // STAGES)
                sim.commit(f"s_full{step & 1}")
                sim.commit("dp_full")
            for k in range(n):
                nxt = k + 1 < n
                s, sb = step % STAGES, step & 1
                if nxt:  # S^T(j+1)
                    yield full(f"q_full{(step + 1) % STAGES}", (step + 1) // STAGES)
                    sim.commit(f"s_full{(step + 1) & 1}")
                yield full(f"p_ready{sb}", step >> 1)  # dV(j)
                if k == 0:
                    yield empty("acc_empty", u)
                if nxt:  # dP^T(j+1)
                    yield full("dp_empty", step)
                    sim.commit("dp_full")
                yield full(f"ds_ready{sb}", step >> 1)  # dK(j), dQ^T(j)
                sim.commit("dq_full")
                sim.commit(f"q_empty{s}")
                step += 1
            if n == 0 and empty_unit_waits:
                yield empty("acc_empty", u)
            sim.commit("kv_empty")
            sim.commit("acc_full")
            sim.arrive(f"list_empty{b}")

    def p_warps():
        step = 0
        for u, n in enumerate(walk):
            b = u & 1
            yield full(f"list_full{b}", u >> 1)
            if n is None:
                break
            for _ in range(n):
                s, sb = step % STAGES, step & 1
                yield full(f"q_full{s}", step // STAGES)
                yield full(f"s_full{sb}", step >> 1)
                sim.arrive(f"p_ready{sb}")
                step += 1
            yield full("acc_full", u)
            sim.arrive("acc_empty")
            sim.arrive(f"list_empty{b}")

    def ds_warps():
        step = 0
        for u, n in enumerate(walk):
            b = u & 1
            yield full(f"list_full{b}", u >> 1)
            if n is None:
                break
            for _ in range(n):
                s, sb = step % STAGES, step & 1
                yield full(f"q_full{s}", step // STAGES)
                yield full(f"p_ready{sb}", step >> 1)
                yield full("dp_full", step)
                sim.arrive("dp_empty")
                yield empty(f"ds_empty{sb}", step >> 1)
                sim.arrive(f"ds_ready{sb}")
                step += 1
            yield full("acc_full", u)
            sim.arrive("acc_empty")
            sim.arrive(f"list_empty{b}")

    def drain():
        step = 0
        if drain_share:
            sim.arrive("ds_ready0")  # its share of step 0, given up front
        for u, n in enumerate(walk):
            b = u & 1
            yield full(f"list_full{b}", u >> 1)
            if n is None:
                break
            for _ in range(n):
                yield full("dq_full", step)
                # dQ^T(j) read: the share of step j+1, then the dS buffer of step j
                sim.arrive(f"ds_ready{(step + 1) & 1}")
                sim.arrive(f"ds_empty{step & 1}")
                step += 1
            sim.arrive(f"list_empty{b}")

    return sim.run({"tma": tma(), "mma": mma(), "p": p_warps(), "ds": ds_warps(), "drain": drain()})


UNIT_PATTERNS = [[10], [4], [1], [2], [3], [10, 10], [3, 5, 1, 2], [0, 4], [7, 0, 2], [0, 0, 3],
                 [1, 1, 1, 1], [5, 0, 0, 5], [0], [0, 0], [2, 0, 1, 0, 3, 0]]


@pytest.mark.parametrize("clc", [False, True], ids=["static", "clc"])
@pytest.mark.parametrize("units", UNIT_PATTERNS, ids=lambda u: "-".join(map(str, u)))
def test_backward_protocol_never_deadlocks_or_aliases(units, clc):
    for seed in range(200):
        stuck = simulate(units, seed, clc=clc)
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
