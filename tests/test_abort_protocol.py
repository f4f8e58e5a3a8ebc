"""The kernels' timeout path, modelled on the interleaving simulator (CPU only).

Every wait in the forward and backward kernels is bounded.  When one runs
out, the role records the timeout, sets the CTA's abort word and leaves its
loop; every other role's next wait sees the word and leaves too.  Before the
CTA exits (and frees its tensor memory), two roles let their own
asynchronous work land, with waits that ignore the abort word:

* the TMA warp waits for the last copy it issued into each K/V (or Q/dO)
  slot and for its last query-tile copy;
* the MMA warp commits every MMA it issued to a drain barrier and waits on it.

The TMA warp drains whether or not its own loop gave up: when a consumer
gives up, the TMA warp may already have issued its last copies and leave its
loop normally, with those copies still landing (the model found this; the
kernels once drained only after a failed wait of their own).

The models below follow the barrier order of ``csrc/fwd_sm100.cu`` and
``csrc/bwd_sm100.cu`` as the protocol models do, plus these exits.  For every
role and every wait index up to a bound, that wait is made to run out, under
random interleavings; the checks are that every role ends (no role waits for
work that can no longer come) and that no copy or MMA is still in flight when
the last role ends.  Planting back either old drain (only after a failed
wait of the TMA warp's own, or skipping the slots' last copies) makes the
check fail.
"""
import pytest

from protocol_sim import Sim

STAGES_BWD = 3


def forward(units, seed, give_up, stages=4, drain_kv=True, drain_always=True, clc=False):
    sim = Sim(seed)
    full, empty, drain = sim.full, sim.empty, sim.drain
    for b in range(2):
        sim.bar(f"list_full{b}", 1)
        sim.bar(f"list_empty{b}", 3)
    for name in ("q_full", "q_empty", "drain", "clc_bar"):
        sim.bar(name, 1)
    walk = list(units) + [None]  # None: the published end of the walk
    for t in range(2):
        for name in ("s_full", "p_full", "o_full", "o_final"):
            sim.bar(f"{name}{t}", 1)
    for s in range(stages):
        sim.bar(f"kv_full{s}", 1)
        sim.bar(f"kv_empty{s}", 1)

    def tma():
        ring, q_loads, uses = 0, 0, [0] * stages
        asked = answered = 0
        ok = True
        for u, steps in enumerate(walk):
            b = u & 1
            ok = yield empty(f"list_empty{b}", u >> 1)
            if not ok:
                break
            sim.arrive(f"list_full{b}")
            if steps is None:
                break
            if clc:
                sim.load("clc_bar")
                asked += 1
            ok = yield empty("q_empty", u)
            if not ok:
                break
            sim.load("q_full")
            q_loads += 1
            for _ in steps:
                for _which in range(2):
                    slot = ring % stages
                    ok = yield empty(f"kv_empty{slot}", ring // stages)
                    if not ok:
                        break
                    sim.load(f"kv_full{slot}")
                    uses[slot] += 1
                    ring += 1
                if not ok:
                    break
            if not ok:
                break
            if clc:
                ok = yield full("clc_bar", u)
                if not ok:
                    break
                answered += 1
        if drain_always or not ok:  # let the copies in flight land
            if asked > answered:
                yield drain("clc_bar", asked - 1)
            for s in range(stages):
                if uses[s] and drain_kv:
                    yield drain(f"kv_full{s}", uses[s] - 1)
            if q_loads:
                yield drain("q_full", q_loads - 1)

    def mma():
        ring, pv = 0, [0, 0]
        ok = True
        for u, steps in enumerate(walk):
            b = u & 1
            ok = yield full(f"list_full{b}", u >> 1)
            if not ok or steps is None:
                break
            n = len(steps)
            ok = yield full("q_full", u)
            if not ok:
                break
            if n > 0:
                slot_k = ring % stages
                ok = yield full(f"kv_full{slot_k}", ring // stages)
                if not ok:
                    break
                for t in range(2):
                    if steps[0][t]:
                        sim.commit(f"s_full{t}")
                sim.commit(f"kv_empty{slot_k}")
                ring += 1
            for j in range(n):
                slot_v, ph_v = ring % stages, ring // stages
                ring += 1
                nxt = j + 1 < n
                slot_kn, ph_kn = ring % stages, ring // stages
                ok = yield full(f"kv_full{slot_v}", ph_v)
                if not ok:
                    break
                for t in range(2):
                    if steps[j][t]:
                        ok = yield full(f"p_full{t}", pv[t])
                        if not ok:
                            break
                        pv[t] += 1
                        sim.commit(f"o_full{t}")
                    if not nxt:
                        sim.commit(f"o_final{t}")
                    if nxt:
                        if t == 0:
                            ok = yield full(f"kv_full{slot_kn}", ph_kn)
                            if not ok:
                                break
                        if steps[j + 1][t]:
                            sim.commit(f"s_full{t}")
                if not ok:
                    break
                if nxt:
                    sim.commit(f"kv_empty{slot_kn}")
                sim.commit(f"kv_empty{slot_v}")
                if nxt:
                    ring += 1
            if not ok:
                break
            sim.commit("q_empty")
            sim.arrive(f"list_empty{b}")
        sim.commit("drain")  # every MMA issued so far completes before this arrival
        yield drain("drain", 0)

    def softmax(t):
        s_cnt = p_cnt = o_units = 0
        for u, steps in enumerate(walk):
            b = u & 1
            if not (yield full(f"list_full{b}", u >> 1)) or steps is None:
                return
            n_act = 0
            for step in steps:
                if not step[t]:
                    continue
                if not (yield full(f"s_full{t}", s_cnt)):
                    return
                s_cnt += 1
                if n_act > 0 and sim.rng.random() < 0.3:
                    if not (yield full(f"o_full{t}", p_cnt - 1)):
                        return
                sim.arrive(f"p_full{t}")
                p_cnt += 1
                n_act += 1
            if steps:
                if not (yield full(f"o_final{t}", o_units)):
                    return
                o_units += 1
            sim.arrive(f"list_empty{b}")

    roles = {"tma": tma(), "mma": mma(), "softmax0": softmax(0), "softmax1": softmax(1)}
    stuck = sim.run(roles, give_up=give_up)
    return stuck, sim.in_flight_at_exit


def backward(units, seed, give_up, drain_stages=True, drain_always=True, clc=False):
    sim = Sim(seed)
    full, empty, drain = sim.full, sim.empty, sim.drain
    S = STAGES_BWD
    for b in range(2):
        sim.bar(f"list_full{b}", 1)
        sim.bar(f"list_empty{b}", 4)
        sim.bar(f"s_full{b}", 1)
        sim.bar(f"p_ready{b}", 1)
        sim.bar(f"ds_ready{b}", 2)
        sim.bar(f"ds_empty{b}", 1)
    for name in ("kv_full", "kv_empty", "dp_full", "dp_empty", "dq_full", "acc_full", "drain", "clc_bar"):
        sim.bar(name, 1)
    walk = list(units) + [None]  # None: the published end of the walk
    sim.bar("acc_empty", 2)
    for s in range(S):
        sim.bar(f"q_full{s}", 1)
        sim.bar(f"q_empty{s}", 1)

    def tma():
        step, kv_loads, uses = 0, 0, [0] * S
        asked = answered = 0
        ok = True
        for u, n in enumerate(walk):
            b = u & 1
            ok = yield empty(f"list_empty{b}", u >> 1)
            if not ok:
                break
            sim.arrive(f"list_full{b}")
            if n is None:
                break
            if clc:
                sim.load("clc_bar")
                asked += 1
            ok = yield empty("kv_empty", u)
            if not ok:
                break
            sim.load("kv_full")
            kv_loads += 1
            for _ in range(n):
                s = step % S
                ok = yield empty(f"q_empty{s}", step // S)
                if not ok:
                    break
                sim.load(f"q_full{s}")
                uses[s] += 1
                step += 1
            if not ok:
                break
            if clc:
                ok = yield full("clc_bar", u)
                if not ok:
                    break
                answered += 1
        if drain_always or not ok:
            if asked > answered:
                yield drain("clc_bar", asked - 1)
            if kv_loads:
                yield drain("kv_full", kv_loads - 1)
            for s in range(S):
                if uses[s] and drain_stages:
                    yield drain(f"q_full{s}", uses[s] - 1)

    def mma():
        step = 0
        ok = True
        for u, n in enumerate(walk):
            b = u & 1
            ok = yield full(f"list_full{b}", u >> 1)
            if not ok or n is None:
                break
            ok = yield full("kv_full", u)
            if not ok:
                break
            if n > 0:
                ok = yield full(f"q_full{step % S}", step // S)
                if not ok:
                    break
                sim.commit(f"s_full{step & 1}")
                sim.commit("dp_full")
            for k in range(n):
                nxt = k + 1 < n
                s, sb = step % S, step & 1
                if nxt:
                    ok = yield full(f"q_full{(step + 1) % S}", (step + 1) // S)
                    if not ok:
                        break
                    sim.commit(f"s_full{(step + 1) & 1}")
                ok = yield full(f"p_ready{sb}", step >> 1)
                if ok and k == 0:
                    ok = yield empty("acc_empty", u)
                if not ok:
                    break
                if nxt:
                    ok = yield full("dp_empty", step)
                    if not ok:
                        break
                    sim.commit("dp_full")
                ok = yield full(f"ds_ready{sb}", step >> 1)
                if not ok:
                    break
                sim.commit("dq_full")
                sim.commit(f"q_empty{s}")
                step += 1
            if not ok:
                break
            if n == 0:
                ok = yield empty("acc_empty", u)
                if not ok:
                    break
            sim.commit("kv_empty")
            sim.commit("acc_full")
            sim.arrive(f"list_empty{b}")
        sim.commit("drain")
        yield drain("drain", 0)

    def p_warps():
        step = 0
        for u, n in enumerate(walk):
            b = u & 1
            if not (yield full(f"list_full{b}", u >> 1)) or n is None:
                return
            for _ in range(n):
                s, sb = step % S, step & 1
                if not ((yield full(f"q_full{s}", step // S)) and (yield full(f"s_full{sb}", step >> 1))):
                    return
                sim.arrive(f"p_ready{sb}")
                step += 1
            if not (yield full("acc_full", u)):
                return
            sim.arrive("acc_empty")
            sim.arrive(f"list_empty{b}")

    def ds_warps():
        step = 0
        for u, n in enumerate(walk):
            b = u & 1
            if not (yield full(f"list_full{b}", u >> 1)) or n is None:
                return
            for _ in range(n):
                s, sb = step % S, step & 1
                ok = (yield full(f"q_full{s}", step // S)) and (yield full(f"p_ready{sb}", step >> 1)) \
                    and (yield full("dp_full", step))
                if not ok:
                    return
                sim.arrive("dp_empty")
                if not (yield empty(f"ds_empty{sb}", step >> 1)):
                    return
                sim.arrive(f"ds_ready{sb}")
                step += 1
            if not (yield full("acc_full", u)):
                return
            sim.arrive("acc_empty")
            sim.arrive(f"list_empty{b}")

    def dq_drain():
        step = 0
        sim.arrive("ds_ready0")
        for u, n in enumerate(walk):
            b = u & 1
            if not (yield full(f"list_full{b}", u >> 1)) or n is None:
                return
            for _ in range(n):
                if not (yield full("dq_full", step)):
                    return
                sim.arrive(f"ds_ready{(step + 1) & 1}")
                sim.arrive(f"ds_empty{step & 1}")
                step += 1
            sim.arrive(f"list_empty{b}")

    roles = {"tma": tma(), "mma": mma(), "p": p_warps(), "ds": ds_warps(), "drain": dq_drain()}
    stuck = sim.run(roles, give_up=give_up)
    return stuck, sim.in_flight_at_exit


BOTH, FIRST = (1, 1), (1, 0)
FWD_UNITS = [[BOTH] * 5, [BOTH, FIRST], [], [BOTH] * 3]
BWD_UNITS = [4, 0, 3, 1]


@pytest.mark.parametrize("clc", [False, True], ids=["static", "clc"])
@pytest.mark.parametrize("role", ["tma", "mma", "softmax0", "softmax1"])
def test_forward_timeout_at_any_wait_ends_clean(role, clc):
    for n in range(0, 40, 3):
        for seed in range(12):
            stuck, left = forward(FWD_UNITS, seed, (role, n), clc=clc)
            assert stuck is None, f"{role} wait {n} seed {seed}: stuck {stuck}"
            assert left == 0, f"{role} wait {n} seed {seed}: {left} copies/MMAs in flight at exit"


@pytest.mark.parametrize("clc", [False, True], ids=["static", "clc"])
@pytest.mark.parametrize("role", ["tma", "mma", "p", "ds", "drain"])
def test_backward_timeout_at_any_wait_ends_clean(role, clc):
    for n in range(0, 40, 3):
        for seed in range(12):
            stuck, left = backward(BWD_UNITS, seed, (role, n), clc=clc)
            assert stuck is None, f"{role} wait {n} seed {seed}: stuck {stuck}"
            assert left == 0, f"{role} wait {n} seed {seed}: {left} copies/MMAs in flight at exit"


def test_without_timeouts_the_models_run_as_before():
    for seed in range(20):
        for clc in (False, True):
            assert forward(FWD_UNITS, seed, None, clc=clc) == (None, 0)
            assert backward(BWD_UNITS, seed, None, clc=clc) == (None, 0)


def test_the_check_notices_copies_left_in_flight():
    """A TMA warp that skipped its K/V (forward) or Q/dO (backward) slots when
    draining would let the CTA exit with copies still landing."""
    left_f = sum(forward(FWD_UNITS, seed, ("mma", n), drain_kv=False)[1] or 0
                 for seed in range(10) for n in range(0, 40, 2))
    left_b = sum(backward(BWD_UNITS, seed, ("mma", n), drain_stages=False)[1] or 0
                 for seed in range(10) for n in range(0, 40, 2))
    assert left_f > 0 and left_b > 0


def test_the_check_notices_a_drain_only_after_own_failure():
    """A TMA warp that drains only when one of its own waits failed exits with
    copies in flight when a consumer gave up after the last copies were issued."""
    left = sum((backward(BWD_UNITS, seed, (role, n), drain_always=False)[1] or 0)
               for role in ("mma", "p", "ds", "drain") for seed in range(10) for n in range(0, 40, 2))
    assert left > 0
