"""A model of the forward kernel's mbarrier protocol, run under random
interleavings of its warp roles (CPU only).

Roles as in ``tiled_attention_25_b200/csrc/fwd_sm100.cu``, with its barrier
counts and phase arithmetic (a group of warps that arrive together is one
arrival here):

* the TMA warp builds each unit's step list, loads the unit's two query
  tiles and streams K and V through a ring of slots;
* the MMA warp issues S_t = Q_t K^T and O_t += P_t V for the two query tiles
  t of the unit, in the ping-pong order, committing s_full, o_full, the ring's
  empty slots, q_empty and, on units with steps, o_final (each tile's right
  after its last PV);
* two softmax warpgroups, one per query tile, turn S_t into P_t (p_full) and
  sometimes rescale O_t, which first waits for the previous PV (o_full);
  the rescale decision depends on the data, so the model draws it.

A step may be active for one query tile only (masked pairs), and units may
have no steps at all (a window with Sq >> Skv).  MMA commits and TMA copies
complete later, at times the simulator picks (``protocol_sim``).  The checks:
no deadlock, and no aliasing (a passing wait sees exactly the phase it wants).
"""
import pytest

from protocol_sim import Sim


def simulate(units, seed, stages=4, final_on_empty_units=False, clc=False):
    """units: per unit, a list of steps (act0, act1).  Returns None, or the
    stuck roles' waits.  final_on_empty_units commits o_final for units
    without steps too, as the kernel once did, to show the model notices."""
    sim = Sim(seed)
    full, empty = sim.full, sim.empty
    for b in range(2):
        sim.bar(f"list_full{b}", 1)
        sim.bar(f"list_empty{b}", 3)      # MMA warp + the two softmax warpgroups
    sim.bar("q_full", 1)
    sim.bar("q_empty", 1)
    sim.bar("clc_bar", 1)                 # the cancel request's response (cluster launch control)
    walk = list(units) + [None]           # None: the published end of the walk
    for t in range(2):
        sim.bar(f"s_full{t}", 1)
        sim.bar(f"p_full{t}", 1)
        sim.bar(f"o_full{t}", 1)
        sim.bar(f"o_final{t}", 1)
    for s in range(stages):
        sim.bar(f"kv_full{s}", 1)
        sim.bar(f"kv_empty{s}", 1)

    def tma():
        ring = 0
        for u, steps in enumerate(walk):
            b = u & 1
            yield empty(f"list_empty{b}", u >> 1)
            sim.arrive(f"list_full{b}")
            if steps is None:
                break
            if clc:
                sim.load("clc_bar")             # ask for the next unit; answered later
            yield empty("q_empty", u)
            sim.load("q_full")                  # both query tiles, one byte count
            for _ in steps:
                for _which in range(2):         # K, then V
                    slot = ring % stages
                    yield empty(f"kv_empty{slot}", ring // stages)
                    sim.load(f"kv_full{slot}")
                    ring += 1
            if clc:
                yield full("clc_bar", u)        # the answer: the next unit, or the end

    def mma():
        ring = 0
        pv = [0, 0]                             # PV products issued per query tile
        for u, steps in enumerate(walk):
            b = u & 1
            yield full(f"list_full{b}", u >> 1)
            if steps is None:
                break
            n = len(steps)
            yield full("q_full", u)
            if n > 0:                           # S_t(0)
                slot_k = ring % stages
                yield full(f"kv_full{slot_k}", ring // stages)
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
                yield full(f"kv_full{slot_v}", ph_v)
                for t in range(2):
                    if steps[j][t]:             # PV_t(j)
                        yield full(f"p_full{t}", pv[t])
                        pv[t] += 1
                        sim.commit(f"o_full{t}")
                    if not nxt:                 # tile t's O is final after its last PV
                        sim.commit(f"o_final{t}")
                    if nxt:                     # S_t(j+1)
                        if t == 0:
                            yield full(f"kv_full{slot_kn}", ph_kn)
                        if steps[j + 1][t]:
                            sim.commit(f"s_full{t}")
                if nxt:
                    sim.commit(f"kv_empty{slot_kn}")
                sim.commit(f"kv_empty{slot_v}")
                if nxt:
                    ring += 1
            sim.commit("q_empty")
            if n == 0 and final_on_empty_units:
                sim.commit("o_final0")
                sim.commit("o_final1")
            sim.arrive(f"list_empty{b}")

    def softmax(t):
        s_cnt = p_cnt = o_units = 0
        for u, steps in enumerate(walk):
            b = u & 1
            yield full(f"list_full{b}", u >> 1)
            if steps is None:
                break
            n_act = 0
            for step in steps:
                if not step[t]:
                    continue
                yield full(f"s_full{t}", s_cnt)
                s_cnt += 1
                if n_act > 0 and sim.rng.random() < 0.3:   # the row max moved: rescale O
                    yield full(f"o_full{t}", p_cnt - 1)
                sim.arrive(f"p_full{t}")
                p_cnt += 1
                n_act += 1
            if steps:
                yield full(f"o_final{t}", o_units)
                o_units += 1
            sim.arrive(f"list_empty{b}")

    return sim.run({"tma": tma(), "mma": mma(), "softmax0": softmax(0), "softmax1": softmax(1)})


BOTH, FIRST, SECOND = (1, 1), (1, 0), (0, 1)
UNIT_PATTERNS = {
    "dense": [[BOTH] * 6, [BOTH] * 6],
    "causal": [[BOTH] * 3 + [FIRST], [BOTH, FIRST], [BOTH] * 5 + [FIRST]],
    "one_tile_steps": [[FIRST, SECOND, BOTH, SECOND], [SECOND], [FIRST]],
    "single_steps": [[BOTH], [BOTH], [BOTH]],
    "empty_units": [[], [BOTH, BOTH], [], [], [FIRST], []],
    "only_empty": [[], []],
    "long": [[BOTH] * 20],
}


@pytest.mark.parametrize("clc", [False, True], ids=["static", "clc"])
@pytest.mark.parametrize("stages", [4, 6])
@pytest.mark.parametrize("name", sorted(UNIT_PATTERNS))
def test_forward_protocol_never_deadlocks_or_aliases(name, stages, clc):
    for seed in range(150):
        stuck = simulate(UNIT_PATTERNS[name], seed, stages=stages, clc=clc)
        assert stuck is None, f"deadlock in {name}, seed {seed}: {stuck}"


def test_the_model_detects_o_final_on_empty_units():
    # committing o_final on units without steps runs its phases ahead of the
    # softmax warps, which wait for it on units with steps only
    failures = 0
    for seed in range(150):
        try:
            failures += simulate(UNIT_PATTERNS["empty_units"], seed, final_on_empty_units=True) is not None
        except AssertionError:
            failures += 1
    assert failures > 0
