"""Both work walks of the persistent kernels (attn_set_work_walk): the static
snake over the longest-first order, and cluster launch control (one CTA per
unit, idle CTAs cancelling not-yet-started ones and taking their units).  A
unit's results do not depend on which CTA computes it, so the forward output
and LSE, and dK, dV, are bitwise equal between the walks; dQ agrees within
rounding and both match the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import Case, check_lse, check_o, host_f64, rel_l2
from synth_inputs import ModParams
from test_gpu_backward import check_grads, run_fwd_bwd, small_params

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    import tiled_attention_25_b200 as m
    yield m
    m.attn_set_work_walk(m.WALK_DEFAULT)


def run_both(ta, c, use_mask=True):
    res = {}
    for walk in (ta.WALK_STATIC, ta.WALK_CLUSTER_LAUNCH_CONTROL):
        ta.attn_set_work_walk(walk)
        mask = ta.new_block_mask(c.mod, c.dev_params, c.B, c.Sq, c.Skv) if use_mask else None
        out = torch.empty_like(c.q)
        lse = torch.empty(c.B, c.Hq, c.Sq, dtype=torch.float32, device="cuda")
        ta.attn_fwd(c.q, c.k, c.v, out, lse, scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params,
                    block_mask=mask)
        torch.cuda.synchronize()
        assert ta.attn_get_status() == 0
        res[walk] = (out, lse, run_fwd_bwd(ta, c, use_mask))
    ta.attn_set_work_walk(ta.WALK_DEFAULT)
    return res[ta.WALK_STATIC], res[ta.WALK_CLUSTER_LAUNCH_CONTROL]


@pytest.mark.parametrize("mod", [oracle.MOD_NONE, oracle.MOD_CAUSAL, oracle.MOD_SLIDING_WINDOW, oracle.MOD_DOCUMENT])
@pytest.mark.parametrize("use_mask", [False, True])
def test_walks_agree_and_match_oracle(ta, mod, use_mask):
    S = 1000
    c = Case(70 + mod, 2, 8, 2, S, S, 128, mod, small_params(mod, S) if mod != oracle.MOD_DOCUMENT else
             ModParams(doc_offsets=[[0, 300, 301, 720, S], [0, 512, S]]))
    (o1, l1, g1), (o2, l2, g2) = run_both(ta, c, use_mask)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1, l2)
    for x, y in zip(g1[1:], g2[1:]):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    assert rel_l2(host_f64(g2[0]), host_f64(g1[0])) < 1e-2
    O, L = c.oracle_fwd()
    check_o(host_f64(o2), O, f"clc mod {mod}")
    check_lse(l2.cpu().double().numpy(), L, f"clc mod {mod}")
    check_grads([host_f64(t) for t in g2], c.oracle_bwd(), f"clc mod {mod}")


def test_many_units_per_sm_and_units_without_work(ta):
    """Far more units than SMs (each CTA cancels many others), including
    backward units that meet no query (causal, Skv >> Sq) and forward units
    that meet no key (window, Sq >> Skv)."""
    for c in (Case(71, 1, 32, 32, 128, 2048, 64, oracle.MOD_CAUSAL),
              Case(72, 1, 32, 8, 2048, 128, 64, oracle.MOD_SLIDING_WINDOW, ModParams(window=16))):
        (o1, l1, g1), (o2, l2, g2) = run_both(ta, c)
        assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
        O, L = c.oracle_fwd()
        check_o(host_f64(o2), O)
        check_grads([host_f64(t) for t in g2], c.oracle_bwd(), "clc, units without work")


def test_deterministic_dq_under_cluster_launch_control(ta):
    """The deterministic backward takes the static walk whatever walk is set
    (its ordered adds need every lower-ranked unit started), so with cluster
    launch control selected dQ is still bitwise the same on every run, and
    equal to the static walk's."""
    from test_gpu_deterministic import run_det, same_bits
    c = Case(73, 4, 8, 4, 2048, 2048, 128, oracle.MOD_CAUSAL)
    ta.attn_set_work_walk(ta.WALK_STATIC)
    try:
        a = run_det(ta, c)
        ta.attn_set_work_walk(ta.WALK_CLUSTER_LAUNCH_CONTROL)
        b = run_det(ta, c)
        d = run_det(ta, c)
    finally:
        ta.attn_set_work_walk(ta.WALK_DEFAULT)
    assert same_bits(a, b) and same_bits(b, d)
