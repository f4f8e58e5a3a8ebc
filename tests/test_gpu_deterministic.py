"""The backward pass with a bitwise reproducible dQ (attn_bwd_deterministic)
on the sm_100a kernels: every gradient is identical bit for bit across runs
and within the tolerances of the fp64 oracle, with and without a block mask,
for masks whose key tiles meet a query tile in different patterns."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import Case, host_f64, rel_l2
from test_gpu_backward import check_grads, small_params

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ta():
    import tiled_attention_25_b200 as m
    return m


def run_det(ta, c, use_mask=True, fill=0x7F):
    mask = ta.new_block_mask(c.mod, c.dev_params, c.B, c.Sq, c.Skv) if use_mask else None
    out = torch.empty_like(c.q)
    lse = torch.empty(c.B, c.Hq, c.Sq, dtype=torch.float32, device="cuda")
    ta.attn_fwd(c.q, c.k, c.v, out, lse, scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params, block_mask=mask)
    ws = ta.new_bwd_workspace(c.B, c.Hq, c.Sq, c.D, deterministic=True)
    ws.fill_(fill)  # contents on entry must not matter
    dq, dk, dv = torch.empty_like(c.q), torch.empty_like(c.k), torch.empty_like(c.v)
    ta.attn_bwd_deterministic(c.q, c.k, c.v, out, lse, c.dout, dq, dk, dv, ws, scale=c.scale, mod_kind=c.mod,
                              mod_params=c.dev_params, block_mask=mask)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    return dq, dk, dv


def same_bits(a, b):
    return all(torch.equal(x.view(torch.int16), y.view(torch.int16)) for x, y in zip(a, b))


@pytest.mark.parametrize("mod", [oracle.MOD_NONE, oracle.MOD_CAUSAL, oracle.MOD_SLIDING_WINDOW,
                                 oracle.MOD_DOCUMENT, oracle.MOD_SOFTCAP])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("use_mask", [False, True])
def test_deterministic_repeats_and_matches_oracle(ta, mod, D, use_mask):
    S = 700  # six key tiles, a ragged tail
    p = small_params(mod, S)
    if p.doc_offsets is not None:  # one list of documents per batch row
        p.doc_offsets = [p.doc_offsets[0], [0, 100, 555, S]]
    c = Case(90 + mod + D, 2, 4, 2, S, S, D, mod, p)
    a = run_det(ta, c, use_mask, fill=0x7F)
    b = run_det(ta, c, use_mask, fill=0x00)
    assert same_bits(a, b)
    check_grads([host_f64(t) for t in a], c.oracle_bwd(), f"deterministic mod {mod} D {D}")


def test_deterministic_many_units_per_cta(ta):
    """More key-tile units than SMs (each CTA runs several, in ascending rank)
    and many key tiles per query tile, under GQA: bitwise repeatable, and
    equal to the atomic-order backward within rounding."""
    c = Case(95, 4, 8, 4, 2048, 2048, 128, oracle.MOD_NONE)  # 256 units
    a = run_det(ta, c, use_mask=True)
    b = run_det(ta, c, use_mask=True)
    assert same_bits(a, b)
    from test_gpu_backward import run_fwd_bwd
    ref = run_fwd_bwd(ta, c)
    assert torch.equal(a[1].view(torch.int16), ref[1].view(torch.int16))  # dK, dV: same order as attn_bwd
    assert torch.equal(a[2].view(torch.int16), ref[2].view(torch.int16))
    assert rel_l2(host_f64(a[0]), host_f64(ref[0])) < 1e-2
    rows = np.array([0, 1, 127, 128, 1000, 2046, 2047])
    exact = c.oracle_bwd(groups=[(3, 1)], q_rows=rows, kv_rows=rows)
    for got, ref_, sel in ((a[0], exact[0], (3, slice(2, 4))), (a[1], exact[1], (3, 1)), (a[2], exact[2], (3, 1))):
        g = host_f64(got)[sel][..., rows, :]
        r = ref_[sel][..., rows, :]
        assert rel_l2(g, r) <= 1e-2


def test_deterministic_unequal_lengths_and_documents(ta):
    for Sq, Skv, mod in ((333, 130, oracle.MOD_CAUSAL), (130, 600, oracle.MOD_NONE), (640, 640, oracle.MOD_DOCUMENT)):
        c = Case(96, 1, 3, 1, Sq, Skv, 64, mod, small_params(mod, Sq) if mod == oracle.MOD_DOCUMENT else None)
        a = run_det(ta, c)
        b = run_det(ta, c)
        assert same_bits(a, b)
        check_grads([host_f64(t) for t in a], c.oracle_bwd(), f"deterministic {Sq}x{Skv} mod {mod}")
