"""Composed mods on the sm_100a kernels (a score mod plus the AND of masks)
against the fp64 oracle, through the C ABI: forward O/LSE, backward dQ/dK/dV
and the block mask, with and without a block mask, on sizes that span several
tiles with a ragged tail and that leave EMPTY, PARTIAL and FULL tiles."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import Case, check_lse, check_o, host_f64, sample_rows
from oracle import (MASK_CAUSAL, MASK_DOCUMENT, MASK_SLIDING_WINDOW, MOD_ALIBI, MOD_CAUSAL,
                    MOD_DOCUMENT, MOD_LOCAL_BOOST, MOD_NONE, MOD_SLIDING_WINDOW, MOD_SOFTCAP)
from synth_inputs import ModParams
from test_gpu_backward import check_grads, run_fwd_bwd
from test_gpu_block_mask import compare as compare_mask
from test_gpu_forward import run_fwd

pytestmark = pytest.mark.gpu

COMPOSED = [
    MOD_ALIBI | MASK_CAUSAL,
    MOD_SOFTCAP | MASK_CAUSAL,
    MOD_LOCAL_BOOST | MASK_SLIDING_WINDOW,
    MOD_SOFTCAP | MASK_SLIDING_WINDOW,
    MOD_ALIBI | MASK_DOCUMENT,
    MOD_SLIDING_WINDOW | MASK_DOCUMENT,
    MOD_LOCAL_BOOST | MASK_SLIDING_WINDOW | MASK_DOCUMENT,
    MOD_NONE | MASK_CAUSAL,
]


@pytest.fixture(scope="module")
def ta():
    import tiled_attention_25_b200 as m
    return m


def params(S, B=1, window=200):
    cut = sorted(set([0, S // 5, S // 2, S // 2 + 1, (9 * S) // 10, S]))
    return ModParams(softcap=20.0, window=window, boost=1.3, boost_radius=96,
                     doc_offsets=[cut] * B if B == 1 else [cut, [0, S]] + [cut] * (B - 2))


@pytest.mark.parametrize("mod", COMPOSED)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("use_mask", [False, True])
def test_forward(ta, mod, D, use_mask):
    S = 600
    c = Case(300 + (mod & 0xFF) + (mod >> 8), 2, 4, 2, S, S, D, mod, params(S, B=2))
    out, lse = run_fwd(ta, c, use_mask=use_mask)
    O, L = c.oracle_fwd()
    check_o(host_f64(out), O, f"mod {mod:#x} D {D}")
    check_lse(lse.cpu().double().numpy(), L, f"mod {mod:#x} D {D}")


@pytest.mark.parametrize("mod", COMPOSED)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("use_mask", [False, True])
def test_backward(ta, mod, D, use_mask):
    S = 600
    c = Case(400 + (mod & 0xFF) + (mod >> 8), 2, 4, 2, S, S, D, mod, params(S, B=2))
    got = [host_f64(t) for t in run_fwd_bwd(ta, c, use_mask)]
    check_grads(got, c.oracle_bwd(), f"mod {mod:#x} D {D}")


@pytest.mark.parametrize("mod", [MOD_SLIDING_WINDOW | MASK_DOCUMENT, MOD_ALIBI | MASK_CAUSAL,
                                 MOD_NONE | MASK_SLIDING_WINDOW | MASK_DOCUMENT])
@pytest.mark.parametrize("S", [129, 600, 2000])
def test_block_mask(ta, mod, S):
    compare_mask(ta, mod, params(S, B=2, window=max(1, S // 4)), 2, S, S)


def test_equivalent_codes_share_a_block_mask(ta):
    # a mask built for one spelling of a mod serves every spelling of it
    S = 520
    c = Case(500, 1, 2, 1, S, S, 128, MOD_SLIDING_WINDOW | MASK_DOCUMENT, params(S))
    mask = ta.new_block_mask(MOD_DOCUMENT | MASK_SLIDING_WINDOW | MASK_CAUSAL, c.dev_params, 1, S, S)
    out = torch.empty_like(c.q)
    lse = torch.empty(1, 2, S, dtype=torch.float32, device="cuda")
    ta.attn_fwd(c.q, c.k, c.v, out, lse, scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params,
                block_mask=mask)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    O, L = c.oracle_fwd()
    check_o(host_f64(out), O, "window|document")
    check_lse(lse.cpu().double().numpy(), L, "window|document")
    # a mask built for another mod is refused
    other = ta.new_block_mask(MOD_DOCUMENT, c.dev_params, 1, S, S)
    with pytest.raises(ta.AttnError):
        ta.attn_fwd(c.q, c.k, c.v, out, lse, scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params,
                    block_mask=other)


def test_single_kind_aliases_are_bit_identical(ta):
    # a kind spelled as flags runs the same kernel on the same tiles
    S = 700
    for kind, alias in ((MOD_CAUSAL, MOD_NONE | MASK_CAUSAL), (MOD_SLIDING_WINDOW, MOD_CAUSAL | MASK_SLIDING_WINDOW),
                        (MOD_DOCUMENT, MOD_CAUSAL | MASK_DOCUMENT)):
        c1 = Case(600, 1, 4, 4, S, S, 128, kind, params(S))
        c2 = Case(600, 1, 4, 4, S, S, 128, alias, params(S))
        o1, l1 = run_fwd(ta, c1, use_mask=True)
        o2, l2 = run_fwd(ta, c2, use_mask=True)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("mod", [MOD_ALIBI | MASK_CAUSAL, MOD_SLIDING_WINDOW | MASK_DOCUMENT])
def test_long_sequence_sampled_rows(ta, mod):
    # 8192 keys, GQA 16/4, block mask on: sampled rows against the oracle
    S = 8192
    offs = [0, 1000, 1001, 3500, 4096, 7000, S]
    c = Case(700 + (mod & 0xFF), 1, 16, 4, S, S, 128, mod,
             ModParams(window=1024, doc_offsets=[offs]))
    out, lse = run_fwd(ta, c, use_mask=True)
    rows = sample_rows(S, 40, 7, extra=[o + d for o in offs[1:-1] for d in (-1, 0, 1)])
    heads = [(0, 0), (0, 5), (0, 15)]
    O, L = c.oracle_fwd(heads=heads, rows=rows)
    og = np.full(O.shape, np.nan)
    lg = np.full(L.shape, np.nan)
    ridx = torch.from_numpy(rows).cuda()
    for b, h in heads:
        og[b, h, rows] = out[b, h].index_select(0, ridx).float().cpu().double().numpy()
        lg[b, h, rows] = lse[b, h].index_select(0, ridx).cpu().double().numpy()
    check_o(og, O, f"{mod:#x}")
    check_lse(lg, L, f"{mod:#x}")
