"""The general (bitmap) mask on the sm_100a kernels against the fp64 oracle,
through the C ABI: forward O/LSE, backward dQ/dK/dV and the block mask, for
shared, per-batch-row and per-head bitmaps, alone and ANDed with other mods."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import Case, check_lse, check_o, host_f64
from oracle import (MASK_BITMAP, MASK_CAUSAL, MASK_DOCUMENT, MASK_SLIDING_WINDOW, MOD_ALIBI, MOD_CAUSAL,
                    MOD_LOCAL_BOOST, MOD_NONE, MOD_SOFTCAP)
from synth_inputs import ModParams, pack_bitmap
from test_gpu_backward import check_grads, run_fwd_bwd
from test_gpu_forward import run_fwd

pytestmark = pytest.mark.gpu

MODS = [MOD_NONE | MASK_BITMAP, MOD_ALIBI | MASK_BITMAP | MASK_CAUSAL, MOD_SOFTCAP | MASK_BITMAP,
        MOD_LOCAL_BOOST | MASK_BITMAP | MASK_SLIDING_WINDOW, MOD_NONE | MASK_BITMAP | MASK_DOCUMENT]


@pytest.fixture(scope="module")
def ta():
    import tiled_attention_25_b200 as m
    return m


def tiled_bitmap(nb, nh, Sq, Skv, seed):
    """Per 128x128 tile: all dropped, all kept, or random bits (density 0.3 to 0.9);
    the diagonal stays kept so that most rows keep a key."""
    rng = np.random.default_rng(seed)
    keep = np.zeros((nb, nh, Sq, Skv), dtype=bool)
    for b in range(nb):
        for h in range(nh):
            for q0 in range(0, Sq, 128):
                for k0 in range(0, Skv, 128):
                    kind = rng.integers(3)
                    blk = keep[b, h, q0:q0 + 128, k0:k0 + 128]
                    if kind == 1:
                        blk[...] = True
                    elif kind == 2:
                        blk[...] = rng.random(blk.shape) < rng.uniform(0.3, 0.9)
    d = np.arange(min(Sq, Skv))
    keep[:, :, d, d] = True
    return keep


def params(bitmap, S, window=200):
    cut = sorted(set([0, S // 5, S // 2, S // 2 + 1, (9 * S) // 10, S]))
    return ModParams(softcap=20.0, window=window, boost=1.3, boost_radius=96, doc_offsets=[cut, [0, S]],
                     bitmap=bitmap)


@pytest.mark.parametrize("mod", MODS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("shape", ["shared", "per_batch", "per_head"])
def test_forward_and_backward(ta, mod, D, shape):
    S, B, Hq, Hkv = 600, 2, 4, 2
    nb, nh = {"shared": (1, 1), "per_batch": (B, 1), "per_head": (B, Hq)}[shape]
    bm = tiled_bitmap(nb, nh, S, S, 800 + D + nh)
    c = Case(810 + (mod & 0xFF) + (mod >> 8), B, Hq, Hkv, S, S, D, mod, params(bm, S))
    out, lse = run_fwd(ta, c, use_mask=True)
    O, L = c.oracle_fwd()
    check_o(host_f64(out), O, f"{mod:#x} {shape} D {D}")
    check_lse(lse.cpu().double().numpy(), L, f"{mod:#x} {shape} D {D}")
    got = [host_f64(t) for t in run_fwd_bwd(ta, c, use_mask=True)]
    check_grads(got, c.oracle_bwd(), f"{mod:#x} {shape} D {D}")


@pytest.mark.parametrize("S", [1, 129, 600])
@pytest.mark.parametrize("shape", [(1, 1), (2, 1), (2, 3)])
def test_block_mask(ta, S, shape):
    nb, nh = shape
    bm = tiled_bitmap(nb, nh, S, S, 900 + S)
    for mod in (MOD_NONE | MASK_BITMAP, MOD_NONE | MASK_BITMAP | MASK_CAUSAL | MASK_SLIDING_WINDOW):
        p = params(bm, S, window=max(1, S // 3))
        dp = ta.ModParams(window=p.window, bitmap=torch.from_numpy(pack_bitmap(bm)).cuda())
        mask = ta.new_block_mask(mod, dp, 2, S, S)
        torch.cuda.synchronize()
        ref = oracle.block_mask(mod, p, 2, S, S)
        for name, arr in ref.items():
            assert np.array_equal(mask.view(name).cpu().numpy(), arr), f"{name} {mod:#x} {shape} S={S}"


def test_lower_triangle_bitmap_is_bit_identical_to_causal(ta):
    S = 700
    i, j = np.arange(S)[:, None], np.arange(S)[None, :]
    tril = np.broadcast_to(j <= i, (1, 1, S, S)).copy()
    c1 = Case(950, 1, 4, 4, S, S, 128, MOD_CAUSAL)
    c2 = Case(950, 1, 4, 4, S, S, 128, MOD_NONE | MASK_BITMAP, ModParams(bitmap=tril))
    o1, l1 = run_fwd(ta, c1, use_mask=True)
    o2, l2 = run_fwd(ta, c2, use_mask=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bitmap_needs_a_block_mask(ta):
    S = 256
    c = Case(960, 1, 2, 2, S, S, 64, MOD_NONE | MASK_BITMAP, ModParams(bitmap=np.ones((1, 1, S, S), bool)))
    out = torch.empty_like(c.q)
    with pytest.raises(ta.AttnError):
        ta.attn_fwd(c.q, c.k, c.v, out, None, scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params)


def test_long_sequence_sampled_rows(ta):
    from gpu_common import sample_rows
    S, Hq, Hkv = 4096, 8, 2
    bm = tiled_bitmap(1, Hq, S, S, 970)
    c = Case(971, 1, Hq, Hkv, S, S, 128, MOD_ALIBI | MASK_BITMAP, ModParams(bitmap=bm))
    out, lse = run_fwd(ta, c, use_mask=True)
    rows = sample_rows(S, 40, 9)
    heads = [(0, 0), (0, 3), (0, 7)]
    O, L = c.oracle_fwd(heads=heads, rows=rows)
    og = np.full(O.shape, np.nan)
    lg = np.full(L.shape, np.nan)
    ridx = torch.from_numpy(rows).cuda()
    for b, h in heads:
        og[b, h, rows] = out[b, h].index_select(0, ridx).float().cpu().double().numpy()
        lg[b, h, rows] = lse[b, h].index_select(0, ridx).cpu().double().numpy()
    check_o(og, O, "alibi|bitmap 4096")
    check_lse(lg, L, "alibi|bitmap 4096")
