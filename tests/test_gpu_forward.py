"""Forward parity of the sm_100a kernel against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import Case, check_lse, check_o, host_f64, sample_rows
from synth_inputs import ModParams, WORKLOADS, doc_lengths, mod_params_for, offsets_from_lengths

pytestmark = pytest.mark.gpu

ALL = [oracle.MOD_NONE, oracle.MOD_CAUSAL, oracle.MOD_ALIBI, oracle.MOD_SOFTCAP,
       oracle.MOD_SLIDING_WINDOW, oracle.MOD_LOCAL_BOOST, oracle.MOD_DOCUMENT]


@pytest.fixture(scope="module")
def ta():
    import tiled_attention_25_b200 as m
    assert torch.cuda.is_available()
    return m


def run_fwd(ta, c, with_lse=True, use_mask=False):
    out = torch.empty_like(c.q)
    lse = torch.empty(c.B, c.Hq, c.Sq, dtype=torch.float32, device="cuda") if with_lse else None
    mask = None
    if use_mask:
        mask = ta.new_block_mask(c.mod, c.dev_params, c.B, c.Sq, c.Skv)
    ta.attn_fwd(c.q, c.k, c.v, out, lse, scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params,
                block_mask=mask)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    return out, lse


def small_params(mod, S):
    p = ModParams(softcap=50.0, window=min(1024, max(3, S // 3)), boost=1.1, boost_radius=min(128, max(2, S // 5)))
    if mod == oracle.MOD_DOCUMENT:
        cut = [0, S // 3, S // 3 + 1, (2 * S) // 3, S] if S >= 8 else [0, S]
        p.doc_offsets = [sorted(set(cut))]
    return p


def test_tiny_workload_full(ta):
    w = WORKLOADS["tiny"]
    c = Case(w.seed, w.B, w.Hq, w.Hkv, w.Sq, w.Skv, w.D, oracle.MOD_NONE)
    out, lse = run_fwd(ta, c)
    O, L = c.oracle_fwd()
    check_o(host_f64(out), O, "tiny")
    check_lse(lse.cpu().double().numpy(), L, "tiny")


@pytest.mark.parametrize("mod", ALL)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("use_mask", [False, True])
def test_mods_ragged(ta, mod, D, use_mask):
    S = 300  # three query tiles, a ragged tail, an odd number of tiles
    c = Case(11 + mod, 1, 4, 2, S, S, D, mod, small_params(mod, S))
    out, lse = run_fwd(ta, c, use_mask=use_mask)
    O, L = c.oracle_fwd()
    check_o(host_f64(out), O, f"mod {mod}")
    check_lse(lse.cpu().double().numpy(), L, f"mod {mod}")


@pytest.mark.parametrize("S", [1, 17, 128, 129, 255, 256, 511])
def test_sizes_causal_and_dense(ta, S):
    for mod in (oracle.MOD_NONE, oracle.MOD_CAUSAL):
        c = Case(100 + S, 2, 2, 2, S, S, 128, mod)
        out, lse = run_fwd(ta, c, use_mask=(mod == oracle.MOD_CAUSAL))
        O, L = c.oracle_fwd()
        check_o(host_f64(out), O, f"S={S}")
        check_lse(lse.cpu().double().numpy(), L, f"S={S}")


@pytest.mark.parametrize("Sq,Skv", [(130, 333), (333, 130), (64, 1000)])
def test_unequal_lengths(ta, Sq, Skv):
    for mod in (oracle.MOD_NONE, oracle.MOD_CAUSAL, oracle.MOD_ALIBI):
        c = Case(7, 1, 3, 1, Sq, Skv, 64, mod)
        out, lse = run_fwd(ta, c)
        O, L = c.oracle_fwd()
        check_o(host_f64(out), O, f"{Sq}x{Skv} mod {mod}")
        check_lse(lse.cpu().double().numpy(), L)


def test_fully_masked_rows_give_zero(ta):
    # window 2 with Sq > Skv: the last rows see no key at all
    c = Case(8, 1, 2, 2, 200, 100, 64, oracle.MOD_SLIDING_WINDOW, ModParams(window=2))
    out, lse = run_fwd(ta, c)
    O, L = c.oracle_fwd()
    check_o(host_f64(out), O)
    got = lse.cpu().double().numpy()
    assert np.isneginf(got[:, :, 150:]).all()
    check_lse(got, L)


def test_units_without_key_tiles(ta):
    # window 16 with Sq >> Skv: every query-tile pair past the first keeps no
    # key, and with more units than SMs a CTA runs several such units in a row
    c = Case(13, 1, 32, 8, 2048, 128, 64, oracle.MOD_SLIDING_WINDOW, ModParams(window=16))
    for use_mask in (False, True):
        out, lse = run_fwd(ta, c, use_mask=use_mask)
        O, L = c.oracle_fwd()
        check_o(host_f64(out), O, f"mask={use_mask}")
        got = lse.cpu().double().numpy()
        assert np.isneginf(got[:, :, 143:]).all()
        check_lse(got, L)


def test_gqa_and_mqa(ta):
    for Hq, Hkv in ((8, 2), (4, 1)):
        c = Case(9, 2, Hq, Hkv, 384, 384, 128, oracle.MOD_CAUSAL)
        out, lse = run_fwd(ta, c, use_mask=True)
        O, L = c.oracle_fwd()
        check_o(host_f64(out), O, f"{Hq}/{Hkv}")
        check_lse(lse.cpu().double().numpy(), L)


@pytest.mark.parametrize("mod", [oracle.MOD_NONE, oracle.MOD_CAUSAL])
def test_out_only_is_bit_identical(ta, mod):
    c = Case(10, 2, 4, 4, 640, 640, 128, mod)
    a, _ = run_fwd(ta, c, with_lse=True, use_mask=True)
    b, _ = run_fwd(ta, c, with_lse=False, use_mask=True)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_mask_and_dense_iteration_agree(ta):
    c = Case(12, 1, 2, 2, 1000, 1000, 128, oracle.MOD_SLIDING_WINDOW, ModParams(window=200))
    a, la = run_fwd(ta, c, use_mask=True)
    b, lb = run_fwd(ta, c, use_mask=False)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(la, lb)


# ------------------------------------------------------------ full-size workloads

def _workload_case(name, mod_name):
    w = WORKLOADS[name]
    mod = {"none": oracle.MOD_NONE, "causal": oracle.MOD_CAUSAL, "alibi": oracle.MOD_ALIBI,
           "softcap": oracle.MOD_SOFTCAP, "sliding_window": oracle.MOD_SLIDING_WINDOW,
           "local_boost": oracle.MOD_LOCAL_BOOST, "document": oracle.MOD_DOCUMENT}[mod_name]
    return w, Case(w.seed, w.B, w.Hq, w.Hkv, w.Sq, w.Skv, w.D, mod, mod_params_for(w, mod_name))


@pytest.mark.parametrize("name,mod_name", [("dense", "none"), ("dense", "causal"), ("gqa_long", "causal"),
                                           ("score_mods", "alibi"), ("score_mods", "softcap"),
                                           ("score_mods", "sliding_window"), ("score_mods", "local_boost"),
                                           ("documents", "document")])
def test_workload_sampled_rows(ta, name, mod_name):
    w, c = _workload_case(name, mod_name)
    out, lse = run_fwd(ta, c, use_mask=True)
    extra = []
    if c.p.doc_offsets is not None:
        for o in c.p.doc_offsets[0][1:-1][:6]:
            extra += [o - 1, o, o + 1]
    rows = sample_rows(w.Sq, 48, w.seed, extra)
    heads = [(w.B - 1, 0), (0, w.Hq - 1)] + [(b, h) for b in range(w.B) for h in range(w.Hq)][1::7]
    O, L = c.oracle_fwd(heads=heads, rows=rows)
    og = np.full(O.shape, np.nan)
    lg = np.full(L.shape, np.nan)
    ridx = torch.from_numpy(rows).cuda()
    for b, h in heads:
        og[b, h, rows] = out[b, h].index_select(0, ridx).float().cpu().double().numpy()
        lg[b, h, rows] = lse[b, h].index_select(0, ridx).cpu().double().numpy()
    check_o(og, O, name)
    check_lse(lg, L, name)


@pytest.mark.parametrize("mod_name", ["none", "causal"])
def test_dense_out_only_sampled_rows(ta, mod_name):
    """The forward without the LSE output (its own kernel variant) at the
    dense 4x8x4096x128 size, against the oracle on sampled rows of several
    heads."""
    w, c = _workload_case("dense", mod_name)
    out, lse = run_fwd(ta, c, with_lse=False, use_mask=True)
    assert lse is None
    rows = sample_rows(w.Sq, 48, 77)
    heads = [(0, 0), (w.B - 1, w.Hq - 1), (1, 3), (2, 6)]
    O, _ = c.oracle_fwd(heads=heads, rows=rows)
    og = np.full(O.shape, np.nan)
    ridx = torch.from_numpy(rows).cuda()
    for b, h in heads:
        og[b, h, rows] = out[b, h].index_select(0, ridx).float().cpu().double().numpy()
    check_o(og, O, f"dense:{mod_name} without LSE")
