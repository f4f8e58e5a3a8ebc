"""Backward parity of the sm_100a kernels against the fp64 oracle (through the C ABI)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import GRAD_REL_L2, Case, host_f64, rel_l2, sample_rows
from synth_inputs import ModParams, WORKLOADS, mod_params_for

pytestmark = pytest.mark.gpu

ALL = [oracle.MOD_NONE, oracle.MOD_CAUSAL, oracle.MOD_ALIBI, oracle.MOD_SOFTCAP,
       oracle.MOD_SLIDING_WINDOW, oracle.MOD_LOCAL_BOOST, oracle.MOD_DOCUMENT]


@pytest.fixture(scope="module")
def ta():
    import tiled_attention_25_b200 as m
    return m


def run_fwd_bwd(ta, c, use_mask=True):
    mask = ta.new_block_mask(c.mod, c.dev_params, c.B, c.Sq, c.Skv) if use_mask else None
    out = torch.empty_like(c.q)
    lse = torch.empty(c.B, c.Hq, c.Sq, dtype=torch.float32, device="cuda")
    ta.attn_fwd(c.q, c.k, c.v, out, lse, scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params, block_mask=mask)
    dq, dk, dv = torch.empty_like(c.q), torch.empty_like(c.k), torch.empty_like(c.v)
    ws = ta.new_bwd_workspace(c.B, c.Hq, c.Sq, c.D)
    ws.fill_(0x7F)  # contents on entry must not matter
    ta.attn_bwd(c.q, c.k, c.v, out, lse, c.dout, dq, dk, dv, ws, scale=c.scale, mod_kind=c.mod,
                mod_params=c.dev_params, block_mask=mask)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    return dq, dk, dv


def check_grads(got, ref, what):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        sel = ~np.isnan(r)
        ref_rms = float(np.sqrt(np.mean(r[sel] ** 2)))
        if ref_rms < 1e-9:
            # the exact gradient vanishes (e.g. one key: softmax is constant), so a
            # relative error is undefined; bound the absolute RMS instead
            err = float(np.sqrt(np.mean((g[sel] - r[sel]) ** 2)))
            assert err <= 1e-4, f"{what} {name} abs-RMS {err:.3e} (zero reference)"
            continue
        e = rel_l2(g, r)
        assert e <= GRAD_REL_L2, f"{what} {name} rel-L2 {e:.3e}"


def small_params(mod, S):
    p = ModParams(softcap=50.0, window=max(3, S // 3), boost=1.1, boost_radius=max(2, S // 5))
    if mod == oracle.MOD_DOCUMENT:
        p.doc_offsets = [sorted(set([0, S // 3, S // 3 + 1, (2 * S) // 3, S]))]
    return p


def test_tiny_workload_full(ta):
    w = WORKLOADS["tiny"]
    c = Case(w.seed, w.B, w.Hq, w.Hkv, w.Sq, w.Skv, w.D, oracle.MOD_NONE)
    got = [host_f64(t) for t in run_fwd_bwd(ta, c, use_mask=False)]
    check_grads(got, c.oracle_bwd(), "tiny")


@pytest.mark.parametrize("mod", ALL)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("use_mask", [False, True])
def test_mods_ragged(ta, mod, D, use_mask):
    S = 300
    c = Case(21 + mod, 1, 4, 2, S, S, D, mod, small_params(mod, S))
    got = [host_f64(t) for t in run_fwd_bwd(ta, c, use_mask)]
    check_grads(got, c.oracle_bwd(), f"mod {mod} D {D}")


@pytest.mark.parametrize("S", [1, 17, 64, 65, 128, 129, 255, 511])
def test_sizes(ta, S):
    for mod in (oracle.MOD_NONE, oracle.MOD_CAUSAL):
        c = Case(200 + S, 2, 2, 1, S, S, 128, mod)
        got = [host_f64(t) for t in run_fwd_bwd(ta, c)]
        check_grads(got, c.oracle_bwd(), f"S={S} mod {mod}")


@pytest.mark.parametrize("Sq,Skv", [(130, 333), (333, 130), (64, 1000)])
def test_unequal_lengths(ta, Sq, Skv):
    for mod in (oracle.MOD_NONE, oracle.MOD_CAUSAL, oracle.MOD_ALIBI):
        c = Case(31, 1, 3, 1, Sq, Skv, 64, mod)
        got = [host_f64(t) for t in run_fwd_bwd(ta, c)]
        check_grads(got, c.oracle_bwd(), f"{Sq}x{Skv} mod {mod}")


def test_key_tiles_without_queries(ta):
    # causal with Skv >> Sq: key tiles past the first meet no query, and with
    # more units than SMs a CTA runs several such units in a row
    c = Case(34, 1, 32, 32, 128, 2048, 64, oracle.MOD_CAUSAL)
    for use_mask in (False, True):
        got = [host_f64(t) for t in run_fwd_bwd(ta, c, use_mask=use_mask)]
        dk, dv = got[1], got[2]
        assert not dk[:, :, 128:].any() and not dv[:, :, 128:].any()
        check_grads(got, c.oracle_bwd(), f"mask={use_mask}")


def test_gqa_mqa(ta):
    for Hq, Hkv in ((8, 2), (4, 1)):
        c = Case(32, 2, Hq, Hkv, 384, 384, 128, oracle.MOD_CAUSAL)
        got = [host_f64(t) for t in run_fwd_bwd(ta, c)]
        check_grads(got, c.oracle_bwd(), f"{Hq}/{Hkv}")


def test_repeat_runs_agree(ta):
    c = Case(33, 1, 4, 4, 512, 512, 128, oracle.MOD_CAUSAL)
    a = run_fwd_bwd(ta, c)
    b = run_fwd_bwd(ta, c)
    # dK, dV have a fixed summation order; dQ is added atomically (order may vary)
    assert torch.equal(a[1].view(torch.int16), b[1].view(torch.int16))
    assert torch.equal(a[2].view(torch.int16), b[2].view(torch.int16))
    assert rel_l2(host_f64(a[0]), host_f64(b[0])) < 1e-2


# ------------------------------------------------------------ full-size workloads

def _case(name, mod_name):
    w = WORKLOADS[name]
    mod = {"none": oracle.MOD_NONE, "causal": oracle.MOD_CAUSAL, "alibi": oracle.MOD_ALIBI,
           "softcap": oracle.MOD_SOFTCAP, "sliding_window": oracle.MOD_SLIDING_WINDOW,
           "local_boost": oracle.MOD_LOCAL_BOOST, "document": oracle.MOD_DOCUMENT}[mod_name]
    return w, Case(w.seed, w.B, w.Hq, w.Hkv, w.Sq, w.Skv, w.D, mod, mod_params_for(w, mod_name))


def _gather(t, b, h, rows):
    return t[b, h].index_select(0, torch.from_numpy(rows).cuda()).float().cpu().double().numpy()


@pytest.mark.parametrize("name,mod_name", [("dense", "none"), ("dense", "causal"), ("score_mods", "alibi"),
                                           ("score_mods", "softcap"), ("score_mods", "sliding_window"),
                                           ("score_mods", "local_boost")])
def test_workload_groups(ta, name, mod_name):
    """Whole KV-head groups: every row of dQ, dK, dV of two groups."""
    w, c = _case(name, mod_name)
    dq, dk, dv = run_fwd_bwd(ta, c)
    groups = [(0, 0), (w.B - 1, w.Hkv - 1)]
    ref = c.oracle_bwd(groups=groups)
    G = w.Hq // w.Hkv
    for b, hk in groups:
        rows = np.arange(w.Sq)
        got_q = np.stack([_gather(dq, b, h, rows) for h in range(hk * G, hk * G + G)])
        e = rel_l2(got_q, ref[0][b, hk * G:hk * G + G])
        assert e <= GRAD_REL_L2, f"{name} dq {e:.3e}"
        for t, r, nm in ((dk, ref[1], "dk"), (dv, ref[2], "dv")):
            e = rel_l2(_gather(t, b, hk, np.arange(w.Skv)), r[b, hk])
            assert e <= GRAD_REL_L2, f"{name} {nm} {e:.3e}"


def test_gqa_long_sampled(ta):
    """32K causal GQA: dQ on sampled rows (each needs only its own row); dK/dV
    of the last two key tiles, which only the last 256 queries see; and dK/dV
    of a middle key tile [16384, 16512) and an early-middle one [8192, 8320),
    which accumulate over thousands of query tiles of all four heads of the
    group.  Causality makes every query before a key's own position
    contribute exactly zero to it, so the oracle sums only the rows from the
    earliest requested key on."""
    w, c = _case("gqa_long", "causal")
    dq, dk, dv = run_fwd_bwd(ta, c)
    G = w.Hq // w.Hkv
    hk = w.Hkv - 1
    tail = np.arange(w.Skv - 256, w.Skv)
    rows = sample_rows(w.Sq, 24, 5)
    ref_q = c.oracle_bwd(groups=[(0, hk)], q_rows=rows, kv_rows=tail[:1], contrib_rows=rows)[0]
    ref_kv = c.oracle_bwd(groups=[(0, hk)], q_rows=tail[-1:], kv_rows=tail, contrib_rows=tail)
    got_q = np.stack([_gather(dq, 0, h, rows) for h in range(hk * G, hk * G + G)])
    assert rel_l2(got_q, ref_q[0, hk * G:hk * G + G][:, rows]) <= GRAD_REL_L2
    assert rel_l2(_gather(dk, 0, hk, tail), ref_kv[1][0, hk, tail]) <= GRAD_REL_L2
    assert rel_l2(_gather(dv, 0, hk, tail), ref_kv[2][0, hk, tail]) <= GRAD_REL_L2
    # interior key tiles, in another KV group
    hk = 2
    mid = np.concatenate([np.arange(8192, 8320), np.arange(16384, 16512)])
    ref_mid = c.oracle_bwd(groups=[(0, hk)], q_rows=mid[-1:], kv_rows=mid,
                           contrib_rows=np.arange(int(mid[0]), w.Sq))
    for lo in (0, 128):
        keys = mid[lo:lo + 128]
        for t, r, nm in ((dk, ref_mid[1], "dk"), (dv, ref_mid[2], "dv")):
            e = rel_l2(_gather(t, 0, hk, keys), r[0, hk, keys])
            assert e <= GRAD_REL_L2, f"keys [{keys[0]}, {keys[-1] + 1}) {nm} {e:.3e}"


def test_documents_sampled_docs(ta):
    """Packed documents: each document is an independent causal problem, so the
    oracle runs on whole documents cut out of the packed sequence: the first,
    a mid-sequence and the last document, in three heads."""
    w, c = _case("documents", "document")
    dq, dk, dv = run_fwd_bwd(ta, c)
    offs = c.p.doc_offsets[0]
    n_docs = len(offs) - 1
    for d in (0, n_docs // 2, n_docs - 1):
        a, b = offs[d], offs[d + 1]
        sub = [x[:, :, a:b] for x in (c.qf, c.kf, c.vf, c.doutf)]
        heads = (3, 8, 15)
        ref = oracle.attention_backward(*sub, c.scale, oracle.MOD_CAUSAL, groups=[(0, h) for h in heads])
        rows = np.arange(a, b)
        for h in heads:
            for t, r, nm in ((dq, ref[0], "dq"), (dk, ref[1], "dk"), (dv, ref[2], "dv")):
                got = _gather(t, 0, h, rows)
                e = rel_l2(got, r[0, h])
                assert e <= GRAD_REL_L2, f"doc {d} head {h} {nm} {e:.3e}"


@pytest.mark.parametrize("D", [64, 128])
def test_alibi_with_given_slopes(ta, D):
    """The caller's ALiBi slopes (attn_mod_params.alibi_slopes), distinct per
    query head, under GQA (query head h reads slope h, KV head h // G) and an
    odd length."""
    S, Hq, Hkv = 301, 8, 2
    slopes = [0.5, 0.05, 0.002, 1.3, 0.25, 0.011, 0.8, 0.0]
    c = Case(180 + D, 2, Hq, Hkv, S, S, D, oracle.MOD_ALIBI, ModParams(alibi_slopes=slopes))
    c.dev_params.alibi_slopes = torch.tensor(slopes, dtype=torch.float32, device="cuda")
    from gpu_common import check_lse, check_o
    for use_mask in (False, True):
        mask = ta.new_block_mask(c.mod, c.dev_params, c.B, c.Sq, c.Skv) if use_mask else None
        out = torch.empty_like(c.q)
        lse = torch.empty(c.B, c.Hq, c.Sq, dtype=torch.float32, device="cuda")
        ta.attn_fwd(c.q, c.k, c.v, out, lse, scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params,
                    block_mask=mask)
        torch.cuda.synchronize()
        O, L = c.oracle_fwd()
        check_o(host_f64(out), O, f"alibi slopes D {D}")
        check_lse(lse.cpu().double().numpy(), L, f"alibi slopes D {D}")
        got = [host_f64(t) for t in run_fwd_bwd(ta, c, use_mask)]
        check_grads(got, c.oracle_bwd(), f"alibi slopes D {D} mask {use_mask}")


@pytest.mark.parametrize("D", [64, 128])
def test_softcap_near_and_far_from_the_cap(ta, D):
    """Softcap with scores on both sides of the kernels' series limit (a warp
    whose raw scores all satisfy |s| <= 0.4 c takes tanh's series, the others
    its exponential form): scale 1 makes the scores N(0, D); with c = 70 (D 64)
    or 100 (D 128) about half the forward chunks and a third to a half of the
    backward steps take the series.  Forward and backward against the oracle."""
    from gpu_common import check_lse, check_o
    S = 300
    c = Case(190 + D, 1, 4, 2, S, S, D, oracle.MOD_SOFTCAP, ModParams(softcap=70.0 if D == 64 else 100.0),
             scale=1.0)
    mask = ta.new_block_mask(c.mod, c.dev_params, c.B, c.Sq, c.Skv)
    out = torch.empty_like(c.q)
    lse = torch.empty(c.B, c.Hq, c.Sq, dtype=torch.float32, device="cuda")
    ta.attn_fwd(c.q, c.k, c.v, out, lse, scale=c.scale, mod_kind=c.mod, mod_params=c.dev_params, block_mask=mask)
    torch.cuda.synchronize()
    O, L = c.oracle_fwd()
    check_o(host_f64(out), O, f"softcap far D {D}")
    check_lse(lse.cpu().double().numpy(), L, f"softcap far D {D}")
    got = [host_f64(t) for t in run_fwd_bwd(ta, c)]
    check_grads(got, c.oracle_bwd(), f"softcap far D {D}")
