"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

None of these retypes the oracle's formulas: each checks a closed form, an
invariant, a special case that reduces to a library routine, brute force, or
a number the pages print.  ``test_oracle_mutants.py`` shows that plausible
mistakes planted in the oracle fail at least one of these pins.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import (MOD_ALIBI, MOD_CAUSAL, MOD_DOCUMENT, MOD_LOCAL_BOOST, MOD_NONE,
                    MOD_SLIDING_WINDOW, MOD_SOFTCAP)
from synth_inputs import ModParams, bf16_bits, bf16_bits_to_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ALL_MODS = [MOD_NONE, MOD_CAUSAL, MOD_ALIBI, MOD_SOFTCAP, MOD_SLIDING_WINDOW,
            MOD_LOCAL_BOOST, MOD_DOCUMENT]


def params_for(mod, S, window=5, radius=3, boost=1.1, softcap=2.0, docs=None):
    p = ModParams(softcap=softcap, window=window, boost=boost, boost_radius=radius)
    if oracle.has_document(mod):
        p.doc_offsets = docs if docs is not None else [[0, S // 3, S // 2 + 1, S]]
    return p


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- input encoding

def test_bf16_rounding_nearest_even():
    x = np.array([1.0, 1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8, -2.5, 3.0e38], dtype=np.float32)
    bits = bf16_bits(x)
    assert list(bits[:4]) == [0x3F80, 0x3F80, 0x3F82, 0xC020]
    back = bf16_bits_to_f64(bits)
    assert back[0] == 1.0 and back[2] == 1.0 + 2.0**-6 and back[3] == -2.5


# ---------------------------------------------------------------- forward closed forms

@pytest.mark.parametrize("mod", ALL_MODS)
def test_constant_values_give_that_row(mod):
    B, H, S, D = 1, 2, 11, 4
    q, k = rand((B, H, S, D), 1), rand((B, H, S, D), 2)
    row = np.array([0.5, -1.25, 3.0, 7.0])
    v = np.broadcast_to(row, (B, H, S, D)).copy()
    O, _ = oracle.attention_forward(q, k, v, 0.7, mod, params_for(mod, S, window=S))
    assert np.allclose(O, row[None, None, None, :], atol=1e-13)


@pytest.mark.parametrize("mod", ALL_MODS)
def test_single_key_gives_v0(mod):
    B, H, Sq, D = 1, 2, 5, 3
    q, k, v = rand((B, H, Sq, D), 3), rand((B, H, 1, D), 4), rand((B, H, 1, D), 5)
    p = params_for(mod, Sq, window=8, docs=[[0, Sq]])
    O, LSE = oracle.attention_forward(q, k, v, 0.5, mod, p)
    assert np.allclose(O, v[:, :, :1, :], atol=1e-14)
    s = 0.5 * np.einsum("bhqd,bhd->bhq", q, k[:, :, 0])
    if mod == MOD_SOFTCAP:
        s = p.softcap * np.tanh(s / p.softcap)
    elif mod == MOD_ALIBI:
        qi = np.arange(Sq)
        s = s - np.array([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)])[None, :, None] * qi
    elif mod == MOD_LOCAL_BOOST:
        qi = np.arange(Sq)
        s = np.where(qi < p.boost_radius, 1.1 * s, s)
    assert np.allclose(LSE, s, atol=1e-13)


def test_causal_first_query_attends_key0():
    B, H, S, D = 2, 3, 9, 5
    q, k, v = rand((B, H, S, D), 6), rand((B, H, S, D), 7), rand((B, H, S, D), 8)
    O, LSE = oracle.attention_forward(q, k, v, 0.3, MOD_CAUSAL)
    assert np.allclose(O[:, :, 0], v[:, :, 0], atol=1e-14)
    assert np.allclose(LSE[:, :, 0], 0.3 * (q[:, :, 0] * k[:, :, 0]).sum(-1), atol=1e-14)


def test_zero_queries_mean_of_values():
    B, H, S, D = 1, 2, 13, 4
    q = np.zeros((B, H, S, D))
    k, v = rand((B, H, S, D), 9), rand((B, H, S, D), 10)
    O, LSE = oracle.attention_forward(q, k, v, 1.0, MOD_NONE)
    assert np.allclose(O, v.mean(axis=2, keepdims=True), atol=1e-14)
    assert np.allclose(LSE, math.log(S), atol=1e-14)
    O, LSE = oracle.attention_forward(q, k, v, 1.0, MOD_CAUSAL)
    prefix = np.cumsum(v, axis=2) / np.arange(1, S + 1)[None, None, :, None]
    assert np.allclose(O, prefix, atol=1e-13)
    assert np.allclose(LSE, np.log(np.arange(1, S + 1))[None, None, :], atol=1e-14)


def test_zero_queries_alibi_geometric_sums():
    B, H, S, D = 1, 4, 17, 2
    q = np.zeros((B, H, S, D))
    k, v = rand((B, H, S, D), 11), rand((B, H, S, D), 12)
    _, LSE = oracle.attention_forward(q, k, v, 1.0, MOD_ALIBI)
    for h in range(H):
        r = math.exp(-(2.0 ** (-8.0 * (h + 1) / H)))
        for i in range(S):
            left = (1 - r ** (i + 1)) / (1 - r)          # distances 0..i
            right = r * (1 - r ** (S - 1 - i)) / (1 - r)  # distances 1..S-1-i
            assert abs(LSE[0, h, i] - math.log(left + right)) < 1e-12


@pytest.mark.parametrize("mod", ALL_MODS)
def test_probability_rows_sum_to_one(mod):
    # V = identity turns O into P itself
    B, H, S = 1, 2, 12
    q, k = rand((B, H, S, 6), 13), rand((B, H, S, 6), 14)
    v = np.broadcast_to(np.eye(S), (B, H, S, S)).copy()
    O, _ = oracle.attention_forward(q, k, v, 0.8, mod, params_for(mod, S, window=4))
    assert (O >= 0).all()
    assert np.allclose(O.sum(-1), 1.0, atol=1e-14)


def test_fully_masked_row_convention():
    q, k, v = rand((1, 1, 6, 3), 15), rand((1, 1, 4, 3), 16), rand((1, 1, 4, 3), 17)
    # sliding window of 2 with Sq > Skv + W leaves the last rows with no key
    O, LSE = oracle.attention_forward(q, k, v, 1.0, MOD_SLIDING_WINDOW, params_for(MOD_SLIDING_WINDOW, 6, window=2))
    assert np.all(O[0, 0, 5] == 0) and LSE[0, 0, 5] == -np.inf
    dq, dk, dv = oracle.attention_backward(q, k, v, rand((1, 1, 6, 3), 18), 1.0, MOD_SLIDING_WINDOW,
                                           params_for(MOD_SLIDING_WINDOW, 6, window=2))
    assert np.all(dq[0, 0, 5] == 0)


# ---------------------------------------------------------------- reductions between mods

def test_mod_reductions():
    B, H, S, D = 2, 2, 20, 4
    q, k, v = rand((B, H, S, D), 19), rand((B, H, S, D), 20), rand((B, H, S, D), 21)
    causal = oracle.attention_forward(q, k, v, 0.6, MOD_CAUSAL)
    wide = oracle.attention_forward(q, k, v, 0.6, MOD_SLIDING_WINDOW, params_for(0, S, window=S))
    one_doc = oracle.attention_forward(q, k, v, 0.6, MOD_DOCUMENT, params_for(MOD_DOCUMENT, S, docs=[[0, S]] * B))
    for a, b in [(causal, wide), (causal, one_doc)]:
        assert np.allclose(a[0], b[0], atol=1e-14) and np.allclose(a[1], b[1], atol=1e-14)
    none = oracle.attention_forward(q, k, v, 0.6, MOD_NONE)
    unit_boost = oracle.attention_forward(q, k, v, 0.6, MOD_LOCAL_BOOST, params_for(0, S, boost=1.0))
    huge_cap = oracle.attention_forward(q, k, v, 0.6, MOD_SOFTCAP, params_for(0, S, softcap=1e7))
    assert np.allclose(none[0], unit_boost[0], atol=1e-14)
    assert np.allclose(none[0], huge_cap[0], atol=1e-10) and np.allclose(none[1], huge_cap[1], atol=1e-10)


def test_window_one_attends_only_self():
    B, H, S, D = 1, 2, 9, 3
    q, k, v = rand((B, H, S, D), 22), rand((B, H, S, D), 23), rand((B, H, S, D), 24)
    O, _ = oracle.attention_forward(q, k, v, 1.0, MOD_SLIDING_WINDOW, params_for(0, S, window=1))
    assert np.allclose(O, v, atol=1e-14)


def test_documents_are_independent_causal_problems():
    S, D = 24, 4
    offs = [0, 7, 15, 24]
    q, k, v = rand((1, 2, S, D), 25), rand((1, 2, S, D), 26), rand((1, 2, S, D), 27)
    O, LSE = oracle.attention_forward(q, k, v, 0.5, MOD_DOCUMENT, params_for(MOD_DOCUMENT, S, docs=[offs]))
    for a, b in zip(offs[:-1], offs[1:]):
        Oc, Lc = oracle.attention_forward(q[:, :, a:b], k[:, :, a:b], v[:, :, a:b], 0.5, MOD_CAUSAL)
        assert np.allclose(O[:, :, a:b], Oc, atol=1e-14) and np.allclose(LSE[:, :, a:b], Lc, atol=1e-14)


def test_gqa_equals_mha_with_repeated_kv():
    B, Hq, Hkv, S, D = 1, 6, 2, 10, 4
    q, k, v = rand((B, Hq, S, D), 28), rand((B, Hkv, S, D), 29), rand((B, Hkv, S, D), 30)
    kr, vr = np.repeat(k, Hq // Hkv, axis=1), np.repeat(v, Hq // Hkv, axis=1)
    for mod in (MOD_NONE, MOD_ALIBI, MOD_CAUSAL):
        a = oracle.attention_forward(q, k, v, 0.4, mod)
        b = oracle.attention_forward(q, kr, vr, 0.4, mod)
        assert np.allclose(a[0], b[0], atol=1e-14) and np.allclose(a[1], b[1], atol=1e-14)
    dout = rand((B, Hq, S, D), 31)
    g = oracle.attention_backward(q, k, v, dout, 0.4, MOD_CAUSAL)
    gr = oracle.attention_backward(q, kr, vr, dout, 0.4, MOD_CAUSAL)
    assert np.allclose(g[0], gr[0], atol=1e-13)
    G = Hq // Hkv
    assert np.allclose(g[1], gr[1].reshape(B, Hkv, G, S, D).sum(2), atol=1e-13)
    assert np.allclose(g[2], gr[2].reshape(B, Hkv, G, S, D).sum(2), atol=1e-13)


def test_joint_key_value_permutation_invariance():
    B, H, S, D = 1, 2, 15, 4
    q, k, v = rand((B, H, S, D), 32), rand((B, H, S, D), 33), rand((B, H, S, D), 34)
    perm = np.random.default_rng(35).permutation(S)
    a = oracle.attention_forward(q, k, v, 0.9, MOD_NONE)
    b = oracle.attention_forward(q, k[:, :, perm], v[:, :, perm], 0.9, MOD_NONE)
    assert np.allclose(a[0], b[0], atol=1e-14) and np.allclose(a[1], b[1], atol=1e-14)


# ---------------------------------------------------------------- online vs two-pass, library

@pytest.mark.parametrize("mod", ALL_MODS)
def test_online_softmax_matches_two_pass(mod):
    B, H, S, D = 1, 2, 37, 5
    q, k, v = rand((B, H, S, D), 36) * 3, rand((B, H, S, D), 37), rand((B, H, S, D), 38)
    p = params_for(mod, S, window=9, radius=6)
    a = oracle.attention_forward(q, k, v, 0.7, mod, p)
    for block in (1, 8, 16):
        b = oracle.online_forward(q, k, v, 0.7, mod, p, block=block)
        assert np.allclose(a[0], b[0], atol=1e-12, rtol=0) and np.allclose(a[1], b[1], atol=1e-12, rtol=0)


@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_sdpa_float64(causal):
    B, H, S, D = 2, 3, 33, 8
    q, k, v = rand((B, H, S, D), 39), rand((B, H, S, D), 40), rand((B, H, S, D), 41)
    O, _ = oracle.attention_forward(q, k, v, 0.25, MOD_CAUSAL if causal else MOD_NONE)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=causal, scale=0.25)
    assert np.allclose(O, ref.numpy(), atol=1e-13)


# ---------------------------------------------------------------- gradients

def _loss(q, k, v, dout, scale, mod, p):
    O, _ = oracle.attention_forward(q, k, v, scale, mod, p)
    return float((O * dout).sum())


@pytest.mark.parametrize("mod", ALL_MODS)
def test_gradients_match_central_differences(mod):
    B, Hq, Hkv, S, D = 1, 2, 1, 7, 3
    q, k, v = rand((B, Hq, S, D), 42), rand((B, Hkv, S, D), 43), rand((B, Hkv, S, D), 44)
    dout = rand((B, Hq, S, D), 45)
    p = params_for(mod, S, window=3, radius=2, softcap=1.5, docs=[[0, 3, S]])
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, 0.8, mod, p)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            fp = _loss(args["q"], args["k"], args["v"], dout, 0.8, mod, p)
            args[name] = xm
            fm = _loss(args["q"], args["k"], args["v"], dout, 0.8, mod, p)
            num[idx] = (fp - fm) / (2 * h)
        err = np.linalg.norm(num - g) / np.linalg.norm(num)
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("mod", [MOD_NONE, MOD_CAUSAL, MOD_ALIBI, MOD_SLIDING_WINDOW, MOD_DOCUMENT])
def test_gradient_sums(mod):
    B, Hq, Hkv, S, D = 2, 4, 2, 19, 5
    q, k, v = rand((B, Hq, S, D), 46), rand((B, Hkv, S, D), 47), rand((B, Hkv, S, D), 48)
    dout = rand((B, Hq, S, D), 49)
    p = params_for(mod, S, window=6, docs=[[0, 5, S], [0, 11, 12, S]])
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, 0.5, mod, p)
    # shifting every score of a row by the same amount leaves softmax unchanged
    assert np.allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    # each query row's probabilities sum to one
    G = Hq // Hkv
    assert np.allclose(dv.sum(axis=2), dout.reshape(B, Hkv, G, S, D).sum(axis=(2, 3)), atol=1e-12)


def test_backward_row_subsets_match_full():
    B, Hq, Hkv, S, D = 1, 4, 2, 30, 4
    q, k, v = rand((B, Hq, S, D), 50), rand((B, Hkv, S, D), 51), rand((B, Hkv, S, D), 52)
    dout = rand((B, Hq, S, D), 53)
    full = oracle.attention_backward(q, k, v, dout, 0.5, MOD_CAUSAL, chunk=7)
    rows = np.array([0, 3, 17, 29])
    part = oracle.attention_backward(q, k, v, dout, 0.5, MOD_CAUSAL, groups=[(0, 1)], q_rows=rows, kv_rows=rows)
    assert np.allclose(part[0][0, 2:4][:, rows], full[0][0, 2:4][:, rows], atol=1e-14)
    assert np.allclose(part[1][0, 1, rows], full[1][0, 1, rows], atol=1e-14)
    assert np.allclose(part[2][0, 1, rows], full[2][0, 1, rows], atol=1e-14)
    fo = oracle.attention_forward(q, k, v, 0.5, MOD_CAUSAL, chunk=5)
    po = oracle.attention_forward(q, k, v, 0.5, MOD_CAUSAL, heads=[(0, 3)], rows=rows)
    assert np.allclose(po[0][0, 3, rows], fo[0][0, 3, rows], atol=1e-14)


# ---------------------------------------------------------------- counts and printed numbers

def test_useful_element_counts_closed_forms():
    S = 300
    assert oracle.useful_elements(MOD_NONE, None, 2, 3, S, S) == 2 * 3 * S * S
    assert oracle.useful_elements(MOD_CAUSAL, None, 2, 3, S, S) == 2 * 3 * S * (S + 1) // 2
    W = 64
    win = sum(min(i + 1, W) for i in range(S))
    assert oracle.useful_elements(MOD_SLIDING_WINDOW, ModParams(window=W), 1, 2, S, S) == 2 * win
    offs = [0, 100, 250, 300]
    docs = sum(L * (L + 1) // 2 for L in (100, 150, 50))
    assert oracle.useful_elements(MOD_DOCUMENT, ModParams(doc_offsets=[offs]), 1, 1, S, S) == docs


def test_flop_convention_reproduces_printed_table():
    with open(os.path.join(GOLDEN, "flashinfer_table.json")) as f:
        table = json.load(f)
    for row in table["rows"]:
        B, H, S, D = row["B"], row["H"], row["S"], row["D"]
        dense = oracle.useful_flops(B * H * S * S, D)
        printed_flop = row["tflops"] * 1e12 * row["ms"] * 1e-3
        expect = dense / 2 if row["causal"] else dense
        assert abs(printed_flop - expect) / expect < 3e-3, row
    # the exact causal count differs from S^2/2 by (S/2) per head: 0.02% at S=4096
    exact = oracle.useful_flops(oracle.useful_elements(MOD_CAUSAL, None, 1, 1, 4096, 4096), 128)
    assert abs(exact / oracle.useful_flops(4096 * 4096 // 2, 128) - 1) < 3e-4


def test_printed_score_count():
    with open(os.path.join(GOLDEN, "score_count.json")) as f:
        g = json.load(f)
    n = oracle.useful_elements(MOD_NONE, None, 1, 1, g["S"], g["S"])
    assert round(n / 1e6) == g["scores_millions_printed"]


def test_backward_contributing_rows_under_causal_mask():
    # keys j >= 200 are seen only by queries i >= j under the causal mask
    B, Hq, Hkv, S, D = 1, 2, 1, 260, 4
    q, k, v = rand((B, Hq, S, D), 54), rand((B, Hkv, S, D), 55), rand((B, Hkv, S, D), 56)
    dout = rand((B, Hq, S, D), 57)
    full = oracle.attention_backward(q, k, v, dout, 0.5, MOD_CAUSAL, chunk=64)
    kv = np.arange(200, S)
    part = oracle.attention_backward(q, k, v, dout, 0.5, MOD_CAUSAL, kv_rows=kv, q_rows=kv,
                                     contrib_rows=np.arange(200, S))
    assert np.allclose(part[1][0, 0, kv], full[1][0, 0, kv], atol=1e-13)
    assert np.allclose(part[2][0, 0, kv], full[2][0, 0, kv], atol=1e-13)
    assert np.allclose(part[0][0, :, kv], full[0][0, :, kv], atol=1e-13)


def test_alibi_with_given_slopes():
    # the default slopes given explicitly reproduce the default; a zero slope
    # removes the bias; Q = 0 gives the geometric sums of each given slope
    B, H, S, D = 1, 3, 15, 4
    q, k, v = rand((B, H, S, D), 60), rand((B, H, S, D), 61), rand((B, H, S, D), 62)
    default = [2.0 ** (-8.0 * (h + 1) / H) for h in range(H)]
    a = oracle.attention_forward(q, k, v, 0.5, MOD_ALIBI, ModParams())
    b = oracle.attention_forward(q, k, v, 0.5, MOD_ALIBI, ModParams(alibi_slopes=default))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    z = oracle.attention_forward(q, k, v, 0.5, MOD_ALIBI, ModParams(alibi_slopes=[0.0] * H))
    n = oracle.attention_forward(q, k, v, 0.5, MOD_NONE)
    assert np.allclose(z[0], n[0], atol=1e-14) and np.allclose(z[1], n[1], atol=1e-14)
    slopes = [0.3, 1.7, 0.05]
    _, L = oracle.attention_forward(np.zeros_like(q), k, v, 1.0, MOD_ALIBI, ModParams(alibi_slopes=slopes))
    for h, sl in enumerate(slopes):
        r = math.exp(-sl)
        for i in range(S):
            total = (1 - r ** (i + 1)) / (1 - r) + r * (1 - r ** (S - 1 - i)) / (1 - r)
            assert abs(L[0, h, i] - math.log(total)) < 1e-12
