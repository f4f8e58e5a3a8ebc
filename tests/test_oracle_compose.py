"""Pins of the oracle's composed mods (a score mod plus the AND of masks).

FlexAttention composes score mods and masks ("PyTorch FlexAttention,
FlashAttention-4 백엔드 도입으로 성능 최대 3.2배 향상", 핵심 요약: any
combination of the mod set).  The oracle's reading: the base kind's score
transform, and an element kept only where every mask keeps it.  Each pin
checks a closed form, a reduction to a single kind, or the restriction
property of softmax; none retypes the oracle's element rule.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import (MASK_CAUSAL, MASK_DOCUMENT, MASK_SLIDING_WINDOW, MOD_ALIBI, MOD_CAUSAL,
                    MOD_DOCUMENT, MOD_LOCAL_BOOST, MOD_NONE, MOD_SLIDING_WINDOW, MOD_SOFTCAP)
from synth_inputs import ModParams

COMPOSED = [MOD_ALIBI | MASK_CAUSAL, MOD_SOFTCAP | MASK_SLIDING_WINDOW, MOD_LOCAL_BOOST | MASK_DOCUMENT,
            MOD_SLIDING_WINDOW | MASK_DOCUMENT, MOD_ALIBI | MASK_SLIDING_WINDOW | MASK_DOCUMENT]


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def params(S, window=4, radius=2, boost=1.3, softcap=1.5, docs=None, B=1):
    return ModParams(softcap=softcap, window=window, boost=boost, boost_radius=radius,
                     doc_offsets=docs if docs is not None else [[0, S // 3, S // 2 + 1, S]] * B)


def test_split_mod():
    assert oracle.split_mod(MOD_ALIBI | MASK_CAUSAL | MASK_DOCUMENT) == (MOD_ALIBI, [MOD_CAUSAL, MOD_DOCUMENT])
    assert oracle.split_mod(MOD_SLIDING_WINDOW) == (MOD_SLIDING_WINDOW, [])
    for bad in (7, 0x2000 | MOD_NONE, 0x4000):
        with pytest.raises(ValueError):
            oracle.split_mod(bad)
    assert oracle.has_mask(MOD_SOFTCAP | MASK_CAUSAL) and not oracle.has_mask(MOD_SOFTCAP)
    assert oracle.has_document(MOD_NONE | MASK_DOCUMENT) and not oracle.has_document(MOD_CAUSAL)


def test_zero_queries_causal_alibi_geometric_sums():
    # Q = 0: scores are the bias alone; causal keeps distances 0..i only
    B, H, S, D = 1, 4, 15, 3
    q = np.zeros((B, H, S, D))
    k, v = rand((B, H, S, D), 1), rand((B, H, S, D), 2)
    O, LSE = oracle.attention_forward(q, k, v, 1.0, MOD_ALIBI | MASK_CAUSAL)
    for h in range(H):
        r = math.exp(-(2.0 ** (-8.0 * (h + 1) / H)))
        for i in range(S):
            w = r ** np.arange(i + 1)            # weight of key i - d at distance d
            assert abs(LSE[0, h, i] - math.log((1 - r ** (i + 1)) / (1 - r))) < 1e-12
            expect = (w[:, None] * v[0, h, i::-1]).sum(0) / w.sum()
            assert np.allclose(O[0, h, i], expect, atol=1e-13)


def test_zero_queries_window_and_documents_count_keys():
    # Q = 0: every kept key weighs the same; row i keeps the keys from
    # max(start of its document, i - W + 1) to i
    S, D, W = 23, 3, 4
    offs = [0, 5, 6, 14, S]
    q = np.zeros((1, 2, S, D))
    k, v = rand((1, 2, S, D), 3), rand((1, 2, S, D), 4)
    for mod in (MOD_SLIDING_WINDOW | MASK_DOCUMENT, MOD_DOCUMENT | MASK_SLIDING_WINDOW,
                MOD_NONE | MASK_SLIDING_WINDOW | MASK_DOCUMENT,
                MOD_SOFTCAP | MASK_CAUSAL | MASK_SLIDING_WINDOW | MASK_DOCUMENT):
        O, LSE = oracle.attention_forward(q, k, v, 1.0, mod, params(S, window=W, docs=[offs]))
        for i in range(S):
            start = max(o for o in offs[:-1] if o <= i)
            first = max(start, i - W + 1)
            assert abs(LSE[0, 0, i] - math.log(i - first + 1)) < 1e-14
            assert np.allclose(O[0, :, i], v[0, :, first:i + 1].mean(axis=1), atol=1e-14)
        assert oracle.useful_elements(mod, params(S, window=W, docs=[offs]), 1, 3, S, S) == \
            3 * sum(min(W, i - max(o for o in offs[:-1] if o <= i) + 1) for i in range(S))


@pytest.mark.parametrize("mod", COMPOSED)
def test_composed_probs_are_restricted_softmax(mod):
    # softmax over a subset of keys = the unmasked softmax restricted to the
    # subset and renormalised; the subset is what each mask alone keeps
    S, D = 17, 5
    base, masks = oracle.split_mod(mod)
    p = params(S)
    q, k = rand((1, 2, S, D), 5), rand((1, 2, S, D), 6)
    score_kind = base if base in (MOD_NONE, MOD_ALIBI, MOD_SOFTCAP, MOD_LOCAL_BOOST) else MOD_NONE
    mask_kinds = masks + ([] if score_kind == base else [base])
    for h in range(2):
        full = oracle.attention_probs(q, k, 0.7, score_kind, p, b=0, h=h)
        keep = np.ones_like(full, dtype=bool)
        for m in mask_kinds:
            keep &= oracle.attention_probs(q, k, 0.7, m, p, b=0, h=h) > 0
        expect = np.where(keep, full, 0.0)
        expect /= expect.sum(axis=1, keepdims=True)
        got = oracle.attention_probs(q, k, 0.7, mod, p, b=0, h=h)
        assert np.allclose(got, expect, atol=1e-14)


def test_composition_reductions():
    B, H, S, D = 2, 2, 21, 4
    q, k, v = rand((B, H, S, D), 7), rand((B, H, S, D), 8), rand((B, H, S, D), 9)
    p = params(S, B=B)
    wide = params(S, window=S, B=B)
    one_doc = params(S, docs=[[0, S]] * B)

    def fwd(mod, pp):
        return oracle.attention_forward(q, k, v, 0.6, mod, pp)

    same = [
        (fwd(MOD_CAUSAL, p), fwd(MOD_NONE | MASK_CAUSAL, p)),
        (fwd(MOD_CAUSAL, p), fwd(MOD_CAUSAL | MASK_CAUSAL, p)),
        (fwd(MOD_SLIDING_WINDOW, p), fwd(MOD_CAUSAL | MASK_SLIDING_WINDOW, p)),
        (fwd(MOD_DOCUMENT, p), fwd(MOD_CAUSAL | MASK_DOCUMENT, p)),
        (fwd(MOD_SLIDING_WINDOW | MASK_DOCUMENT, p), fwd(MOD_DOCUMENT | MASK_SLIDING_WINDOW, p)),
        (fwd(MOD_ALIBI | MASK_SLIDING_WINDOW, wide), fwd(MOD_ALIBI | MASK_CAUSAL, wide)),
        (fwd(MOD_SOFTCAP | MASK_DOCUMENT, one_doc), fwd(MOD_SOFTCAP | MASK_CAUSAL, one_doc)),
        (fwd(MOD_SLIDING_WINDOW | MASK_DOCUMENT, wide), fwd(MOD_DOCUMENT, wide)),
        (fwd(MOD_LOCAL_BOOST | MASK_CAUSAL, params(S, boost=1.0, B=B)), fwd(MOD_CAUSAL, p)),
    ]
    for a, b in same:
        assert np.allclose(a[0], b[0], atol=1e-14) and np.allclose(a[1], b[1], atol=1e-14)
    # a window of one key inside any document keeps only the query's own key
    O, _ = fwd(MOD_ALIBI | MASK_SLIDING_WINDOW | MASK_DOCUMENT, params(S, window=1, B=B))
    assert np.allclose(O, v, atol=1e-14)


def _loss(q, k, v, dout, scale, mod, p):
    O, _ = oracle.attention_forward(q, k, v, scale, mod, p)
    return float((O * dout).sum())


@pytest.mark.parametrize("mod", COMPOSED)
def test_composed_gradients_match_central_differences(mod):
    B, Hq, Hkv, S, D = 1, 2, 1, 8, 3
    q, k, v = rand((B, Hq, S, D), 10), rand((B, Hkv, S, D), 11), rand((B, Hkv, S, D), 12)
    dout = rand((B, Hq, S, D), 13)
    p = params(S, window=3, radius=2, docs=[[0, 3, S]])
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, 0.8, mod, p)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
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


def test_composed_block_mask_reduces_and_brackets():
    # window >= S leaves the document classes; a composed tile is never
    # kept where either mask alone empties it
    S = 700
    docs = [[0, 130, 300, 301, 555, S]]
    wide = oracle.classify_tiles(MOD_SLIDING_WINDOW | MASK_DOCUMENT, params(S, window=S, docs=docs), 1, S, S)
    assert np.array_equal(wide, oracle.classify_tiles(MOD_DOCUMENT, params(S, docs=docs), 1, S, S))
    p = params(S, window=200, docs=docs)
    comp = oracle.classify_tiles(MOD_SLIDING_WINDOW | MASK_DOCUMENT, p, 1, S, S)
    win = oracle.classify_tiles(MOD_SLIDING_WINDOW, p, 1, S, S)
    doc = oracle.classify_tiles(MOD_DOCUMENT, p, 1, S, S)
    assert np.all(comp <= np.minimum(win, doc))
    assert np.all((comp == 2) == ((win == 2) & (doc == 2)))
