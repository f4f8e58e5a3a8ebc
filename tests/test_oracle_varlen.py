"""Pins of the oracle's packed variable-length mask (MASK_VARLEN): each
sequence's queries attend exactly to that sequence's keys, whatever the two
lengths are.  The pins cut the packed tensors into the independent problems
the mask describes and compare with the plain definition on each."""
import numpy as np
import pytest

import oracle
from oracle import MASK_CAUSAL, MASK_DOCUMENT, MASK_VARLEN, MOD_ALIBI, MOD_NONE, MOD_SOFTCAP
from synth_inputs import ModParams


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


QO = [0, 5, 5, 17, 30]     # query lengths 5, 0, 12, 13
KO = [0, 9, 12, 14, 41]    # key lengths 9, 3, 2, 27


def params(**kw):
    return ModParams(q_offsets=[QO, [0, 30]], k_offsets=[KO, [0, 41]], softcap=2.0, **kw)


@pytest.mark.parametrize("mod", [MOD_NONE | MASK_VARLEN, MOD_SOFTCAP | MASK_VARLEN])
def test_sequences_are_independent_problems(mod):
    B, H, D = 2, 2, 4
    q, k, v = rand((B, H, 30, D), 1), rand((B, H, 41, D), 2), rand((B, H, 41, D), 3)
    O, L = oracle.attention_forward(q, k, v, 0.7, mod, params())
    base = mod & 0xFF
    for b, (qo, ko) in enumerate(((QO, KO), ([0, 30], [0, 41]))):
        for d in range(len(qo) - 1):
            a, e, c, f = qo[d], qo[d + 1], ko[d], ko[d + 1]
            if a == e:
                continue
            if c == f:  # a sequence without keys keeps nothing
                assert np.all(O[b, :, a:e] == 0) and np.all(L[b, :, a:e] == -np.inf)
                continue
            Oc, Lc = oracle.attention_forward(q[b:b + 1, :, a:e], k[b:b + 1, :, c:f], v[b:b + 1, :, c:f], 0.7,
                                              base, params())
            assert np.allclose(O[b:b + 1, :, a:e], Oc, atol=1e-14) and np.allclose(L[b:b + 1, :, a:e], Lc, atol=1e-14)


def test_equal_offsets_with_causal_per_sequence_reduce_to_documents():
    # one batch row, equal query and key offsets: the varlen mask is the
    # document mask without its causal part
    S, D = 24, 3
    offs = [0, 7, 15, 24]
    q, k, v = rand((1, 2, S, D), 4), rand((1, 2, S, D), 5), rand((1, 2, S, D), 6)
    p = ModParams(q_offsets=[offs], k_offsets=[offs], doc_offsets=[offs])
    keep_varlen = oracle.attention_probs(q, k, 1.0, MOD_NONE | MASK_VARLEN, p) > 0
    keep_doc = oracle.attention_probs(q, k, 1.0, MOD_NONE | MASK_DOCUMENT, p) > 0
    i, j = np.arange(S)[:, None], np.arange(S)[None, :]
    assert np.array_equal(keep_doc, keep_varlen & (j <= i))


def test_counts_and_classes():
    n = oracle.useful_elements(MOD_NONE | MASK_VARLEN, params(), 2, 3, 30, 41)
    lens = lambda o: np.diff(o)
    expect = int(np.dot(lens(QO), lens(KO))) + 30 * 41
    assert n == 3 * expect
    # tile classes on a bigger packing: FULL tiles lie inside one sequence's rectangle
    qo, ko = [0, 100, 300, 301, 700], [0, 250, 260, 500, 900]
    p = ModParams(q_offsets=[qo], k_offsets=[ko])
    cls = oracle.classify_tiles(MOD_NONE | MASK_VARLEN, p, 1, 700, 900)[0]
    for qt in range(cls.shape[0]):
        for kt in range(cls.shape[1]):
            r0, r1, c0, c1 = qt * 128, min(700, qt * 128 + 128), kt * 128, min(900, kt * 128 + 128)
            inside = [(max(r0, qo[d]) < min(r1, qo[d + 1])) and (max(c0, ko[d]) < min(c1, ko[d + 1]))
                      for d in range(4)]
            if not any(inside):
                assert cls[qt, kt] == 0
            full = any(qo[d] <= r0 and r1 <= qo[d + 1] and ko[d] <= c0 and c1 <= ko[d + 1] for d in range(4))
            assert (cls[qt, kt] == 2) == full


def test_varlen_takes_no_other_mask():
    for bad in (MASK_VARLEN | MASK_CAUSAL, MASK_VARLEN | MASK_DOCUMENT, oracle.MOD_CAUSAL | MASK_VARLEN):
        with pytest.raises(ValueError):
            oracle.split_mod(bad)
    assert oracle.split_mod(MOD_ALIBI | MASK_VARLEN) == (MOD_ALIBI, [oracle.attention._VARLEN])


def test_varlen_gradients_match_central_differences():
    B, Hq, Hkv, D = 1, 2, 1, 3
    qo, ko = [0, 3, 7], [0, 4, 6]
    p = ModParams(q_offsets=[qo], k_offsets=[ko])
    q, k, v = rand((B, Hq, 7, D), 7), rand((B, Hkv, 6, D), 8), rand((B, Hkv, 6, D), 9)
    dout = rand((B, Hq, 7, D), 10)
    mod = MOD_NONE | MASK_VARLEN
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
            fp = float((oracle.attention_forward(args["q"], args["k"], args["v"], 0.8, mod, p)[0] * dout).sum())
            args[name] = xm
            fm = float((oracle.attention_forward(args["q"], args["k"], args["v"], 0.8, mod, p)[0] * dout).sum())
            num[idx] = (fp - fm) / (2 * h)
        assert np.linalg.norm(num - g) / np.linalg.norm(num) < 1e-6, name
