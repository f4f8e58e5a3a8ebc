"""Pins of the oracle's general mask (a bitmap of mask_mod values).

FlexAttention accepts an arbitrary mask_mod ("PyTorch FlexAttention,
FlashAttention-4 백엔드 도입으로 성능 최대 3.2배 향상", 핵심 요약); the
oracle takes its values as a boolean array [B or 1][H or 1][Sq][Skv] and
keeps exactly the true elements (ANDed with any other mask of the mod).
Each pin reduces a bitmap to a kind with its own closed form, or checks the
restriction property of softmax against the raw array.
"""
import numpy as np
import pytest

import oracle
from oracle import (MASK_BITMAP, MASK_CAUSAL, MASK_SLIDING_WINDOW, MOD_ALIBI, MOD_CAUSAL, MOD_NONE,
                    MOD_SLIDING_WINDOW, MOD_SOFTCAP)
from synth_inputs import ModParams


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def random_bitmap(B, H, Sq, Skv, seed, density=0.5):
    bm = np.random.default_rng(seed).random((B, H, Sq, Skv)) < density
    bm[..., np.arange(Sq), np.minimum(np.arange(Sq), Skv - 1)] = True  # every row keeps a key
    return bm


def same(a, b, tol=1e-14):
    return np.allclose(a[0], b[0], atol=tol) and np.allclose(a[1], b[1], atol=tol)


def test_bitmaps_of_known_masks_reduce_to_them():
    B, H, S, D = 2, 2, 19, 4
    q, k, v = rand((B, H, S, D), 1), rand((B, H, S, D), 2), rand((B, H, S, D), 3)
    i, j = np.arange(S)[:, None], np.arange(S)[None, :]
    tril = np.broadcast_to(j <= i, (1, 1, S, S))
    band = np.broadcast_to((i - j >= 0) & (i - j < 5), (1, 1, S, S))
    ones = np.ones((1, 1, S, S), dtype=bool)
    fwd = lambda mod, bm: oracle.attention_forward(q, k, v, 0.7, mod, ModParams(window=5, bitmap=bm))
    assert same(fwd(MOD_NONE | MASK_BITMAP, tril), fwd(MOD_CAUSAL, None))
    assert same(fwd(MOD_NONE | MASK_BITMAP, band), fwd(MOD_SLIDING_WINDOW, None))
    assert same(fwd(MOD_ALIBI | MASK_BITMAP, ones), fwd(MOD_ALIBI, None))
    assert same(fwd(MOD_SLIDING_WINDOW | MASK_BITMAP, tril), fwd(MOD_SLIDING_WINDOW, None))


@pytest.mark.parametrize("mod", [MOD_NONE | MASK_BITMAP, MOD_ALIBI | MASK_BITMAP,
                                 MOD_SOFTCAP | MASK_BITMAP | MASK_CAUSAL])
def test_random_bitmap_is_restricted_softmax(mod):
    # probabilities = the unmasked score mod's softmax restricted to the kept
    # elements (read straight from the array) and renormalised
    S, D = 15, 5
    bm = random_bitmap(1, 1, S, S, 4)
    p = ModParams(softcap=1.5, bitmap=bm)
    q, k = rand((1, 2, S, D), 5), rand((1, 2, S, D), 6)
    score = mod & 0xFF
    i, j = np.arange(S)[:, None], np.arange(S)[None, :]
    keep = bm[0, 0] & ((j <= i) if mod & MASK_CAUSAL else True)
    for h in range(2):
        full = oracle.attention_probs(q, k, 0.9, score, p, b=0, h=h)
        expect = np.where(keep, full, 0.0)
        expect /= expect.sum(axis=1, keepdims=True)
        assert np.allclose(oracle.attention_probs(q, k, 0.9, mod, p, b=0, h=h), expect, atol=1e-14)


def test_per_head_bitmap_equals_separate_heads():
    B, H, S, D = 2, 3, 13, 4
    q, k, v = rand((B, H, S, D), 7), rand((B, 1, S, D), 8), rand((B, 1, S, D), 9)
    bm = random_bitmap(B, H, S, S, 10)
    O, L = oracle.attention_forward(q, k, v, 0.5, MOD_NONE | MASK_BITMAP, ModParams(bitmap=bm))
    for b in range(B):
        for h in range(H):
            Oh, Lh = oracle.attention_forward(q[b:b + 1, h:h + 1], k[b:b + 1], v[b:b + 1], 0.5,
                                              MOD_NONE | MASK_BITMAP, ModParams(bitmap=bm[b:b + 1, h:h + 1]))
            assert np.allclose(O[b, h], Oh[0, 0], atol=1e-14) and np.allclose(L[b, h], Lh[0, 0], atol=1e-14)


def test_bitmap_and_window_compose():
    # window flag ANDed with a bitmap = the bitmap with the band applied by hand
    B, H, S, D = 1, 2, 17, 3
    q, k, v = rand((B, H, S, D), 11), rand((B, H, S, D), 12), rand((B, H, S, D), 13)
    bm = random_bitmap(1, 1, S, S, 14, density=0.7)
    i, j = np.arange(S)[:, None], np.arange(S)[None, :]
    banded = bm & ((i - j >= 0) & (i - j < 4))[None, None]
    banded[..., np.arange(S), np.arange(S)] = True
    bm2 = bm.copy()
    bm2[..., np.arange(S), np.arange(S)] = True
    a = oracle.attention_forward(q, k, v, 0.8, MOD_NONE | MASK_SLIDING_WINDOW | MASK_BITMAP,
                                 ModParams(window=4, bitmap=bm2))
    b = oracle.attention_forward(q, k, v, 0.8, MOD_NONE | MASK_BITMAP, ModParams(bitmap=banded))
    assert same(a, b)


def test_row_without_kept_keys_follows_the_convention():
    S = 6
    bm = np.ones((1, 1, S, S), dtype=bool)
    bm[0, 0, 3] = False
    q, k, v = rand((1, 1, S, 3), 15), rand((1, 1, S, 3), 16), rand((1, 1, S, 3), 17)
    O, L = oracle.attention_forward(q, k, v, 1.0, MOD_NONE | MASK_BITMAP, ModParams(bitmap=bm))
    assert np.all(O[0, 0, 3] == 0) and L[0, 0, 3] == -np.inf
    dq, _, _ = oracle.attention_backward(q, k, v, rand((1, 1, S, 3), 18), 1.0, MOD_NONE | MASK_BITMAP,
                                         ModParams(bitmap=bm))
    assert np.all(dq[0, 0, 3] == 0)


@pytest.mark.parametrize("mod", [MOD_NONE | MASK_BITMAP, MOD_SOFTCAP | MASK_BITMAP | MASK_CAUSAL])
def test_bitmap_gradients_match_central_differences(mod):
    B, Hq, Hkv, S, D = 1, 2, 1, 7, 3
    q, k, v = rand((B, Hq, S, D), 19), rand((B, Hkv, S, D), 20), rand((B, Hkv, S, D), 21)
    dout = rand((B, Hq, S, D), 22)
    p = ModParams(softcap=1.5, bitmap=random_bitmap(1, Hq, S, S, 23))
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


def test_bitmap_block_classes():
    S = 300
    i, j = np.arange(S)[:, None], np.arange(S)[None, :]
    tril = np.broadcast_to(j <= i, (1, 1, S, S))
    assert np.array_equal(oracle.classify_tiles(MOD_NONE | MASK_BITMAP, ModParams(bitmap=tril), 2, S, S),
                          oracle.classify_tiles(MOD_CAUSAL, ModParams(), 2, S, S))
    ones = np.ones((1, 1, S, S), dtype=bool)
    assert (oracle.classify_tiles(MOD_NONE | MASK_BITMAP, ModParams(bitmap=ones), 1, S, S) == 2).all()
    # a bitmap that keeps one element of tile (0, 2) only
    one = np.zeros((1, 1, S, S), dtype=bool)
    one[0, 0, 5, 260] = True
    cls = oracle.classify_tiles(MOD_NONE | MASK_BITMAP, ModParams(bitmap=one), 1, S, S)
    assert cls[0, 0, 2] == 1 and cls.sum() == 1


def test_per_head_bitmap_classes_hold_for_every_head():
    # head 0 causal, head 1 everything: below the diagonal both keep all
    # (FULL), above it only head 1 keeps (PARTIAL); no tile is EMPTY
    S = 384
    i, j = np.arange(S)[:, None], np.arange(S)[None, :]
    bm = np.stack([j <= i, np.ones((S, S), dtype=bool)])[None]
    cls = oracle.classify_tiles(MOD_NONE | MASK_BITMAP, ModParams(bitmap=bm), 1, S, S)[0]
    assert (cls[np.tril_indices(3, -1)] == 2).all()
    assert (cls[np.triu_indices(3)] == 1).all()
    # counting kept elements sums the heads separately
    n = oracle.useful_elements(MOD_NONE | MASK_BITMAP, ModParams(bitmap=bm), 1, 2, S, S)
    assert n == S * (S + 1) // 2 + S * S
