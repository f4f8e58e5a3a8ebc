"""Pins of the brute-force block mask against closed-form tile classes."""
import numpy as np
import pytest

import oracle
from oracle import MOD_ALIBI, MOD_CAUSAL, MOD_DOCUMENT, MOD_NONE, MOD_SLIDING_WINDOW
from synth_inputs import ModParams

T = 128


def interval_class(q0, q1, k0, k1, lo_of, hi_of):
    """Class of tile rows [q0,q1) x cols [k0,k1) when row i keeps cols [lo(i), hi(i)]."""
    n_keep = 0
    for i in range(q0, q1):
        a, b = max(k0, lo_of(i)), min(k1 - 1, hi_of(i))
        n_keep += max(0, b - a + 1)
    if n_keep == 0:
        return 0
    return 2 if n_keep == (q1 - q0) * (k1 - k0) else 1


@pytest.mark.parametrize("S", [128, 384, 385, 1000])
def test_causal_tiles(S):
    bm = oracle.block_mask(MOD_CAUSAL, None, 1, S, S)
    n = -(-S // T)
    for qi in range(n):
        for kt in range(n):
            q0, q1 = qi * T, min(S, qi * T + T)
            k0, k1 = kt * T, min(S, kt * T + T)
            expect = 2 if kt < qi else (0 if kt > qi else (2 if q1 - q0 == 1 else 1))
            assert bm["tile_class"][0, qi, kt] == expect
            assert expect == interval_class(q0, q1, k0, k1, lambda i: 0, lambda i: i)
    assert list(bm["kv_count"][0]) == [qi + 1 for qi in range(n)]


def test_single_row_tail_tile_is_full():
    bm = oracle.block_mask(MOD_CAUSAL, None, 1, 257, 257)
    assert bm["tile_class"][0, 2, 2] == 2


@pytest.mark.parametrize("W", [1, 100, 128, 1024])
def test_window_tiles(W):
    S = 1100
    bm = oracle.block_mask(MOD_SLIDING_WINDOW, ModParams(window=W), 1, S, S)
    n = -(-S // T)
    for qi in range(n):
        for kt in range(n):
            c = interval_class(qi * T, min(S, qi * T + T), kt * T, min(S, kt * T + T),
                               lambda i: i - W + 1, lambda i: i)
            assert bm["tile_class"][0, qi, kt] == c


def test_documents_tiles_and_lists():
    S = 1000
    offs = [[0, 130, 600, 1000], [0, 1000]]
    bm = oracle.block_mask(MOD_DOCUMENT, ModParams(doc_offsets=offs), 2, S, S)
    causal = oracle.block_mask(MOD_CAUSAL, None, 1, S, S)
    assert np.array_equal(bm["tile_class"][1], causal["tile_class"][0])
    starts = np.repeat(np.array(offs[0][:-1]), np.diff(offs[0]))
    n = -(-S // T)
    for qi in range(n):
        for kt in range(n):
            c = interval_class(qi * T, min(S, qi * T + T), kt * T, min(S, kt * T + T),
                               lambda i: int(starts[i]), lambda i: i)
            assert bm["tile_class"][0, qi, kt] == c
    for b in range(2):
        for qi in range(n):
            nz = np.nonzero(bm["tile_class"][b, qi])[0]
            assert bm["kv_count"][b, qi] == len(nz)
            assert list(bm["kv_index"][b, qi, :len(nz)]) == list(nz)
            assert (bm["kv_index"][b, qi, len(nz):] == -1).all()
        for kt in range(n):
            nz = np.nonzero(bm["tile_class"][b, :, kt])[0]
            assert bm["q_count"][b, kt] == len(nz)
            assert list(bm["q_index"][b, kt, :len(nz)]) == list(nz)


@pytest.mark.parametrize("mod", [MOD_NONE, MOD_ALIBI])
def test_unmasked_mods_all_full(mod):
    bm = oracle.block_mask(mod, None, 2, 300, 500)
    assert (bm["tile_class"] == 2).all()
    assert list(bm["fwd_order"]) == list(range(2 * 2))
    assert list(bm["bwd_order"]) == list(range(2 * 4))


def test_orders_are_lpt_permutations():
    S = 1300
    bm = oracle.block_mask(MOD_CAUSAL, None, 2, S, S)
    n = -(-S // T)
    nP = -(-n // 2)
    order = list(bm["fwd_order"])
    assert sorted(order) == list(range(2 * nP))
    # causal pair p of query tiles (2p, 2p+1) touches kv tiles 0..2p+1
    cost = [min(n, 2 * (u % nP) + 2) for u in order]
    assert cost == sorted(cost, reverse=True)
    # ties in ascending unit id
    for a, b in zip(order, order[1:]):
        if min(n, 2 * (a % nP) + 2) == min(n, 2 * (b % nP) + 2):
            assert a < b
    border = list(bm["bwd_order"])
    assert sorted(border) == list(range(2 * n))
    qc = [n - (u % n) for u in border]
    assert qc == sorted(qc, reverse=True)
