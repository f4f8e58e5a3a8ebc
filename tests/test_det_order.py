"""CPU model of the deterministic dQ ordering of the backward kernel.

The kernel makes every key tile add its dQ part into a block of query rows
only once the key tiles before it (those that meet the same query tile)
have added theirs: a counter per row block, and a position per (key tile,
query tile) taken from the block mask's key-tile lists or, without one, by
counting the earlier key tiles with a non-empty dense class.  These tests
check, without a GPU, that

  * the positions are exactly the ranks of the key tiles among the units
    that visit each query tile (so every counter reaches every wait value,
    and the order of the adds is ascending key tiles), for both sources;
  * the unit walk (ascending key tiles, each CTA taking ascending ranks in
    the snake order) cannot deadlock: a simulation with random progress of
    the CTAs always finishes, for grids smaller and larger than the work.
"""
import random

import numpy as np
import pytest

import oracle
from synth_inputs import ModParams

TILE = 128
M_CAUSAL, M_WINDOW, M_DOC, M_VARLEN = 1, 2, 4, 16
CAUSAL_BITS = M_CAUSAL | M_WINDOW | M_DOC


def dense_tile_class(mask, window, q0, q1, k0, k1):
    """The kernels' class of a tile without a block mask (mods.cuh)."""
    if mask == 0:
        return 2
    if mask & M_VARLEN:
        return 1
    w = window if mask & M_WINDOW else 1 << 30
    first, last = q0, q1 - 1
    if not (k0 <= last and k1 - 1 >= first - w + 1):
        return 0
    full = k1 - 1 <= first and k0 >= last - w + 1
    return 2 if full and not mask & M_DOC else 1


def unit_list(kt, mask, window, Sq, Skv, tile_class=None, b=0):
    """Query tiles the unit of key tile kt visits (build_kv_qtiles)."""
    nQ = -(-Sq // TILE)
    q_begin = kt if (tile_class is None and mask & CAUSAL_BITS) else 0
    k0, k1 = kt * TILE, min(Skv, kt * TILE + TILE)
    out = []
    for qt in range(q_begin, nQ):
        if tile_class is not None:
            c = int(tile_class[b, qt, kt])
        else:
            c = dense_tile_class(mask, window, qt * TILE, min(Sq, qt * TILE + TILE), k0, k1)
        if c:
            out.append(qt)
    return out


def position(kt, qt, mask, window, Sq, Skv, kv_index=None, kv_count=None, b=0):
    """The kernel's position of key tile kt in query tile qt's add order."""
    if kv_index is not None:
        row = kv_index[b, qt, :kv_count[b, qt]]
        return int(np.searchsorted(row, kt, side="left"))
    q0, q1 = qt * TILE, min(Sq, qt * TILE + TILE)
    return sum(dense_tile_class(mask, window, q0, q1, k2 * TILE, min(Skv, k2 * TILE + TILE)) != 0
               for k2 in range(kt))


CASES = [
    (0, 1024, 700, 700, None),
    (M_CAUSAL, 1024, 700, 700, None),
    (M_CAUSAL | M_WINDOW, 200, 1000, 1000, None),
    (M_CAUSAL | M_WINDOW, 129, 333, 333, None),
    (M_CAUSAL | M_DOC, 1024, 640, 640, [0, 213, 214, 426, 640]),
    (M_CAUSAL, 1024, 333, 130, None),
    (0, 1024, 130, 600, None),
    (M_CAUSAL, 1024, 128, 1000, None),
]


def _oracle_mask_code(mask):
    code = oracle.MOD_NONE
    if mask & M_CAUSAL:
        code |= oracle.MASK_CAUSAL
    if mask & M_WINDOW:
        code |= oracle.MASK_SLIDING_WINDOW
    if mask & M_DOC:
        code |= oracle.MASK_DOCUMENT
    return code


@pytest.mark.parametrize("mask,window,Sq,Skv,docs", CASES)
@pytest.mark.parametrize("with_block_mask", [False, True])
def test_positions_are_ranks_of_visiting_units(mask, window, Sq, Skv, docs, with_block_mask):
    nK = -(-Skv // TILE)
    cls = kvi = kvc = None
    if with_block_mask:
        p = ModParams(window=window, doc_offsets=[docs] if docs else None)
        bm = oracle.block_mask(_oracle_mask_code(mask), p, 1, Sq, Skv)
        cls, kvi, kvc = bm["tile_class"], bm["kv_index"], bm["kv_count"]
    visitors = {}
    for kt in range(nK):
        for qt in unit_list(kt, mask, window, Sq, Skv, cls):
            visitors.setdefault(qt, []).append(kt)
    for qt, kts in visitors.items():
        assert kts == sorted(kts)
        for rank, kt in enumerate(kts):
            assert position(kt, qt, mask, window, Sq, Skv, kvi, kvc) == rank, (qt, kt)


def snake_ranks(n_units, grid):
    """The ranks CTA c walks, in order (kernel_common.cuh snake_unit)."""
    out = [[] for _ in range(grid)]
    k = 0
    while True:
        any_ = False
        for c in range(grid):
            r = k * grid + (grid - 1 - c if k & 1 else c)
            if r < n_units:
                out[c].append(r)
                any_ = True
        if not any_:
            return out
        k += 1


def simulate(B, Hkv, G, Sq, Skv, mask, window, grid, seed, descending=False):
    """Random-progress run of the ordered adds; returns True if every unit finishes."""
    nK = -(-Skv // TILE)
    n_units = B * nK * Hkv
    # unit rank u -> (b, kt, hk), ascending key tiles (decode_bwd_unit, deterministic mode)
    def decode(u):
        pair, hk = divmod(u, Hkv)
        kt, b = divmod(pair, B)
        return b, (nK - 1 - kt) if descending else kt, hk
    steps = {}
    for u in range(n_units):
        b, kt, hk = decode(u)
        seq = []
        qts = unit_list(kt, mask, window, Sq, Skv)
        for g in range(G):
            for qt in qts:
                for half in range(2):
                    if qt * TILE + half * 64 < Sq:
                        block = (b, hk * G + g, qt * 2 + half)
                        seq.append((block, position(kt, qt, mask, window, Sq, Skv)))
        steps[u] = seq
    walk = snake_ranks(n_units, grid)
    sem = {}
    at = [0] * grid        # index into the CTA's walk
    step = [0] * grid      # step within the current unit
    rng = random.Random(seed)
    while True:
        live = [c for c in range(grid) if at[c] < len(walk[c])]
        if not live:
            return True
        progressed = False
        rng.shuffle(live)
        for c in live:
            u = walk[c][at[c]]
            seq = steps[u]
            if step[c] == len(seq):
                at[c] += 1
                step[c] = 0
                progressed = True
                continue
            block, pos = seq[step[c]]
            if sem.get(block, 0) == pos:
                sem[block] = pos + 1
                step[c] += 1
                progressed = True
                if rng.random() < 0.5:
                    break
        if not progressed:
            return False


@pytest.mark.parametrize("B,Hkv,G,Sq,mask,window,grid", [
    (2, 2, 2, 1000, 0, 1024, 3),
    (2, 2, 2, 1000, 0, 1024, 16),
    (1, 2, 4, 1300, M_CAUSAL, 1024, 5),
    (3, 1, 1, 900, M_CAUSAL | M_WINDOW, 300, 4),
    (4, 2, 1, 700, 0, 1024, 148),
])
def test_ordered_adds_never_deadlock(B, Hkv, G, Sq, mask, window, grid):
    for seed in range(20):
        assert simulate(B, Hkv, G, Sq, Sq, mask, window, grid, seed)


def test_descending_order_would_deadlock():
    """The check has teeth: with the key tiles walked in descending order, a
    CTA's unit waits on a unit that some CTA only reaches later."""
    assert not simulate(2, 1, 1, 1000, 1000, 0, 1024, 3, seed=0, descending=True)
