"""Brute-force block mask and work order (fp64 oracle package; test infrastructure only).

The FlexAttention FA4 backend skips KV blocks that the mask empties entirely
and balances the remaining, data-dependent work over the SMs ("PyTorch
FlexAttention, FlashAttention-4 백엔드 도입으로 성능 최대 3.2배 향상",
섹션별 상세: block-sparse iteration and Cluster Launch Control; 실무 Takeaway:
load balance under data-dependent masks).  This module classifies every
128x128 tile by evaluating the mask on each of its elements, one by one in
vectorised form, with no shortcut.

Contract (byte-for-byte what the CUDA ``build_block_mask`` must produce):
  tile_class [B][nQ][nK] uint8: 0 EMPTY (no in-range element kept),
      2 FULL (every in-range element kept), 1 PARTIAL otherwise.  Elements past
      Sq or Skv are out of range and take no part in the classification.
  kv_count [B][nQ] int32, kv_index [B][nQ][nK] int32: the non-EMPTY KV tiles
      of each query tile in ascending order, padded with -1.
  q_count [B][nK] int32, q_index [B][nK][nQ] int32: the transpose.
  fwd_order [B * nP] int32, nP = ceil(nQ / 2): forward work pairs
      u = b * nP + p (query tiles 2p and 2p+1) sorted by descending cost,
      cost = number of KV tiles non-EMPTY for either query tile; ties keep
      ascending u (longest-processing-time-first order).
  bwd_order [B * nK] int32: backward units u = b * nK + kv tile sorted by
      descending q_count; ties keep ascending u.
"""
from __future__ import annotations

import numpy as np

from .attention import has_bitmap, has_mask, score_mod

TILE = 128


def classify_tiles(mod, params, B, Sq, Skv, tile=TILE):
    """Tile classes; with a per-head bitmap the classes hold for every head at
    once: EMPTY where no head keeps an element, FULL where every head keeps
    every in-range element, PARTIAL otherwise."""
    nQ = -(-Sq // tile)
    nK = -(-Skv // tile)
    cls = np.full((B, nQ, nK), 2, dtype=np.uint8)
    if not has_mask(mod):
        return cls
    heads = np.asarray(params.bitmap).shape[1] if has_bitmap(mod) else 1
    kj = np.arange(Skv, dtype=np.int64)[None, :]
    for b in range(B):
        for qi in range(nQ):
            rows = np.arange(qi * tile, min(Sq, (qi + 1) * tile), dtype=np.int64)[:, None]
            keeps = [score_mod(np.zeros((rows.shape[0], Skv)), mod, params, b, h, heads, rows, kj)[1]
                     for h in range(heads)]
            for kt in range(nK):
                blocks = [keep[:, kt * tile:min(Skv, (kt + 1) * tile)] for keep in keeps]
                counts = [int(blk.sum()) for blk in blocks]
                if max(counts) == 0:
                    cls[b, qi, kt] = 0
                elif min(counts) == blocks[0].size:
                    cls[b, qi, kt] = 2
                else:
                    cls[b, qi, kt] = 1
    return cls


def block_mask(mod, params, B, Sq, Skv, tile=TILE):
    cls = classify_tiles(mod, params, B, Sq, Skv, tile)
    _, nQ, nK = cls.shape
    kv_count = np.zeros((B, nQ), dtype=np.int32)
    kv_index = np.full((B, nQ, nK), -1, dtype=np.int32)
    q_count = np.zeros((B, nK), dtype=np.int32)
    q_index = np.full((B, nK, nQ), -1, dtype=np.int32)
    for b in range(B):
        for qi in range(nQ):
            nz = [kt for kt in range(nK) if cls[b, qi, kt] != 0]
            kv_count[b, qi] = len(nz)
            kv_index[b, qi, :len(nz)] = nz
        for kt in range(nK):
            nz = [qi for qi in range(nQ) if cls[b, qi, kt] != 0]
            q_count[b, kt] = len(nz)
            q_index[b, kt, :len(nz)] = nz
    nP = -(-nQ // 2)
    pair_cost = []
    for b in range(B):
        for p in range(nP):
            live = set()
            for qi in (2 * p, 2 * p + 1):
                if qi < nQ:
                    live.update(kt for kt in range(nK) if cls[b, qi, kt] != 0)
            pair_cost.append(len(live))
    fwd_order = np.array(sorted(range(B * nP), key=lambda u: (-pair_cost[u], u)), dtype=np.int32)
    unit_cost = [int(q_count[b, kt]) for b in range(B) for kt in range(nK)]
    bwd_order = np.array(sorted(range(B * nK), key=lambda u: (-unit_cost[u], u)), dtype=np.int32)
    return {
        "tile_class": cls,
        "kv_count": kv_count,
        "kv_index": kv_index,
        "q_count": q_count,
        "q_index": q_index,
        "fwd_order": fwd_order,
        "bwd_order": bwd_order,
    }
