"""Useful-work counts for throughput reporting (host-side integer arithmetic).

Only unmasked score elements count as useful work.  Every mask of the set,
and every composition of them, keeps an interval of keys per query row, so
the counts are sums of interval lengths.  Forward useful FLOPs are 4 D per
element (two GEMMs, 2 flop per multiply-add), the convention of the
FlashInfer benchmark table ("FlashInfer SM120 NVFP4 어텐션 최적화", 성능:
4 B H S^2 D); backward counts five GEMMs, 10 D per element.
"""
from __future__ import annotations

import numpy as np

from .abi import (MASK_BITMAP, MASK_CAUSAL, MASK_DOCUMENT, MASK_SLIDING_WINDOW, MOD_CAUSAL, MOD_DOCUMENT,
                  MOD_SLIDING_WINDOW)


def mask_parts(mod_kind):
    """(causal, window, document) masks present in a mod code (kind | mask flags)."""
    base, flags = int(mod_kind) & 0xFF, int(mod_kind) & ~0xFF
    window = base == MOD_SLIDING_WINDOW or bool(flags & MASK_SLIDING_WINDOW)
    document = base == MOD_DOCUMENT or bool(flags & MASK_DOCUMENT)
    causal = base == MOD_CAUSAL or bool(flags & MASK_CAUSAL) or window or document
    return causal, window, document


def useful_elements(mod_kind, B, Hq, Sq, Skv, window=None, doc_offsets=None) -> int:
    """Unmasked (b, h, q, kv) elements; doc_offsets: per-batch-row offset lists.
    Interval masks only: a bitmap mask's count is the number of its set bits."""
    if int(mod_kind) & MASK_BITMAP:
        raise ValueError("count a bitmap mask from its bits")
    if int(mod_kind) & 0x1000:
        raise ValueError("count a varlen mask as the sum over sequences of query length x key length")
    causal, win, doc = mask_parts(mod_kind)
    i = np.arange(Sq, dtype=np.int64)
    hi = np.minimum(i, Skv - 1) if causal else np.full(Sq, Skv - 1, dtype=np.int64)
    lo = np.maximum(i - window + 1, 0) if win else np.zeros(Sq, dtype=np.int64)
    total = 0
    for b in range(B):
        lo_b = lo
        if doc:
            offs = np.asarray(doc_offsets[b], dtype=np.int64)
            start = offs[np.searchsorted(offs, i, side="right") - 1]
            lo_b = np.maximum(lo, start)
        total += int(np.maximum(hi - lo_b + 1, 0).sum())
    return Hq * total


def useful_flops(n_elements: int, D: int, backward: bool = False) -> float:
    return float(n_elements) * D * (10.0 if backward else 4.0)
