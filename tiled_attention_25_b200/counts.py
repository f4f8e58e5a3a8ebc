"""Useful-work counts for throughput reporting (host-side integer arithmetic).

Only unmasked score elements count as useful work.  Every mask of the set
keeps an interval of keys per query row, so the counts are sums of interval
lengths.  Forward useful FLOPs are 4 D per element (two GEMMs, 2 flop per
multiply-add), the convention of the FlashInfer benchmark table ("FlashInfer
SM120 NVFP4 어텐션 최적화", 성능: 4 B H S^2 D); backward counts five GEMMs,
10 D per element.
"""
from __future__ import annotations

from .abi import MOD_CAUSAL, MOD_DOCUMENT, MOD_SLIDING_WINDOW


def _interval_sum(Sq, Skv, lo_of):
    total = 0
    for i in range(Sq):
        hi = min(i, Skv - 1)
        lo = max(0, lo_of(i))
        if hi >= lo:
            total += hi - lo + 1
    return total


def useful_elements(mod_kind, B, Hq, Sq, Skv, window=None, doc_offsets=None) -> int:
    """Unmasked (b, h, q, kv) elements; doc_offsets: per-batch-row offset lists."""
    if mod_kind == MOD_CAUSAL:
        per_b = [sum(min(i + 1, Skv) for i in range(Sq))] * B
    elif mod_kind == MOD_SLIDING_WINDOW:
        per_b = [_interval_sum(Sq, Skv, lambda i: i - window + 1)] * B
    elif mod_kind == MOD_DOCUMENT:
        per_b = []
        for offs in doc_offsets:
            per_b.append(sum((e - s) * (e - s + 1) // 2 for s, e in zip(offs[:-1], offs[1:])))
    else:
        per_b = [Sq * Skv] * B
    return Hq * sum(per_b)


def useful_flops(n_elements: int, D: int, backward: bool = False) -> float:
    return float(n_elements) * D * (10.0 if backward else 4.0)
