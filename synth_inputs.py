"""Seeded synthetic inputs shared by the fp64 oracle, the tests and bench.py.

This module holds no attention arithmetic: it only draws random numbers,
rounds them to bfloat16 bit patterns and describes the workloads.  Both the
oracle (``oracle/``) and the CUDA path take their inputs from here, and
neither imports the other.

Recipe (stated once, used everywhere):
  * workload ``k`` draws from ``numpy.random.default_rng(k)``;
  * Q, K, V and dO are drawn in that order as float32 ``standard_normal`` of
    shapes ``[B][Hq][Sq][D]``, ``[B][Hkv][Skv][D]`` (twice) and
    ``[B][Hq][Sq][D]``, then rounded to bfloat16 (round-to-nearest-even);
  * document lengths for the packed-document workload come from
    ``default_rng(100 + k)``: uniform integers in [512, 4096] until the
    sequence is filled, the last one truncated to fit;
  * the general (bitmap) mask of workload ``k`` comes from
    ``default_rng(200 + k)``: each 128 x 128 tile is dropped, kept whole or
    kept element by element with a density drawn from [0.3, 0.9], with equal
    odds, and the diagonal is always kept; one mask serves every batch row
    and head.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# Score-mod identifiers; the same numbering as ``attn_mod_kind`` in
# include/attn25.h (a C enum cannot be shared with Python without a parser).
MOD_NONE = 0
MOD_CAUSAL = 1
MOD_ALIBI = 2
MOD_SOFTCAP = 3
MOD_SLIDING_WINDOW = 4
MOD_LOCAL_BOOST = 5
MOD_DOCUMENT = 6
# Mask flags ORed onto a kind to compose mods (the ATTN_MASK_* values).
MASK_CAUSAL = 0x100
MASK_SLIDING_WINDOW = 0x200
MASK_DOCUMENT = 0x400
MASK_BITMAP = 0x800

MOD_NAMES = {
    "none": MOD_NONE,
    "causal": MOD_CAUSAL,
    "alibi": MOD_ALIBI,
    "softcap": MOD_SOFTCAP,
    "sliding_window": MOD_SLIDING_WINDOW,
    "local_boost": MOD_LOCAL_BOOST,
    "document": MOD_DOCUMENT,
    # compositions: a score mod with the AND of masks
    "alibi+causal": MOD_ALIBI | MASK_CAUSAL,
    "softcap+sliding_window": MOD_SOFTCAP | MASK_SLIDING_WINDOW,
    "sliding_window+document": MOD_SLIDING_WINDOW | MASK_DOCUMENT,
    # a general mask given by its values
    "bitmap": MOD_NONE | MASK_BITMAP,
}


@dataclasses.dataclass
class ModParams:
    """Runtime scalars of the score mods (host-side description)."""

    softcap: float = 50.0
    window: int = 1024
    boost: float = 1.1
    boost_radius: int = 128
    # per batch row, the ascending document start offsets plus the end (S)
    doc_offsets: list | None = None
    # general mask values: bool [B or 1][H or 1][Sq][Skv], True = keep
    bitmap: np.ndarray | None = None
    # ALiBi slopes per query head, or None for 2^(-8 (h + 1) / Hq)
    alibi_slopes: list | None = None
    # packed sequences with their own query and key lengths: per batch row,
    # ascending query and key start offsets plus the ends (Sq, Skv)
    q_offsets: list | None = None
    k_offsets: list | None = None


@dataclasses.dataclass
class Workload:
    name: str
    seed: int
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Skv: int
    D: int
    mods: tuple

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


# The five workloads the method is measured on (shapes and mods of the
# FlexAttention / FlashAttention workloads described by the pages).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 2, 2, 256, 256, 64, ("none",)),
    "dense": Workload("dense", 2, 4, 8, 8, 4096, 4096, 128, ("none", "causal")),
    "gqa_long": Workload("gqa_long", 3, 1, 32, 8, 32768, 32768, 128, ("causal",)),
    "score_mods": Workload("score_mods", 4, 2, 16, 16, 8192, 8192, 128,
                           ("alibi", "softcap", "sliding_window", "local_boost")),
    "documents": Workload("documents", 5, 1, 16, 16, 32768, 32768, 128, ("document",)),
    # the composed and general masks on the score-mod shape
    "composed": Workload("composed", 6, 2, 16, 16, 8192, 8192, 128,
                         ("alibi+causal", "softcap+sliding_window", "sliding_window+document", "bitmap")),
}


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest-even); return the uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def draw_qkv(seed: int, B: int, Hq: int, Hkv: int, Sq: int, Skv: int, D: int,
             with_dout: bool = True) -> dict:
    """Q, K, V (and dO) as bfloat16 bit patterns, drawn in the order Q, K, V, dO."""
    rng = np.random.default_rng(seed)
    out = {}
    out["q"] = bf16_bits(rng.standard_normal((B, Hq, Sq, D), dtype=np.float32))
    out["k"] = bf16_bits(rng.standard_normal((B, Hkv, Skv, D), dtype=np.float32))
    out["v"] = bf16_bits(rng.standard_normal((B, Hkv, Skv, D), dtype=np.float32))
    if with_dout:
        out["dout"] = bf16_bits(rng.standard_normal((B, Hq, Sq, D), dtype=np.float32))
    return out


def draw_workload(w: Workload, with_dout: bool = True) -> dict:
    return draw_qkv(w.seed, w.B, w.Hq, w.Hkv, w.Sq, w.Skv, w.D, with_dout)


def doc_lengths(seed: int, S: int, lo: int = 512, hi: int = 4096) -> list:
    """Document lengths drawn uniformly from [lo, hi] until S is filled; the last is truncated."""
    rng = np.random.default_rng(seed)
    lengths = []
    total = 0
    while total < S:
        n = int(rng.integers(lo, hi, endpoint=True))
        n = min(n, S - total)
        lengths.append(n)
        total += n
    return lengths


def offsets_from_lengths(lengths) -> list:
    """Start offsets of consecutive documents plus the final end."""
    offs = [0]
    for n in lengths:
        offs.append(offs[-1] + int(n))
    return offs


def doc_offsets_for(w: Workload) -> list:
    """Per-batch-row document offsets of a workload (every row gets its own draw)."""
    return [offsets_from_lengths(doc_lengths(100 + w.seed + 1000 * b, w.Skv)) for b in range(w.B)]


def pad_offsets(offsets_per_b) -> tuple:
    """Pack ragged per-row offset lists into an int32 [B][num_docs+1] array.

    Rows with fewer documents repeat their final offset (empty documents).
    Returns (array, num_docs).
    """
    num_docs = max(len(o) - 1 for o in offsets_per_b)
    arr = np.empty((len(offsets_per_b), num_docs + 1), dtype=np.int32)
    for b, o in enumerate(offsets_per_b):
        arr[b, : len(o)] = o
        arr[b, len(o):] = o[-1]
    return arr, num_docs


def block_bitmap(seed: int, Sq: int, Skv: int) -> np.ndarray:
    """Bool [1][1][Sq][Skv] general mask: per 128 x 128 tile, dropped, kept, or
    kept element by element at a random density, with equal odds; the
    diagonal always kept."""
    rng = np.random.default_rng(seed)
    keep = np.zeros((Sq, Skv), dtype=bool)
    for q0 in range(0, Sq, 128):
        for k0 in range(0, Skv, 128):
            kind = int(rng.integers(3))
            blk = keep[q0:q0 + 128, k0:k0 + 128]
            if kind == 1:
                blk[...] = True
            elif kind == 2:
                blk[...] = rng.random(blk.shape) < rng.uniform(0.3, 0.9)
    d = np.arange(min(Sq, Skv))
    keep[d, d] = True
    return keep[None, None]


def mod_params_for(w: Workload, mod: str) -> ModParams:
    p = ModParams()
    if "document" in mod.split("+"):
        p.doc_offsets = doc_offsets_for(w)
    if mod == "bitmap":
        p.bitmap = block_bitmap(200 + w.seed, w.Sq, w.Skv)
    return p


def pack_bitmap(keep: np.ndarray) -> np.ndarray:
    """Bool [B'][H'][Sq][Skv] -> int32 words [B'][H'][Sq][4 ceil(Skv / 128)]: bit
    (j & 31) of word j >> 5 is element j; padding bits are zero."""
    keep = np.asarray(keep, dtype=bool)
    nb, nh, sq, skv = keep.shape
    rw = 4 * (-(-skv // 128))
    padded = np.zeros((nb, nh, sq, rw * 32), dtype=bool)
    padded[..., :skv] = keep
    bits = np.packbits(padded.reshape(nb, nh, sq, rw, 32), axis=-1, bitorder="little")
    return bits.reshape(nb, nh, sq, rw * 4).view(np.uint32).view(np.int32).copy()
