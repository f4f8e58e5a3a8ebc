"""Plain fp64 CPU oracle for exact scaled-dot-product attention with score mods.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this package; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
arm of ``bench.py`` use it.  It shares no code with the CUDA library.

What it computes (the plain definition, no tiling, no online softmax):

* Standard attention ``softmax(Q K^T * scale) V`` with the full score matrix
  formed element by element ("FlashAttention 설명", §1 어텐션의 실제 비용;
  "FlashAttention-2 — GPU attention의 사실상 표준", §2).  The tiled kernels
  are claimed to reach exactly this result, not an approximation
  ("FlashAttention 설명", §4 and §5), so the definition itself is the oracle.
* A FlexAttention-style score mod applied to the *scaled* score, then the mask
  (masked scores are -inf) ("PyTorch FlexAttention, FlashAttention-4 백엔드
  도입으로 성능 최대 3.2배 향상", 섹션별 상세: the ``local_boost`` and
  ``tanh_softcap`` examples take the score and the raw q/kv indices).
* Two-pass softmax per query row; outputs O and the natural-log logsumexp
  ``LSE = max + ln(sum)`` of the modded, scaled scores ("FlashInfer SM120
  NVFP4 어텐션 최적화", 코드 분석 1-2: the optional LSE output).
* The backward pass: the pages only say that scores are recomputed instead of
  stored ("FlashAttention-2 — GPU attention의 사실상 표준", §3 Recomputation);
  the plainest reading is the exact gradient of O with respect to Q, K, V,
  written out below.

Readings where the pages are silent:
  * mods see ``scale * q.k``; the mask is applied after the mod;
  * causal uses absolute indices, keep ``kv <= q``;
  * sliding window keeps ``0 <= q - kv < W``;
  * ALiBi bias ``-slope_h * |q - kv|`` with ``slope_h = 2^(-8 (h+1) / Hq)``,
    h counted from 0, on both sides of the diagonal, or the caller's slopes
    (``params.alibi_slopes[h]``) when given;
  * local boost multiplies by ``boost`` where ``|q - kv| < radius``;
  * document mask keeps ``doc(q) == doc(kv) and kv <= q``;
  * GQA: query head ``h`` reads KV head ``h // (Hq // Hkv)``;
  * a fully masked row has O = 0, LSE = -inf and zero gradient;
  * composition (FlexAttention composes score and mask mods, "PyTorch
    FlexAttention, FlashAttention-4 백엔드 …", 핵심 요약 and 섹션별 상세):
    a mod code is one of the seven kinds, optionally ORed with mask flags
    (``MASK_CAUSAL``, ``MASK_SLIDING_WINDOW``, ``MASK_DOCUMENT``).  The score
    transform is the base kind's; an element is kept only where the base kind
    and every flagged mask keep it (the logical AND of the masks);
  * a general mask_mod ("PyTorch FlexAttention, …", 핵심 요약: arbitrary
    mask functions) is given as its values: ``MASK_BITMAP`` keeps (b, h, i, j)
    where ``params.bitmap[b', h', i, j]`` is true, with b' = b and h' = h, or 0
    where the array's batch or head extent is 1 (shared by all);
  * packed variable-length sequences with their own query and key lengths
    (the pages' separate query and key lengths, "FlashInfer SM120 NVFP4 …",
    코드 분석 1-2): ``MASK_VARLEN`` keeps (i, j) where query i and key j
    belong to the same sequence d, i.e. q_offsets[b][d] <= i < q_offsets[b][d+1]
    and k_offsets[b][d] <= j < k_offsets[b][d+1]; it is not causal (a causal
    packing with equal lengths is the document mask) and takes no other mask.
"""
from __future__ import annotations

import numpy as np

MOD_NONE = 0
MOD_CAUSAL = 1
MOD_ALIBI = 2
MOD_SOFTCAP = 3
MOD_SLIDING_WINDOW = 4
MOD_LOCAL_BOOST = 5
MOD_DOCUMENT = 6

# Mask flags ORed onto a base kind to compose mods.
MASK_CAUSAL = 0x100
MASK_SLIDING_WINDOW = 0x200
MASK_DOCUMENT = 0x400
MASK_BITMAP = 0x800
MASK_VARLEN = 0x1000
_BITMAP = 0x100  # pseudo-kinds of the bitmap and varlen masks (never base kinds)
_VARLEN = 0x101
_FLAG_KIND = ((MASK_CAUSAL, MOD_CAUSAL), (MASK_SLIDING_WINDOW, MOD_SLIDING_WINDOW),
              (MASK_DOCUMENT, MOD_DOCUMENT), (MASK_BITMAP, _BITMAP), (MASK_VARLEN, _VARLEN))


def split_mod(mod):
    """(base kind, [mask kinds of the flags]) of a mod code; rejects unknown bits."""
    base, flags = int(mod) & 0xFF, int(mod) & ~0xFF
    if base > MOD_DOCUMENT or flags & ~(MASK_CAUSAL | MASK_SLIDING_WINDOW | MASK_DOCUMENT | MASK_BITMAP |
                                        MASK_VARLEN):
        raise ValueError(f"unknown mod {mod:#x}")
    masks = [kind for flag, kind in _FLAG_KIND if flags & flag]
    if _VARLEN in masks and (len(masks) > 1 or base in (MOD_CAUSAL, MOD_SLIDING_WINDOW, MOD_DOCUMENT)):
        raise ValueError(f"the varlen mask takes no other mask: {mod:#x}")
    return base, masks


def has_mask(mod) -> bool:
    """True when the mod masks any element (some kind in it is a mask)."""
    base, masks = split_mod(mod)
    return bool(masks) or base in (MOD_CAUSAL, MOD_SLIDING_WINDOW, MOD_DOCUMENT)


def has_bitmap(mod) -> bool:
    return bool(int(mod) & MASK_BITMAP)


def has_document(mod) -> bool:
    base, masks = split_mod(mod)
    return base == MOD_DOCUMENT or MOD_DOCUMENT in masks


def alibi_slope(h: int, Hq: int) -> float:
    """ALiBi slope of query head h (0-based): 2^(-8 (h+1) / Hq)."""
    return 2.0 ** (-8.0 * (h + 1) / Hq)


def doc_ids(offsets, S: int) -> np.ndarray:
    """Document index of every position 0..S-1 given ascending start offsets (+ end)."""
    ids = np.empty(S, dtype=np.int64)
    for d in range(len(offsets) - 1):
        ids[offsets[d]:offsets[d + 1]] = d
    return ids


def score_mod(s, mod, params, b, h, Hq, qi, kj):
    """Apply the score mod and the mask to scaled scores.

    s  : float64 [rows, cols] scaled scores scale * q.k
    qi : int64 [rows, 1] absolute query indices; kj : int64 [1, cols] key indices
    mod: a kind, optionally ORed with mask flags (composition)
    Returns (s_mod, keep, dmod): the modded score, the keep mask and the
    derivative d s_mod / d s (used by the backward pass).
    """
    base, masks = split_mod(mod)
    s_mod, keep, dmod = _single_mod(s, base, params, b, h, Hq, qi, kj)
    for kind in masks:
        _, keep_m, _ = _single_mod(s, kind, params, b, h, Hq, qi, kj)
        keep = keep & keep_m
    return s_mod, keep, dmod


def _single_mod(s, mod, params, b, h, Hq, qi, kj):
    """One kind of the set: (modded score, keep mask, d s_mod / d s)."""
    keep = np.ones(np.broadcast_shapes(s.shape, qi.shape, kj.shape), dtype=bool)
    dmod = np.ones_like(s)
    s_mod = s
    if mod == MOD_NONE:
        pass
    elif mod == MOD_CAUSAL:
        keep = kj <= qi
    elif mod == MOD_ALIBI:
        slopes = getattr(params, "alibi_slopes", None) if params is not None else None
        slope = alibi_slope(h, Hq) if slopes is None else float(slopes[h])
        s_mod = s - slope * np.abs(qi - kj)
    elif mod == MOD_SOFTCAP:
        c = params.softcap
        t = np.tanh(s / c)
        s_mod = c * t
        dmod = 1.0 - t * t
    elif mod == MOD_SLIDING_WINDOW:
        diff = qi - kj
        keep = (diff >= 0) & (diff < params.window)
    elif mod == MOD_LOCAL_BOOST:
        inside = np.abs(qi - kj) < params.boost_radius
        s_mod = np.where(inside, s * params.boost, s)
        dmod = np.where(inside, params.boost, 1.0) * np.ones_like(s)
    elif mod == _VARLEN:
        qo, ko = params.q_offsets[b], params.k_offsets[b]
        # sequence index of every query and key; positions past the last
        # offset belong to no sequence (-1 for queries, -2 for keys)
        seq_q = np.full(max(int(qi.max(initial=0)) + 1, qo[-1]), -1, dtype=np.int64)
        seq_k = np.full(max(int(kj.max(initial=0)) + 1, ko[-1]), -2, dtype=np.int64)
        for d in range(len(qo) - 1):
            seq_q[qo[d]:qo[d + 1]] = d
            seq_k[ko[d]:ko[d + 1]] = d
        keep = seq_q[qi] == seq_k[kj]
    elif mod == _BITMAP:
        bm = np.asarray(params.bitmap, dtype=bool)
        keep = bm[b if bm.shape[0] > 1 else 0, h if bm.shape[1] > 1 else 0][qi, kj]
    elif mod == MOD_DOCUMENT:
        offs = params.doc_offsets[b]
        S = int(max(qi.max(initial=0), kj.max(initial=0))) + 1
        ids = doc_ids(offs, max(S, offs[-1]))
        keep = (ids[qi] == ids[kj]) & (kj <= qi)
    else:
        raise ValueError(f"unknown mod {mod}")
    keep = np.broadcast_to(keep, s.shape)
    return s_mod, keep, dmod


def _row_softmax(s_mod, keep):
    """Two-pass softmax of one block of full rows; returns (P, LSE)."""
    x = np.where(keep, s_mod, -np.inf)
    m = x.max(axis=1)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(x - m_safe[:, None])
    l = e.sum(axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        P = np.where(l[:, None] > 0, e / l[:, None], 0.0)
        lse = np.where(l > 0, m_safe + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return P, lse


def _kv_head(h, Hq, Hkv):
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (Hq // Hkv)


def _chunks(rows, chunk):
    for i in range(0, len(rows), chunk):
        yield rows[i:i + chunk]


def attention_forward(q, k, v, scale, mod=MOD_NONE, params=None, heads=None,
                      rows=None, chunk=1024):
    """O and LSE of attention by the plain definition.

    q: float64 [B][Hq][Sq][D]; k, v: float64 [B][Hkv][Skv][D].
    heads: optional list of (b, h) pairs to compute (default all);
    rows:  optional sorted int array of query rows to compute (default all).
    Returns (O, LSE) with O [B][Hq][Sq][D] and LSE [B][Hq][Sq]; entries not
    computed are NaN.
    """
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, Dv = v.shape
    O = np.full((B, Hq, Sq, Dv), np.nan)
    LSE = np.full((B, Hq, Sq), np.nan)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(Hq)]
    row_ids = np.arange(Sq) if rows is None else np.asarray(rows, dtype=np.int64)
    kj = np.arange(Skv, dtype=np.int64)[None, :]
    for b, h in heads:
        hk = _kv_head(h, Hq, Hkv)
        for r in _chunks(row_ids, chunk):
            s = scale * (q[b, h, r] @ k[b, hk].T)
            s_mod, keep, _ = score_mod(s, mod, params, b, h, Hq, r[:, None], kj)
            P, lse = _row_softmax(s_mod, keep)
            O[b, h, r] = P @ v[b, hk]
            LSE[b, h, r] = lse
    return O, LSE


def attention_probs(q, k, scale, mod=MOD_NONE, params=None, b=0, h=0):
    """The full probability matrix P of one (b, h) (small inputs only)."""
    B, Hq, Sq, D = q.shape
    Hkv, Skv = k.shape[1], k.shape[2]
    hk = _kv_head(h, Hq, Hkv)
    s = scale * (q[b, h] @ k[b, hk].T)
    s_mod, keep, _ = score_mod(s, mod, params, b, h, Hq,
                               np.arange(Sq)[:, None], np.arange(Skv)[None, :])
    P, _ = _row_softmax(s_mod, keep)
    return P


def attention_backward(q, k, v, dout, scale, mod=MOD_NONE, params=None,
                       groups=None, q_rows=None, kv_rows=None, chunk=1024,
                       contrib_rows=None):
    """dQ, dK, dV of L = sum(dO * O) by the exact gradient formulas.

    With s = scale q.k, s' = mod(s), P = softmax_row(s' masked), O = P V:
        dV_j  = sum_{h in group} sum_i P_ij dO_i
        dP_ij = dO_i . v_j
        D_i   = sum_j P_ij dP_ij
        dS'_ij = P_ij (dP_ij - D_i),  dS_ij = dS'_ij * ds'/ds
        dQ_i  = scale sum_j dS_ij k_j
        dK_j  = scale sum_{h in group} sum_i dS_ij q_i
    groups: optional list of (b, hk) KV-head groups to compute (default all);
    q_rows / kv_rows: optional sorted index arrays restricting which rows of
    dQ and of dK/dV are returned (all query rows still enter dK/dV).
    contrib_rows: optional sorted query rows whose terms are summed into
    dK/dV (default: all rows).  Only for callers that know every other row's
    P_ij is exactly zero for the requested keys (e.g. causal masks, keys past
    the last excluded query), so that the sum is unchanged.
    Entries not computed are NaN.
    """
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, Dv = v.shape
    G = Hq // Hkv
    dq = np.full(q.shape, np.nan)
    dk = np.full(k.shape, np.nan)
    dv = np.full(v.shape, np.nan)
    if groups is None:
        groups = [(b, hk) for b in range(B) for hk in range(Hkv)]
    all_rows = np.arange(Sq, dtype=np.int64) if contrib_rows is None else np.asarray(contrib_rows, dtype=np.int64)
    kv_sel = np.arange(Skv) if kv_rows is None else np.asarray(kv_rows, dtype=np.int64)
    q_sel = None if q_rows is None else set(int(x) for x in q_rows)
    kj = np.arange(Skv, dtype=np.int64)[None, :]
    for b, hk in groups:
        dk_acc = np.zeros((len(kv_sel), D))
        dv_acc = np.zeros((len(kv_sel), Dv))
        for h in range(hk * G, (hk + 1) * G):
            for r in _chunks(all_rows, chunk):
                s = scale * (q[b, h, r] @ k[b, hk].T)
                s_mod, keep, dmod = score_mod(s, mod, params, b, h, Hq, r[:, None], kj)
                P, _ = _row_softmax(s_mod, keep)
                dP = dout[b, h, r] @ v[b, hk].T
                Di = (P * dP).sum(axis=1)
                dS = P * (dP - Di[:, None]) * dmod
                if q_sel is None:
                    dq[b, h, r] = scale * (dS @ k[b, hk])
                else:
                    pick = np.array([i for i, x in enumerate(r) if int(x) in q_sel], dtype=np.int64)
                    if len(pick):
                        dq[b, h, r[pick]] = scale * (dS[pick] @ k[b, hk])
                dk_acc += scale * (dS[:, kv_sel].T @ q[b, h, r])
                dv_acc += P[:, kv_sel].T @ dout[b, h, r]
        dk[b, hk, kv_sel] = dk_acc
        dv[b, hk, kv_sel] = dv_acc
    return dq, dk, dv


def online_forward(q, k, v, scale, mod=MOD_NONE, params=None, block=16):
    """Block-by-block online softmax (running max, running sum, rescaled output).

    Used only to check that the streaming update reaches the two-pass result
    ("FlashAttention 설명", §4 running statistics and §5 온라인 소프트맥스: when
    a block arrives the maximum is updated and earlier values are rescaled).
    The page's list of update steps is cut off after the rescale; the
    remaining steps are the standard ones: l <- l e^{m-m'} + sum e^{s-m'} and
    acc <- acc e^{m-m'} + sum e^{s-m'} v.  Small inputs only.
    """
    B, Hq, Sq, D = q.shape
    _, Hkv, Skv, Dv = v.shape
    O = np.zeros((B, Hq, Sq, Dv))
    LSE = np.zeros((B, Hq, Sq))
    qi = np.arange(Sq, dtype=np.int64)[:, None]
    for b in range(B):
        for h in range(Hq):
            hk = _kv_head(h, Hq, Hkv)
            m = np.full(Sq, -np.inf)
            l = np.zeros(Sq)
            acc = np.zeros((Sq, Dv))
            for j0 in range(0, Skv, block):
                kj = np.arange(j0, min(Skv, j0 + block), dtype=np.int64)[None, :]
                s = scale * (q[b, h] @ k[b, hk, j0:j0 + block].T)
                s_mod, keep, _ = score_mod(s, mod, params, b, h, Hq, qi, kj)
                x = np.where(keep, s_mod, -np.inf)
                m_new = np.maximum(m, x.max(axis=1))
                m_safe = np.where(np.isfinite(m_new), m_new, 0.0)
                alpha = np.where(np.isfinite(m), np.exp(m - m_safe), 0.0)
                p = np.exp(x - m_safe[:, None])
                l = l * alpha + p.sum(axis=1)
                acc = acc * alpha[:, None] + p @ v[b, hk, j0:j0 + block]
                m = m_new
            with np.errstate(invalid="ignore", divide="ignore"):
                O[b, h] = np.where(l[:, None] > 0, acc / np.where(l > 0, l, 1.0)[:, None], 0.0)
                LSE[b, h] = np.where(l > 0, np.where(np.isfinite(m), m, 0.0) + np.log(np.where(l > 0, l, 1.0)), -np.inf)
    return O, LSE


def useful_elements(mod, params, B, Hq, Sq, Skv) -> int:
    """Number of unmasked (b, h, q, kv) score elements (the useful-work count)."""
    qi = np.arange(Sq, dtype=np.int64)[:, None]
    kj = np.arange(Skv, dtype=np.int64)[None, :]
    # a per-head bitmap differs between heads; every other mask is shared by them
    per_head = has_bitmap(mod) and np.asarray(params.bitmap).shape[1] > 1
    total = 0
    for b in range(B):
        for h in range(Hq if per_head else 1):
            if has_mask(mod):
                n = 0
                for r0 in range(0, Sq, 2048):
                    r = qi[r0:r0 + 2048]
                    _, keep, _ = score_mod(np.zeros((len(r), Skv)), mod, params, b, h, Hq, r, kj)
                    n += int(keep.sum())
            else:
                n = Sq * Skv
            total += n * (1 if per_head else Hq)
    return total


def useful_flops(n_useful: int, D: int, backward: bool = False) -> float:
    """Useful FLOPs: two GEMMs (QK^T, PV) x 2 flop per MAC forward = 4 D per element.

    Backward counts five GEMMs (QK^T recompute, dP, dV, dK, dQ) = 10 D per element.
    The forward convention is the one the FlashInfer benchmark table uses
    ("FlashInfer SM120 NVFP4 어텐션 최적화", 성능: 4 B H S^2 D, causal halved).
    """
    return float(n_useful) * D * (10.0 if backward else 4.0)
