// Score mods and masks applied inline on score tiles, plus tile classification.
//
// The mods are the FlexAttention-style score_mod / mask_mod set of "PyTorch
// FlexAttention, FlashAttention-4 백엔드 도입으로 성능 최대 3.2배 향상"
// (섹션별 상세: local_boost and tanh_softcap take the score and the raw
// q/kv indices; 핵심 요약: ALiBi, sliding window, document masks, and their
// composition, and arbitrary mask functions).  A mod is one score transform
// (none, ALiBi, softcap, local boost) and the AND of any of four masks.  Three
// keep, for query row i, an interval of keys: causal j <= i; sliding window
// i - W < j <= i; document: j <= i in i's document.  An intersection of
// intervals is an interval, so they keep one interval [lo(i), hi(i)] per row
// (and, transposed, one interval of queries per key).  The fourth is a bitmap
// of a general mask's values, read on PARTIAL tiles only.  The kind numbers
// are those of the C interface; only the score transforms are used here.
// Scores are handled in the base-2 domain: x = s' * log2(e), so that
// exp(s' - m) = 2^(x - m2).
#pragma once

#include <cstdint>

namespace attn25 {

constexpr int MOD_NONE = 0;
constexpr int MOD_ALIBI = 2;
constexpr int MOD_SOFTCAP = 3;
constexpr int MOD_BOOST = 5;

constexpr int TILE = 128;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

// Mask bits of a normalised mod (window and document imply causal).
constexpr int kMaskCausal = 1;
constexpr int kMaskWindow = 2;
constexpr int kMaskDoc = 4;
constexpr int kMaskBitmap = 8;  // a general mask given by its values, one bit per element
constexpr int kMaskVarlen = 16; // packed sequences with their own query and key lengths
// the masks that keep only keys at or before the query (kv <= q)
constexpr int kMaskCausalBits = kMaskCausal | kMaskWindow | kMaskDoc;

// Kernel specialisation key: the score transform (MOD_NONE, MOD_ALIBI,
// MOD_SOFTCAP or MOD_BOOST) plus kKeyMasked when any mask is present, and
// kKeyBitmap (always with kKeyMasked) when a bitmap mask is; which interval
// masks, and all parameters, are runtime values.
constexpr int kKeyMasked = 16;
constexpr int kKeyBitmap = 32;
__host__ __device__ constexpr int score_of(int key) { return key & (kKeyMasked - 1); }
__host__ __device__ constexpr bool masked(int key) { return (key & kKeyMasked) != 0; }
__host__ __device__ constexpr bool has_bitmap(int key) { return (key & kKeyBitmap) != 0; }

struct ModDev {
  int kind;                 // score transform: MOD_NONE, MOD_ALIBI, MOD_SOFTCAP or MOD_BOOST
  int mask;                 // kMask* bits
  float softcap;            // c
  int window;               // W (1 << 30 without the window mask)
  float boost;              // local boost factor
  int boost_radius;         // |i - j| < radius gets the boost
  const float* alibi_slopes;  // [Hq] or nullptr (then 2^(-8(h+1)/Hq))
  const int32_t* doc_offsets; // [B][num_docs + 1], nullptr without the document mask
  int num_docs;
  const uint32_t* bitmap;     // keep bits, nullptr without the bitmap mask
  int bm_row_words;           // words per query row (a multiple of 4)
  long long bm_head_stride;   // words between heads (0: shared)
  long long bm_batch_stride;  // words between batch rows (0: shared)
  const int32_t* vq_offsets;  // varlen mask: [B][n_seqs + 1] query and key starts plus ends
  const int32_t* vk_offsets;
  int n_seqs;
};

// First word of query row i of head h, batch row b in the keep bitmap.
__device__ __forceinline__ const uint32_t* bitmap_row(const ModDev& m, int b, int h, int i) {
  return m.bitmap + b * m.bm_batch_stride + h * m.bm_head_stride +
         static_cast<long long>(i) * m.bm_row_words;
}

// First key of the document that holds position i (offsets ascending, offs[0] = 0).
__device__ __forceinline__ int doc_start(const int32_t* offs, int num_docs, int i) {
  int lo = 0, hi = num_docs;  // invariant: offs[lo] <= i, answer index in [lo, hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(offs + mid) <= i) lo = mid; else hi = mid;
  }
  return __ldg(offs + lo);
}

// Index of the segment [offs[d], offs[d+1]) that holds position i (offsets
// ascending; empty segments repeat an offset and never hold a position).
__device__ __forceinline__ int segment_of(const int32_t* offs, int n, int i) {
  int lo = 0, hi = n;  // invariant: offs[lo] <= i, answer in [lo, hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(offs + mid) <= i) lo = mid; else hi = mid;
  }
  return lo;
}

// Kept key interval [lo, hi] of query row i (hi already clipped to Skv - 1):
// the intersection of the masks' intervals.  The varlen mask keeps the key
// range of the sequence that holds i.
__device__ __forceinline__ void row_interval(int mask, int window, const int32_t* offs_b,
                                             int num_docs, const int32_t* vq_b, const int32_t* vk_b,
                                             int n_seqs, int i, int Skv, int& lo, int& hi) {
  lo = 0;
  hi = Skv - 1;
  if (mask & kMaskCausalBits) hi = min(hi, i);
  if (mask & kMaskWindow) lo = max(lo, i - window + 1);
  if (mask & kMaskDoc) lo = max(lo, doc_start(offs_b, num_docs, i));
  if (mask & kMaskVarlen) {
    const int d = segment_of(vq_b, n_seqs, i);
    lo = max(lo, __ldg(vk_b + d));
    hi = min(hi, __ldg(vk_b + d + 1) - 1);
  }
}

__device__ __forceinline__ void row_interval(const ModDev& m, int b, int i, int Skv, int& lo,
                                             int& hi) {
  const size_t vb = static_cast<size_t>(b) * (m.n_seqs + 1);
  row_interval(m.mask, m.window,
               m.doc_offsets == nullptr ? nullptr
                                        : m.doc_offsets + static_cast<size_t>(b) * (m.num_docs + 1),
               m.num_docs, m.vq_offsets == nullptr ? nullptr : m.vq_offsets + vb,
               m.vk_offsets == nullptr ? nullptr : m.vk_offsets + vb, m.n_seqs, i, Skv, lo, hi);
}

__device__ __forceinline__ float alibi_slope(const ModDev& m, int h, int Hq) {
  if (m.alibi_slopes != nullptr) return __ldg(m.alibi_slopes + h);
  return exp2f(-8.0f * static_cast<float>(h + 1) / static_cast<float>(Hq));
}

// Class of the tile rows [q0, q1) x keys [k0, k1) (both already clipped to the
// sequence lengths) without a block mask: 0 EMPTY, 1 PARTIAL, 2 FULL, exact
// for the causal and window masks (kept iff i - W < j <= i), and with the
// document mask never FULL (its intervals need the offsets; PARTIAL tiles take
// the per-element predicate, which is always exact).
__host__ __device__ inline int dense_tile_class(int mask, int window, int q0, int q1, int k0,
                                                int k1) {
  if (mask == 0) return 2;
  if (mask & kMaskVarlen) return 1;  // the sequences' rectangles need the offsets
  const int W = (mask & kMaskWindow) ? window : (1 << 30);
  const int first_row = q0, last_row = q1 - 1;
  const bool any = (k0 <= last_row) && (k1 - 1 >= first_row - W + 1);
  if (!any) return 0;
  const bool all = (k1 - 1 <= first_row) && (k0 >= last_row - W + 1);
  return (all && !(mask & kMaskDoc)) ? 2 : 1;
}

}  // namespace attn25
