// Score mods and masks applied inline on score tiles, plus tile classification.
//
// The mods are the FlexAttention-style score_mod / mask_mod set of "PyTorch
// FlexAttention, FlashAttention-4 백엔드 도입으로 성능 최대 3.2배 향상"
// (섹션별 상세: local_boost and tanh_softcap take the score and the raw
// q/kv indices; 핵심 요약: ALiBi, sliding window, document masks).  Every
// mask of the set keeps, for query row i, an interval of keys
// [lo(i), hi(i)]:  causal lo = 0, hi = i;  sliding window lo = i - W + 1,
// hi = i;  document lo = start of the document holding i, hi = i.  Mods
// without a mask keep [0, Skv).  Scores are handled in the base-2 domain:
// x = s' * log2(e), so that exp(s' - m) = 2^(x - m2).
#pragma once

#include <cstdint>

namespace attn25 {

constexpr int MOD_NONE = 0;
constexpr int MOD_CAUSAL = 1;
constexpr int MOD_ALIBI = 2;
constexpr int MOD_SOFTCAP = 3;
constexpr int MOD_WINDOW = 4;
constexpr int MOD_BOOST = 5;
constexpr int MOD_DOCUMENT = 6;

constexpr int TILE = 128;
constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

__host__ __device__ constexpr bool is_interval_mask(int mod) {
  return mod == MOD_CAUSAL || mod == MOD_WINDOW || mod == MOD_DOCUMENT;
}

struct ModDev {
  int kind;
  float softcap;            // c
  int window;               // W
  float boost;              // local boost factor
  int boost_radius;         // |i - j| < radius gets the boost
  const float* alibi_slopes;  // [Hq] or nullptr (then 2^(-8(h+1)/Hq))
  const int32_t* doc_offsets; // [B][num_docs + 1]
  int num_docs;
};

// First key of the document that holds position i (offsets ascending, offs[0] = 0).
__device__ __forceinline__ int doc_start(const int32_t* offs, int num_docs, int i) {
  int lo = 0, hi = num_docs;  // invariant: offs[lo] <= i, answer index in [lo, hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(offs + mid) <= i) lo = mid; else hi = mid;
  }
  return __ldg(offs + lo);
}

// Kept key interval [lo, hi] of query row i (hi already clipped to Skv - 1).
__device__ __forceinline__ void row_interval(const ModDev& m, int b, int i, int Skv, int& lo,
                                             int& hi) {
  lo = 0;
  hi = Skv - 1;
  if (m.kind == MOD_CAUSAL) {
    hi = min(hi, i);
  } else if (m.kind == MOD_WINDOW) {
    hi = min(hi, i);
    lo = max(0, i - m.window + 1);
  } else if (m.kind == MOD_DOCUMENT) {
    hi = min(hi, i);
    lo = doc_start(m.doc_offsets + static_cast<size_t>(b) * (m.num_docs + 1), m.num_docs, i);
  }
}

__device__ __forceinline__ float alibi_slope(const ModDev& m, int h, int Hq) {
  if (m.alibi_slopes != nullptr) return __ldg(m.alibi_slopes + h);
  return exp2f(-8.0f * static_cast<float>(h + 1) / static_cast<float>(Hq));
}

// Class of the tile rows [q0, q1) x keys [k0, k1) (both already clipped to the
// sequence lengths) for interval masks, by exact counting of kept elements:
// 0 EMPTY, 1 PARTIAL, 2 FULL.  Used where the row intervals have closed forms.
__host__ __device__ inline int interval_tile_class(int kind, int window, int q0, int q1, int k0,
                                                   int k1) {
  if (kind == MOD_CAUSAL || kind == MOD_WINDOW) {
    // kept iff lo(i) <= j <= i with lo(i) = 0 (causal) or i - W + 1
    const int first_row = q0, last_row = q1 - 1;
    const bool any = (k0 <= last_row) &&
                     (kind == MOD_CAUSAL || k1 - 1 >= first_row - window + 1);
    if (!any) return 0;
    const bool all = (k1 - 1 <= first_row) &&
                     (kind == MOD_CAUSAL || k0 >= last_row - window + 1);
    return all ? 2 : 1;
  }
  return 1;
}

}  // namespace attn25
