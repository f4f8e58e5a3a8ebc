// Shared pieces of the forward and backward kernels: the per-unit step lists
// built from the block mask (or, without one, from the masks' closed forms).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "mods.cuh"
#include "sm100.cuh"

namespace attn25 {

// ------------------------------------------------------------------ work walk
//
// The k-th unit a CTA processes, in the block mask's longest-first order:
// wave k covers ranks [k G, k G + G) (G = gridDim.x), CTA c takes rank
// k G + c on even waves and k G + G - 1 - c on odd ones.  Reversing every
// other wave pairs each CTA's long units with short ones, so per-CTA totals
// stay level when unit lengths fall steadily (causal, sliding-window and
// document masks); a plain round-robin gives CTA 0 the longest unit of every
// wave.  Every role of a CTA computes the same sequence; only the last wave
// can be partial, so the walk ends at the first rank past the unit count.
__device__ __forceinline__ int snake_unit(int k) {
  const int base = k * static_cast<int>(gridDim.x);
  return (k & 1) ? base + static_cast<int>(gridDim.x - 1 - blockIdx.x) : base + static_cast<int>(blockIdx.x);
}

// ------------------------------------------------------------------ step lists
//
// The TMA warp writes each work unit's list of steps into shared memory once
// (all 32 lanes, coalesced reads of the block mask), and every other role
// reads its steps from there: no role walks global memory per step.
constexpr int kMaxSteps = 2048;  // list capacity: key tiles (forward) / query tiles (backward)

// Forward step entry: key tile in bits 0-19; bit 20/21: query tile 0/1 has
// work there; bit 22/23: query tile 0/1 needs the element predicate.
constexpr uint32_t kStepAct0 = 1u << 20, kStepAct1 = 1u << 21;
constexpr uint32_t kStepPrt0 = 1u << 22, kStepPrt1 = 1u << 23;

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Executed by a whole warp; returns the number of steps (all lanes).
// tile_class == nullptr: dense iteration with closed-form classes.
__device__ __forceinline__ int build_pair_steps(const uint8_t* tile_class, int b, int p, int nQ,
                                                int nK, int Sq, int Skv, int mask, int window,
                                                uint32_t* list) {
  const int lane = threadIdx.x & 31;
  const int qt0 = 2 * p, qt1 = 2 * p + 1;
  const bool has1 = qt1 < nQ;
  const int q0a = qt0 * TILE, q1a = min(Sq, q0a + TILE);
  const int q0b = qt1 * TILE, q1b = has1 ? min(Sq, q0b + TILE) : q0b;
  int k_begin = 0, k_end = nK;
  if (tile_class == nullptr && (mask & kMaskCausalBits)) {
    k_end = min(nK, (max(q1a, q1b) - 1) / TILE + 1);
    if (mask & kMaskWindow) k_begin = max(0, (q0a - window + 1) / TILE);
  }
  const bool tail = (Skv % TILE) != 0;
  const uint8_t* r0 = tile_class == nullptr ? nullptr
                                            : tile_class + (static_cast<size_t>(b) * nQ + qt0) * nK;
  int n = 0;
  for (int base = k_begin; base < k_end; base += 32) {
    const int kt = base + lane;
    int c0 = 0, c1 = 0;
    if (kt < k_end) {
      if (r0 != nullptr) {
        c0 = __ldg(r0 + kt);
        c1 = has1 ? __ldg(r0 + nK + kt) : 0;
      } else {
        const int k0 = kt * TILE, k1 = min(Skv, k0 + TILE);
        c0 = dense_tile_class(mask, window, q0a, q1a, k0, k1);
        c1 = has1 ? dense_tile_class(mask, window, q0b, q1b, k0, k1) : 0;
      }
    }
    const bool active = (c0 | c1) != 0;
    const uint32_t ballot = __ballot_sync(0xffffffffu, active);
    if (active) {
      const int pos = n + __popc(ballot & lanemask_lt());
      const bool t = tail && kt == nK - 1;
      uint32_t e = static_cast<uint32_t>(kt);
      if (c0) e |= kStepAct0 | ((c0 == 1 || t) ? kStepPrt0 : 0u);
      if (c1) e |= kStepAct1 | ((c1 == 1 || t) ? kStepPrt1 : 0u);
      if (pos < kMaxSteps) list[pos] = e;
    }
    n += __popc(ballot);
  }
  return min(n, kMaxSteps);
}

// Backward step source: the query tiles (and their class) a key tile meets.
// Entries are 16 bits: the query-tile index, and bit 15 when the tile needs
// the element predicate.
constexpr uint32_t kQtPred16 = 1u << 15;
constexpr uint32_t kQtIndexMask = kQtPred16 - 1;
static_assert(kMaxSteps <= static_cast<int>(kQtIndexMask) + 1, "query-tile index width");

__device__ __forceinline__ int build_kv_qtiles(const uint8_t* tile_class, int b, int kt, int nQ,
                                               int nK, int Sq, int Skv, int mask, int window,
                                               uint16_t* list) {
  const int lane = threadIdx.x & 31;
  int q_begin = 0;
  if (tile_class == nullptr && (mask & kMaskCausalBits)) q_begin = kt;  // these masks keep q >= kv
  const bool tail_kv = (Skv % TILE) != 0 && kt == nK - 1;
  const int k0 = kt * TILE, k1 = min(Skv, k0 + TILE);
  int n = 0;
  for (int base = q_begin; base < nQ; base += 32) {
    const int qt = base + lane;
    int c = 0;
    if (qt < nQ) {
      if (tile_class != nullptr) {
        c = __ldg(tile_class + (static_cast<size_t>(b) * nQ + qt) * nK + kt);
      } else {
        c = dense_tile_class(mask, window, qt * TILE, min(Sq, qt * TILE + TILE), k0, k1);
      }
    }
    const uint32_t ballot = __ballot_sync(0xffffffffu, c != 0);
    if (c != 0) {
      const int pos = n + __popc(ballot & lanemask_lt());
      if (pos < kMaxSteps) list[pos] = static_cast<uint16_t>(static_cast<uint32_t>(qt) | ((c == 1 || tail_kv) ? kQtPred16 : 0u));
    }
    n += __popc(ballot);
  }
  return min(n, kMaxSteps);
}

}  // namespace attn25
