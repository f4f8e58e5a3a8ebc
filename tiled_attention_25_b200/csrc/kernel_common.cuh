// Shared pieces of the forward and backward kernels: work-list iteration over
// the block mask and per-row score transforms.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "mods.cuh"
#include "sm100.cuh"

namespace attn25 {

// Walks the KV tiles one 256-row query pair (query tiles qt0 = 2p, qt1 = 2p+1)
// must visit: the union of the two tiles' non-EMPTY KV lists, ascending.
// Every warp role runs its own copy and gets the same sequence.
struct PairIter {
  const int32_t* L0;  // kv_index row of qt0 (list mode) or nullptr (dense mode)
  const int32_t* L1;
  const uint8_t* C0;  // tile_class rows
  const uint8_t* C1;
  int n0, n1, i0, i1;
  // dense mode
  int k, k_end;
  int kind, window;
  int q0a, q1a, q0b, q1b;  // clipped row ranges of the two tiles (empty if q0 >= q1)
  int Skv, nK;
  bool tail;  // Skv is not a multiple of the tile
  bool list_mode;

  __device__ void init(const uint8_t* tile_class, const int32_t* kv_count, const int32_t* kv_index,
                       int b, int p, int nQ, int nK_, int Sq, int Skv_, int kind_, int window_) {
    nK = nK_;
    Skv = Skv_;
    kind = kind_;
    window = window_;
    tail = (Skv % TILE) != 0;
    const int qt0 = 2 * p, qt1 = 2 * p + 1;
    q0a = qt0 * TILE;
    q1a = min(Sq, q0a + TILE);
    q0b = qt1 * TILE;
    q1b = min(Sq, q0b + TILE);
    if (q1b < q0b) q1b = q0b;
    i0 = i1 = 0;
    list_mode = tile_class != nullptr;
    if (list_mode) {
      const size_t r0 = static_cast<size_t>(b) * nQ + qt0;
      L0 = kv_index + r0 * nK;
      C0 = tile_class + r0 * nK;
      n0 = __ldg(kv_count + r0);
      if (qt1 < nQ) {
        L1 = kv_index + (r0 + 1) * nK;
        C1 = tile_class + (r0 + 1) * nK;
        n1 = __ldg(kv_count + r0 + 1);
      } else {
        L1 = nullptr;
        C1 = nullptr;
        n1 = 0;
      }
      k = 0;
      k_end = 0;
    } else {
      L0 = L1 = nullptr;
      C0 = C1 = nullptr;
      n0 = n1 = 0;
      k = 0;
      k_end = nK;
      if (kind == MOD_CAUSAL || kind == MOD_WINDOW || kind == MOD_DOCUMENT) {
        const int last_row = max(q1a, q1b) - 1;
        k_end = min(nK, last_row / TILE + 1);
        if (kind == MOD_WINDOW) k = max(0, (q0a - window + 1) / TILE);
      }
    }
  }

  __device__ __forceinline__ int dense_class(int q0, int q1, int kt) const {
    if (q0 >= q1) return 0;
    if (kind == MOD_CAUSAL || kind == MOD_WINDOW)
      return interval_tile_class(kind, window, q0, q1, kt * TILE, min(Skv, kt * TILE + TILE));
    if (kind == MOD_DOCUMENT) return 1;
    return 2;
  }

  // Next step: KV tile kt; act0/act1: the query tile has work there;
  // part0/part1: the per-element predicate is needed there.
  __device__ bool next(int& kt, bool& act0, bool& act1, bool& part0, bool& part1) {
    const bool tail_tile_flag = tail;
    if (list_mode) {
      const int a = (i0 < n0) ? __ldg(L0 + i0) : 0x7fffffff;
      const int c = (i1 < n1) ? __ldg(L1 + i1) : 0x7fffffff;
      if (a == 0x7fffffff && c == 0x7fffffff) return false;
      kt = min(a, c);
      act0 = (a == kt);
      act1 = (c == kt);
      if (act0) ++i0;
      if (act1) ++i1;
      const bool t = tail_tile_flag && kt == nK - 1;
      part0 = act0 && (t || __ldg(C0 + kt) == 1);
      part1 = act1 && (t || __ldg(C1 + kt) == 1);
      return true;
    }
    while (k < k_end) {
      const int kk = k++;
      const int c0 = dense_class(q0a, q1a, kk);
      const int c1 = dense_class(q0b, q1b, kk);
      if (c0 == 0 && c1 == 0) continue;
      kt = kk;
      act0 = c0 != 0;
      act1 = c1 != 0;
      const bool t = tail_tile_flag && kt == nK - 1;
      part0 = act0 && (t || c0 == 1);
      part1 = act1 && (t || c1 == 1);
      return true;
    }
    return false;
  }
};

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
                                                int nK, int Sq, int Skv, int kind, int window,
                                                uint32_t* list) {
  const int lane = threadIdx.x & 31;
  const int qt0 = 2 * p, qt1 = 2 * p + 1;
  const bool has1 = qt1 < nQ;
  const int q0a = qt0 * TILE, q1a = min(Sq, q0a + TILE);
  const int q0b = qt1 * TILE, q1b = has1 ? min(Sq, q0b + TILE) : q0b;
  int k_begin = 0, k_end = nK;
  if (tile_class == nullptr && is_interval_mask(kind)) {
    k_end = min(nK, (max(q1a, q1b) - 1) / TILE + 1);
    if (kind == MOD_WINDOW) k_begin = max(0, (q0a - window + 1) / TILE);
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
        if (kind == MOD_CAUSAL || kind == MOD_WINDOW) {
          c0 = interval_tile_class(kind, window, q0a, q1a, k0, k1);
          c1 = has1 ? interval_tile_class(kind, window, q0b, q1b, k0, k1) : 0;
        } else {
          c0 = kind == MOD_DOCUMENT ? 1 : 2;
          c1 = has1 ? c0 : 0;
        }
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
                                               int nK, int Sq, int Skv, int kind, int window,
                                               uint16_t* list) {
  const int lane = threadIdx.x & 31;
  int q_begin = 0;
  if (tile_class == nullptr && is_interval_mask(kind)) q_begin = kt;  // every mask keeps q >= kv
  const bool tail_kv = (Skv % TILE) != 0 && kt == nK - 1;
  const int k0 = kt * TILE, k1 = min(Skv, k0 + TILE);
  int n = 0;
  for (int base = q_begin; base < nQ; base += 32) {
    const int qt = base + lane;
    int c = 0;
    if (qt < nQ) {
      if (tile_class != nullptr) {
        c = __ldg(tile_class + (static_cast<size_t>(b) * nQ + qt) * nK + kt);
      } else if (kind == MOD_CAUSAL || kind == MOD_WINDOW) {
        c = interval_tile_class(kind, window, qt * TILE, min(Sq, qt * TILE + TILE), k0, k1);
      } else {
        c = kind == MOD_DOCUMENT ? 1 : 2;
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
