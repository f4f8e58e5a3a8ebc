// Backward attention kernels for sm_100a.
//
// The scores are recomputed from Q, K and the saved logsumexp instead of
// being stored ("FlashAttention-2 — GPU attention의 사실상 표준", §3 item 2
// Recomputation, and §4 Architecture, its Backward item).  With s' = mod(scale q.k) and
// P = exp(s' - LSE), the exact gradient of O = P V is
//     dV = P^T dO,  dP = dO V^T,  Delta_i = rowsum(dO_i * O_i),
//     dS = P * (dP - Delta) * ds'/ds,  dQ = scale dS K,  dK = scale dS^T Q.
//
// Three kernels run on the stream:
//   bwd_prep     Delta and LSE * log2(e) per row; zero the fp32 dQ accumulator
//   bwd_main     persistent over (batch row, KV head, 128-key tile) units
//   bwd_dq_cast  dQ accumulator * scale -> bf16
// bwd_main keeps K and V of its key tile in shared memory and dK, dV in
// tensor memory while it walks every query head of the KV head's group and
// every non-empty 64-row query sub-tile.  Per step it computes, in the
// transposed (key-major) orientation so that one thread owns one key row:
//     S^T = K Q^T,  dP^T = V dO^T               (tcgen05, smem x smem)
//     P^T, dS^T                                  (4 warps, thread = key row)
//     dV += P^T dO  (P^T from tensor memory),  dK += dS^T Q,
//     dQ^T = K^T dS^T                            (tcgen05)
// and adds dQ into the fp32 accumulator with coalesced reductions performed
// in L2 (the order of the adds, and the last bits of dQ, vary run to run).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kernel_common.cuh"
#include "launch.h"


// Profiling builds: clock64 of event `id` of step `st` on CTA 0, written by
// lane 0 of the first warp of each role, for a window of steps.
#if defined(ATTN25_TRACE)
#define BWD_EV(st, id)                                                                          \
  do {                                                                                          \
    if (blockIdx.x == 0 && lane == 0 && ((warp & 3) == 0 || warp >= 12) && (st) >= ev_step0 && \
        (st) < ev_step0 + kEvSteps && a.trace != nullptr)                                       \
      a.trace[kTraceCounters - 128 + ((st) - ev_step0) * kEvPerStep + (id)] = clock64();         \
  } while (0)
#else
#define BWD_EV(st, id) \
  do {                 \
  } while (0)
#endif

namespace attn25 {

namespace {

constexpr int kBwdThreads = 512;
constexpr int BM = 64;  // query rows per step
static_assert(BM == 64, "the bitmap mask fetches two 32-query words per lane");
// Warpgroups: 0 = P^T, 1 = dS^T, 2 = dQ drain, 3 = MMA (warp 12), TMA (warp 13).
// No setmaxnreg split: every thread keeps the launch allocation (at most 128
// registers at 512 threads).  Without the split, ptxas can keep the polling
// loops of the waits out of line (one copy instead of one per wait site);
// the smaller code was measured 49% faster on the dense 4x8x4096x128
// workload (820 vs 550 TFLOP/s), the kernel being bound by instruction
// fetch with four distinct warp roles.

template <int D>
struct BwdCfg {
  static constexpr int kKVBytes = TILE * D * 2;           // one 128-key tile of K or V
  static constexpr int kQBytes = BM * D * 2;              // one 64-row tile of Q or dO
  static constexpr int kStageBytes = 2 * kQBytes + 1024;  // Q, dO, LSE2 and Delta rows
  static constexpr int kStages = 3;  // Q / dO / statistics stages
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKVBytes;
  static constexpr int kStageOff = 2 * kKVBytes;
  static constexpr int kDSOff = kStageOff + kStages * kStageBytes;  // two 128 x 64 bf16 buffers
  static constexpr int kDSBytes = TILE * BM * 2;
  static constexpr int kBarOff = kDSOff + 2 * kDSBytes;
  static constexpr int kListOff = kBarOff + 1024;  // two query-tile lists (16-bit entries)
  // deterministic dQ: for each list entry, how many key tiles before this
  // unit's add into that query tile (16-bit entries, two lists)
  static constexpr int kPosOff = kListOff + 2 * kMaxSteps * 2;
  static constexpr int kSmemBytes = kPosOff + 2 * kMaxSteps * 2;
  static constexpr int kAllocBytes = kSmemBytes + 1024;
  static_assert(kAllocBytes <= 232448, "shared memory");
  // TMEM columns: two S^T buffers (P^T overwrites their first 32 columns), dP^T,
  // the dV and dK accumulators, dQ^T
  static constexpr int kColS = 0, kColDP = 128, kColDV = 192, kColDK = 192 + D, kColDQ = 192 + 2 * D;
  static_assert(kColDQ + BM <= 512, "TMEM columns");
  static constexpr uint32_t kIdescST = idesc_bf16_f32(128, BM, false, false);   // K Q^T, V dO^T
  static constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, false, true);    // P^T dO, dS^T Q
  static constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, BM, true, true);     // K^T dS^T
};

struct BwdBarriers {
  alignas(16) uint32_t clc_resp[4];  // cluster launch control response (the next unit)
  uint64_t clc_bar;
  uint64_t list_full[2], list_empty[2];
  uint64_t kv_full, kv_empty;
  uint64_t q_full[4], q_empty[4];
  uint64_t s_full[2], p_ready[2];
  uint64_t dp_full, dp_empty, ds_ready[2];
  uint64_t ds_empty[2];
  uint64_t dq_full;
  uint64_t acc_full, acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort_flag;
  uint32_t never_set;  // abort word for drain waits that must not stop early
  int32_t list_n[2];   // lengths of the two query-tile lists
  int32_t list_unit[2];  // cluster launch control: the unit of each list; -1 ends the walk
};

// Consumers of a query-tile list: the MMA warp and the P, dS and drain warps
// (lane 0 each).
constexpr int kBwdListConsumers = 13;
constexpr int kDrainWarps = 4;

struct BwdUnit {
  int b, hk, kt;
};

template <int MOD>
__device__ __forceinline__ BwdUnit decode_bwd_unit(const BwdArgs& a, int u) {
  const int pair_idx = u / a.Hkv;
  BwdUnit r;
  r.hk = u - pair_idx * a.Hkv;
  if (a.dq_sem != nullptr) {
    // deterministic dQ: ascending key tiles (across batch rows and KV heads),
    // so that every unit waits only on units of lower rank
    r.kt = pair_idx / a.B;
    r.b = pair_idx - r.kt * a.B;
    return r;
  }
  // The block mask's longest-first order of (batch row, key tile), with the
  // KV head either inside it (units of equal length for every head run side
  // by side: the balance that causal and sliding-window masks need) or
  // outside it (the units running side by side share their query heads, so
  // the Q and dO tiles and dQ accumulator rows they stream stay in L2: no
  // mask, or documents, whose units of many heads would otherwise stream many
  // documents' rows at once).  Measured on one B200, backward TFLOP/s, head
  // outside against inside: dense 835 -> 854, documents 472 -> 537, ALiBi
  // 812 -> 849, local boost 781 -> 796; causal 680 -> 606 and sliding window
  // 558 -> 518 (the balance), softcap 706 -> 643 (its slower steps keep the
  // units of one head in step, all adding into the same dQ rows at once).
  int pi;
  if (score_of(MOD) == MOD_SOFTCAP || ((a.mod.mask & kMaskCausal) != 0 && (a.mod.mask & kMaskDoc) == 0)) {
    pi = pair_idx;
  } else {
    const int n_pairs = a.B * a.nK;
    r.hk = u / n_pairs;
    pi = u - r.hk * n_pairs;
  }
  const int pair = (a.bwd_order != nullptr) ? __ldg(a.bwd_order + pi) : pi;
  r.b = pair / a.nK;
  r.kt = pair - r.b * a.nK;
  return r;
}

// Walks the steps of one unit from its query-tile list in shared memory: for
// each query head of the group, each listed 128-row query tile, and each
// 64-row half of it that starts inside Sq.
struct StepIter {
  const uint16_t* list;
  int n, G, Sq;
  int g, j, half;
  uint32_t cur;

  __device__ __forceinline__ void init(const uint16_t* list_, int n_, int G_, int Sq_) {
    list = list_;
    n = n_;
    G = G_;
    Sq = Sq_;
    g = 0;
    j = 0;
    half = 2;
    cur = 0;
  }

  // Next step: head offset g_out in the group, first query row q0, and
  // whether the element predicate is needed.
  __device__ __forceinline__ bool next(int& g_out, int& q0, bool& pred) {
    while (true) {
      if (half >= 2) {
        if (j >= n) {
          j = 0;
          if (++g >= G) return false;
          if (n == 0) return false;
        }
        cur = list[j++];
        half = 0;
      }
      const int start = static_cast<int>(cur & kQtIndexMask) * TILE + (half++) * BM;
      if (start >= Sq) continue;
      g_out = g;
      q0 = start;
      pred = (cur & kQtPred16) != 0;
      return true;
    }
  }

  // List index of the entry of the last step next() returned.
  __device__ __forceinline__ int entry() const { return j - 1; }
};

// ------------------------------------------------------------------ deterministic dQ
//
// Every key tile that meets a query tile adds its dQ part into the fp32
// accumulator; to make the sum's order fixed, the adds into each block of 64
// query rows (and each 32-column slice, one per drain warp) are ordered by
// key tile: a counter per (row block, slice) holds how many key tiles have
// added, and the unit of key tile kt waits until it equals the number of
// key tiles before kt that meet the query tile (its position).  Units are
// walked in ascending key-tile order and each CTA takes them in ascending
// rank, so a unit only ever waits on units of lower rank, which are running
// or done on other CTAs (all CTAs are resident: one per SM).

// Positions of the list entries of key tile kt (whole warp): the lower bound
// of kt in the block mask's ascending key-tile list of each query tile, or,
// without a block mask, the count of earlier key tiles with a non-empty dense
// class (the same classes the units' step lists come from).
__device__ __forceinline__ void build_positions(const BwdArgs& a, int b, int kt, const uint16_t* lst,
                                                int n, uint16_t* pos) {
  __syncwarp();  // the list entries were written by other lanes
  for (int j = threadIdx.x & 31; j < n; j += 32) {
    const int qt = static_cast<int>(lst[j] & kQtIndexMask);
    int p = 0;
    if (a.kv_index != nullptr) {
      const size_t r = static_cast<size_t>(b) * a.nQ + qt;
      const int32_t* row = a.kv_index + r * a.nK;
      int hi = __ldg(a.kv_count + r);
      while (p < hi) {
        const int mid = (p + hi) >> 1;
        if (__ldg(row + mid) < kt) p = mid + 1; else hi = mid;
      }
    } else {
      const int q0 = qt * TILE, q1 = min(a.Sq, q0 + TILE);
      for (int k2 = 0; k2 < kt; ++k2)
        p += dense_tile_class(a.mod.mask, a.mod.window, q0, q1, k2 * TILE, min(a.Skv, k2 * TILE + TILE)) != 0;
    }
    pos[j] = static_cast<uint16_t>(p);
  }
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Warp-collective: wait (bounded) until the counter equals `want`; every lane
// then holds an acquire of it, so its reductions follow the earlier adds.
static __device__ __noinline__ bool sem_wait_eq(const unsigned* sem, unsigned want, WaitCtl w) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) {
    uint64_t t0 = 0;
    bool timed = false;
    while (ld_acquire_gpu(sem) != want) {
      if (aborted(w)) {
        ok = false;
        break;
      }
      const uint64_t t = globaltimer();
      if (!timed) {
        t0 = t;
        timed = true;
      } else if (t - t0 > w.limit_ns) {
        record_error(kErrTimeout, w);
        ok = false;
        break;
      }
    }
  }
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok) (void)ld_acquire_gpu(sem);
  return ok;
}

// Warp-collective: publish this warp's adds (each lane fences its own), then count them.
__device__ __forceinline__ void sem_release(unsigned* sem) {
  __threadfence();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) atomicAdd(sem, 1u);
}

// Tiles of head h of batch row b through 4-D tensor maps (D, S, H, B).
template <int D>
__device__ __forceinline__ void load_kv_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                             int row0, int h, int b) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) tma_load_4d(dst + c * (TILE * 128), map, bar, c * 64, row0, h, b);
}

template <int D>
__device__ __forceinline__ void load_q_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int row0, int h, int b) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) tma_load_4d(dst + c * (BM * 128), map, bar, c * 64, row0, h, b);
}

__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes,
                                             uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// A (M=128 rows) x B^T with both operands K-major, 128-byte swizzle; the
// M-side tile has 128 rows (chunk stride 16 KB), the N-side 64 rows (8 KB).
template <int D>
__device__ __forceinline__ void issue_st(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t ka = (kk >> 2) * (TILE * 128) + (kk & 3) * 32;
    const uint32_t kb = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
    mma_ss_w(d_tmem, smem_desc_sw128(a_smem + ka, 16, 1024), smem_desc_sw128(b_smem + kb, 16, 1024),
             BwdCfg<D>::kIdescST, kk > 0 ? 1u : 0u);
  }
}


// Kept query interval of key row kv (the transposed form of the row
// intervals, intersected over the masks): every mask keeps q >= kv; the
// window keeps q < kv + W; the document keeps q before the end of kv's
// document; key rows past Skv keep nothing.
template <int MOD>
__device__ __forceinline__ void key_interval(const BwdArgs& a, int b, int kv, int& qlo, int& qhi) {
  qlo = 0;
  qhi = a.Sq - 1;
  if constexpr (masked(MOD)) {
    const int mask = a.mod.mask;
    if (mask & kMaskCausalBits) qlo = kv;
    if (mask & kMaskWindow) qhi = min(qhi, kv + a.mod.window - 1);
    if (mask & kMaskDoc) {
      const int32_t* offs = a.mod.doc_offsets + static_cast<size_t>(b) * (a.mod.num_docs + 1);
      const int kvc = min(kv, a.Skv - 1);
      int lo = 0, hi = a.mod.num_docs;  // the document holding kvc, then its end
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(offs + mid) <= kvc) lo = mid; else hi = mid;
      }
      qhi = min(qhi, __ldg(offs + lo + 1) - 1);
    }
    if (mask & kMaskVarlen) {  // the query range of the sequence that holds the key
      const size_t vb = static_cast<size_t>(b) * (a.mod.n_seqs + 1);
      const int d = segment_of(a.mod.vk_offsets + vb, a.mod.n_seqs, min(kv, a.Skv - 1));
      qlo = max(qlo, __ldg(a.mod.vq_offsets + vb + d));
      qhi = min(qhi, __ldg(a.mod.vq_offsets + vb + d + 1) - 1);
    }
  }
  if (kv >= a.Skv) qhi = qlo - 1;
}

__device__ __forceinline__ float4 lds128(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

// Whether query q0 + c is kept for this thread's key on a PARTIAL step: inside
// the key's query interval and, with the bitmap mask, set in the bitmap.
// wa / wb hold (lane l) the keep-bit word of query q0 + l / q0 + 32 + l over
// this warp's 32 keys; bit (key & 31) keeps.  The whole warp must call it.
template <int MOD>
__device__ __forceinline__ bool keep_query(int c, int q0, int qlo, int qhi, uint32_t wa, uint32_t wb) {
  const int qq = q0 + c;
  bool keep = qq >= qlo && qq <= qhi;
  if constexpr (has_bitmap(MOD)) {
    const uint32_t w = __shfl_sync(0xffffffffu, c < 32 ? wa : wb, c & 31);
    keep = keep && ((w >> (threadIdx.x & 31)) & 1u) != 0u;
  }
  return keep;
}

// Whether the local boost band |q - kv| < radius meets any of this warp's
// steps (dq0 = q0 - kv of the thread's key); warp-uniform.
__device__ __forceinline__ bool boost_band_meets(const BwdArgs& a, float dq0) {
  const float rad = static_cast<float>(a.mod.boost_radius);
  return !__all_sync(0xffffffffu, dq0 >= rad || dq0 + static_cast<float>(BM - 1) <= -rad);
}

// One key row of S^T (raw q.k for 64 queries) -> P^T = 2^(x - LSE2) in place;
// nl2_addr is the shared address of the 64 negated base-2 LSEs.  Every mod
// shares one exponential loop: the boost multiplies the raw scores in a pass
// of its own that runs only where the band meets the warp's step, and the
// mask runs after the exponentials (P = 0 where masked, the same as 2^-inf).
template <int MOD>
__device__ __forceinline__ void probs_t(float (&x)[BM], const BwdArgs& a, int h, float dq0, int q0, int qlo,
                                        int qhi, bool pred, uint32_t nl2_addr, uint32_t wa, uint32_t wb) {
  float aux = 0.f;
  if constexpr (score_of(MOD) == MOD_ALIBI) aux = alibi_slope(a.mod, h, a.Hq) * LOG2E;
  if constexpr (score_of(MOD) == MOD_BOOST) {
    if (boost_band_meets(a, dq0)) {
      // columns c with |dq0 + c| < radius: c_lo <= c <= c_hi
      const int d = static_cast<int>(dq0), rad = a.mod.boost_radius;
      const int c_lo = -rad - d + 1, c_hi = rad - d - 1;
#pragma unroll
      for (int c = 0; c < BM; ++c) x[c] *= (c >= c_lo && c <= c_hi) ? a.mod.boost : 1.f;
    }
  }
  const float2 sl2 = make_float2(a.sl2, a.sl2);
#pragma unroll
  for (int c4 = 0; c4 < BM / 4; ++c4) {
    const float4 l = lds128(nl2_addr + c4 * 16);
#pragma unroll
    for (int hp = 0; hp < 2; ++hp) {
      const int c = c4 * 4 + hp * 2;
      const float2 nl = hp == 0 ? make_float2(l.x, l.y) : make_float2(l.z, l.w);
      float2 v;
      if constexpr (score_of(MOD) == MOD_ALIBI) {
        v.x = fmaf(x[c], a.sl2, -aux * fabsf(dq0 + static_cast<float>(c))) + nl.x;
        v.y = fmaf(x[c + 1], a.sl2, -aux * fabsf(dq0 + static_cast<float>(c + 1))) + nl.y;
      } else {
        v = __ffma2_rn(make_float2(x[c], x[c + 1]), sl2, nl);
      }
      x[c] = ex2_approx(v.x);  // 0 on padding rows (-LSE2 = -inf)
      x[c + 1] = ex2_approx(v.y);
    }
  }
  if (pred) {  // PARTIAL steps only
#pragma unroll
    for (int c = 0; c < BM; ++c) x[c] = keep_query<MOD>(c, q0, qlo, qhi, wa, wb) ? x[c] : 0.f;
  }
}

// Softcap keeps each 32-query half of an S^T buffer as [P^T | P ds'/ds]: 16
// columns of P^T bf16 pairs (the A operand of dV += P^T dO) and 16 of
// P (1 - tanh^2), the factor the dS warps take (the derivative of
// c tanh(s / c)); the other mods keep P^T in the buffer's first 32 columns.
template <int MOD>
constexpr bool kSoftcapHalves = score_of(MOD) == MOD_SOFTCAP;
// TMEM column, within an S^T buffer, of P^T's 16-query K-chunk kk
template <int MOD>
__device__ __forceinline__ constexpr uint32_t p_col(int kk) {
  return kSoftcapHalves<MOD> ? static_cast<uint32_t>((kk >> 1) * 32 + (kk & 1) * 8) : static_cast<uint32_t>(kk * 8);
}

// Softcap, one 32-query half (columns t_half ...) of a key row of S^T:
// P = 2^(c log2(e) tanh(scale x / c) - LSE2) and P (1 - tanh^2), masked on
// PARTIAL steps, stored as bf16 pairs over the half's columns.  One loop body
// serves both halves (the warp's hot code stays small).
template <int MOD>
__device__ __forceinline__ void softcap_half(uint32_t t_half, int hf, const BwdArgs& a, int q0, int qlo,
                                             int qhi, bool pred, uint32_t nl2_addr, uint32_t wa, uint32_t wb) {
  float x[32];
  tmem_ld32(t_half, reinterpret_cast<uint32_t(&)[32]>(x[0]));
  tmem_wait_ld();
  const float aux = a.scale / a.mod.softcap, aux2 = a.mod.softcap * LOG2E;
  uint32_t pk[16], pd[16];
#pragma unroll
  for (int c4 = 0; c4 < 8; ++c4) {
    const float4 l = lds128(nl2_addr + (hf * 8 + c4) * 16);
#pragma unroll
    for (int hp = 0; hp < 2; ++hp) {
      const int c = c4 * 4 + hp * 2;
      const float2 nl = hp == 0 ? make_float2(l.x, l.y) : make_float2(l.z, l.w);
      const float t0 = tanh_ex2(x[c] * aux), t1 = tanh_ex2(x[c + 1] * aux);
      const float p0 = ex2_approx(fmaf(aux2, t0, nl.x)), p1 = ex2_approx(fmaf(aux2, t1, nl.y));  // 0 on padding rows
      pk[c >> 1] = pack_bf16x2(p0, p1);
      pd[c >> 1] = pack_bf16x2(p0 * fmaf(-t0, t0, 1.f), p1 * fmaf(-t1, t1, 1.f));
    }
  }
  if (pred) {  // PARTIAL steps only
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t keep = (keep_query<MOD>(hf * 32 + 2 * e, q0, qlo, qhi, wa, wb) ? 0x0000ffffu : 0u) |
                            (keep_query<MOD>(hf * 32 + 2 * e + 1, q0, qlo, qhi, wa, wb) ? 0xffff0000u : 0u);
      pk[e] &= keep;
      pd[e] &= keep;
    }
  }
  tmem_st16(t_half, pk);
  tmem_st16(t_half + 16, pd);
}

// One accumulator row (dV or dK) of this thread's key: TMEM fp32 -> mul -> bf16 -> global.
// N 32-column chunks per TMEM round trip (two, except where the kernel's
// registers allow only one); 32-byte stores where the row allows them.
template <int D, int N>
__device__ __forceinline__ void store_acc_rows(__nv_bfloat16* dst, uint32_t src, float mul, bool have,
                                               bool row_ok) {
  const bool wide = (reinterpret_cast<uintptr_t>(dst) & 31u) == 0;
#pragma unroll
  for (int c2 = 0; c2 < D / (32 * N); ++c2) {
    uint32_t o[N][32];
#pragma unroll
    for (int h = 0; h < N; ++h) {
      if (have) {
        tmem_ld32(src + (N * c2 + h) * 32, o[h]);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[h][e] = 0u;
      }
    }
    if (have) tmem_wait_ld();
#pragma unroll
    for (int h = 0; h < N; ++h) {
      const int c = N * c2 + h;
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pk[e] = pack_bf16x2(__uint_as_float(o[h][2 * e]) * mul, __uint_as_float(o[h][2 * e + 1]) * mul);
      if (row_ok) {
        if (wide) {
#pragma unroll
          for (int e = 0; e < 2; ++e) st_global_v8(dst + c * 32 + e * 16, &pk[8 * e]);
        } else {
          uint4* p = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) p[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
    }
  }
}

template <int D, int MOD, bool CLC>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const BwdArgs a) {
  using Cfg = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  BwdBarriers* bars = reinterpret_cast<BwdBarriers*>(smem + Cfg::kBarOff);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t k_smem = sbase + Cfg::kKOff;
  const uint32_t v_smem = sbase + Cfg::kVOff;
  uint16_t* lists = reinterpret_cast<uint16_t*>(smem + Cfg::kListOff);
  uint16_t* positions = reinterpret_cast<uint16_t*>(smem + Cfg::kPosOff);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->list_full[i]), 32);
      mbar_init(smem_u32(&bars->list_empty[i]), kBwdListConsumers);
    }
    mbar_init(smem_u32(&bars->kv_full), 1);
    mbar_init(smem_u32(&bars->kv_empty), 1);
    mbar_init(smem_u32(&bars->clc_bar), 1);
    for (int b = 0; b < Cfg::kStages; ++b) {
      mbar_init(smem_u32(&bars->q_full[b]), 1);
      mbar_init(smem_u32(&bars->q_empty[b]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->ds_empty[b]), kDrainWarps);
      mbar_init(smem_u32(&bars->s_full[b]), 1);
      mbar_init(smem_u32(&bars->p_ready[b]), 128);
    }
    mbar_init(smem_u32(&bars->dp_full), 1);
    mbar_init(smem_u32(&bars->dp_empty), 128);
    // one slot per step parity: 128 dS threads (dS^T(j) stored) and 128 drain
    // threads (dQ^T(j-1) read)
    for (int b = 0; b < 2; ++b) mbar_init(smem_u32(&bars->ds_ready[b]), 256);
    mbar_init(smem_u32(&bars->dq_full), 1);
    mbar_init(smem_u32(&bars->acc_full), 1);
    mbar_init(smem_u32(&bars->acc_empty), 256);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort_flag = 0;
    bars->never_set = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == 13 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl wc{a.wait_ns, smem_u32(&bars->abort_flag), a.status};
  long long tr[12] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0};
  (void)tr;
  // first step of the event window (profiling builds): the host stores it in
  // the last backward counter word
  ATTN25_TRACE_ONLY(const int ev_step0 = a.trace != nullptr ? static_cast<int>(a.trace[127]) : 0;)
  ATTN25_TRACE_ONLY(const long long t_start = clock64();)

  if (warp >= 12) {
    if (warp == 13) {
      // ---------------------------------------------------------- TMA producer
      // all lanes build the query-tile lists; lane 0 issues the copies
      int unit_iter = 0, step = 0;
      uint32_t kv_loads = 0, clc_asked = 0, clc_read = 0;
      const uint32_t clc_resp = smem_u32(bars->clc_resp), clc_bar = smem_u32(&bars->clc_bar);
      bool ok = true;
      // The static walk: the snake over the order.  Cluster launch control (one
      // CTA launched per unit): this CTA's own unit, then the unit of each
      // not-yet-started CTA the hardware cancels for it; each list is published
      // with its unit's rank, and rank -1 ends every role's walk.
      for (int u = CLC ? static_cast<int>(blockIdx.x) : snake_unit(0); ok; ++unit_iter) {
        if constexpr (!CLC) {
          if (u >= a.n_units) break;
        }
        const int buf = unit_iter & 1;
        uint16_t* lst = lists + buf * kMaxSteps;
        BwdUnit un{};
        if constexpr (!CLC) un = decode_bwd_unit<MOD>(a, u);
        if (!mbar_wait_warp_ool(smem_u32(&bars->list_empty[buf]), ((unit_iter >> 1) & 1) ^ 1, wc)) { ok = false; break; }
        int n = 0;
        if constexpr (CLC) {
          if (u >= a.n_units) u = -1;
          if (u >= 0) un = decode_bwd_unit<MOD>(a, u);
          if (lane == 0) bars->list_unit[buf] = u;
        }
        if (u >= 0) {
          n = build_kv_qtiles(a.tile_class, un.b, un.kt, a.nQ, a.nK, a.Sq, a.Skv, a.mod.mask, a.mod.window, lst);
          if (a.dq_sem != nullptr) build_positions(a, un.b, un.kt, lst, n, positions + buf * kMaxSteps);
        }
        if (lane == 0) bars->list_n[buf] = n;
        mbar_arrive(smem_u32(&bars->list_full[buf]));
        if constexpr (CLC) {
          if (u < 0) break;
          if (lane == 0) {  // ask for the next unit now; the answer lands while this one streams
            mbar_arrive_expect_tx(clc_bar, 16);
            clc_try_cancel(clc_resp, clc_bar);
            ++clc_asked;
          }
        }
        if (lane == 0) {
          if (!ATTN25_TIMED(tr[1], mbar_wait_thread_ool(smem_u32(&bars->kv_empty), (unit_iter & 1) ^ 1, wc))) {
            ok = false;
          } else {
            mbar_arrive_expect_tx(smem_u32(&bars->kv_full), 2 * Cfg::kKVBytes);
            ++kv_loads;
            load_kv_tile<D>(k_smem, &tm_k, smem_u32(&bars->kv_full), un.kt * TILE, un.hk, un.b);
            load_kv_tile<D>(v_smem, &tm_v, smem_u32(&bars->kv_full), un.kt * TILE, un.hk, un.b);
            StepIter it;
            it.init(lst, n, a.G, a.Sq);
            int g, q0;
            bool pred;
            while (it.next(g, q0, pred)) {
              const int s = step % Cfg::kStages;
              if (!ATTN25_TIMED(tr[2], mbar_wait_thread_ool(smem_u32(&bars->q_empty[s]), ((step / Cfg::kStages) & 1) ^ 1, wc))) { ok = false; break; }
              const uint32_t st = sbase + Cfg::kStageOff + s * Cfg::kStageBytes;
              const uint32_t bar = smem_u32(&bars->q_full[s]);
              mbar_arrive_expect_tx(bar, 2 * Cfg::kQBytes + 2 * BM * 4);
              const int bh = un.b * a.Hq + un.hk * a.G + g;
              BWD_EV(step, 0);
              load_q_tile<D>(st, &tm_q, bar, q0, un.hk * a.G + g, un.b);
              load_q_tile<D>(st + Cfg::kQBytes, &tm_do, bar, q0, un.hk * a.G + g, un.b);
              const size_t row = static_cast<size_t>(bh) * a.Sq_pad + q0;
              bulk_load_1d(st + 2 * Cfg::kQBytes, a.lse2 + row, BM * 4, bar);
              bulk_load_1d(st + 2 * Cfg::kQBytes + 512, a.delta + row, BM * 4, bar);
              ++step;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if constexpr (CLC) {  // the next unit: the rank of the cancelled CTA, or -1
          if (!mbar_wait_warp_ool(clc_bar, clc_read & 1, wc)) { ok = false; break; }
          ++clc_read;
          u = clc_cancelled_x(clc_resp);
        } else {
          u = snake_unit(unit_iter + 1);
        }
      }
      if (lane == 0) {
        // let the copies in flight land before the CTA exits (also after a
        // normal end: a consumer that gave up may have left them unconsumed)
        const WaitCtl dwc{drain_limit(a.wait_ns), smem_u32(&bars->never_set), a.status};
        if (clc_asked > clc_read) mbar_wait_thread_ool(clc_bar, (clc_asked - 1) & 1, dwc);
        if (kv_loads) mbar_wait_thread_ool(smem_u32(&bars->kv_full), (kv_loads - 1) & 1, dwc);
        // stage s took the loads of steps s, s + kStages, ... below `step`
        for (int s = 0; s < Cfg::kStages && s < step; ++s)
          mbar_wait_thread_ool(smem_u32(&bars->q_full[s]), ((step - 1 - s) / Cfg::kStages) & 1, dwc);
      }
      ATTN25_TRACE_ONLY(tr[0] = clock64() - t_start;)
      trace_flush(a.trace, 48, tr);
    } else if (warp == 12) {
      // ---------------------------------------------------------- MMA issuer
      // Per step j (global step counter; S^T buffer j & 1, stage j % 3), four
      // barrier waits:
      //   q_full(j+1):  Q(j+1) has landed -> S^T(j+1) into the other buffer
      //   p_ready(j):   P^T(j) is in TMEM -> dV += P^T(j) dO
      //   dp_empty(j):  the dS warps have read dP^T(j) -> dP^T(j+1)
      //   ds_ready(j):  dS^T(j) is in shared memory and the drain warps have
      //                 read dQ^T(j-1) -> dK += dS^T Q, dQ^T(j) = K^T dS^T
      // so that dP^T(j+1) runs while the dS warps still work on step j.
      // S^T(j+1) overwrites the buffer of step j-1, whose P^T the dV MMA of
      // step j-1 (issued earlier by this warp) and the dS warps (before
      // their arrival on ds_ready(j-1)) have read.  The whole warp runs the
      // loop; one elected lane issues.
      const uint32_t t_dp = tmem + Cfg::kColDP;
      const uint32_t t_dv = tmem + Cfg::kColDV, t_dk = tmem + Cfg::kColDK, t_dq = tmem + Cfg::kColDQ;
      int unit_iter = 0, step = 0;
      bool ok = true;
#define MMA_WAIT(wait_expr) \
  {                         \
    if (!(wait_expr)) {     \
      ok = false;           \
      break;                \
    }                       \
  }
      for (;; ++unit_iter) {
        const int buf = unit_iter & 1;
        if constexpr (CLC) {
          MMA_WAIT(mbar_wait_warp_ool(smem_u32(&bars->list_full[buf]), (unit_iter >> 1) & 1, wc));
          if (bars->list_unit[buf] < 0) break;
          MMA_WAIT(ATTN25_TIMED(tr[1], mbar_wait_warp_ool(smem_u32(&bars->kv_full), unit_iter & 1, wc)));
        } else {
          if (snake_unit(unit_iter) >= a.n_units) break;
          MMA_WAIT(mbar_wait_warp_ool(smem_u32(&bars->list_full[buf]), (unit_iter >> 1) & 1, wc) &&
                   ATTN25_TIMED(tr[1], mbar_wait_warp_ool(smem_u32(&bars->kv_full), unit_iter & 1, wc)));
        }
        StepIter it;
        it.init(lists + buf * kMaxSteps, bars->list_n[buf], a.G, a.Sq);
        int g, q0;
        bool pred;
        bool has = it.next(g, q0, pred);
        int n_steps = 0;
        if (has) {  // S^T and dP^T of the unit's first step
          const int s = step % Cfg::kStages, sb = step & 1;
          MMA_WAIT(ATTN25_TIMED(tr[3], mbar_wait_warp_ool(smem_u32(&bars->q_full[s]), (step / Cfg::kStages) & 1, wc)));
          tc_fence_after();
          const uint32_t st = sbase + Cfg::kStageOff + s * Cfg::kStageBytes;
          issue_st<D>(tmem + Cfg::kColS + sb * BM, k_smem, st);
          mma_commit_w(smem_u32(&bars->s_full[sb]));
          issue_st<D>(t_dp, v_smem, st + Cfg::kQBytes);
          mma_commit_w(smem_u32(&bars->dp_full));
        }
        while (has) {
          const int s = step % Cfg::kStages, sb = step & 1;  // stage and S^T buffer of this step
          const uint32_t st = sbase + Cfg::kStageOff + s * Cfg::kStageBytes;
          int g_n, q0_n;
          bool pred_n;
          const bool has_n = it.next(g_n, q0_n, pred_n);
          const int s_n = (step + 1) % Cfg::kStages, sb_n = (step + 1) & 1;
          const uint32_t st_n = sbase + Cfg::kStageOff + s_n * Cfg::kStageBytes;
          if (has_n) {  // S^T of the next step into the other buffer
            MMA_WAIT(ATTN25_TIMED(tr[3], mbar_wait_warp_ool(smem_u32(&bars->q_full[s_n]), ((step + 1) / Cfg::kStages) & 1, wc)));
            tc_fence_after();
            BWD_EV(step + 1, 1);
            issue_st<D>(tmem + Cfg::kColS + sb_n * BM, k_smem, st_n);
            mma_commit_w(smem_u32(&bars->s_full[sb_n]));
          }
          // dV += P^T dO once P^T is in tensor memory (and, on the unit's first
          // step, once the previous unit's epilogue has read the accumulators)
          MMA_WAIT(ATTN25_TIMED(tr[4], mbar_wait_warp_ool(smem_u32(&bars->p_ready[sb]), (step >> 1) & 1, wc)) &&
                   (n_steps > 0 ||
                    ATTN25_TIMED(tr[2], mbar_wait_warp_ool(smem_u32(&bars->acc_empty), (unit_iter & 1) ^ 1, wc))));
          tc_fence_after();
          BWD_EV(step, 2);
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            mma_ts_w(t_dv, tmem + Cfg::kColS + sb * BM + p_col<MOD>(kk),
                     smem_desc_sw128(st + Cfg::kQBytes + kk * 2048, BM * 128, 1024), Cfg::kIdescAcc,
                     (n_steps > 0 || kk > 0) ? 1u : 0u);
          BWD_EV(step, 3);
          // dP^T of the next step once the dS warps have read this step's
          if (has_n) {
            MMA_WAIT(ATTN25_TIMED(tr[8], mbar_wait_warp_ool(smem_u32(&bars->dp_empty), step & 1, wc)));
            tc_fence_after();
            BWD_EV(step, 4);
            issue_st<D>(t_dp, v_smem, st_n + Cfg::kQBytes);
            mma_commit_w(smem_u32(&bars->dp_full));
          }
          // dK += dS^T Q once dS^T is in shared memory; the same barrier slot also
          // counts the drain warps' read of dQ^T(step - 1), so dQ^T(step) may follow
          const uint32_t ds_smem = sbase + Cfg::kDSOff + sb * Cfg::kDSBytes;
          MMA_WAIT(ATTN25_TIMED(tr[5], mbar_wait_warp_ool(smem_u32(&bars->ds_ready[sb]), (step >> 1) & 1, wc)));
          tc_fence_after();
          BWD_EV(step, 5);
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            mma_ss_w(t_dk, smem_desc_sw128(ds_smem + kk * 32, 16, 1024),
                     smem_desc_sw128(st + kk * 2048, BM * 128, 1024), Cfg::kIdescAcc,
                     (n_steps > 0 || kk > 0) ? 1u : 0u);
          BWD_EV(step, 6);
#pragma unroll
          for (int kk = 0; kk < TILE / 16; ++kk)
            mma_ss_w(t_dq, smem_desc_sw128(k_smem + kk * 2048, TILE * 128, 1024),
                     smem_desc_sw128(ds_smem + kk * 2048, BM * 128, 1024), Cfg::kIdescDQ,
                     kk > 0 ? 1u : 0u);
          mma_commit_w(smem_u32(&bars->dq_full));
          mma_commit_w(smem_u32(&bars->q_empty[s]));
          BWD_EV(step, 7);
          ++n_steps;
          ++step;
          has = has_n;
          g = g_n;
          q0 = q0_n;
          pred = pred_n;
        }
        if (!ok) break;
        // a unit without steps still hands the accumulators over in turn: its
        // (empty) dV/dK may only be announced once the previous unit's
        // epilogue has read them, or acc_full would run a phase ahead
        if (n_steps == 0)
          MMA_WAIT(ATTN25_TIMED(tr[2], mbar_wait_warp_ool(smem_u32(&bars->acc_empty), (unit_iter & 1) ^ 1, wc)));
        mma_commit_w(smem_u32(&bars->kv_empty));
        mma_commit_w(smem_u32(&bars->acc_full));
        if (lane == 0) mbar_arrive(smem_u32(&bars->list_empty[buf]));
        __syncwarp();
      }
#undef MMA_WAIT
      mma_commit_w(smem_u32(&bars->drain));
      mbar_wait_warp_ool(smem_u32(&bars->drain), 0, WaitCtl{drain_limit(a.wait_ns), smem_u32(&bars->never_set), a.status});
      ATTN25_TRACE_ONLY(tr[0] = clock64() - t_start; tr[7] = step;)
      trace_flush(a.trace, 32, tr);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ P^T (thread = key row)
    const int r = threadIdx.x;  // TMEM lane = key row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t t_dv = tmem + Cfg::kColDV + lane_off;
    int unit_iter = 0, step = 0;
    bool ok = true;
    for (;; ++unit_iter) {
      const int buf = unit_iter & 1;
      int u;
      if constexpr (CLC) {
        if (!mbar_wait_warp_ool(smem_u32(&bars->list_full[buf]), (unit_iter >> 1) & 1, wc)) { ok = false; break; }
        u = bars->list_unit[buf];
        if (u < 0) break;
      } else {
        u = snake_unit(unit_iter);
        if (u >= a.n_units) break;
      }
      const BwdUnit un = decode_bwd_unit<MOD>(a, u);
      const int kv = un.kt * TILE + r;
      int qlo, qhi;
      key_interval<MOD>(a, un.b, kv, qlo, qhi);
      if constexpr (!CLC) {
        if (!mbar_wait_warp_ool(smem_u32(&bars->list_full[buf]), (unit_iter >> 1) & 1, wc)) { ok = false; break; }
      }
      StepIter it;
      it.init(lists + buf * kMaxSteps, bars->list_n[buf], a.G, a.Sq);
      int g, q0;
      bool pred;
      int n_steps = 0;
      while (it.next(g, q0, pred)) {
        const int s = step % Cfg::kStages, sb = step & 1;
        const uint32_t nl2_s = sbase + Cfg::kStageOff + s * Cfg::kStageBytes + 2 * Cfg::kQBytes;
        const uint32_t t_s = tmem + Cfg::kColS + sb * BM + lane_off;
        // bitmap mask on PARTIAL steps: lane l fetches the word of queries q0 + l
        // and q0 + 32 + l over this warp's 32 keys (issued before the waits)
        uint32_t wa = 0u, wb = 0u;
        if constexpr (has_bitmap(MOD)) {
          if (pred) {
            const int lane = threadIdx.x & 31;
            const uint32_t* col = bitmap_row(a.mod, un.b, un.hk * a.G + g, 0) + un.kt * 4 + (r >> 5);
            const int qa = q0 + lane, qb = q0 + 32 + lane;
            if (qa < a.Sq) wa = __ldg(col + static_cast<long long>(qa) * a.mod.bm_row_words);
            if (qb < a.Sq) wb = __ldg(col + static_cast<long long>(qb) * a.mod.bm_row_words);
          }
        }
        if (!ATTN25_TIMED(tr[1], mbar_wait_warp_ool(smem_u32(&bars->q_full[s]), (step / Cfg::kStages) & 1, wc))) { ok = false; break; }
        if (!ATTN25_TIMED(tr[2], mbar_wait_warp_ool(smem_u32(&bars->s_full[sb]), (step >> 1) & 1, wc))) { ok = false; break; }
        tc_fence_after();
        BWD_EV(step, 8);
        ATTN25_TRACE_ONLY(const long long t_p = clock64();)
        const int h = un.hk * a.G + g;
        if constexpr (kSoftcapHalves<MOD>) {
          (void)h;
#pragma unroll 1
          for (int hf = 0; hf < 2; ++hf) softcap_half<MOD>(t_s + hf * 32, hf, a, q0, qlo, qhi, pred, nl2_s, wa, wb);
          ATTN25_TRACE_ONLY(const long long t_p2 = clock64(); tr[5] += t_p2 - t_p;)
          tmem_wait_st();
          ATTN25_TRACE_ONLY(tr[6] += clock64() - t_p2;)
        } else {
          float x[BM];
          tmem_ld32(t_s, reinterpret_cast<uint32_t(&)[32]>(x[0]));
          tmem_ld32(t_s + 32, reinterpret_cast<uint32_t(&)[32]>(x[32]));
          tmem_wait_ld();
          ATTN25_TRACE_ONLY(const long long t_p1 = clock64(); tr[4] += t_p1 - t_p;)
          probs_t<MOD>(x, a, h, static_cast<float>(q0 - kv), q0, qlo, qhi, pred, nl2_s, wa, wb);
          // P^T (bf16 pairs) over the first 32 columns of this S^T buffer
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
          ATTN25_TRACE_ONLY(const long long t_p2 = clock64(); tr[5] += t_p2 - t_p1;)
          tmem_st32(t_s, pk);
          tmem_wait_st();
          ATTN25_TRACE_ONLY(tr[6] += clock64() - t_p2;)
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&bars->p_ready[sb]));
        BWD_EV(step, 9);
        ATTN25_TRACE_ONLY(tr[3] += clock64() - t_p;)
        ++n_steps;
        ++step;
      }
      if (!ok) break;
      // ---- unit epilogue: dV -> bf16
      if (!ATTN25_TIMED(tr[7], mbar_wait_warp_ool(smem_u32(&bars->acc_full), unit_iter & 1, wc))) { ok = false; break; }
      tc_fence_after();
      ATTN25_TRACE_ONLY(const long long t_e = clock64();)
      store_acc_rows<D, kSoftcapHalves<MOD> ? 1 : 2>(a.dv + un.b * a.dv_st.b + un.hk * a.dv_st.h + static_cast<long long>(kv) * a.dv_st.s, t_dv, 1.f,
                        n_steps > 0, kv < a.Skv);
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->acc_empty));
      if (lane == 0) mbar_arrive(smem_u32(&bars->list_empty[buf]));
      ATTN25_TRACE_ONLY(tr[8] += clock64() - t_e;)
    }
    ATTN25_TRACE_ONLY(tr[0] = clock64() - t_start;)
    trace_flush(a.trace, 0, tr);
  } else if (warp < 8) {
    // ------------------------------------------------------------ dS^T (thread = key row)
    const int r = threadIdx.x - 128;
    const uint32_t lane_off = static_cast<uint32_t>((warp - 4) * 32) << 16;
    const uint32_t t_dp = tmem + Cfg::kColDP + lane_off, t_dk = tmem + Cfg::kColDK + lane_off;
    int unit_iter = 0, step = 0;
    bool ok = true;
    for (;; ++unit_iter) {
      const int buf = unit_iter & 1;
      int u;
      if constexpr (CLC) {
        if (!mbar_wait_warp_ool(smem_u32(&bars->list_full[buf]), (unit_iter >> 1) & 1, wc)) { ok = false; break; }
        u = bars->list_unit[buf];
        if (u < 0) break;
      } else {
        u = snake_unit(unit_iter);
        if (u >= a.n_units) break;
      }
      const BwdUnit un = decode_bwd_unit<MOD>(a, u);
      const int kv = un.kt * TILE + r;
      if constexpr (!CLC) {
        if (!mbar_wait_warp_ool(smem_u32(&bars->list_full[buf]), (unit_iter >> 1) & 1, wc)) { ok = false; break; }
      }
      StepIter it;
      it.init(lists + buf * kMaxSteps, bars->list_n[buf], a.G, a.Sq);
      int g, q0;
      bool pred;
      int n_steps = 0;
      while (it.next(g, q0, pred)) {
        const int s = step % Cfg::kStages, sb = step & 1;
        const uint32_t stats = sbase + Cfg::kStageOff + s * Cfg::kStageBytes + 2 * Cfg::kQBytes;
        const uint32_t t_p = tmem + Cfg::kColS + sb * BM + lane_off;
        if (!ATTN25_TIMED(tr[1], mbar_wait_warp_ool(smem_u32(&bars->q_full[s]), (step / Cfg::kStages) & 1, wc))) { ok = false; break; }
        if (!ATTN25_TIMED(tr[2], mbar_wait_warp_ool(smem_u32(&bars->p_ready[sb]), (step >> 1) & 1, wc))) { ok = false; break; }
        if (!ATTN25_TIMED(tr[4], mbar_wait_warp_ool(smem_u32(&bars->dp_full), step & 1, wc))) { ok = false; break; }
        tc_fence_after();
        BWD_EV(step, 10);
        ATTN25_TRACE_ONLY(const long long t_ds = clock64();)
        float dp[BM];
        uint32_t pb[32];
        tmem_ld32(t_dp, reinterpret_cast<uint32_t(&)[32]>(dp[0]));
        tmem_ld32(t_dp + 32, reinterpret_cast<uint32_t(&)[32]>(dp[32]));
        if constexpr (kSoftcapHalves<MOD>) {  // the factor P (1 - tanh^2) the P warps stored beside P^T
          tmem_ld16(t_p + 16, reinterpret_cast<uint32_t(&)[16]>(pb[0]));
          tmem_ld16(t_p + 48, reinterpret_cast<uint32_t(&)[16]>(pb[16]));
        } else {
          tmem_ld32(t_p, pb);
        }
        tmem_wait_ld();
        ATTN25_TRACE_ONLY(tr[3] += clock64() - t_ds;)
        // dP^T has been read: the next step's dP^T may overwrite it.  (P^T of
        // this buffer is released through ds_ready below.)
        tc_fence_before();
        mbar_arrive(smem_u32(&bars->dp_empty));
        BWD_EV(step, 11);
        // the dS buffer is free once the drain warps have staged dQ of two steps ago through it
        if (!ATTN25_TIMED(tr[5], mbar_wait_warp_ool(smem_u32(&bars->ds_empty[sb]), ((step >> 1) & 1) ^ 1, wc))) { ok = false; break; }
        uint8_t* ds_row = smem + Cfg::kDSOff + sb * Cfg::kDSBytes + r * 128;
        // local boost: dS carries the boost inside the band, folded into dP
        // there, (dP' - Delta) = boost (dP - Delta) with dP' = boost dP + (boost - 1)(-Delta)
        if constexpr (score_of(MOD) == MOD_BOOST) {
          const float dq0 = static_cast<float>(q0 - kv);
          if (boost_band_meets(a, dq0)) {
            const float rad = static_cast<float>(a.mod.boost_radius), bst = a.mod.boost;
#pragma unroll
            for (int c4 = 0; c4 < BM / 4; ++c4) {
              const float4 n4 = lds128(stats + 512 + c4 * 16);
              const float nd4[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = c4 * 4 + e;
                if (fabsf(dq0 + static_cast<float>(c)) < rad) dp[c] = fmaf(dp[c], bst, (bst - 1.f) * nd4[e]);
              }
            }
          }
        }
#pragma unroll
        for (int c16 = 0; c16 < 8; ++c16) {  // 8 columns (16 bytes) at a time
          const float4 nd0 = lds128(stats + 512 + c16 * 32), nd1 = lds128(stats + 512 + c16 * 32 + 16);
          const float nd[8] = {nd0.x, nd0.y, nd0.z, nd0.w, nd1.x, nd1.y, nd1.z, nd1.w};
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = c16 * 8 + 2 * e;
            const uint32_t pp = pb[c >> 1];
            const float2 pr = make_float2(__uint_as_float(pp << 16), __uint_as_float(pp & 0xffff0000u));
            // dS = P (dP - Delta) (softcap: P (1 - tanh^2) (dP - Delta))
            const float2 d = __fmul2_rn(pr, __fadd2_rn(make_float2(dp[c], dp[c + 1]), make_float2(nd[2 * e], nd[2 * e + 1])));
            w[e] = pack_bf16x2(d.x, d.y);
          }
          // 128-byte swizzle: 16-byte chunk c16 of row r lands at chunk c16 ^ (r % 8)
          *reinterpret_cast<uint4*>(ds_row + ((c16 ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(smem_u32(&bars->ds_ready[sb]));
        BWD_EV(step, 12);
        ATTN25_TRACE_ONLY(tr[6] += clock64() - t_ds;)
        ++n_steps;
        ++step;
      }
      if (!ok) break;
      // ---- unit epilogue: scale * dK -> bf16
      if (!ATTN25_TIMED(tr[7], mbar_wait_warp_ool(smem_u32(&bars->acc_full), unit_iter & 1, wc))) { ok = false; break; }
      tc_fence_after();
      ATTN25_TRACE_ONLY(const long long t_e = clock64();)
      store_acc_rows<D, kSoftcapHalves<MOD> ? 1 : 2>(a.dk + un.b * a.dk_st.b + un.hk * a.dk_st.h + static_cast<long long>(kv) * a.dk_st.s, t_dk, a.scale,
                        n_steps > 0, kv < a.Skv);
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->acc_empty));
      if (lane == 0) mbar_arrive(smem_u32(&bars->list_empty[buf]));
      ATTN25_TRACE_ONLY(tr[8] += clock64() - t_e;)
    }
    ATTN25_TRACE_ONLY(tr[0] = clock64() - t_start;)
    trace_flush(a.trace, 64, tr);
  } else {
    // ------------------------------------------------------------ dQ drain (thread = head-dim lane)
    // dQ^T leaves TMEM row by row (lane = head dim d) and is added into the
    // fp32 accumulator [B*Hq][Sq_pad][D] with reductions performed in L2: one
    // instruction covers 32 consecutive d of one query row (128 bytes, one
    // L1 wavefront).  (Four-wide reductions into a transposed accumulator
    // need 32 wavefronts per instruction and starve the tensor core of
    // shared-memory bandwidth; staging through shared memory for bulk
    // reductions costs twice the wavefronts.)
    const int w = warp - 8;      // TMEM lane quarter = 32-row block of D
    const uint32_t lane_off = static_cast<uint32_t>(w * 32) << 16;
    const uint32_t t_dq = tmem + Cfg::kColDQ + lane_off;
    const bool active = w * 32 < D;
    int unit_iter = 0, step = 0;
    bool ok = true;
    // ds_ready of step j counts the drain's read of dQ^T(j-1); step 0 has no
    // predecessor, so its share is given up front
    mbar_arrive(smem_u32(&bars->ds_ready[0]));
    for (;; ++unit_iter) {
      const int buf = unit_iter & 1;
      int u;
      if constexpr (CLC) {
        if (!mbar_wait_warp_ool(smem_u32(&bars->list_full[buf]), (unit_iter >> 1) & 1, wc)) { ok = false; break; }
        u = bars->list_unit[buf];
        if (u < 0) break;
      } else {
        u = snake_unit(unit_iter);
        if (u >= a.n_units) break;
      }
      const BwdUnit un = decode_bwd_unit<MOD>(a, u);
      if constexpr (!CLC) {
        if (!mbar_wait_warp_ool(smem_u32(&bars->list_full[buf]), (unit_iter >> 1) & 1, wc)) { ok = false; break; }
      }
      StepIter it;
      it.init(lists + buf * kMaxSteps, bars->list_n[buf], a.G, a.Sq);
      int g, q0;
      bool pred;
      while (it.next(g, q0, pred)) {
        const int sb = step & 1;
        if (!ATTN25_TIMED(tr[1], mbar_wait_warp_ool(smem_u32(&bars->dq_full), step & 1, wc))) { ok = false; break; }
        tc_fence_after();
        BWD_EV(step, 13);
        float v[BM];
        tmem_ld32(t_dq, reinterpret_cast<uint32_t(&)[32]>(v[0]));
        tmem_ld32(t_dq + 32, reinterpret_cast<uint32_t(&)[32]>(v[32]));
        tmem_wait_ld();
        tc_fence_before();
        // dQ^T(step) has been read: its columns may take dQ^T(step + 1), which the
        // MMA warp issues after waiting for ds_ready of step + 1
        mbar_arrive(smem_u32(&bars->ds_ready[(step + 1) & 1]));
        BWD_EV(step, 14);
        ATTN25_TRACE_ONLY(const long long t_r = clock64();)
        // the dS buffer is free already (dK and dQ^T of this step completed)
        if (lane == 0) mbar_arrive(smem_u32(&bars->ds_empty[sb]));
        if (active) {
          const int bh = un.b * a.Hq + un.hk * a.G + g;
          float* dst = a.dq_acc + (static_cast<size_t>(bh) * a.Sq_pad + q0) * D + w * 32 + lane;
          unsigned* sem = nullptr;
          if (a.dq_sem != nullptr) {  // deterministic dQ: wait for this unit's turn
            sem = a.dq_sem + (static_cast<size_t>(bh) * (a.Sq_pad / BM) + q0 / BM) * 4 + w;
            if (!sem_wait_eq(sem, positions[buf * kMaxSteps + it.entry()], wc)) {
              ok = false;
              break;
            }
          }
#pragma unroll
          for (int c = 0; c < BM; ++c) atomicAdd(dst + static_cast<size_t>(c) * D, v[c]);
          if (sem != nullptr) sem_release(sem);
        }
        ATTN25_TRACE_ONLY(tr[2] += clock64() - t_r;)
        BWD_EV(step, 15);
        ++step;
      }
      if (!ok) break;
      if (lane == 0) mbar_arrive(smem_u32(&bars->list_empty[buf]));
    }
    ATTN25_TRACE_ONLY(tr[0] = clock64() - t_start;)
    trace_flush(a.trace, 16, tr);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 12) tmem_dealloc(tmem, 512);
}

// -Delta_i = -sum_d dO_id O_id and -LSE_i log2(e) (-inf where the row kept
// nothing or lies past Sq), and zero the fp32 dQ accumulator.  One warp per row.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdArgs a) {
  const long long total_rows = static_cast<long long>(a.B) * a.Hq * a.Sq_pad;
  const int lane = threadIdx.x & 31;
  for (long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       row < total_rows; row += (static_cast<long long>(gridDim.x) * blockDim.x) >> 5) {
    const long long bh = row / a.Sq_pad;
    const int q = static_cast<int>(row - bh * a.Sq_pad);
    float acc = 0.f;
    if (q < a.Sq) {
      const long long b = bh / a.Hq, h = bh - b * a.Hq;
      const __nv_bfloat16* orow = a.out + b * a.o_st.b + h * a.o_st.h + q * a.o_st.s;
      const __nv_bfloat16* grow = a.dout + b * a.do_st.b + h * a.do_st.h + q * a.do_st.s;
      for (int d = lane * 2; d < D; d += 64) {
        const __nv_bfloat162 o2 = *reinterpret_cast<const __nv_bfloat162*>(orow + d);
        const __nv_bfloat162 g2 = *reinterpret_cast<const __nv_bfloat162*>(grow + d);
        acc = fmaf(__bfloat162float(o2.x), __bfloat162float(g2.x), acc);
        acc = fmaf(__bfloat162float(o2.y), __bfloat162float(g2.y), acc);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    float4* z = reinterpret_cast<float4*>(a.dq_acc + static_cast<size_t>(row) * D);
    for (int i = lane; i < D / 4; i += 32) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    // deterministic dQ: the counters of this 64-row block start at zero
    if (a.dq_sem != nullptr && (q % BM) == 0 && lane < 4) a.dq_sem[(row / BM) * 4 + lane] = 0u;
    if (lane == 0) {
      // stored negated, so that the main kernel's exponent is one FFMA:
      // -LSE log2(e), or -inf where the row keeps nothing or lies past Sq (P = 0)
      float nl2 = -INFINITY;
      if (q < a.Sq) {
        const float l = a.lse[static_cast<size_t>(bh) * a.Sq + q];
        nl2 = (l == -INFINITY) ? -INFINITY : -l * LOG2E;
      }
      a.lse2[row] = nl2;
      a.delta[row] = q < a.Sq ? -acc : 0.f;
    }
  }
}

// dQ = scale * accumulator, rounded to bf16; 8 elements per thread.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_cast_kernel(const BwdArgs a) {
  const long long n8 = static_cast<long long>(a.B) * a.Hq * a.Sq * (D / 8);
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long e = i * 8;
    const long long row = e / D;
    const int d = static_cast<int>(e - row * D);
    const long long bh = row / a.Sq;
    const int q = static_cast<int>(row - bh * a.Sq);
    const float4* src = reinterpret_cast<const float4*>(a.dq_acc + (static_cast<size_t>(bh) * a.Sq_pad + q) * D + d);
    const float4 x0 = src[0], x1 = src[1];
    uint4 o;
    o.x = pack_bf16x2(x0.x * a.scale, x0.y * a.scale);
    o.y = pack_bf16x2(x0.z * a.scale, x0.w * a.scale);
    o.z = pack_bf16x2(x1.x * a.scale, x1.y * a.scale);
    o.w = pack_bf16x2(x1.z * a.scale, x1.w * a.scale);
    const long long b = bh / a.Hq, h = bh - b * a.Hq;
    *reinterpret_cast<uint4*>(a.dq + b * a.dq_st.b + h * a.dq_st.h + q * a.dq_st.s + d) = o;
  }
}

template <int D, int MOD>
cudaError_t launch_bwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const CUtensorMap& tdo, const BwdArgs& a, int grid, cudaStream_t stream) {
  const long long rows = static_cast<long long>(a.B) * a.Hq * a.Sq_pad;
  int prep_blocks = static_cast<int>((rows * 32 + 255) / 256);
  if (prep_blocks > a.num_sms * 16) prep_blocks = a.num_sms * 16;  // two waves of 8 resident blocks per SM
  bwd_prep_kernel<D><<<prep_blocks, 256, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  auto kernel = a.clc ? attn_bwd_kernel<D, MOD, true> : attn_bwd_kernel<D, MOD, false>;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, BwdCfg<D>::kAllocBytes);
  if (e != cudaSuccess) return e;
  kernel<<<grid, kBwdThreads, BwdCfg<D>::kAllocBytes, stream>>>(tq, tk, tv, tdo, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long n8 = static_cast<long long>(a.B) * a.Hq * a.Sq * (D / 8);
  int cast_blocks = static_cast<int>((n8 + 255) / 256);
  if (cast_blocks > a.num_sms * 16) cast_blocks = a.num_sms * 16;
  bwd_dq_cast_kernel<D><<<cast_blocks, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_mod(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& tdo, const BwdArgs& a, int key, int grid, cudaStream_t s) {
  constexpr int M = kKeyMasked, MB = kKeyMasked | kKeyBitmap;
  switch (key) {
    case MOD_NONE: return launch_bwd_t<D, MOD_NONE>(tq, tk, tv, tdo, a, grid, s);
    case MOD_ALIBI: return launch_bwd_t<D, MOD_ALIBI>(tq, tk, tv, tdo, a, grid, s);
    case MOD_SOFTCAP: return launch_bwd_t<D, MOD_SOFTCAP>(tq, tk, tv, tdo, a, grid, s);
    case MOD_BOOST: return launch_bwd_t<D, MOD_BOOST>(tq, tk, tv, tdo, a, grid, s);
    case M | MOD_NONE: return launch_bwd_t<D, M | MOD_NONE>(tq, tk, tv, tdo, a, grid, s);
    case M | MOD_ALIBI: return launch_bwd_t<D, M | MOD_ALIBI>(tq, tk, tv, tdo, a, grid, s);
    case M | MOD_SOFTCAP: return launch_bwd_t<D, M | MOD_SOFTCAP>(tq, tk, tv, tdo, a, grid, s);
    case M | MOD_BOOST: return launch_bwd_t<D, M | MOD_BOOST>(tq, tk, tv, tdo, a, grid, s);
    case MB | MOD_NONE: return launch_bwd_t<D, MB | MOD_NONE>(tq, tk, tv, tdo, a, grid, s);
    case MB | MOD_ALIBI: return launch_bwd_t<D, MB | MOD_ALIBI>(tq, tk, tv, tdo, a, grid, s);
    case MB | MOD_SOFTCAP: return launch_bwd_t<D, MB | MOD_SOFTCAP>(tq, tk, tv, tdo, a, grid, s);
    case MB | MOD_BOOST: return launch_bwd_t<D, MB | MOD_BOOST>(tq, tk, tv, tdo, a, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const BwdArgs& a, int D, int key, int grid,
                       cudaStream_t stream) {
  if (D == 128) return launch_bwd_mod<128>(tq, tk, tv, tdo, a, key, grid, stream);
  if (D == 64) return launch_bwd_mod<64>(tq, tk, tv, tdo, a, key, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace attn25
