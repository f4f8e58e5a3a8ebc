// Block-mask construction and work ordering (plain CUDA, integer only).
//
// Classifies every 128x128 (query tile, key tile) pair as EMPTY / PARTIAL /
// FULL so that the attention kernels can skip empty KV tiles and run the
// element predicate only on partial ones ("PyTorch FlexAttention,
// FlashAttention-4 백엔드 …", 섹션별 상세: block-sparse iteration; "FlashInfer
// SM120 NVFP4 어텐션 최적화", 코드 분석 4: masking only where the tile needs
// it).  Every mask of the set, and every intersection of them, keeps an
// interval of keys [lo(i), hi(i)] per query row, so the kept count of a tile row is a closed-form interval
// length; summing it over the tile's rows counts kept elements exactly, which
// is the same classification as testing every element.
//
// Then the work orders: query-tile pairs and key tiles sorted longest first
// (stable counting sort), the longest-processing-time-first order that the
// persistent kernels walk ("PyTorch FlexAttention, …", 실무 Takeaway: load
// balance across SMs under data-dependent masks).
#include <cuda_runtime.h>

#include "launch.h"
#include "mods.cuh"

namespace attn25 {

namespace {

__device__ __forceinline__ void row_keep_interval(const MaskArgs& a, int b, int i, int& lo,
                                                  int& hi) {
  const size_t vb = static_cast<size_t>(b) * (a.n_seqs + 1);
  row_interval(a.mask, a.window,
               a.doc_offsets == nullptr ? nullptr
                                        : a.doc_offsets + static_cast<size_t>(b) * (a.num_docs + 1),
               a.num_docs, a.vq_offsets == nullptr ? nullptr : a.vq_offsets + vb,
               a.vk_offsets == nullptr ? nullptr : a.vk_offsets + vb, a.n_seqs, i, a.Skv, lo, hi);
}

// grid (nQ, B): classify one query-tile row of tiles and write its KV list.
__global__ void __launch_bounds__(256) classify_kernel(const MaskArgs a) {
  const int qt = blockIdx.x, b = blockIdx.y;
  __shared__ int s_lo[TILE], s_hi[TILE];
  __shared__ uint8_t s_cls[1024];
  const int q0 = qt * TILE, q1 = min(a.Sq, q0 + TILE);
  for (int r = threadIdx.x; r < TILE; r += blockDim.x) {
    int lo = 0, hi = -1;
    if (q0 + r < q1) row_keep_interval(a, b, q0 + r, lo, hi);
    s_lo[r] = lo;
    s_hi[r] = hi;
  }
  __syncthreads();
  const size_t row = static_cast<size_t>(b) * a.nQ + qt;
  for (int kt = threadIdx.x; kt < a.nK; kt += blockDim.x) {
    const int k0 = kt * TILE, k1 = min(a.Skv, k0 + TILE);
    const long long total = static_cast<long long>(q1 - q0) * (k1 - k0);
    long long kept_min, kept_max;  // over the heads the masks distinguish
    if (a.bitmap == nullptr) {
      long long kept = 0;
      for (int r = 0; r < q1 - q0; ++r) {
        const int lo = max(s_lo[r], k0), hi = min(s_hi[r], k1 - 1);
        kept += max(0, hi - lo + 1);
      }
      kept_min = kept_max = kept;
    } else {
      // kept = set bits of the row's 128-key word group inside its interval
      kept_min = total;
      kept_max = 0;
      for (int h = 0; h < a.bm_heads; ++h) {
        const uint32_t* base = a.bitmap + b * a.bm_batch_stride + h * a.bm_head_stride;
        long long kept = 0;
        for (int r = 0; r < q1 - q0; ++r) {
          const int lo = max(s_lo[r], k0) - k0, hi = min(s_hi[r], k1 - 1) - k0;  // tile columns
          if (hi < lo) continue;
          const uint4 w = __ldg(reinterpret_cast<const uint4*>(
                                    base + static_cast<long long>(q0 + r) * a.bm_row_words) + kt);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int clo = max(lo - 32 * c, 0), chi = min(hi - 32 * c, 31);
            if (chi < clo) continue;
            const uint32_t in = (0xffffffffu >> (31 - chi)) & (0xffffffffu << clo);
            kept += __popc(ws[c] & in);
          }
        }
        kept_min = min(kept_min, kept);
        kept_max = max(kept_max, kept);
      }
    }
    const uint8_t c = kept_max == 0 ? 0 : (kept_min == total ? 2 : 1);
    a.tile_class[row * a.nK + kt] = c;
    if (kt < 1024) s_cls[kt] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int n = 0;
    int32_t* list = a.kv_index + row * a.nK;
    for (int kt = 0; kt < a.nK; ++kt) {
      const uint8_t c = (kt < 1024) ? s_cls[kt] : a.tile_class[row * a.nK + kt];
      if (c != 0) list[n++] = kt;
    }
    a.kv_count[row] = n;
    for (int kt = n; kt < a.nK; ++kt) list[kt] = -1;
  }
}

// grid (nK, B): the transposed lists (query tiles per key tile).
__global__ void __launch_bounds__(32) transpose_kernel(const MaskArgs a) {
  const int kt = blockIdx.x, b = blockIdx.y;
  if (threadIdx.x != 0) return;
  const size_t col = static_cast<size_t>(b) * a.nK + kt;
  int32_t* list = a.q_index + col * a.nQ;
  int n = 0;
  for (int qt = 0; qt < a.nQ; ++qt)
    if (a.tile_class[(static_cast<size_t>(b) * a.nQ + qt) * a.nK + kt] != 0) list[n++] = qt;
  a.q_count[col] = n;
  for (int qt = n; qt < a.nQ; ++qt) list[qt] = -1;
}

__device__ __forceinline__ int pair_cost(const MaskArgs& a, int u) {
  const int b = u / a.nP, p = u - b * a.nP;
  const uint8_t* r0 = a.tile_class + (static_cast<size_t>(b) * a.nQ + 2 * p) * a.nK;
  const bool has1 = 2 * p + 1 < a.nQ;
  int cost = 0;
  for (int kt = 0; kt < a.nK; ++kt) cost += (r0[kt] != 0 || (has1 && r0[a.nK + kt] != 0));
  return cost;
}

// One block: the forward pairs and the backward units, each sorted by
// descending cost with ties in ascending id.  Costs go to shared memory and
// every thread places its units at their rank: the number of units that sort
// before them.
constexpr int kOrderSmemUnits = 16384;

__global__ void __launch_bounds__(1024) order_kernel(const MaskArgs a) {
  extern __shared__ int s_cost[];  // kOrderSmemUnits entries
  for (int pass = 0; pass < 2; ++pass) {
    const int n = pass == 0 ? a.B * a.nP : a.B * a.nK;
    int32_t* out = pass == 0 ? a.fwd_order : a.bwd_order;
    for (int u = threadIdx.x; u < n; u += blockDim.x)
      s_cost[u] = pass == 0 ? pair_cost(a, u) : a.q_count[u];
    __syncthreads();
    for (int u = threadIdx.x; u < n; u += blockDim.x) {
      const int c = s_cost[u];
      int rank = 0;
      for (int v = 0; v < n; ++v) {
        const int cv = s_cost[v];
        rank += (cv > c) || (cv == c && v < u);
      }
      out[rank] = u;
    }
    __syncthreads();
  }
}

// The same order for unit counts beyond the shared-memory table: a stable
// counting sort by one thread over costs in [0, max(nQ, nK)].
__global__ void __launch_bounds__(32) order_serial_kernel(const MaskArgs a) {
  if (threadIdx.x != 0) return;
  extern __shared__ int s_hist[];  // max(nQ, nK) + 2 counters
  const int max_cost = a.nQ > a.nK ? a.nQ : a.nK;
  for (int pass = 0; pass < 2; ++pass) {
    const int n = pass == 0 ? a.B * a.nP : a.B * a.nK;
    int32_t* out = pass == 0 ? a.fwd_order : a.bwd_order;
    for (int c = 0; c <= max_cost + 1; ++c) s_hist[c] = 0;
    for (int u = 0; u < n; ++u) ++s_hist[pass == 0 ? pair_cost(a, u) : a.q_count[u]];
    int start = 0;
    for (int c = max_cost; c >= 0; --c) {
      const int cnt = s_hist[c];
      s_hist[c] = start;
      start += cnt;
    }
    for (int u = 0; u < n; ++u) out[s_hist[pass == 0 ? pair_cost(a, u) : a.q_count[u]]++] = u;
  }
}

}  // namespace

cudaError_t launch_block_mask(const MaskArgs& a, cudaStream_t stream) {
  classify_kernel<<<dim3(a.nQ, a.B), 256, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  transpose_kernel<<<dim3(a.nK, a.B), 32, 0, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n_max = a.B * (a.nP > a.nK ? a.nP : a.nK);
  if (n_max <= kOrderSmemUnits) {
    const int smem = n_max * static_cast<int>(sizeof(int));
    if (smem > 48 * 1024) {
      e = cudaFuncSetAttribute(order_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kOrderSmemUnits * static_cast<int>(sizeof(int)));
      if (e != cudaSuccess) return e;
    }
    order_kernel<<<1, 1024, smem, stream>>>(a);
  } else {
    order_serial_kernel<<<1, 32, ((a.nQ > a.nK ? a.nQ : a.nK) + 2) * sizeof(int), stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace attn25
