// Forward attention kernel for sm_100a.
//
// One persistent CTA per SM walks work units (batch row, query head, pair of
// 128-row query tiles).  Warp roles:
//   warps 0-3  softmax for query tile 0 of the pair (thread = query row)
//   warps 4-7  softmax for query tile 1
//   warp  8    MMA issuer (the whole warp runs the issue code; one lane,
//              chosen by elect.sync, issues each tcgen05.mma)
//   warp  9    TMA producer
// Scores S_t = Q_t K^T accumulate in tensor memory (TMEM), the softmax warps
// read them with tcgen05.ld, write the bf16 probabilities P_t back over S_t,
// and O_t += P_t V runs with P_t taken straight from TMEM.  The two query
// tiles ping-pong: while one tile's softmax runs, the tensor core works on the
// other tile's products (the ping-pong pipeline of "PyTorch FlexAttention,
// FlashAttention-4 백엔드 …", 섹션별 상세, and the warp-specialised
// producer/consumer split of "FlashAttention-3 (KO)", 비동기 실행 및 워프 특화).
//
// Online softmax ("FlashAttention 설명", §5; "FlashAttention-2 …", §4): per
// row a running maximum m, running sum l and the accumulator O in TMEM.  The
// running maximum is only moved when a new score exceeds it by more than
// 2^8 (in the base-2 domain), and only then is O rescaled; otherwise the
// stale maximum stays the reference.  Every term keeps the same reference,
// so O / l is unchanged while rescales become rare.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "exp2_poly.h"
#include "kernel_common.cuh"
#include "launch.h"

namespace attn25 {

namespace {

constexpr int kFwdThreads = 384;  // 2 softmax warpgroups + 1 control warpgroup
// Register split (setmaxnreg): the launch gives 168 per thread (384 x 168 =
// 64512 in the CTA pool); the control warpgroup drops to 104 so that the two
// softmax warpgroups can rise to 200: 2 x 128 x 200 + 128 x 104 = 64512.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 200;
constexpr int kControlRegs = 104;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kFwdThreads * kLaunchRegs, "register split");
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct FwdCfg {
  static constexpr int kTileBytes = TILE * D * 2;           // one 128 x D bf16 tile
  static constexpr int kStages = (D == 128) ? 4 : 6;        // K/V ring slots
  static constexpr int kQOff = 0;                           // Q0, Q1
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kBarOff = kRingOff + kStages * kTileBytes;
  static constexpr int kListOff = kBarOff + 1024;           // two step lists
  static constexpr int kSmemBytes = kListOff + 2 * kMaxSteps * 4;
  static constexpr int kAllocBytes = kSmemBytes + 1024;     // + alignment slack
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, false, false);
  static constexpr uint32_t kIdescQK8 = idesc_e4m3_f32(128, 128, false, false);
  static constexpr int kTileBytes8 = TILE * D;             // one 128 x D e4m3 tile
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, false, true);
};

struct FwdBarriers {
  alignas(16) uint32_t clc_resp[4];  // cluster launch control response (the next unit)
  uint64_t clc_bar;
  uint64_t list_full[2], list_empty[2];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_full[2], o_full[2], o_final[2];
  uint64_t drain;
  uint64_t kv_full[8], kv_empty[8];
  uint32_t tmem_base;
  uint32_t abort_flag;
  uint32_t never_set;  // abort word for drain waits that must not stop early
  int32_t list_n[2];   // step counts of the two step lists
  int32_t list_unit[2];  // cluster launch control: the unit of each list; -1 ends the walk
};

// Consumers of a step list: the MMA warp and the 8 softmax warps (lane 0 each).
constexpr int kListConsumers = 9;

struct UnitCoord {
  int b, h, p;
};

__device__ __forceinline__ UnitCoord decode_unit(const FwdArgs& a, int u) {
  const int pair_idx = u / a.Hq;
  const int h = u - pair_idx * a.Hq;
  const int pair = (a.fwd_order != nullptr) ? __ldg(a.fwd_order + pair_idx) : pair_idx;
  UnitCoord c;
  c.b = pair / a.nP;
  c.p = pair - c.b * a.nP;
  c.h = h;
  return c;
}

// Load the tile rows [row0, row0+128) of head h of batch row b (all D
// columns) as D/64 boxes of 64 columns, each 128 rows x 128 bytes with
// 128-byte swizzle; the tensor map is 4-D (D, S, H, B) with the tensor's strides.
template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                          int row0, int h, int b) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) tma_load_4d(dst + c * (TILE * 128), map, bar, c * 64, row0, h, b);
}

template <int D, bool FP8 = false>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_smem, uint32_t k_smem) {
  if constexpr (FP8) {
    // e4m3 rows of D = 128 bytes fill one 128-byte swizzle row: 4 MMAs of K = 32
    static_assert(D == 128, "FP8 scores need D = 128");
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) {
      const uint32_t off = kk * 32;
      mma_ss_f8_w(d_tmem, smem_desc_sw128(q_smem + off, 16, 1024), smem_desc_sw128(k_smem + off, 16, 1024),
                  FwdCfg<D>::kIdescQK8, kk > 0 ? 1u : 0u);
    }
  } else {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = (kk >> 2) * (TILE * 128) + (kk & 3) * 32;
      mma_ss_w(d_tmem, smem_desc_sw128(q_smem + off, 16, 1024), smem_desc_sw128(k_smem + off, 16, 1024),
               FwdCfg<D>::kIdescQK, kk > 0 ? 1u : 0u);
    }
  }
}

// Q or K tile: bf16 (D/64 boxes of 64 columns) or e4m3 (one box of D = 128
// bytes per row), through 4-D tensor maps (D, S, H, B).
template <int D, bool FP8>
__device__ __forceinline__ void load_qk_tile(uint32_t dst, const CUtensorMap* map, uint32_t bar, int row0,
                                             int h, int b) {
  if constexpr (FP8) {
    tma_load_4d(dst, map, bar, 0, row0, h, b);
  } else {
    load_tile<D>(dst, map, bar, row0, h, b);
  }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_smem,
                                         bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < TILE / 16; ++kk) {
    mma_ts_w(d_tmem, p_tmem + kk * 8, smem_desc_sw128(v_smem + kk * 2048, TILE * 128, 1024),
             FwdCfg<D>::kIdescPV, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Per-row constants of one work unit.
struct RowCtx {
  int row;      // absolute query index
  int lo, hi;   // kept key interval
  float sl2;    // scale * log2(e)
  float aux;    // ALiBi: slope * log2(e); softcap: scale / c; boost: boost * sl2
  float aux2;   // softcap: c * log2(e)
  float lim;    // softcap: raw scores up to this size take tanh's series (|s / c| <= 0.4)
  const uint32_t* bits;  // bitmap mask: this row's keep bits (nullptr on padding rows)
};

// Three-input maximum (one instruction).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Raw scores of one row (32 columns starting at key k0 + c0) -> base-2 modded scores.
template <int MOD>
__device__ __forceinline__ void transform32(float (&x)[32], const RowCtx& r, const ModDev& md,
                                            int k0, int c0, bool pred) {
  const float di = static_cast<float>(r.row - k0 - c0);
  if constexpr (score_of(MOD) == MOD_SOFTCAP) {
    // scores well below the cap everywhere in the warp's chunk take tanh from
    // its series on the FMA pipe, the others from its exponential form (MUFU)
    // (largest |x| of the chunk: four chains of three-input maxima)
    float m0 = max3(fabsf(x[0]), fabsf(x[1]), fabsf(x[2])), m1 = max3(fabsf(x[3]), fabsf(x[4]), fabsf(x[5]));
    float m2 = max3(fabsf(x[6]), fabsf(x[7]), fabsf(x[8])), m3 = max3(fabsf(x[9]), fabsf(x[10]), fabsf(x[11]));
#pragma unroll
    for (int e = 12; e < 28; e += 8) {
      m0 = max3(m0, fabsf(x[e]), fabsf(x[e + 1]));
      m1 = max3(m1, fabsf(x[e + 2]), fabsf(x[e + 3]));
      m2 = max3(m2, fabsf(x[e + 4]), fabsf(x[e + 5]));
      m3 = max3(m3, fabsf(x[e + 6]), fabsf(x[e + 7]));
    }
    m0 = max3(m0, fabsf(x[28]), fabsf(x[29]));
    m1 = max3(m1, fabsf(x[30]), fabsf(x[31]));
    if (__all_sync(0xffffffffu, fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) <= r.lim)) {
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float2 t = tanh_series2(make_float2(x[c], x[c + 1]), r.aux, r.aux2);
        x[c] = t.x;
        x[c + 1] = t.y;
      }
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] = r.aux2 * tanh_ex2(x[c] * r.aux);
    }
  } else if constexpr (score_of(MOD) == MOD_BOOST) {
    // the boost band |i - j| < radius covers the warp's chunk wholly, or
    // misses it wholly, except near its edges
    const float rad = static_cast<float>(md.boost_radius);
    const bool all_in = fabsf(di) < rad && fabsf(di - 31.f) < rad;
    const bool all_out = di - 31.f >= rad || di <= -rad;
    if (__all_sync(0xffffffffu, all_in)) {
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] *= r.aux;
    } else if (__all_sync(0xffffffffu, all_out)) {
#pragma unroll
      for (int c = 0; c < 32; ++c) x[c] *= r.sl2;
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const bool inside = fabsf(di - static_cast<float>(c)) < rad;
        x[c] *= inside ? r.aux : r.sl2;
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      float v = x[c];
      if constexpr (score_of(MOD) == MOD_ALIBI) {
        v = fmaf(v, r.sl2, -r.aux * fabsf(di - static_cast<float>(c)));
      } else {
        v = v * r.sl2;
      }
      x[c] = v;
    }
  }
  if (pred) {
    const int jlo = r.lo - k0 - c0, jhi = r.hi - k0 - c0;
#pragma unroll
    for (int c = 0; c < 32; ++c) x[c] = (c >= jlo && c <= jhi) ? x[c] : -INFINITY;
  }
}

// Scores whose transform is the plain scale (no score mod, any masks) stay
// raw until the exponent: the row maximum is taken on raw scores and the
// scale is folded into the exponent's FFMA.
__host__ __device__ constexpr bool pure_scale(int key) { return score_of(key) == MOD_NONE; }


// Apply mask (and, for the other mods, the mod itself) to one row of raw
// scores; return the row maximum in the base-2 domain.
template <int MOD, bool PRED>
__device__ __forceinline__ float row_scores(float (&x)[4][32], const RowCtx& rc, const ModDev& md,
                                            int k0, const uint4& bw) {
  float mx = -INFINITY;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if constexpr (pure_scale(MOD)) {
      if constexpr (PRED) {
        const int jlo = rc.lo - k0 - c * 32, jhi = rc.hi - k0 - c * 32;
#pragma unroll
        for (int e = 0; e < 32; ++e) x[c][e] = (e >= jlo && e <= jhi) ? x[c][e] : -INFINITY;
      }
    } else {
      transform32<MOD>(x[c], rc, md, k0, c * 32, PRED);
    }
    if constexpr (PRED && has_bitmap(MOD)) {
      // the bitmap mask: bit e of word c keeps key k0 + 32 c + e
      const uint32_t w = c == 0 ? bw.x : (c == 1 ? bw.y : (c == 2 ? bw.z : bw.w));
#pragma unroll
      for (int e = 0; e < 32; ++e) x[c][e] = ((w >> e) & 1u) ? x[c][e] : -INFINITY;
    }
    // three-input max: 16 instructions per 32 columns, 4 independent chains
    float m0 = max3(x[c][0], x[c][1], x[c][2]), m1 = max3(x[c][3], x[c][4], x[c][5]);
    float m2 = max3(x[c][6], x[c][7], x[c][8]), m3 = max3(x[c][9], x[c][10], x[c][11]);
#pragma unroll
    for (int e = 12; e < 28; e += 8) {
      m0 = max3(m0, x[c][e], x[c][e + 1]);
      m1 = max3(m1, x[c][e + 2], x[c][e + 3]);
      m2 = max3(m2, x[c][e + 4], x[c][e + 5]);
      m3 = max3(m3, x[c][e + 6], x[c][e + 7]);
    }
    m0 = max3(m0, x[c][28], x[c][29]);
    m1 = max3(m1, x[c][30], x[c][31]);
    mx = max3(mx, max3(m0, m1, m2), m3);
  }
  if constexpr (pure_scale(MOD)) mx *= rc.sl2;  // -inf stays -inf
  return mx;
}

// 2^(x0, x1) on the FMA pipe with packed fp32 pairs (finite inputs only),
// the same range reduction and polynomial as exp2_poly.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  const float2 t = __fadd2_rn(x, magic);
  const float2 n = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), x);
  float2 p = __ffma2_rn(make_float2(kExp2C3, kExp2C3), f, make_float2(kExp2C2, kExp2C2));
  p = __ffma2_rn(p, f, make_float2(kExp2C1, kExp2C1));
  p = __ffma2_rn(p, f, make_float2(kExp2C0, kExp2C0));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// P = 2^(x - m) for one row, written as bf16 pairs over the first 64 TMEM
// columns of the row's S tile; returns the fp32 row sum.  Scale, shift and
// the row sum use packed fp32 pairs.  With EMUL, 5 of every 16 pairs take the
// FMA-pipe polynomial instead of the MUFU ex2, balancing the two pipes.
template <int MOD, bool EMUL>
__device__ __forceinline__ float row_probs(float (&x)[4][32], const RowCtx& rc, float m_use,
                                           uint32_t s_addr) {
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
  const float2 neg_m = make_float2(-m_use, -m_use);
  const float2 sl2 = make_float2(rc.sl2, rc.sl2);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const float2 xs = make_float2(x[c][e], x[c][e + 1]);
      float2 arg;
      if constexpr (pure_scale(MOD)) {
        arg = __ffma2_rn(xs, sl2, neg_m);
      } else {
        arg = __fadd2_rn(xs, neg_m);
      }
      float2 pr;
      if (EMUL && ((e >> 1) % 3) == 2) {
        pr = exp2_poly2(arg);
      } else {
        pr = make_float2(ex2_approx(arg.x), ex2_approx(arg.y));
      }
      if ((e >> 1) & 1) acc1 = __fadd2_rn(acc1, pr);
      else acc0 = __fadd2_rn(acc0, pr);
      pk[e >> 1] = pack_bf16x2(pr.x, pr.y);
    }
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(s_addr + c * 16),
        "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3]), "r"(pk[4]), "r"(pk[5]), "r"(pk[6]),
        "r"(pk[7]), "r"(pk[8]), "r"(pk[9]), "r"(pk[10]), "r"(pk[11]), "r"(pk[12]),
        "r"(pk[13]), "r"(pk[14]), "r"(pk[15])
        : "memory");
  }
  const float2 acc = __fadd2_rn(acc0, acc1);
  return acc.x + acc.y;
}

template <int D, int MOD, bool HAS_LSE, bool FP8, bool CLC>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
  using Cfg = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzled tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  FwdBarriers* bars = reinterpret_cast<FwdBarriers*>(smem + Cfg::kBarOff);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_smem[2] = {sbase + Cfg::kQOff, sbase + Cfg::kQOff + Cfg::kTileBytes};
  const uint32_t ring = sbase + Cfg::kRingOff;
  uint32_t* lists = reinterpret_cast<uint32_t*>(smem + Cfg::kListOff);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->list_full[i]), 32);
      mbar_init(smem_u32(&bars->list_empty[i]), kListConsumers);
    }
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->q_empty), 1);
    mbar_init(smem_u32(&bars->clc_bar), 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&bars->s_full[t]), 1);
      mbar_init(smem_u32(&bars->p_full[t]), 128);
      mbar_init(smem_u32(&bars->o_full[t]), 1);
      mbar_init(smem_u32(&bars->o_final[t]), 1);
    }
    mbar_init(smem_u32(&bars->drain), 1);
    for (int s = 0; s < Cfg::kStages; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), 1);
    }
    bars->abort_flag = 0;
    bars->never_set = 0;
    fence_mbar_init();
  }
  if (warp == 8) {  // allocate all 512 TMEM columns (one CTA per SM)
    tmem_alloc(smem_u32(&bars->tmem_base), 512);
    tmem_relinquish();
  }
  if (warp == 9 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtl wc{a.wait_ns, smem_u32(&bars->abort_flag), a.status};
  long long tr[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  (void)tr;
  ATTN25_TRACE_ONLY(const long long t_start = clock64();)

  // every kernel takes the register split (the softcap and boost transforms
  // have warp-uniform fast paths that fit in the softmax warps' registers)
  constexpr bool kSplitRegs = true;
  if (warp >= 8) {
  if constexpr (kSplitRegs) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
  if (warp == 9) {
    // ------------------------------------------------------------ TMA producer
    // all lanes build the step lists; lane 0 issues the copies
    uint32_t slot_uses[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int ring_pos = 0;
    int unit_iter = 0;
    uint32_t q_loads = 0, clc_asked = 0, clc_read = 0;
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
      UnitCoord uc{};
      if constexpr (!CLC) uc = decode_unit(a, u);
      const int buf = unit_iter & 1;
      uint32_t* lst = lists + buf * kMaxSteps;
      if (!mbar_wait_warp(smem_u32(&bars->list_empty[buf]), ((unit_iter >> 1) & 1) ^ 1, wc)) { ok = false; break; }
      int n = 0;
      if constexpr (CLC) {
        if (u >= a.n_units) u = -1;
        if (u >= 0) uc = decode_unit(a, u);
        if (lane == 0) bars->list_unit[buf] = u;
      }
      if (u >= 0)
        n = build_pair_steps(a.tile_class, uc.b, uc.p, a.nQ, a.nK, a.Sq, a.Skv, a.mod.mask, a.mod.window, lst);
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
      const int hk = uc.h / a.G;
      if (lane == 0) {
        // Q buffers are free once the previous unit's QK^T products finished
        if (!ATTN25_TIMED(tr[1], mbar_wait_thread(smem_u32(&bars->q_empty), (unit_iter & 1) ^ 1, wc))) {
          ok = false;
        } else {
          constexpr int kQKBytes = FP8 ? Cfg::kTileBytes8 : Cfg::kTileBytes;
          mbar_arrive_expect_tx(smem_u32(&bars->q_full), 2 * kQKBytes);
          ++q_loads;
          load_qk_tile<D, FP8>(q_smem[0], &tm_q, smem_u32(&bars->q_full), (2 * uc.p) * TILE, uc.h, uc.b);
          load_qk_tile<D, FP8>(q_smem[1], &tm_q, smem_u32(&bars->q_full), (2 * uc.p + 1) * TILE, uc.h, uc.b);
          for (int j2 = 0; j2 < n && ok; ++j2) {
            const int kt = static_cast<int>(lst[j2] & 0xFFFFFu);
#pragma unroll
            for (int which = 0; which < 2; ++which) {  // K then V
              const int slot = ring_pos % Cfg::kStages;
              const uint32_t phase = (ring_pos / Cfg::kStages) & 1;
              if (!ATTN25_TIMED(tr[2], mbar_wait_thread(smem_u32(&bars->kv_empty[slot]), phase ^ 1, wc))) { ok = false; break; }
              const uint32_t bar = smem_u32(&bars->kv_full[slot]);
              if (which == 0) {  // K: e4m3 or bf16
                mbar_arrive_expect_tx(bar, kQKBytes);
                load_qk_tile<D, FP8>(ring + slot * Cfg::kTileBytes, &tm_k, bar, kt * TILE, hk, uc.b);
              } else {           // V: bf16
                mbar_arrive_expect_tx(bar, Cfg::kTileBytes);
                load_tile<D>(ring + slot * Cfg::kTileBytes, &tm_v, bar, kt * TILE, hk, uc.b);
              }
              ++slot_uses[slot];
              ++ring_pos;
            }
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      if constexpr (CLC) {  // the next unit: the rank of the cancelled CTA, or -1
        if (!mbar_wait_warp(clc_bar, clc_read & 1, wc)) { ok = false; break; }
        ++clc_read;
        u = clc_cancelled_x(clc_resp);
      } else {
        u = snake_unit(unit_iter + 1);
      }
    }
    if (lane == 0) {
      // let the copies in flight land before the CTA exits: after a failed wait
      // of this warp, and also after a normal end, since a consumer that gave
      // up may have left the last copies unconsumed (instant otherwise)
      const WaitCtl drain_wc{drain_limit(a.wait_ns), smem_u32(&bars->never_set), a.status};
      if (clc_asked > clc_read) mbar_wait_thread(clc_bar, (clc_asked - 1) & 1, drain_wc);
      for (int s2 = 0; s2 < Cfg::kStages; ++s2) {
        if (slot_uses[s2] == 0) continue;
        mbar_wait_thread(smem_u32(&bars->kv_full[s2]), (slot_uses[s2] - 1) & 1, drain_wc);
      }
      if (q_loads > 0)
        mbar_wait_thread(smem_u32(&bars->q_full), (q_loads - 1) & 1, drain_wc);
    }
    ATTN25_TRACE_ONLY(tr[0] = clock64() - t_start;)
    trace_flush(a.trace, 48, tr);
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    // all lanes run the loop (waits are warp-collective); lane 0 issues
    int ring_pos = 0;
    int unit_iter = 0;
    uint32_t p_cnt[2] = {0, 0};
    bool ok = true;
    const uint32_t s_tmem[2] = {tmem, tmem + 128};
    const uint32_t o_tmem[2] = {tmem + 256, tmem + 256 + D};
    for (;; ++unit_iter) {
      if constexpr (!CLC) {
        if (snake_unit(unit_iter) >= a.n_units) break;
      }
      const int buf = unit_iter & 1;
      const uint32_t* lst = lists + buf * kMaxSteps;
      if (!mbar_wait_warp(smem_u32(&bars->list_full[buf]), (unit_iter >> 1) & 1, wc)) { ok = false; break; }
      if constexpr (CLC) {
        if (bars->list_unit[buf] < 0) break;
      }
      const int n_steps = bars->list_n[buf];
      if (!ATTN25_TIMED(tr[1], mbar_wait_warp(smem_u32(&bars->q_full), unit_iter & 1, wc))) { ok = false; break; }
      tc_fence_after();
      int j = 0;
      bool act[2];
      bool has = n_steps > 0;
      if (has) {
        const uint32_t e = lst[0];
        act[0] = (e & kStepAct0) != 0;
        act[1] = (e & kStepAct1) != 0;
      }
      bool o_started[2] = {false, false};
      if (has) {
        const int slot_k = ring_pos % Cfg::kStages;
        if (!ATTN25_TIMED(tr[2], mbar_wait_warp(smem_u32(&bars->kv_full[slot_k]), (ring_pos / Cfg::kStages) & 1, wc))) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (act[t]) {
            issue_qk<D, FP8>(s_tmem[t], q_smem[t], ring + slot_k * Cfg::kTileBytes);
            mma_commit_w(smem_u32(&bars->s_full[t]));
          }
        mma_commit_w(smem_u32(&bars->kv_empty[slot_k]));
        ++ring_pos;
      }
      while (has && ok) {
        const int slot_v = ring_pos % Cfg::kStages;
        const uint32_t ph_v = (ring_pos / Cfg::kStages) & 1;
        ++ring_pos;
        bool act_n[2] = {false, false};
        const bool has_n = j + 1 < n_steps;
        if (has_n) {
          const uint32_t e = lst[j + 1];
          act_n[0] = (e & kStepAct0) != 0;
          act_n[1] = (e & kStepAct1) != 0;
        }
        const int slot_kn = ring_pos % Cfg::kStages;
        const uint32_t ph_kn = (ring_pos / Cfg::kStages) & 1;
        if (!ATTN25_TIMED(tr[3], mbar_wait_warp(smem_u32(&bars->kv_full[slot_v]), ph_v, wc))) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (act[t]) {
            if (!ATTN25_TIMED(tr[4 + t], mbar_wait_warp(smem_u32(&bars->p_full[t]), p_cnt[t] & 1, wc))) { ok = false; break; }
            ++p_cnt[t];
            tc_fence_after();
            issue_pv<D>(o_tmem[t], s_tmem[t], ring + slot_v * Cfg::kTileBytes, o_started[t]);
            mma_commit_w(smem_u32(&bars->o_full[t]));
            o_started[t] = true;
          }
          // the unit's last step: tile t's O is final once this PV completes, so its
          // epilogue need not wait for the other tile's last softmax.  (o_final
          // counts units with at least one step only, so that units without key
          // tiles cannot run its phases ahead of the epilogues.)
          if (!has_n) mma_commit_w(smem_u32(&bars->o_final[t]));
          if (has_n) {
            if (t == 0) {
              if (!ATTN25_TIMED(tr[2], mbar_wait_warp(smem_u32(&bars->kv_full[slot_kn]), ph_kn, wc))) { ok = false; break; }
              tc_fence_after();
            }
            if (act_n[t]) {
              issue_qk<D, FP8>(s_tmem[t], q_smem[t], ring + slot_kn * Cfg::kTileBytes);
              mma_commit_w(smem_u32(&bars->s_full[t]));
            }
          }
        }
        if (!ok) break;
        if (has_n) mma_commit_w(smem_u32(&bars->kv_empty[slot_kn]));
        mma_commit_w(smem_u32(&bars->kv_empty[slot_v]));
        if (has_n) ++ring_pos;
        has = has_n;
        ++j;
        act[0] = act_n[0];
        act[1] = act_n[1];
      }
      if (!ok) break;
      mma_commit_w(smem_u32(&bars->q_empty));
      if (lane == 0) mbar_arrive(smem_u32(&bars->list_empty[buf]));
      __syncwarp();
    }
    // drain: wait until every MMA this warp issued has completed
    mma_commit_w(smem_u32(&bars->drain));
    mbar_wait_warp(smem_u32(&bars->drain), 0, WaitCtl{drain_limit(a.wait_ns), smem_u32(&bars->never_set), a.status});
    ATTN25_TRACE_ONLY(tr[0] = clock64() - t_start;)
    trace_flush(a.trace, 32, tr);
  }
  } else {
    if constexpr (kSplitRegs) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
    // ------------------------------------------------------------ softmax warpgroups
    const int t = warp >> 2;                  // query tile of the pair
    const int r = threadIdx.x & 127;          // row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + t * 128 + lane_off;
    const uint32_t o_addr = tmem + 256 + t * D + lane_off;
    uint32_t s_cnt = 0, p_cnt = 0;
    int unit_iter = 0;
    uint32_t o_units = 0;  // units with at least one step seen so far (o_final phases)
    bool ok = true;
    for (;; ++unit_iter) {
      const int buf = unit_iter & 1;
      int u;
      if constexpr (CLC) {
        if (!mbar_wait_warp(smem_u32(&bars->list_full[buf]), (unit_iter >> 1) & 1, wc)) { ok = false; break; }
        u = bars->list_unit[buf];
        if (u < 0) break;
      } else {
        u = snake_unit(unit_iter);
        if (u >= a.n_units) break;
      }
      const UnitCoord uc = decode_unit(a, u);
      RowCtx rc;
      rc.row = (2 * uc.p + t) * TILE + r;
      rc.sl2 = a.sl2;
      if constexpr (FP8) {  // the scores come out of the MMA in code units: dequantise in the exponent's scale
        static_assert(score_of(MOD) == MOD_NONE, "FP8 scores take masks only");
        rc.sl2 *= __ldg(a.q_scales + uc.b * a.Hq + uc.h) * __ldg(a.k_scales + uc.b * a.Hkv + uc.h / a.G);
      }
      rc.aux = 0.f;
      rc.aux2 = 0.f;
      rc.lim = 0.f;
      if constexpr (score_of(MOD) == MOD_ALIBI) rc.aux = alibi_slope(a.mod, uc.h, a.Hq) * LOG2E;
      if constexpr (score_of(MOD) == MOD_SOFTCAP) {
        rc.aux = a.scale / a.mod.softcap;
        rc.aux2 = a.mod.softcap * LOG2E;
        rc.lim = kTanhSeriesLimit * a.mod.softcap / a.scale;
      }
      if constexpr (score_of(MOD) == MOD_BOOST) rc.aux = a.mod.boost * a.sl2;
      if constexpr (masked(MOD)) {
        row_interval(a.mod, uc.b, min(rc.row, a.Sq - 1), a.Skv, rc.lo, rc.hi);
      } else {
        rc.lo = 0;
        rc.hi = a.Skv - 1;
      }
      if (rc.row >= a.Sq) rc.hi = rc.lo - 1;  // padding rows keep nothing
      rc.bits = nullptr;
      if constexpr (has_bitmap(MOD)) {
        if (rc.row < a.Sq) rc.bits = bitmap_row(a.mod, uc.b, uc.h, rc.row);
      }

      float m_run = -INFINITY, l_run = 0.f;
      int n_act = 0;
      const uint32_t* lst = lists + buf * kMaxSteps;
      if constexpr (!CLC) {
        if (!mbar_wait_warp(smem_u32(&bars->list_full[buf]), (unit_iter >> 1) & 1, wc)) { ok = false; break; }
      }
      const int n_steps = bars->list_n[buf];
      const uint32_t act_bit = t == 0 ? kStepAct0 : kStepAct1;
      const uint32_t prt_bit = t == 0 ? kStepPrt0 : kStepPrt1;
      for (int j = 0; j < n_steps; ++j) {
        const uint32_t e = lst[j];
        if (!(e & act_bit)) continue;
        const int kt = static_cast<int>(e & 0xFFFFFu);
        const bool prt_t = (e & prt_bit) != 0;
        uint4 bw = make_uint4(0u, 0u, 0u, 0u);  // keep bits of this row's 128 keys (PARTIAL tiles)
        if constexpr (has_bitmap(MOD)) {
          if (prt_t && rc.bits != nullptr) bw = __ldg(reinterpret_cast<const uint4*>(rc.bits) + kt);
        }
        if (!ATTN25_TIMED(tr[1], mbar_wait_warp(smem_u32(&bars->s_full[t]), s_cnt & 1, wc))) { ok = false; break; }
        ++s_cnt;
        ATTN25_TRACE_ONLY(const long long t_tile = clock64(); tr[7] += 1;)
        tc_fence_after();
        const int k0 = kt * TILE;
        float x[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(s_addr + c * 32, reinterpret_cast<uint32_t(&)[32]>(x[c]));
        tmem_wait_ld();
        // local boost: a tile whose keys lie outside every row's band (the warp's
        // rows, warp-uniform) takes the plain-scale path of the masks-only key
        constexpr int kPlain = MOD & ~(kKeyMasked - 1);
        bool plain = false;
        if constexpr (score_of(MOD) == MOD_BOOST) {
          const float rad = static_cast<float>(a.mod.boost_radius), di = static_cast<float>(rc.row - k0);
          plain = __all_sync(0xffffffffu, di - static_cast<float>(TILE - 1) >= rad || di <= -rad);
        }
        float mx;
        if (plain) {
          mx = prt_t ? row_scores<kPlain, true>(x, rc, a.mod, k0, bw) : row_scores<kPlain, false>(x, rc, a.mod, k0, bw);
        } else {
          mx = prt_t ? row_scores<MOD, true>(x, rc, a.mod, k0, bw) : row_scores<MOD, false>(x, rc, a.mod, k0, bw);
        }
        const float m_new = fmaxf(m_run, mx);
        const bool need = m_new > m_run + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_new);
          if (n_act > 0) {
            // O must be complete (previous P V finished) before it is rescaled
            if (!mbar_wait_warp(smem_u32(&bars->o_full[t]), (p_cnt - 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < D / 16; ++c) {
              uint32_t o[16];
              tmem_ld16(o_addr + c * 16, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st16(o_addr + c * 16, o);
            }
          }
          l_run *= alpha;
          m_run = m_new;
          ATTN25_TRACE_ONLY(tr[6] += 1;)
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        ATTN25_TRACE_ONLY(const long long t_mid = clock64(); tr[2] += t_mid - t_tile;)
        // full tiles hold no -inf, so part of their exponentials can run on the FMA
        // pipe (not with softcap, whose tanh series already loads that pipe)
        float lsum;
        if constexpr (score_of(MOD) == MOD_SOFTCAP) lsum = row_probs<MOD, false>(x, rc, m_use, s_addr);
        else if (plain) lsum = prt_t ? row_probs<kPlain, false>(x, rc, m_use, s_addr) : row_probs<kPlain, true>(x, rc, m_use, s_addr);
        else lsum = prt_t ? row_probs<MOD, false>(x, rc, m_use, s_addr) : row_probs<MOD, true>(x, rc, m_use, s_addr);
        l_run += lsum;
        ATTN25_TRACE_ONLY(tr[3] += clock64() - t_mid;)
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&bars->p_full[t]));
        ++p_cnt;
        ++n_act;
      }
      if (!ok) break;
      // ---- epilogue of this unit: O / l -> bf16, LSE
      if (n_steps > 0) {
        if (!ATTN25_TIMED(tr[4], mbar_wait_warp(smem_u32(&bars->o_final[t]), o_units & 1, wc))) { ok = false; break; }
        ++o_units;
      }
      ATTN25_TRACE_ONLY(const long long t_epi = clock64();)
      tc_fence_after();
      const bool row_valid = rc.row < a.Sq;
      const size_t row_idx = (static_cast<size_t>(uc.b) * a.Hq + uc.h) * a.Sq + rc.row;
      __nv_bfloat16* orow = a.out + uc.b * a.o_st.b + uc.h * a.o_st.h + static_cast<long long>(rc.row) * a.o_st.s;
      const float inv_l = (l_run > 0.f) ? 1.0f / l_run : 0.f;
      // 32-byte stores where the row allows them (a full L2 sector per lane)
      const bool wide = (reinterpret_cast<uintptr_t>(orow) & 31u) == 0;
#pragma unroll
      for (int c2 = 0; c2 < D / 64; ++c2) {  // two 32-column chunks per TMEM round trip
        uint32_t o[2][32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (n_act > 0) {
            tmem_ld32(o_addr + (2 * c2 + h) * 32, o[h]);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[h][e] = 0u;
          }
        }
        if (n_act > 0) tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c = 2 * c2 + h;
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(o[h][2 * e]) * inv_l, __uint_as_float(o[h][2 * e + 1]) * inv_l);
          if (row_valid) {
            if (wide) {
#pragma unroll
              for (int e = 0; e < 2; ++e) st_global_v8(orow + c * 32 + e * 16, &pk[8 * e]);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
              for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            }
          }
        }
      }
      if constexpr (HAS_LSE) {
        if (row_valid)
          a.lse[row_idx] = (l_run > 0.f) ? (m_run + __log2f(l_run)) * LN2 : -INFINITY;
      }
      tc_fence_before();
      if (lane == 0) mbar_arrive(smem_u32(&bars->list_empty[buf]));
      ATTN25_TRACE_ONLY(tr[5] += clock64() - t_epi;)
    }
    ATTN25_TRACE_ONLY(tr[0] = clock64() - t_start;)
    trace_flush(a.trace, 16 * t, tr);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 8) tmem_dealloc(tmem, 512);
}

}  // namespace

}  // namespace attn25

namespace attn25 {

namespace {

template <int D, int MOD, bool LSE, bool FP8, bool CLC>
cudaError_t launch_fwd_k(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const FwdArgs& a, int grid, cudaStream_t stream) {
  auto kernel = attn_fwd_kernel<D, MOD, LSE, FP8, CLC>;
  // The register split assumes the kernel launches with kLaunchRegs per
  // thread; with fewer, setmaxnreg.inc could wait forever, so refuse.
  static int launch_regs = -1;
  if (launch_regs < 0) {
    cudaFuncAttributes attr;
    cudaError_t e0 = cudaFuncGetAttributes(&attr, kernel);
    if (e0 != cudaSuccess) return e0;
    launch_regs = attr.numRegs;
  }
  if (launch_regs < kLaunchRegs) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       FwdCfg<D>::kAllocBytes);
  if (e != cudaSuccess) return e;
  kernel<<<grid, kFwdThreads, FwdCfg<D>::kAllocBytes, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

template <int D, int MOD, bool LSE, bool FP8 = false>
cudaError_t launch_fwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                         const FwdArgs& a, int grid, cudaStream_t stream) {
  return a.clc ? launch_fwd_k<D, MOD, LSE, FP8, true>(tq, tk, tv, a, grid, stream)
               : launch_fwd_k<D, MOD, LSE, FP8, false>(tq, tk, tv, a, grid, stream);
}

template <int D, bool LSE>
cudaError_t launch_fwd_mod(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const FwdArgs& a, int key, int grid, cudaStream_t s) {
  constexpr int M = kKeyMasked, MB = kKeyMasked | kKeyBitmap;
  switch (key) {
    case MOD_NONE: return launch_fwd_t<D, MOD_NONE, LSE>(tq, tk, tv, a, grid, s);
    case MOD_ALIBI: return launch_fwd_t<D, MOD_ALIBI, LSE>(tq, tk, tv, a, grid, s);
    case MOD_SOFTCAP: return launch_fwd_t<D, MOD_SOFTCAP, LSE>(tq, tk, tv, a, grid, s);
    case MOD_BOOST: return launch_fwd_t<D, MOD_BOOST, LSE>(tq, tk, tv, a, grid, s);
    case M | MOD_NONE: return launch_fwd_t<D, M | MOD_NONE, LSE>(tq, tk, tv, a, grid, s);
    case M | MOD_ALIBI: return launch_fwd_t<D, M | MOD_ALIBI, LSE>(tq, tk, tv, a, grid, s);
    case M | MOD_SOFTCAP: return launch_fwd_t<D, M | MOD_SOFTCAP, LSE>(tq, tk, tv, a, grid, s);
    case M | MOD_BOOST: return launch_fwd_t<D, M | MOD_BOOST, LSE>(tq, tk, tv, a, grid, s);
    case MB | MOD_NONE: return launch_fwd_t<D, MB | MOD_NONE, LSE>(tq, tk, tv, a, grid, s);
    case MB | MOD_ALIBI: return launch_fwd_t<D, MB | MOD_ALIBI, LSE>(tq, tk, tv, a, grid, s);
    case MB | MOD_SOFTCAP: return launch_fwd_t<D, MB | MOD_SOFTCAP, LSE>(tq, tk, tv, a, grid, s);
    case MB | MOD_BOOST: return launch_fwd_t<D, MB | MOD_BOOST, LSE>(tq, tk, tv, a, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const FwdArgs& a, int key, bool has_lse, int grid, cudaStream_t s) {
  constexpr int M = kKeyMasked, MB = kKeyMasked | kKeyBitmap;
  switch (key) {
    case MOD_NONE:
      return has_lse ? launch_fwd_t<128, MOD_NONE, true, true>(tq, tk, tv, a, grid, s)
                     : launch_fwd_t<128, MOD_NONE, false, true>(tq, tk, tv, a, grid, s);
    case M | MOD_NONE:
      return has_lse ? launch_fwd_t<128, M | MOD_NONE, true, true>(tq, tk, tv, a, grid, s)
                     : launch_fwd_t<128, M | MOD_NONE, false, true>(tq, tk, tv, a, grid, s);
    case MB | MOD_NONE:
      return has_lse ? launch_fwd_t<128, MB | MOD_NONE, true, true>(tq, tk, tv, a, grid, s)
                     : launch_fwd_t<128, MB | MOD_NONE, false, true>(tq, tk, tv, a, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdArgs& a, int D, int key, bool has_lse, int grid,
                       cudaStream_t stream) {
  if (D == 128)
    return has_lse ? launch_fwd_mod<128, true>(tq, tk, tv, a, key, grid, stream)
                   : launch_fwd_mod<128, false>(tq, tk, tv, a, key, grid, stream);
  if (D == 64)
    return has_lse ? launch_fwd_mod<64, true>(tq, tk, tv, a, key, grid, stream)
                   : launch_fwd_mod<64, false>(tq, tk, tv, a, key, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace attn25
