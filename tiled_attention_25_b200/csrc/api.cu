// The C ABI of libattn25.so: argument checks, TMA descriptor encoding and
// kernel dispatch.  Every exported function is declared in include/attn25.h.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "attn25.h"
#include "kernel_common.cuh"
#include "launch.h"

namespace attn25 {

// One status word per device that loads the library.
__device__ int g_attn_status;

#if defined(ATTN25_TRACE)
// Profiling builds: per-role cycle counters (forward at 0, backward at 128),
// then the backward's per-step event clocks.
__device__ unsigned long long g_attn_trace[kTraceWords];
#endif

// Backward workspace for attn_bwd_noalloc: a fixed block of device memory
// that every GPU loading this library holds until the process exits, so
// that callers without an allocator can still run the backward pass.
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_bwd_scratch[kNoAllocScratchBytes];

namespace {

std::atomic<uint32_t> g_wait_ms{4000};
std::atomic<int> g_work_walk{1};  // ATTN_WALK_CLUSTER_LAUNCH_CONTROL (default) or ATTN_WALK_STATIC

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  bool usable = false;
  int sms = 0;
  int* status = nullptr;
  unsigned long long* trace = nullptr;
  void* scratch = nullptr;  // device address of g_bwd_scratch (nullptr if unavailable)
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int current_device(DeviceInfo** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    d.ready = true;
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    void* p = nullptr;
    const bool sym_ok = cudaGetSymbolAddress(&p, g_attn_status) == cudaSuccess;
    d.status = static_cast<int*>(p);
    // Host code must not use g_bwd_scratch's name as a device address: look
    // up the real address once, with this device current.
    void* sp = nullptr;
    if (cudaGetSymbolAddress(&sp, g_bwd_scratch) == cudaSuccess) d.scratch = sp;
#if defined(ATTN25_TRACE)
    void* tp = nullptr;
    if (cudaGetSymbolAddress(&tp, g_attn_trace) == cudaSuccess) d.trace = static_cast<unsigned long long*>(tp);
#endif
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
              cudaSuccess &&
          q == cudaDriverEntryPointSuccess)
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.usable = (major == 10) && sym_ok && d.sms > 0 && g_encode != nullptr;
    cudaGetLastError();  // do not leak a sticky-free error from the probes
  }
  if (!d.usable) return ATTN_ERR_DEVICE;
  *out = &d;
  return ATTN_OK;
}

// bf16 tensor [outer][rows][inner] with rows x 64-column boxes, 128-byte swizzle.
// A [B][H][S][D] bf16 tensor whose D elements are contiguous, as the 4-D map
// (D, S, H, B) with the tensor's own strides; boxes of 64 x box_rows x 1 x 1.
bool encode_bf16_4d(CUtensorMap* m, const void* base, int D, int S, int H, int B, const Strides& st,
                    int box_rows) {
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(st.s) * 2, static_cast<cuuint64_t>(st.h) * 2,
                           static_cast<cuuint64_t>(st.b) * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Contiguous [B][H][S][D = 128] e4m3 codes as the 4-D map (D, S, H, B): one
// box of 128 bytes x box_rows rows, 128-byte swizzle.
bool encode_u8_4d(CUtensorMap* m, const void* base, int D, int S, int H, int B, int box_rows) {
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S) * D,
                           static_cast<cuuint64_t>(H) * S * D};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The strides of a tensor: the caller's, or those of contiguous [B][H][S][D].
bool layout_of(const attn_strides* given, int H, int S, int D, Strides& st) {
  if (given == nullptr) {
    st = Strides{static_cast<long long>(H) * S * D, static_cast<long long>(S) * D, D};
    return true;
  }
  st = Strides{given->b, given->h, given->s};
  // the tensor maps take strides of whole 16-byte units
  return st.b >= 8 && st.h >= 8 && st.s >= 8 && st.b % 8 == 0 && st.h % 8 == 0 && st.s % 8 == 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int cdiv(int a, int b) { return (a + b - 1) / b; }

uint64_t wait_ns() { return static_cast<uint64_t>(g_wait_ms.load()) * 1000000ull; }

// One warp waits, with the kernels' bounded wait, on a barrier that nothing
// arrives at: after the wait limit it records ATTN_ERR_TIMEOUT in the status
// word and returns, the same path a kernel takes when one of its waits runs out.
__global__ void wait_check_kernel(uint64_t limit_ns, int* status) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_word;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_word = 0;
    fence_mbar_init();
  }
  __syncwarp();
  const WaitCtl wc{limit_ns, smem_u32(&abort_word), status};
  (void)mbar_wait_warp(smem_u32(&bar), 0, wc);
}

// A mod code split into its score transform and mask bits (composition:
// one of the seven kinds, optionally ORed with ATTN_MASK_* flags).
struct ModSpec {
  int score;      // MOD_NONE, MOD_ALIBI, MOD_SOFTCAP or MOD_BOOST
  int mask;       // kMask* bits; window and document imply causal
  int key;        // kernel specialisation key
  int canonical;  // score | ATTN_MASK_* flags: equal for codes that mean the same mod
};

bool split_mod(int code, ModSpec& m) {
  const int base = code & 0xFF, flags = code & ~0xFF;
  if (base < ATTN_MOD_NONE || base > ATTN_MOD_DOCUMENT) return false;
  if (flags & ~(ATTN_MASK_CAUSAL | ATTN_MASK_SLIDING_WINDOW | ATTN_MASK_DOCUMENT | ATTN_MASK_BITMAP |
                ATTN_MASK_VARLEN))
    return false;
  // the varlen mask takes no other mask (a causal packing of equal lengths is the document mask)
  if ((flags & ATTN_MASK_VARLEN) &&
      ((flags & ~ATTN_MASK_VARLEN) || base == ATTN_MOD_CAUSAL || base == ATTN_MOD_SLIDING_WINDOW ||
       base == ATTN_MOD_DOCUMENT))
    return false;
  m.score = MOD_NONE;
  m.mask = 0;
  switch (base) {
    case ATTN_MOD_CAUSAL: m.mask |= kMaskCausal; break;
    case ATTN_MOD_ALIBI: m.score = MOD_ALIBI; break;
    case ATTN_MOD_SOFTCAP: m.score = MOD_SOFTCAP; break;
    case ATTN_MOD_SLIDING_WINDOW: m.mask |= kMaskCausal | kMaskWindow; break;
    case ATTN_MOD_LOCAL_BOOST: m.score = MOD_BOOST; break;
    case ATTN_MOD_DOCUMENT: m.mask |= kMaskCausal | kMaskDoc; break;
    default: break;
  }
  if (flags & ATTN_MASK_CAUSAL) m.mask |= kMaskCausal;
  if (flags & ATTN_MASK_SLIDING_WINDOW) m.mask |= kMaskCausal | kMaskWindow;
  if (flags & ATTN_MASK_DOCUMENT) m.mask |= kMaskCausal | kMaskDoc;
  if (flags & ATTN_MASK_BITMAP) m.mask |= kMaskBitmap;
  if (flags & ATTN_MASK_VARLEN) m.mask |= kMaskVarlen;
  m.key = m.score | (m.mask != 0 ? kKeyMasked : 0) | ((m.mask & kMaskBitmap) ? kKeyBitmap : 0);
  m.canonical = m.score | ((m.mask & kMaskCausal) ? ATTN_MASK_CAUSAL : 0) |
                ((m.mask & kMaskWindow) ? ATTN_MASK_SLIDING_WINDOW : 0) |
                ((m.mask & kMaskDoc) ? ATTN_MASK_DOCUMENT : 0) |
                ((m.mask & kMaskBitmap) ? ATTN_MASK_BITMAP : 0) |
                ((m.mask & kMaskVarlen) ? ATTN_MASK_VARLEN : 0);
  return true;
}

// Shared validation of shapes, mod and mask.
int check_common(int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale, int mod_kind,
                 const attn_mod_params* mp, const attn_block_mask* bm) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Skv < 1) return ATTN_ERR_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return ATTN_ERR_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  // coordinates and unit counts stay well inside int32
  if (static_cast<long long>(B) * Hq * (cdiv(Sq, TILE) + 1) >= (1ll << 30)) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Hq >= (1ll << 30)) return ATTN_ERR_UNSUPPORTED;
  // per-unit step lists live in shared memory: at most kMaxSteps tiles each way
  if (cdiv(Sq, TILE) > kMaxSteps || cdiv(Skv, TILE) > kMaxSteps) return ATTN_ERR_UNSUPPORTED;
  ModSpec ms;
  if (!split_mod(mod_kind, ms)) return ATTN_ERR_ARG;
  if (ms.score == MOD_SOFTCAP &&
      (mp == nullptr || !(mp->softcap > 0.f) || !std::isfinite(mp->softcap)))
    return ATTN_ERR_ARG;
  if (ms.score == MOD_BOOST && (mp == nullptr || !std::isfinite(mp->boost) || mp->boost_radius < 0))
    return ATTN_ERR_ARG;
  if (ms.score == MOD_ALIBI && mp != nullptr && mp->alibi_slopes != nullptr &&
      (reinterpret_cast<uintptr_t>(mp->alibi_slopes) & 3u))
    return ATTN_ERR_ALIGN;
  if ((ms.mask & kMaskWindow) && (mp == nullptr || mp->window < 1)) return ATTN_ERR_ARG;
  if (ms.mask & kMaskDoc) {
    if (mp == nullptr || mp->doc_offsets == nullptr || mp->num_docs < 1 || mp->num_docs > 4096)
      return ATTN_ERR_ARG;
    if (Sq != Skv) return ATTN_ERR_UNSUPPORTED;
    if (reinterpret_cast<uintptr_t>(mp->doc_offsets) & 3u) return ATTN_ERR_ALIGN;
  }
  if (ms.mask & kMaskVarlen) {
    if (mp == nullptr || mp->q_offsets == nullptr || mp->k_offsets == nullptr || mp->num_seqs < 1 ||
        mp->num_seqs > 65536)
      return ATTN_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(mp->q_offsets) & 3u) || (reinterpret_cast<uintptr_t>(mp->k_offsets) & 3u))
      return ATTN_ERR_ALIGN;
  }
  if (ms.mask & kMaskBitmap) {
    if (mp == nullptr || mp->bitmap == nullptr) return ATTN_ERR_ARG;
    if (!aligned16(mp->bitmap)) return ATTN_ERR_ALIGN;
    if (mp->bitmap_row_words < cdiv(Skv, 32) || (mp->bitmap_row_words & 3)) return ATTN_ERR_ARG;
    if (mp->bitmap_heads < 1 || mp->bitmap_head_stride < 0 || mp->bitmap_batch_stride < 0 ||
        (mp->bitmap_head_stride & 3) || (mp->bitmap_batch_stride & 3))
      return ATTN_ERR_ARG;
    if (mp->bitmap_heads == 1 && mp->bitmap_head_stride != 0) return ATTN_ERR_ARG;
  }
  if (bm != nullptr) {
    if (bm->tile_class == nullptr || bm->kv_count == nullptr || bm->kv_index == nullptr ||
        bm->q_count == nullptr || bm->q_index == nullptr || bm->fwd_order == nullptr ||
        bm->bwd_order == nullptr)
      return ATTN_ERR_ARG;
    if (bm->B != B || bm->Sq != Sq || bm->Skv != Skv || bm->nq_tiles != cdiv(Sq, TILE) ||
        bm->nk_tiles != cdiv(Skv, TILE) || bm->mod_kind != ms.canonical)
      return ATTN_ERR_ARG;
  }
  return ATTN_OK;
}

// The bitmap mask's extra rules for attn_fwd / attn_bwd: its heads are the
// call's query heads (or one shared mask), and a block mask, which is the
// only place its tile classes come from, is given.
int check_bitmap_call(int mod_kind, int Hq, const attn_mod_params* mp, const attn_block_mask* bm) {
  ModSpec ms;
  split_mod(mod_kind, ms);
  if (!(ms.mask & kMaskBitmap)) return ATTN_OK;
  if (bm == nullptr) return ATTN_ERR_ARG;
  if (mp->bitmap_heads != 1 && mp->bitmap_heads != Hq) return ATTN_ERR_ARG;
  return ATTN_OK;
}

// Device view of a validated mod code.
ModDev make_mod(int mod_kind, const attn_mod_params* mp) {
  ModSpec ms;
  split_mod(mod_kind, ms);
  ModDev m{};
  m.kind = ms.score;
  m.mask = ms.mask;
  m.window = 1 << 30;
  if (mp != nullptr) {
    m.softcap = mp->softcap;
    m.boost = mp->boost;
    m.boost_radius = mp->boost_radius;
    m.alibi_slopes = mp->alibi_slopes;
    if (ms.mask & kMaskWindow) m.window = mp->window;
    if (ms.mask & kMaskDoc) {
      m.doc_offsets = mp->doc_offsets;
      m.num_docs = mp->num_docs;
    }
    if (ms.mask & kMaskVarlen) {
      m.vq_offsets = mp->q_offsets;
      m.vk_offsets = mp->k_offsets;
      m.n_seqs = mp->num_seqs;
    }
    if (ms.mask & kMaskBitmap) {
      m.bitmap = mp->bitmap;
      m.bm_row_words = mp->bitmap_row_words;
      m.bm_head_stride = mp->bitmap_head_stride;
      m.bm_batch_stride = mp->bitmap_batch_stride;
    }
  }
  return m;
}

int mod_key(int mod_kind) {
  ModSpec ms;
  split_mod(mod_kind, ms);
  return ms.key;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct MaskLayout {
  size_t off[7];
  size_t total;
};

MaskLayout mask_layout(int B, int Sq, int Skv) {
  const size_t nQ = cdiv(Sq, TILE), nK = cdiv(Skv, TILE), nP = (nQ + 1) / 2;
  const size_t sizes[7] = {B * nQ * nK,      B * nQ * 4, B * nQ * nK * 4, B * nK * 4,
                           B * nK * nQ * 4, B * nP * 4, B * nK * 4};
  MaskLayout L;
  size_t o = 0;
  for (int i = 0; i < 7; ++i) {
    L.off[i] = o;
    o += align256(sizes[i]);
  }
  L.total = o;
  return L;
}

}  // namespace

}  // namespace attn25

using namespace attn25;

extern "C" {

const char* attn_strerror(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported shape or option";
    case ATTN_ERR_ALIGN: return "pointer not 16-byte aligned";
    case ATTN_ERR_WORKSPACE: return "workspace or mask buffer too small";
    case ATTN_ERR_LAUNCH: return "CUDA launch failed";
    case ATTN_ERR_TIMEOUT: return "kernel timed out waiting on an internal barrier";
    case ATTN_ERR_DEVICE: return "no usable sm_100 device";
    default: return "unknown status";
  }
}

void attn_set_wait_limit_ms(uint32_t ms) { g_wait_ms.store(ms < 1 ? 1 : ms); }

int attn_set_work_walk(int walk) {
  if (walk != ATTN_WALK_STATIC && walk != ATTN_WALK_CLUSTER_LAUNCH_CONTROL) return ATTN_ERR_ARG;
  g_work_walk.store(walk);
  return ATTN_OK;
}

int attn_check_wait_timeout(attn_stream_t stream) {
  DeviceInfo* d = nullptr;
  const int rc = current_device(&d);
  if (rc != ATTN_OK) return rc;
  wait_check_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(wait_ns(), d->status);
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

int attn_get_status(attn_stream_t stream) {
  DeviceInfo* d = nullptr;
  int rc = current_device(&d);
  if (rc != ATTN_OK) return rc;
  int value = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&value, d->status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ATTN_ERR_LAUNCH;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (value != 0) {
    const int zero = 0;
    cudaMemcpyAsync(d->status, &zero, sizeof(int), cudaMemcpyHostToDevice, s);
    cudaStreamSynchronize(s);
  }
  return value;
}

size_t attn_block_mask_bytes(int B, int Sq, int Skv) {
  if (B < 1 || Sq < 1 || Skv < 1) return 0;
  return mask_layout(B, Sq, Skv).total;
}

int attn_block_mask_bind(void* buffer, size_t bytes, int B, int Sq, int Skv,
                         attn_block_mask* out) {
  if (buffer == nullptr || out == nullptr || B < 1 || Sq < 1 || Skv < 1) return ATTN_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(buffer) & 255u) return ATTN_ERR_ALIGN;
  const MaskLayout L = mask_layout(B, Sq, Skv);
  if (bytes < L.total) return ATTN_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(buffer);
  out->tile_class = base + L.off[0];
  out->kv_count = reinterpret_cast<int32_t*>(base + L.off[1]);
  out->kv_index = reinterpret_cast<int32_t*>(base + L.off[2]);
  out->q_count = reinterpret_cast<int32_t*>(base + L.off[3]);
  out->q_index = reinterpret_cast<int32_t*>(base + L.off[4]);
  out->fwd_order = reinterpret_cast<int32_t*>(base + L.off[5]);
  out->bwd_order = reinterpret_cast<int32_t*>(base + L.off[6]);
  out->B = B;
  out->Sq = Sq;
  out->Skv = Skv;
  out->nq_tiles = cdiv(Sq, TILE);
  out->nk_tiles = cdiv(Skv, TILE);
  out->mod_kind = -1;
  return ATTN_OK;
}

int build_block_mask(int mod_kind, const attn_mod_params* mod_params, int B, int Sq, int Skv,
                     attn_block_mask* mask, attn_stream_t stream) {
  if (mask == nullptr) return ATTN_ERR_ARG;
  if (mask->tile_class == nullptr || mask->B != B || mask->Sq != Sq || mask->Skv != Skv)
    return ATTN_ERR_ARG;
  int rc = check_common(B, 1, 1, Sq, Skv, 64, 1.f, mod_kind, mod_params, nullptr);
  if (rc != ATTN_OK) return rc;
  DeviceInfo* d = nullptr;
  rc = current_device(&d);
  if (rc != ATTN_OK) return rc;
  const ModDev md = make_mod(mod_kind, mod_params);
  ModSpec ms;
  split_mod(mod_kind, ms);
  MaskArgs a{};
  a.mask = md.mask;
  a.window = md.window;
  a.doc_offsets = md.doc_offsets;
  a.num_docs = md.num_docs;
  a.bitmap = md.bitmap;
  a.bm_row_words = md.bm_row_words;
  a.bm_heads = md.bitmap != nullptr ? mod_params->bitmap_heads : 0;
  a.bm_head_stride = md.bm_head_stride;
  a.bm_batch_stride = md.bm_batch_stride;
  a.vq_offsets = md.vq_offsets;
  a.vk_offsets = md.vk_offsets;
  a.n_seqs = md.n_seqs;
  a.B = B;
  a.Sq = Sq;
  a.Skv = Skv;
  a.nQ = cdiv(Sq, TILE);
  a.nK = cdiv(Skv, TILE);
  a.nP = (a.nQ + 1) / 2;
  a.tile_class = mask->tile_class;
  a.kv_count = mask->kv_count;
  a.kv_index = mask->kv_index;
  a.q_count = mask->q_count;
  a.q_index = mask->q_index;
  a.fwd_order = mask->fwd_order;
  a.bwd_order = mask->bwd_order;
  if (launch_block_mask(a, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_LAUNCH;
  mask->mod_kind = ms.canonical;
  return ATTN_OK;
}

// The forward: bf16 Q and K (strided), or (fp8) contiguous e4m3 codes of Q
// and K with their per-head scales.
static int fwd_impl(const void* q, const void* k, const attn_bf16* v, attn_bf16* out, float* lse,
                    const float* q_scales, const float* k_scales, bool fp8, int B, int Hq, int Hkv, int Sq,
                    int Skv, int D, float scale, int mod_kind, const attn_mod_params* mod_params,
                    const attn_block_mask* block_mask, const attn_layouts* layouts, attn_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return ATTN_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return ATTN_ERR_ALIGN;
  int rc = check_common(B, Hq, Hkv, Sq, Skv, D, scale, mod_kind, mod_params, block_mask);
  if (rc == ATTN_OK) rc = check_bitmap_call(mod_kind, Hq, mod_params, block_mask);
  if (rc != ATTN_OK) return rc;
  DeviceInfo* d = nullptr;
  rc = current_device(&d);
  if (rc != ATTN_OK) return rc;

  Strides sq, sk, sv, so;
  if (!layout_of(layouts ? &layouts->q : nullptr, Hq, Sq, D, sq) ||
      !layout_of(layouts ? &layouts->k : nullptr, Hkv, Skv, D, sk) ||
      !layout_of(layouts ? &layouts->v : nullptr, Hkv, Skv, D, sv) ||
      !layout_of(layouts ? &layouts->out : nullptr, Hq, Sq, D, so))
    return ATTN_ERR_ALIGN;
  CUtensorMap tq, tk, tv;
  const bool qk_ok = fp8 ? encode_u8_4d(&tq, q, D, Sq, Hq, B, TILE) && encode_u8_4d(&tk, k, D, Skv, Hkv, B, TILE)
                         : encode_bf16_4d(&tq, q, D, Sq, Hq, B, sq, TILE) &&
                               encode_bf16_4d(&tk, k, D, Skv, Hkv, B, sk, TILE);
  if (!qk_ok || !encode_bf16_4d(&tv, v, D, Skv, Hkv, B, sv, TILE)) return ATTN_ERR_ARG;

  FwdArgs a{};
  a.out = reinterpret_cast<__nv_bfloat16*>(out);
  a.o_st = so;
  a.lse = lse;
  a.q_scales = q_scales;
  a.k_scales = k_scales;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.Sq = Sq;
  a.Skv = Skv;
  a.nQ = cdiv(Sq, TILE);
  a.nK = cdiv(Skv, TILE);
  a.nP = (a.nQ + 1) / 2;
  a.n_units = B * a.nP * Hq;
  a.scale = scale;
  a.sl2 = scale * LOG2E;
  a.mod = make_mod(mod_kind, mod_params);
  if (block_mask != nullptr) {
    a.tile_class = block_mask->tile_class;
    a.kv_count = block_mask->kv_count;
    a.kv_index = block_mask->kv_index;
    a.fwd_order = block_mask->fwd_order;
  }
  a.wait_ns = wait_ns();
  a.status = d->status;
  a.trace = d->trace;
  // cluster launch control launches one CTA per unit; the static walk one per SM
  a.clc = g_work_walk.load() == ATTN_WALK_CLUSTER_LAUNCH_CONTROL ? 1 : 0;
  const int grid = a.clc ? a.n_units : (a.n_units < d->sms ? a.n_units : d->sms);
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e = fp8 ? launch_fwd_fp8(tq, tk, tv, a, mod_key(mod_kind), lse != nullptr, grid, st)
                            : launch_fwd(tq, tk, tv, a, D, mod_key(mod_kind), lse != nullptr, grid, st);
  return e == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

int attn_fwd_strided(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* out,
                     float* lse, int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
                     int mod_kind, const attn_mod_params* mod_params, const attn_block_mask* block_mask,
                     const attn_layouts* layouts, attn_stream_t stream) {
  return fwd_impl(q, k, v, out, lse, nullptr, nullptr, false, B, Hq, Hkv, Sq, Skv, D, scale, mod_kind,
                  mod_params, block_mask, layouts, stream);
}

int attn_fwd_fp8(const uint8_t* q8, const uint8_t* k8, const float* q_scales, const float* k_scales,
                 const attn_bf16* v, attn_bf16* out, float* lse, int B, int Hq, int Hkv, int Sq, int Skv,
                 int D, float scale, int mod_kind, const attn_mod_params* mod_params,
                 const attn_block_mask* block_mask, attn_stream_t stream) {
  if (q_scales == nullptr || k_scales == nullptr) return ATTN_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(q_scales) & 3u) || (reinterpret_cast<uintptr_t>(k_scales) & 3u))
    return ATTN_ERR_ALIGN;
  if (D != 128) return ATTN_ERR_UNSUPPORTED;
  ModSpec ms;
  if (split_mod(mod_kind, ms) && ms.score != MOD_NONE) return ATTN_ERR_UNSUPPORTED;  // masks only
  return fwd_impl(q8, k8, v, out, lse, q_scales, k_scales, true, B, Hq, Hkv, Sq, Skv, D, scale, mod_kind,
                  mod_params, block_mask, nullptr, stream);
}

int attn_fp8_rotate_quantize(const attn_bf16* x, const int8_t* signs, uint8_t* codes, float* scales, int B,
                             int H, int S, int D, attn_stream_t stream) {
  if (x == nullptr || signs == nullptr || codes == nullptr || scales == nullptr) return ATTN_ERR_ARG;
  if (B < 1 || H < 1 || S < 1) return ATTN_ERR_ARG;
  if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 65535) return ATTN_ERR_UNSUPPORTED;  // one grid row per head
  if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3u)) return ATTN_ERR_ALIGN;
  DeviceInfo* d = nullptr;
  const int rc = current_device(&d);
  if (rc != ATTN_OK) return rc;
  return launch_fp8_prep(x, signs, codes, scales, B * H, S, D, d->sms, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? ATTN_OK
             : ATTN_ERR_LAUNCH;
}

int attn_fwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, attn_bf16* out,
             float* lse, int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
             int mod_kind, const attn_mod_params* mod_params, const attn_block_mask* block_mask,
             attn_stream_t stream) {
  return attn_fwd_strided(q, k, v, out, lse, B, Hq, Hkv, Sq, Skv, D, scale, mod_kind, mod_params, block_mask,
                          nullptr, stream);
}

size_t attn_bwd_workspace_size(int B, int Hq, int Sq, int D) {
  if (B < 1 || Hq < 1 || Sq < 1 || (D != 64 && D != 128)) return 0;
  const size_t rows = static_cast<size_t>(B) * Hq * (cdiv(Sq, TILE) * TILE);
  return align256(rows * D * 4) + 2 * align256(rows * 4);
}

size_t attn_bwd_deterministic_workspace_size(int B, int Hq, int Sq, int D) {
  const size_t base = attn_bwd_workspace_size(B, Hq, Sq, D);
  if (base == 0) return 0;
  // four counters per block of 64 query rows (one per 32-column slice of dQ)
  const size_t blocks = static_cast<size_t>(B) * Hq * (cdiv(Sq, TILE) * TILE / 64);
  return base + align256(blocks * 4 * sizeof(unsigned));
}

// The backward pass: det selects the ordered (bitwise reproducible) dQ sum.
static int bwd_impl(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, const attn_bf16* out,
                    const float* lse, const attn_bf16* dout, attn_bf16* dq, attn_bf16* dk, attn_bf16* dv,
                    void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int Sq, int Skv,
                    int D, float scale, int mod_kind, const attn_mod_params* mod_params,
                    const attn_block_mask* block_mask, const attn_layouts* layouts, bool det,
                    attn_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || lse == nullptr ||
      dout == nullptr || dq == nullptr || dk == nullptr || dv == nullptr || workspace == nullptr)
    return ATTN_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return ATTN_ERR_ALIGN;
  int rc = check_common(B, Hq, Hkv, Sq, Skv, D, scale, mod_kind, mod_params, block_mask);
  if (rc == ATTN_OK) rc = check_bitmap_call(mod_kind, Hq, mod_params, block_mask);
  if (rc != ATTN_OK) return rc;
  const size_t need = det ? attn_bwd_deterministic_workspace_size(B, Hq, Sq, D)
                         : attn_bwd_workspace_size(B, Hq, Sq, D);
  if (workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  rc = current_device(&d);
  if (rc != ATTN_OK) return rc;

  const int Sq_pad = cdiv(Sq, TILE) * TILE;
  const size_t rows = static_cast<size_t>(B) * Hq * Sq_pad;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BwdArgs a{};
  a.out = reinterpret_cast<const __nv_bfloat16*>(out);
  a.dout = reinterpret_cast<const __nv_bfloat16*>(dout);
  a.lse = lse;
  a.dq_acc = reinterpret_cast<float*>(ws);
  a.lse2 = reinterpret_cast<float*>(ws + align256(rows * D * 4));
  a.delta = reinterpret_cast<float*>(ws + align256(rows * D * 4) + align256(rows * 4));
  a.dq = reinterpret_cast<__nv_bfloat16*>(dq);
  a.dk = reinterpret_cast<__nv_bfloat16*>(dk);
  a.dv = reinterpret_cast<__nv_bfloat16*>(dv);
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.G = Hq / Hkv;
  a.Sq = Sq;
  a.Skv = Skv;
  a.Sq_pad = Sq_pad;
  a.nQ = cdiv(Sq, TILE);
  a.nK = cdiv(Skv, TILE);
  a.n_units = B * Hkv * a.nK;
  a.num_sms = d->sms;
  a.scale = scale;
  a.sl2 = scale * LOG2E;
  a.mod = make_mod(mod_kind, mod_params);
  if (block_mask != nullptr) {
    a.tile_class = block_mask->tile_class;
    a.q_count = block_mask->q_count;
    a.q_index = block_mask->q_index;
    a.bwd_order = block_mask->bwd_order;
  }
  if (det) {
    a.dq_sem = reinterpret_cast<unsigned*>(ws + attn_bwd_workspace_size(B, Hq, Sq, D));
    if (block_mask != nullptr) {
      a.kv_count = block_mask->kv_count;
      a.kv_index = block_mask->kv_index;
    }
  }
  a.wait_ns = wait_ns();
  a.status = d->status;
  a.trace = d->trace == nullptr ? nullptr : d->trace + 128;

  Strides sq, sk, sv;
  if (!layout_of(layouts ? &layouts->q : nullptr, Hq, Sq, D, sq) ||
      !layout_of(layouts ? &layouts->k : nullptr, Hkv, Skv, D, sk) ||
      !layout_of(layouts ? &layouts->v : nullptr, Hkv, Skv, D, sv) ||
      !layout_of(layouts ? &layouts->out : nullptr, Hq, Sq, D, a.o_st) ||
      !layout_of(layouts ? &layouts->dout : nullptr, Hq, Sq, D, a.do_st) ||
      !layout_of(layouts ? &layouts->dq : nullptr, Hq, Sq, D, a.dq_st) ||
      !layout_of(layouts ? &layouts->dk : nullptr, Hkv, Skv, D, a.dk_st) ||
      !layout_of(layouts ? &layouts->dv : nullptr, Hkv, Skv, D, a.dv_st))
    return ATTN_ERR_ALIGN;
  CUtensorMap tq, tk, tv, tdo;
  if (!encode_bf16_4d(&tq, q, D, Sq, Hq, B, sq, 64) || !encode_bf16_4d(&tk, k, D, Skv, Hkv, B, sk, TILE) ||
      !encode_bf16_4d(&tv, v, D, Skv, Hkv, B, sv, TILE) || !encode_bf16_4d(&tdo, dout, D, Sq, Hq, B, a.do_st, 64))
    return ATTN_ERR_ARG;
  // The ordered adds need every unit of lower rank started before a unit waits
  // on it: only the static walk's resident CTAs (one per SM, ascending ranks)
  // guarantee that, so the deterministic backward always takes it.
  a.clc = !det && g_work_walk.load() == ATTN_WALK_CLUSTER_LAUNCH_CONTROL ? 1 : 0;
  const int grid = a.clc ? a.n_units : (a.n_units < d->sms ? a.n_units : d->sms);
  if (launch_bwd(tq, tk, tv, tdo, a, D, mod_key(mod_kind), grid,
                 reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ATTN_ERR_LAUNCH;
  return ATTN_OK;
}

int attn_bwd_strided(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, const attn_bf16* out,
                     const float* lse, const attn_bf16* dout, attn_bf16* dq, attn_bf16* dk, attn_bf16* dv,
                     void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int Sq, int Skv,
                     int D, float scale, int mod_kind, const attn_mod_params* mod_params,
                     const attn_block_mask* block_mask, const attn_layouts* layouts, attn_stream_t stream) {
  return bwd_impl(q, k, v, out, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, Sq, Skv, D,
                  scale, mod_kind, mod_params, block_mask, layouts, false, stream);
}

int attn_bwd_deterministic(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, const attn_bf16* out,
                           const float* lse, const attn_bf16* dout, attn_bf16* dq, attn_bf16* dk,
                           attn_bf16* dv, void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                           int Sq, int Skv, int D, float scale, int mod_kind,
                           const attn_mod_params* mod_params, const attn_block_mask* block_mask,
                           attn_stream_t stream) {
  return bwd_impl(q, k, v, out, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, Sq, Skv, D,
                  scale, mod_kind, mod_params, block_mask, nullptr, true, stream);
}

int attn_bwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v, const attn_bf16* out,
             const float* lse, const attn_bf16* dout, attn_bf16* dq, attn_bf16* dk, attn_bf16* dv,
             void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int Sq, int Skv,
             int D, float scale, int mod_kind, const attn_mod_params* mod_params,
             const attn_block_mask* block_mask, attn_stream_t stream) {
  return attn_bwd_strided(q, k, v, out, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, Hq, Hkv, Sq, Skv,
                          D, scale, mod_kind, mod_params, block_mask, nullptr, stream);
}

size_t attn_bwd_noalloc_max_workspace(void) { return kNoAllocScratchBytes; }

int attn_bwd_noalloc(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v,
                     const attn_bf16* out, const float* lse, const attn_bf16* dout, attn_bf16* dq,
                     attn_bf16* dk, attn_bf16* dv, int B, int Hq, int Hkv, int Sq, int Skv, int D,
                     float scale, int mod_kind, const attn_mod_params* mod_params,
                     const attn_block_mask* block_mask, attn_stream_t stream) {
  const size_t need = attn_bwd_workspace_size(B, Hq, Sq, D);
  if (need == 0) return (D != 64 && D != 128) ? ATTN_ERR_UNSUPPORTED : ATTN_ERR_ARG;
  if (need > kNoAllocScratchBytes) return ATTN_ERR_WORKSPACE;
  DeviceInfo* d = nullptr;
  const int rc = current_device(&d);
  if (rc != ATTN_OK) return rc;
  if (d->scratch == nullptr) return ATTN_ERR_DEVICE;
  // the backward's first kernel rewrites every word of the workspace it reads
  // later (it zeroes the dQ accumulator), so stale contents do not matter
  return attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, d->scratch, kNoAllocScratchBytes, B, Hq, Hkv,
                  Sq, Skv, D, scale, mod_kind, mod_params, block_mask, stream);
}

#if defined(ATTN25_TRACE)
ATTN25_API int attn_trace_read(unsigned long long* host_out, int n) {
  DeviceInfo* d = nullptr;
  int rc = current_device(&d);
  if (rc != ATTN_OK) return rc;
  if (host_out == nullptr || n < 0 || n > kTraceWords || d->trace == nullptr) return ATTN_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (cudaMemcpy(host_out, d->trace, n * sizeof(unsigned long long), cudaMemcpyDeviceToHost) != cudaSuccess)
    return ATTN_ERR_LAUNCH;
  return ATTN_OK;
}

ATTN25_API int attn_trace_reset(void) {
  DeviceInfo* d = nullptr;
  int rc = current_device(&d);
  if (rc != ATTN_OK) return rc;
  if (d->trace == nullptr) return ATTN_ERR_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return ATTN_ERR_LAUNCH;
  return cudaMemset(d->trace, 0, kTraceWords * sizeof(unsigned long long)) == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

ATTN25_API int attn_trace_window(int first_step) {
  DeviceInfo* d = nullptr;
  int rc = current_device(&d);
  if (rc != ATTN_OK) return rc;
  if (d->trace == nullptr || first_step < 0) return ATTN_ERR_ARG;
  const unsigned long long v = static_cast<unsigned long long>(first_step);
  return cudaMemcpy(d->trace + kTraceCounters - 1, &v, sizeof(v), cudaMemcpyHostToDevice) == cudaSuccess
             ? ATTN_OK
             : ATTN_ERR_LAUNCH;
}
#endif

}  // extern "C"
