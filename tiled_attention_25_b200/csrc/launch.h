// Kernel argument blocks and launchers shared between the kernels and the C ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mods.cuh"

namespace attn25 {

// Element strides of a [B][H][S][D] tensor whose D elements are contiguous.
struct Strides {
  long long b, h, s;
};

struct FwdArgs {
  __nv_bfloat16* out;
  const float* q_scales;  // FP8 scores: per (b, query head) and per (b, KV head) scales of the
  const float* k_scales;  // e4m3 Q and K codes (nullptr for bf16 Q and K)
  Strides o_st;  // of out
  float* lse;
  int B, Hq, Hkv, G, Sq, Skv;
  int nQ, nK, nP, n_units;
  float scale;  // softmax scale
  float sl2;    // scale * log2(e)
  ModDev mod;
  const uint8_t* tile_class;  // block mask (all nullptr for dense iteration)
  const int32_t* kv_count;
  const int32_t* kv_index;
  const int32_t* fwd_order;
  int clc;                    // work walk: 0 static snake over the order, 1 cluster launch control
  uint64_t wait_ns;
  int* status;
  unsigned long long* trace;  // profiling builds only (else nullptr)
};

struct BwdArgs {
  const __nv_bfloat16* out;   // forward output O
  const __nv_bfloat16* dout;  // dO
  const float* lse;           // forward LSE (natural log)
  float* dq_acc;              // [B*Hq][Sq_pad][D] fp32
  float* lse2;                // [B*Hq][Sq_pad]: -LSE * log2(e), -inf where the row keeps nothing
  float* delta;               // [B*Hq][Sq_pad]: -rowsum(dO * O)
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  Strides o_st, do_st, dq_st, dk_st, dv_st;  // of out, dout, dq, dk, dv
  int B, Hq, Hkv, G, Sq, Skv, Sq_pad;
  int nQ, nK, n_units;
  int num_sms;  // SMs of the device (grid caps of the prep and cast kernels)
  float scale, sl2;
  ModDev mod;
  const uint8_t* tile_class;
  const int32_t* q_count;
  const int32_t* q_index;
  const int32_t* bwd_order;
  // Deterministic dQ: per (row block of 64 queries, 32-column slice of dQ)
  // counters [B*Hq][Sq_pad/64][4] of the key tiles that have added their
  // part, so that the parts enter the fp32 sum in ascending key-tile order
  // (nullptr: reductions in any order).  The positions come from the block
  // mask's key-tile lists (kv_count / kv_index) or, without one, from the
  // dense tile classes.
  unsigned int* dq_sem;
  const int32_t* kv_count;
  const int32_t* kv_index;
  int clc;                    // work walk: 0 static snake over the order, 1 cluster launch control
  uint64_t wait_ns;
  int* status;
  unsigned long long* trace;  // profiling builds only (else nullptr)
};

struct MaskArgs {
  int mask;      // kMask* bits
  int window;    // W (1 << 30 without the window mask)
  const int32_t* doc_offsets;
  int num_docs;
  const uint32_t* bitmap;  // keep bits (bitmap mask) or nullptr
  int bm_row_words, bm_heads;
  long long bm_head_stride, bm_batch_stride;
  const int32_t* vq_offsets;  // varlen mask or nullptr
  const int32_t* vk_offsets;
  int n_seqs;
  int B, Sq, Skv, nQ, nK, nP;
  uint8_t* tile_class;
  int32_t* kv_count;
  int32_t* kv_index;
  int32_t* q_count;
  int32_t* q_index;
  int32_t* fwd_order;
  int32_t* bwd_order;
};

// Each returns cudaSuccess or the launch error.
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdArgs& a, int D, int key, bool has_lse, int grid,
                       cudaStream_t stream);
// The forward with e4m3 Q and K (D = 128; masks, no score transform).
cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const FwdArgs& a, int key, bool has_lse, int grid, cudaStream_t stream);
// FP8 incoherent processing of x [BH][S][D] bf16 -> e4m3 codes and one scale per row of BH.
cudaError_t launch_fp8_prep(const void* x, const int8_t* signs, uint8_t* codes, float* scales, int BH, int S,
                            int D, int sms, cudaStream_t stream);
cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const BwdArgs& a, int D, int key, int grid,
                       cudaStream_t stream);
cudaError_t launch_block_mask(const MaskArgs& a, cudaStream_t stream);


}  // namespace attn25
