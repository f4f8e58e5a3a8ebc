/*
 * attn25 — exact fused scaled-dot-product attention for NVIDIA B200 (sm_100a).
 *
 * C ABI of libattn25.so.  Every pointer argument named "device" is a CUDA
 * device pointer; every call is asynchronous on the given stream and returns
 * before the GPU work ends.  The caller owns and allocates every buffer
 * (inputs, outputs, the backward workspace, the block mask); the library
 * keeps only one device status word per GPU.
 *
 * What is computed.  For each batch row b, query head h (KV head
 * hk = h / (Hq / Hkv)), query i and key j:
 *     s_ij  = scale * sum_d q_id k_jd
 *     s'_ij = mod(s_ij; b, h, i, j), masked entries are -inf
 *     O_i   = sum_j softmax_j(s'_i.) v_j,   LSE_i = ln sum_j exp(s'_ij)
 * i.e. standard attention softmax(Q K^T * scale) V ("FlashAttention 설명",
 * §1) with a FlexAttention-style score mod or mask ("PyTorch FlexAttention,
 * FlashAttention-4 백엔드 도입으로 성능 최대 3.2배 향상", 섹션별 상세), computed
 * tile by tile with an online softmax so that the score matrix never reaches
 * global memory ("FlashAttention-2 — GPU attention의 사실상 표준", §3-§4;
 * "FlashAttention 설명", §3-§6).  The backward pass recomputes the scores from
 * the saved LSE ("FlashAttention-2 …", §3 Recomputation).
 *
 * Layouts.  Q, O, dQ, dO: bf16 [B][Hq][Sq][D]; K, V, dK, dV: bf16
 * [B][Hkv][Skv][D]; LSE: fp32 [B][Hq][Sq] (natural log), contiguous, D
 * innermost.  Supported: D in {64, 128}; 1 <= Sq, Skv <= 262144; Hq a
 * multiple of Hkv.  Every tensor base pointer must be 16-byte aligned.
 *
 * Errors.  Functions return ATTN_OK (0) or a negative attn_status; arguments
 * are checked on the host before anything is launched.  A kernel that waits
 * longer than the wait limit on one of its internal barriers stops, writes
 * ATTN_ERR_TIMEOUT into the device status word and returns; the host reads
 * (and clears) it with attn_get_status().
 */
#ifndef ATTN25_H
#define ATTN25_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN25_API __attribute__((visibility("default")))
#else
#define ATTN25_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without including the CUDA headers (the same handle type). */
typedef struct CUstream_st* attn_stream_t;

/* A bfloat16 value as its 16-bit pattern. */
typedef uint16_t attn_bf16;

typedef enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_ARG = -1,          /* NULL pointer, bad size, Hq % Hkv != 0 */
  ATTN_ERR_UNSUPPORTED = -2,  /* D not in {64,128}, or a mod/param combination not supported */
  ATTN_ERR_ALIGN = -3,        /* a base pointer is not 16-byte aligned */
  ATTN_ERR_WORKSPACE = -4,    /* workspace or block-mask buffer too small */
  ATTN_ERR_LAUNCH = -5,       /* a CUDA call or kernel launch failed */
  ATTN_ERR_TIMEOUT = -6,      /* a kernel gave up waiting on an internal barrier */
  ATTN_ERR_DEVICE = -7        /* no usable sm_100 device, or the kernel image failed to load */
} attn_status;

/*
 * Score mods and masks (the fixed set; each is applied to the scaled score
 * s = scale * q.k of query i and key j, absolute indices, 0-based).
 * The FlexAttention page shows score_mod(score, b, h, q_idx, kv_idx) with the
 * local boost and tanh softcap examples ("PyTorch FlexAttention, …",
 * 섹션별 상세) and names ALiBi, sliding window and document masking (핵심 요약).
 */
typedef enum attn_mod_kind {
  ATTN_MOD_NONE = 0,            /* s' = s */
  ATTN_MOD_CAUSAL = 1,          /* keep j <= i */
  ATTN_MOD_ALIBI = 2,           /* s' = s - slope_h |i - j| */
  ATTN_MOD_SOFTCAP = 3,         /* s' = c tanh(s / c) */
  ATTN_MOD_SLIDING_WINDOW = 4,  /* keep 0 <= i - j < W */
  ATTN_MOD_LOCAL_BOOST = 5,     /* s' = boost * s if |i - j| < radius, else s */
  ATTN_MOD_DOCUMENT = 6         /* keep doc(i) == doc(j) and j <= i */
} attn_mod_kind;

/*
 * Composition (FlexAttention composes score and mask mods, "PyTorch
 * FlexAttention, …", 핵심 요약).  A mod_kind argument is one attn_mod_kind,
 * optionally ORed with any of these flags: the score transform is the kind's
 * (s' = s for the three mask kinds), and an element is kept only where the
 * kind and every flagged mask keep it.  Examples:
 *   ATTN_MOD_ALIBI | ATTN_MASK_CAUSAL          causal ALiBi
 *   ATTN_MOD_SOFTCAP | ATTN_MASK_SLIDING_WINDOW  softcapped sliding window
 *   ATTN_MOD_SLIDING_WINDOW | ATTN_MASK_DOCUMENT window inside each document
 * Each component reads its own fields of attn_mod_params.  Unknown bits or
 * kinds return ATTN_ERR_ARG.
 */
enum {
  ATTN_MASK_CAUSAL = 0x100,
  ATTN_MASK_SLIDING_WINDOW = 0x200,
  ATTN_MASK_DOCUMENT = 0x400,
  ATTN_MASK_BITMAP = 0x800,     /* a general mask given by its values (attn_mod_params.bitmap);
                                   attn_fwd / attn_bwd then need a block mask built for it */
  ATTN_MASK_VARLEN = 0x1000     /* packed sequences with their own query and key lengths:
                                   query i and key j interact only within one sequence; not
                                   causal, and combined with no other mask */
};

/*
 * Runtime scalars of the mods; a change needs no recompilation (the page
 * notes that its JIT backend recompiles when such a scalar changes).
 * Fields that the chosen mod does not use are ignored.
 */
typedef struct attn_mod_params {
  float softcap;               /* ATTN_MOD_SOFTCAP: c > 0 (e.g. 50) */
  int32_t window;              /* ATTN_MOD_SLIDING_WINDOW / ATTN_MASK_SLIDING_WINDOW: W >= 1 (e.g. 1024) */
  float boost;                 /* ATTN_MOD_LOCAL_BOOST: factor (e.g. 1.1) */
  int32_t boost_radius;        /* ATTN_MOD_LOCAL_BOOST: radius >= 0 (e.g. 128) */
  const float* alibi_slopes;   /* ATTN_MOD_ALIBI: device fp32 [Hq] (4-byte aligned), or NULL for
                                  2^(-8 (h+1) / Hq) */
  const int32_t* doc_offsets;  /* ATTN_MOD_DOCUMENT / ATTN_MASK_DOCUMENT: device int32 (4-byte aligned) [B][num_docs+1]: ascending document
                                  starts, offsets[b][0] = 0, offsets[b][num_docs] = Skv; repeat the last
                                  value to pad rows with fewer documents.  Queries and keys share the
                                  offsets (packed self-attention, Sq == Skv required). */
  int32_t num_docs;            /* ATTN_MOD_DOCUMENT / ATTN_MASK_DOCUMENT: 1 <= num_docs <= 4096 */
  /* ATTN_MASK_BITMAP: the values of a general mask_mod, one bit per element.
   * Element (b, h, i, j) is kept when bit (j & 31) of word
   *   b * bitmap_batch_stride + h * bitmap_head_stride + i * bitmap_row_words + (j >> 5)
   * is set.  Device memory, 16-byte aligned, read only; bits at j >= Skv are ignored. */
  const uint32_t* bitmap;
  int32_t bitmap_row_words;     /* a multiple of 4, >= ceil(Skv / 32) */
  int32_t bitmap_heads;         /* 1 (one mask for all heads, head stride 0) or Hq */
  int64_t bitmap_head_stride;   /* words, a multiple of 4; 0 when bitmap_heads == 1 */
  int64_t bitmap_batch_stride;  /* words, a multiple of 4; 0 = one mask for all batch rows */
  /* ATTN_MASK_VARLEN: device int32 [B][num_seqs + 1] ascending starts of each sequence's
   * queries and keys, plus the ends (Sq and Skv); repeat an offset for an empty sequence. */
  const int32_t* q_offsets;
  const int32_t* k_offsets;
  int32_t num_seqs;             /* 1 <= num_seqs <= 65536 */
} attn_mod_params;

/*
 * Block mask over 128x128 tiles ("PyTorch FlexAttention, …", 섹션별 상세:
 * block-sparse iteration that skips fully masked blocks).  All arrays are
 * device memory inside one caller-allocated buffer (attn_block_mask_bytes),
 * laid out by attn_block_mask_bind and filled by build_block_mask:
 *   tile_class [B][nq][nk] uint8: 0 EMPTY, 1 PARTIAL, 2 FULL over in-range elements
 *   kv_count [B][nq], kv_index [B][nq][nk]: non-EMPTY KV tiles per query tile, ascending, -1 padded
 *   q_count [B][nk], q_index [B][nk][nq]: non-EMPTY query tiles per KV tile, ascending, -1 padded
 *   fwd_order [B * ceil(nq/2)]: forward work pairs (query tiles 2p, 2p+1 of row b, id b*np+p)
 *       in longest-first order of their non-EMPTY KV tile count, ties by id
 *   bwd_order [B * nk]: backward units (id b*nk+kv tile) longest-first by q_count, ties by id
 */
typedef struct attn_block_mask {
  uint8_t* tile_class;
  int32_t* kv_count;
  int32_t* kv_index;
  int32_t* q_count;
  int32_t* q_index;
  int32_t* fwd_order;
  int32_t* bwd_order;
  int32_t B, Sq, Skv, nq_tiles, nk_tiles;
  int32_t mod_kind;            /* the mod it was built for, in canonical form (score kind |
                                  ATTN_MASK_* flags, so equal for codes that mean the same mod);
                                  attn_fwd/attn_bwd check it */
} attn_block_mask;

/*
 * Forward pass.  q, k, v: device bf16 inputs; out: device bf16 output;
 * lse: device fp32 [B][Hq][Sq] or NULL (then a kernel specialisation that
 * neither computes nor writes it runs, as the FlashInfer page's out-only
 * path: "FlashInfer SM120 NVFP4 어텐션 최적화", 코드 분석 2-4).
 * block_mask: NULL for dense iteration (causal and sliding-window tiles are
 * then classified on the fly, document masks test every element), or a mask
 * built by build_block_mask for the same mod and sizes.
 * mod_params may be NULL when no component reads it (none, causal, ALiBi with the
 * default slopes).
 */
ATTN25_API int attn_fwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v,
             attn_bf16* out, float* lse,
             int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
             int mod_kind, const attn_mod_params* mod_params,
             const attn_block_mask* block_mask, attn_stream_t stream);

/* Bytes of device workspace attn_bwd needs (fp32 dQ accumulator and row statistics). */
ATTN25_API size_t attn_bwd_workspace_size(int B, int Hq, int Sq, int D);

/*
 * Backward pass: dq, dk, dv (device bf16) from q, k, v, out, lse (as written
 * by attn_fwd with the same arguments; required) and dout.  workspace:
 * device memory of at least attn_bwd_workspace_size bytes, 256-byte aligned;
 * its contents on entry do not matter.  dQ is accumulated in fp32 with
 * atomic adds, so its last bits may differ from run to run.
 */
ATTN25_API int attn_bwd(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v,
             const attn_bf16* out, const float* lse, const attn_bf16* dout,
             attn_bf16* dq, attn_bf16* dk, attn_bf16* dv,
             void* workspace, size_t workspace_bytes,
             int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
             int mod_kind, const attn_mod_params* mod_params,
             const attn_block_mask* block_mask, attn_stream_t stream);

/*
 * attn_bwd without a workspace argument, for callers that cannot allocate
 * device memory when they call it: for example a plugin host that hands its
 * kernels no workspace, or an application whose device memory is carved up
 * in advance by its own pool and must not grow.  The library itself holds a
 * fixed 32 MiB block of device memory for this (reserved on every GPU that
 * loads the library, until the process exits) and runs the same kernels as
 * attn_bwd on it; this function allocates nothing.  The paper has no
 * counterpart; it exists for this deployment constraint only.
 *
 * - Problems whose attn_bwd_workspace_size exceeds
 *   attn_bwd_noalloc_max_workspace() are rejected with ATTN_ERR_WORKSPACE.
 * - The first call of the library on a device (this one included) looks up
 *   the block's device address; make that first call before any stream
 *   capture.
 * - All calls share the one block.  Calls whose GPU work overlaps in time
 *   (two streams, or two host threads) race and corrupt each other's
 *   results; serialise them on one stream.  Contents left by an earlier call
 *   are rewritten before use, so back-to-back calls are fine.
 */
ATTN25_API int attn_bwd_noalloc(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v,
             const attn_bf16* out, const float* lse, const attn_bf16* dout,
             attn_bf16* dq, attn_bf16* dk, attn_bf16* dv,
             int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
             int mod_kind, const attn_mod_params* mod_params,
             const attn_block_mask* block_mask, attn_stream_t stream);

/* Largest workspace attn_bwd_noalloc can use (bytes). */
ATTN25_API size_t attn_bwd_noalloc_max_workspace(void);

/* Bytes of device memory one block mask for (B, Sq, Skv) occupies. */
ATTN25_API size_t attn_block_mask_bytes(int B, int Sq, int Skv);

/* Lay out a block mask inside a caller buffer (device, 256-byte aligned); no GPU work. */
ATTN25_API int attn_block_mask_bind(void* buffer, size_t bytes, int B, int Sq, int Skv,
                         attn_block_mask* out);

/*
 * Classify every 128x128 tile for the mod and fill all arrays of a bound
 * block mask (bit-exact with a per-element classification).  With a per-head
 * bitmap the classes hold for every head: EMPTY where no head keeps an
 * element of the tile, FULL where every head keeps all of its in-range
 * elements, PARTIAL otherwise.
 */
ATTN25_API int build_block_mask(int mod_kind, const attn_mod_params* mod_params,
                     int B, int Sq, int Skv, attn_block_mask* mask,
                     attn_stream_t stream);

/*
 * Strided tensors.  Each bf16 tensor is a [B][H][S][D] view whose D elements
 * are contiguous; these are its element strides between batch rows, heads
 * and sequence positions (each a positive multiple of 8, so that a row
 * starts on 16 bytes).  Contiguous [B][H][S][D] has {H*S*D, S*D, D}; the
 * common [B][S][H][D] storage has {S*H*D, D, H*D}.
 */
typedef struct attn_strides {
  int64_t b, h, s;
} attn_strides;

typedef struct attn_layouts {
  attn_strides q, k, v, out, dout, dq, dk, dv;  /* attn_fwd_strided reads q, k, v, out */
} attn_layouts;

/* attn_fwd and attn_bwd on strided tensors (layouts NULL: contiguous);
 * bad strides return ATTN_ERR_ALIGN.  LSE stays contiguous [B][Hq][Sq], the
 * shape the FlashInfer page allocates for it ("FlashInfer SM120 NVFP4 어텐션
 * 최적화", 코드 분석 1); the pages fix no layout for Q, K, V and O, so the
 * library takes the two common ones and any strides between. */
ATTN25_API int attn_fwd_strided(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v,
                                attn_bf16* out, float* lse,
                                int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
                                int mod_kind, const attn_mod_params* mod_params,
                                const attn_block_mask* block_mask, const attn_layouts* layouts,
                                attn_stream_t stream);
ATTN25_API int attn_bwd_strided(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v,
                                const attn_bf16* out, const float* lse, const attn_bf16* dout,
                                attn_bf16* dq, attn_bf16* dk, attn_bf16* dv,
                                void* workspace, size_t workspace_bytes,
                                int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
                                int mod_kind, const attn_mod_params* mod_params,
                                const attn_block_mask* block_mask, const attn_layouts* layouts,
                                attn_stream_t stream);

/*
 * The backward pass with a bitwise reproducible dQ.  With Q, K and V split
 * into blocks ("FlashAttention-2 — GPU attention의 사실상 표준", §3 item 1,
 * Tiling) and the backward recomputing the scores block by block (§3 item 2
 * and §4, the Backward item), dQ of a query row is a sum of one term per key
 * tile that meets it; attn_bwd adds those terms into its fp32 accumulator in
 * whatever order the key tiles finish, so dQ's last bits vary from run to
 * run.  Here every key tile waits for its turn before adding, and the terms
 * enter each row's sum in ascending key-tile order, so dQ (like dK and dV)
 * is the same bit for bit on every run, with or without a block mask.
 *
 * Arguments as attn_bwd (contiguous tensors).  workspace: device memory of
 * attn_bwd_deterministic_workspace_size bytes, 256-byte aligned: the
 * attn_bwd workspace plus four 32-bit counters per block of 64 query rows;
 * its contents on entry do not matter.  The key tiles run in ascending order
 * (not longest first), and a key tile may wait for the tiles before it: the
 * kernel relies on all its CTAs being resident at once (one per SM), which
 * holds unless other work shares the GPU's SMs at the same time (then a
 * wait runs out and the call reports ATTN_ERR_TIMEOUT through
 * attn_get_status instead of hanging).
 */
ATTN25_API size_t attn_bwd_deterministic_workspace_size(int B, int Hq, int Sq, int D);
ATTN25_API int attn_bwd_deterministic(const attn_bf16* q, const attn_bf16* k, const attn_bf16* v,
                                      const attn_bf16* out, const float* lse, const attn_bf16* dout,
                                      attn_bf16* dq, attn_bf16* dk, attn_bf16* dv,
                                      void* workspace, size_t workspace_bytes,
                                      int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
                                      int mod_kind, const attn_mod_params* mod_params,
                                      const attn_block_mask* block_mask, attn_stream_t stream);

/*
 * FP8 incoherent processing of queries or keys ("FlashAttention-3 …",
 * FlashAttention-3의 기술적 혁신, item 3).  Each row of x (device bf16
 * [B][H][S][D], D = 64 or 128, 16-byte aligned) is rotated by
 * diag(signs) H_D / sqrt(D), H_D the Sylvester Hadamard matrix and signs
 * (device int8 [D]) a vector of +-1 that the caller draws once; then every
 * (b, h) is quantised to OCP e4m3 (round to nearest even, saturating at 448)
 * with one scale, its absolute maximum / 448.
 *   codes:  device uint8 [B][H][S][D] (16-byte aligned): the e4m3 values;
 *   scales: device fp32 [B][H]: x rotated ~= codes * scales.
 * The steps are exactly rounded fp32 operations in a fixed order (sign flip,
 * Walsh-Hadamard butterflies h = 1, 2, ..., D/2, one product by fp32
 * 1/sqrt(D), IEEE division by the scale), so the codes are reproducible.
 * B * H must not exceed 65535.
 */
ATTN25_API int attn_fp8_rotate_quantize(const attn_bf16* x, const int8_t* signs, uint8_t* codes,
                                        float* scales, int B, int H, int S, int D,
                                        attn_stream_t stream);

/*
 * The forward pass with FP8 scores: q8 and k8 are the e4m3 codes that
 * attn_fp8_rotate_quantize made of Q and K (device uint8 [B][Hq][Sq][D] and
 * [B][Hkv][Skv][D], 16-byte aligned, rotated by the same signs), and
 * q_scales [B][Hq], k_scales [B][Hkv] their fp32 scales.  S = Q8 K8^T is
 * formed by tcgen05 MMAs of kind f8f6f4 and dequantised in the softmax's
 * scale; v, out, lse, the masks and the block mask are as in attn_fwd.
 * D must be 128; mod_kind may hold masks but no score transform
 * (ATTN_ERR_UNSUPPORTED otherwise).
 */
ATTN25_API int attn_fwd_fp8(const uint8_t* q8, const uint8_t* k8, const float* q_scales,
                            const float* k_scales, const attn_bf16* v, attn_bf16* out, float* lse,
                            int B, int Hq, int Hkv, int Sq, int Skv, int D, float scale,
                            int mod_kind, const attn_mod_params* mod_params,
                            const attn_block_mask* block_mask, attn_stream_t stream);

/* Synchronise the stream, then return and clear the device status word. */
ATTN25_API int attn_get_status(attn_stream_t stream);

/* Set the per-wait time limit of the kernels in milliseconds (default 4000). */
ATTN25_API void attn_set_wait_limit_ms(uint32_t ms);

/*
 * How the persistent forward and backward kernels take their work units
 * (query-tile pairs forward, key tiles backward), which they always take in
 * the block mask's longest-first order (ascending key tiles for
 * attn_bwd_deterministic, which always takes the static walk: its ordered dQ
 * adds need every unit of lower rank started, which the static walk's
 * resident CTAs guarantee):
 *   ATTN_WALK_STATIC: one CTA per SM; wave k of the order goes to the CTAs
 *     in turn, every other wave reversed (a snake), fixed in advance;
 *   ATTN_WALK_CLUSTER_LAUNCH_CONTROL (default): one CTA per unit is launched; a CTA that
 *     finishes its unit asks the hardware (Blackwell's cluster launch control)
 *     to cancel the next CTA that has not started and does that CTA's unit, so
 *     the walk adapts to data-dependent unit lengths as it runs ("PyTorch
 *     FlexAttention, FlashAttention-4 백엔드 …", 섹션별 상세 and 실무
 *     Takeaway: dynamic scheduling through CLC balances the SMs under
 *     data-dependent masks).
 * Applies to calls made after it; returns ATTN_ERR_ARG for another value.
 */
enum { ATTN_WALK_STATIC = 0, ATTN_WALK_CLUSTER_LAUNCH_CONTROL = 1 };
ATTN25_API int attn_set_work_walk(int walk);

/*
 * Self-check of the timeout path (the pages have no counterpart: it exists
 * so that a caller can see the error path work on its own GPU).  Launches on
 * the stream a kernel whose one wait is on a barrier that nothing arrives at;
 * after the current wait limit it gives up, records ATTN_ERR_TIMEOUT in the
 * device status word and returns, as an attention kernel does when one of
 * its waits runs out.  attn_get_status then returns ATTN_ERR_TIMEOUT (and
 * clears it); the context stays usable.  Returns ATTN_OK once launched.
 */
ATTN25_API int attn_check_wait_timeout(attn_stream_t stream);

/* A static description of an attn_status value. */
ATTN25_API const char* attn_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* ATTN25_H */
