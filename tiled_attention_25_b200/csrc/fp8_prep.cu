// FP8 incoherent processing: rotate each row of Q or K by diag(signs) H_D /
// sqrt(D) (H_D the Sylvester Hadamard matrix) and quantise every (b, head)
// to e4m3 with one scale, its absolute maximum / 448 ("FlashAttention-3 …",
// FlashAttention-3의 기술적 혁신, item 3: a random orthogonal rotation
// before FP8 quantisation spreads outlier coordinates and cancels in QK^T).
//
// Every value is formed by the same exactly rounded fp32 steps in both
// passes, so the two passes agree and the codes are reproducible:
//   1. the sign flip;  2. the fast Walsh-Hadamard butterflies, stages
//   h = 1, 2, ..., D/2, each pair (y[i], y[i+h]) of a block of 2h becoming
//   (y[i] + y[i+h], y[i] - y[i+h]);  3. one product by fp32 1/sqrt(D);
//   4. scale = absmax / 448 (IEEE division);  5. e4m3(y / scale), rounded
//   to nearest with ties to even, saturating at +-448.
// One warp holds one row: lane l holds the V = D/32 consecutive elements
// l V .. l V + V - 1, so stages h < V run in registers and stages h >= V
// pair lane l with lane l ^ (h / V).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "launch.h"

namespace attn25 {

namespace {

constexpr int kPrepThreads = 256;
constexpr int kPrepRows = 4;  // rows a warp has in flight

// Lane l of a warp holds elements l V .. l V + V - 1 (V = D / 32) of a row.
template <int D>
struct RowBits {
  uint32_t w[D / 64];  // V bf16, two per word
};

template <int D>
__device__ __forceinline__ RowBits<D> load_row(const __nv_bfloat16* row) {
  const int lane = threadIdx.x & 31;
  RowBits<D> r;
  if constexpr (D == 128) {  // 8 bytes per lane
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(row) + lane);
    r.w[0] = v.x;
    r.w[1] = v.y;
  } else {  // 4 bytes per lane
    r.w[0] = __ldg(reinterpret_cast<const uint32_t*>(row) + lane);
  }
  return r;
}

// The lane's signs of the sign flip, as floats.
template <int D>
__device__ __forceinline__ void load_signs(const int8_t* signs, float (&sg)[D / 32]) {
  constexpr int V = D / 32;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < V; ++j) sg[j] = static_cast<float>(__ldg(signs + lane * V + j));
}

// The sign flip, the butterflies and the 1/sqrt(D) product of one row.
template <int D>
__device__ __forceinline__ void rotate_row(const RowBits<D>& bits, const float (&sg)[D / 32], float inv_sqrt_d,
                                           float (&y)[D / 32]) {
  constexpr int V = D / 32;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const uint32_t wd = bits.w[j >> 1];
    y[j] = __uint_as_float((j & 1) ? (wd & 0xffff0000u) : (wd << 16)) * sg[j];
  }
#pragma unroll
  for (int h = 1; h < V; h *= 2) {  // pairs inside the lane
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if (!(j & h)) {
        const float a = y[j], b = y[j + h];
        y[j] = a + b;
        y[j + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int h = V; h < D; h *= 2) {  // pairs across lanes
    const int d = h / V;
    // this lane holds the y[i + h] half (p - y) or the y[i] half (y + p): one
    // fused multiply-add by -1 or +1, exact product and one rounding, the same
    // value as the subtraction or the addition
    const float sg = (lane & d) != 0 ? -1.f : 1.f;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const float p = __shfl_xor_sync(0xffffffffu, y[j], d);
      y[j] = fmaf(sg, y[j], p);
    }
  }
#pragma unroll
  for (int j = 0; j < V; ++j) y[j] *= inv_sqrt_d;
}

// grid (row blocks, B*H): the absolute maximum of each (b, head) after the
// rotation, as float bits (non-negative floats order like unsigned ints).
// Each warp takes kPrepRows rows at a time, their loads issued together.
template <int D>
__global__ void __launch_bounds__(kPrepThreads) fp8_amax_kernel(const __nv_bfloat16* x, const int8_t* signs,
                                                                 uint32_t* amax, int S, float inv_sqrt_d) {
  const int bh = blockIdx.y, warp = threadIdx.x >> 5;
  constexpr int kWarps = kPrepThreads / 32;
  float sg[D / 32];
  load_signs<D>(signs, sg);
  float m = 0.f;
  for (int r0 = (blockIdx.x * kWarps + warp) * kPrepRows; r0 < S; r0 += gridDim.x * kWarps * kPrepRows) {
    RowBits<D> bits[kPrepRows];
#pragma unroll
    for (int i = 0; i < kPrepRows; ++i)
      if (r0 + i < S) bits[i] = load_row<D>(x + (static_cast<size_t>(bh) * S + r0 + i) * D);
#pragma unroll
    for (int i = 0; i < kPrepRows; ++i) {
      if (r0 + i < S) {
        float y[D / 32];
        rotate_row<D>(bits[i], sg, inv_sqrt_d, y);
#pragma unroll
        for (int j = 0; j < D / 32; ++j) m = fmaxf(m, fabsf(y[j]));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float wmax[kWarps];
  if ((threadIdx.x & 31) == 0) wmax[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) b = fmaxf(b, wmax[w]);
    atomicMax(amax + bh, __float_as_uint(b));
  }
}

__device__ __forceinline__ float head_scale(uint32_t amax_bits) {
  const float a = __uint_as_float(amax_bits);
  return a > 0.f ? a / 448.f : 1.f;
}

// two e4m3 codes, lo in the low byte
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

template <int D>
__global__ void __launch_bounds__(kPrepThreads) fp8_quantize_kernel(const __nv_bfloat16* x, const int8_t* signs,
                                                                     const uint32_t* amax, uint8_t* codes, int S,
                                                                     float inv_sqrt_d) {
  constexpr int V = D / 32;
  const int bh = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kWarps = kPrepThreads / 32;
  const float scale = head_scale(__ldg(amax + bh));
  float sg[V];
  load_signs<D>(signs, sg);
  for (int r0 = (blockIdx.x * kWarps + warp) * kPrepRows; r0 < S; r0 += gridDim.x * kWarps * kPrepRows) {
    RowBits<D> bits[kPrepRows];
#pragma unroll
    for (int i = 0; i < kPrepRows; ++i)
      if (r0 + i < S) bits[i] = load_row<D>(x + (static_cast<size_t>(bh) * S + r0 + i) * D);
#pragma unroll
    for (int i = 0; i < kPrepRows; ++i) {
      if (r0 + i < S) {
        const size_t row = static_cast<size_t>(bh) * S + r0 + i;
        float y[V];
        rotate_row<D>(bits[i], sg, inv_sqrt_d, y);
        uint8_t* out = codes + row * D + lane * V;
        if constexpr (V == 4) {
          const uint32_t lo = e4m3x2(y[0] / scale, y[1] / scale), hi = e4m3x2(y[2] / scale, y[3] / scale);
          *reinterpret_cast<uint32_t*>(out) = lo | (hi << 16);
        } else {
          *reinterpret_cast<uint16_t*>(out) = e4m3x2(y[0] / scale, y[1] / scale);
        }
      }
    }
  }
}

// amax bits -> fp32 scale, in place
__global__ void fp8_scale_kernel(uint32_t* amax_scale, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float s = head_scale(amax_scale[i]);
    amax_scale[i] = __float_as_uint(s);
  }
}

template <int D>
cudaError_t launch_fp8_prep_t(const __nv_bfloat16* x, const int8_t* signs, uint8_t* codes, float* scales, int BH,
                              int S, float inv_sqrt_d, int row_blocks, cudaStream_t stream) {
  uint32_t* amax = reinterpret_cast<uint32_t*>(scales);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(uint32_t) * BH, stream);
  if (e != cudaSuccess) return e;
  const dim3 grid(row_blocks, BH);
  fp8_amax_kernel<D><<<grid, kPrepThreads, 0, stream>>>(x, signs, amax, S, inv_sqrt_d);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  fp8_quantize_kernel<D><<<grid, kPrepThreads, 0, stream>>>(x, signs, amax, codes, S, inv_sqrt_d);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  fp8_scale_kernel<<<(BH + 255) / 256, 256, 0, stream>>>(amax, BH);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fp8_prep(const void* x, const int8_t* signs, uint8_t* codes, float* scales, int BH, int S,
                            int D, int sms, cudaStream_t stream) {
  // about eight blocks per SM over all heads, each block taking whole rows
  const int rows_per_block = kPrepThreads / 32 * kPrepRows;
  long long want = (8LL * sms + BH - 1) / BH;
  const long long most = (S + rows_per_block - 1) / rows_per_block;
  const int row_blocks = static_cast<int>(want < 1 ? 1 : (want > most ? most : want));
  const float inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (D == 128) return launch_fp8_prep_t<128>(xb, signs, codes, scales, BH, S, inv_sqrt_d, row_blocks, stream);
  if (D == 64) return launch_fp8_prep_t<64>(xb, signs, codes, scales, BH, S, inv_sqrt_d, row_blocks, stream);
  return cudaErrorInvalidValue;
}

}  // namespace attn25
