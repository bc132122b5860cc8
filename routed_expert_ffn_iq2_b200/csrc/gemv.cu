// gemv.cu -- the decode-GEMV family for the projection formats of the model
// the pages run ("Red Lite dev15 -- DeltaNet projection bring-up", section
// "Field-derived recurrent dimensions": ssm_ba Q8_0 (2048,64), ssm_out Q4_K
// (4096,2048); "Red Lite dev16", section "Pinned full-attention graph":
// attn_k / attn_v Q4_K (2048,512), attn_output Q4_K (4096,2048)).
//
// y[t][r] = sum_c W[r][c] x[t][c] for up to 8 token vectors, fp32.  Block
// layouts (include/redlite_moe.h):
//   Q8_0-style  34 bytes / 32 weights: fp16 d, int8 q[32]; w = d q
//   Q4_K-style 144 bytes / 256 weights: fp16 d, fp16 dmin, a 96-bit field
//               of eight 6-bit scales (bit 6j) and minima (bit 48 + 6j),
//               4-bit q in weight order; w = d sc q - dmin m
// One warp per output row, 256 inputs per step: lane l takes inputs
// 8l..8l+7 of the step, so each step reads the row's bytes for those 256
// inputs with coalesced loads; x is read through L1 (every row of a CTA
// reads the same x).
#include "internal.cuh"

namespace redlite {

constexpr int kGemvWarps = 8;
constexpr int kGemvMaxTok = 8;

__device__ __forceinline__ void add_x(float acc[kGemvMaxTok], int ntok, const float *x, int64_t k, int64_t c0,
                                      const float w[8]) {
#pragma unroll
  for (int t = 0; t < kGemvMaxTok; ++t)
    if (t < ntok) {
      const float4 *xp = reinterpret_cast<const float4 *>(x + t * k + c0);
      const float4 a = __ldg(xp), b = __ldg(xp + 1);
      acc[t] += w[0] * a.x + w[1] * a.y + w[2] * a.z + w[3] * a.w + w[4] * b.x + w[5] * b.y + w[6] * b.z +
                w[7] * b.w;
    }
}

template <int QT>
__global__ void __launch_bounds__(32 * kGemvWarps) gemv_proj_kernel(const uint8_t *__restrict__ W, int64_t rows,
                                                                   int64_t k, const float *__restrict__ x,
                                                                   int ntok, float *__restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * kGemvWarps + (threadIdx.x >> 5);
  if (r >= rows) return;
  float acc[kGemvMaxTok];
#pragma unroll
  for (int t = 0; t < kGemvMaxTok; ++t) acc[t] = 0.f;
  const int64_t steps = k / 256;
  if constexpr (QT == 3) {
    const uint8_t *row = W + r * (k / 32) * 34;
    for (int64_t s = 0; s < steps; ++s) {
      // inputs 8l..8l+7 of the step: block 8s + l/4, values 8(l%4)..+7
      const uint8_t *blk = row + (8 * s + lane / 4) * 34;
      const float d = __half2float(__ushort_as_half(__ldg(reinterpret_cast<const unsigned short *>(blk))));
      const unsigned short *qv = reinterpret_cast<const unsigned short *>(blk + 2 + 8 * (lane & 3));
      float w[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const unsigned short two = __ldg(qv + i);
        w[2 * i] = d * (float)(int8_t)(two & 0xFF);
        w[2 * i + 1] = d * (float)(int8_t)(two >> 8);
      }
      add_x(acc, ntok, x, k, 256 * s + 8 * lane, w);
    }
  } else {
    const uint8_t *row = W + r * steps * 144;
    for (int64_t s = 0; s < steps; ++s) {
      const uint8_t *blk = row + s * 144;
      const uint32_t dd = __ldg(reinterpret_cast<const uint32_t *>(blk));
      const uint32_t f0 = __ldg(reinterpret_cast<const uint32_t *>(blk + 4));
      const uint32_t f1 = __ldg(reinterpret_cast<const uint32_t *>(blk + 8));
      const uint32_t f2 = __ldg(reinterpret_cast<const uint32_t *>(blk + 12));
      const uint32_t q = __ldg(reinterpret_cast<const uint32_t *>(blk + 16) + lane);
      const int j = lane >> 2;  // sub-block of inputs 8l..8l+7
      const uint64_t lo = (uint64_t)f0 | ((uint64_t)f1 << 32), hi = (uint64_t)f1 | ((uint64_t)f2 << 32);
      const int sc = (int)((lo >> (6 * j)) & 63u), mn = (int)((hi >> (16 + 6 * j)) & 63u);
      const float d = __half2float(__ushort_as_half((unsigned short)(dd & 0xFFFFu)));
      const float dmin = __half2float(__ushort_as_half((unsigned short)(dd >> 16)));
      const float a = d * (float)sc, b = dmin * (float)mn;
      float w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = a * (float)((q >> (4 * i)) & 15u) - b;
      add_x(acc, ntok, x, k, 256 * s + 8 * lane, w);
    }
  }
#pragma unroll
  for (int t = 0; t < kGemvMaxTok; ++t) {
    float v = acc[t];
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0 && t < ntok) y[t * rows + r] = v;
  }
}

}  // namespace redlite

using namespace redlite;

extern "C" size_t redlite_proj_matrix_bytes(int32_t qtype, int64_t rows, int64_t k) {
  if (rows <= 0 || k <= 0 || k % 256) return 0;
  if (qtype == REDLITE_Q_Q8_0_STYLE) return (size_t)(rows * (k / 32) * 34);
  if (qtype == REDLITE_Q_Q4_K_STYLE) return (size_t)(rows * (k / 256) * 144);
  return 0;
}

extern "C" int redlite_proj_gemv(int32_t qtype, const void *W, int64_t rows, int64_t k, const float *x,
                                 int32_t n_tokens, float *y, void *stream) {
  if (qtype != REDLITE_Q_Q8_0_STYLE && qtype != REDLITE_Q_Q4_K_STYLE) return REDLITE_EINVAL;
  if (rows <= 0 || k <= 0 || n_tokens < 0 || n_tokens > kGemvMaxTok) return REDLITE_EINVAL;
  if (k % 256) return REDLITE_EUNSUPPORTED;
  if (n_tokens == 0) return REDLITE_OK;
  if (!W || !x || !y) return REDLITE_EINVAL;
  if ((((uintptr_t)W) & (qtype == REDLITE_Q_Q4_K_STYLE ? 15 : 1)) || ((uintptr_t)x & 15) || ((uintptr_t)y & 3))
    return REDLITE_EINVAL;
  const unsigned blocks = (unsigned)((rows + kGemvWarps - 1) / kGemvWarps);
  cudaStream_t s = (cudaStream_t)stream;
  if (qtype == REDLITE_Q_Q8_0_STYLE)
    gemv_proj_kernel<3><<<blocks, 32 * kGemvWarps, 0, s>>>((const uint8_t *)W, rows, k, x, n_tokens, y);
  else
    gemv_proj_kernel<4><<<blocks, 32 * kGemvWarps, 0, s>>>((const uint8_t *)W, rows, k, x, n_tokens, y);
  return cudaGetLastError() == cudaSuccess ? REDLITE_OK : REDLITE_ECUDA;
}
