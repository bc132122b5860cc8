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
// 256 inputs per step: lane l takes inputs 8l..8l+7 of the step, so a step
// reads the row's bytes for those 256 inputs with coalesced loads; x is
// read through L1 (every row reads the same x).
#include "internal.cuh"

namespace redlite {

constexpr int kGemvWarps = 8;
constexpr int kGemvMaxTok = 8;

constexpr int kGemvRows = 4;    // output rows per CTA; its 8 warps split the inputs of each
constexpr int kGemvUnroll = 2;  // steps a warp loads before it computes

// The packed words of one row's 256-input step that lane l (inputs
// 8l..8l+7) needs: Q8_0-style w0 = d, w1..w4 = the 8 int8 values;
// Q4_K-style w0..w3 = d | dmin, the 96-bit scale/minimum field, w4 = the 8
// nibbles.
template <int QT>
__device__ __forceinline__ void step_load(const uint8_t *row, int64_t s, int lane, uint32_t wd[5]) {
  if constexpr (QT == 3) {
    const uint8_t *blk = row + (8 * s + lane / 4) * 34;  // block 8s + l/4, values 8(l%4)..+7
    const unsigned short *qv = reinterpret_cast<const unsigned short *>(blk + 2 + 8 * (lane & 3));
    wd[0] = __ldg(reinterpret_cast<const unsigned short *>(blk));
#pragma unroll
    for (int i = 0; i < 4; ++i) wd[1 + i] = __ldg(qv + i);
  } else {
    const uint8_t *blk = row + s * 144;
    const uint4 hd = __ldg(reinterpret_cast<const uint4 *>(blk));
    wd[0] = hd.x, wd[1] = hd.y, wd[2] = hd.z, wd[3] = hd.w;
    wd[4] = __ldg(reinterpret_cast<const uint32_t *>(blk + 16) + lane);
  }
}

// The lane's 8 weights from the words of step_load.
template <int QT>
__device__ __forceinline__ void step_weights(const uint32_t wd[5], int lane, float w[8]) {
  if constexpr (QT == 3) {
    const float d = __half2float(__ushort_as_half((unsigned short)wd[0]));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      w[2 * i] = d * (float)(int8_t)(wd[1 + i] & 0xFF);
      w[2 * i + 1] = d * (float)(int8_t)((wd[1 + i] >> 8) & 0xFF);
    }
  } else {
    const int j = lane >> 2;  // sub-block of inputs 8l..8l+7
    const uint64_t lo = (uint64_t)wd[1] | ((uint64_t)wd[2] << 32), hi = (uint64_t)wd[2] | ((uint64_t)wd[3] << 32);
    const int sc = (int)((lo >> (6 * j)) & 63u), mn = (int)((hi >> (16 + 6 * j)) & 63u);
    const float d = __half2float(__ushort_as_half((unsigned short)(wd[0] & 0xFFFFu)));
    const float dmin = __half2float(__ushort_as_half((unsigned short)(wd[0] >> 16)));
    const float av = d * (float)sc, bv = dmin * (float)mn;
#pragma unroll
    for (int i = 0; i < 8; ++i) w[i] = av * (float)((wd[4] >> (4 * i)) & 15u) - bv;
  }
}

// A CTA computes rows r0..r0+3 for NT token vectors (ntok <= NT): warp w
// takes the 256-input steps w, w + 8, ... of those rows, loading kGemvUnroll
// steps of all four rows before it computes (their loads in flight
// together); the warps' partial sums of a row meet in shared memory.
template <int QT, int NT>
__global__ void __launch_bounds__(32 * kGemvWarps) gemv_proj_kernel(const uint8_t *__restrict__ W, int64_t rows,
                                                                   int64_t k, const float *__restrict__ x,
                                                                   int ntok, float *__restrict__ y) {
  __shared__ float red[kGemvWarps][kGemvRows][NT];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t r0 = (int64_t)blockIdx.x * kGemvRows;
  const int64_t steps = k / 256;
  const size_t row_bytes = QT == 3 ? (size_t)(k / 32) * 34 : (size_t)steps * 144;
  float acc[kGemvRows][NT];
#pragma unroll
  for (int h = 0; h < kGemvRows; ++h)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[h][t] = 0.f;
  for (int64_t s0 = warp; s0 < steps; s0 += kGemvWarps * kGemvUnroll) {
    uint32_t wd[kGemvUnroll][kGemvRows][5];
#pragma unroll
    for (int u = 0; u < kGemvUnroll; ++u)
#pragma unroll
      for (int h = 0; h < kGemvRows; ++h) {
        const int64_t s = s0 + (int64_t)u * kGemvWarps, r = r0 + h;
        if (s < steps && r < rows) {
          step_load<QT>(W + r * row_bytes, s, lane, wd[u][h]);
        } else {
#pragma unroll
          for (int i = 0; i < 5; ++i) wd[u][h][i] = 0u;  // all-zero words decode to zero weights
        }
      }
#pragma unroll
    for (int u = 0; u < kGemvUnroll; ++u) {
      const int64_t s = s0 + (int64_t)u * kGemvWarps;
      if (s >= steps) break;
      float4 xa[NT], xb[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t)
        if (t < ntok) {
          const float4 *xp = reinterpret_cast<const float4 *>(x + t * k + 256 * s + 8 * lane);
          xa[t] = __ldg(xp), xb[t] = __ldg(xp + 1);
        }
#pragma unroll
      for (int h = 0; h < kGemvRows; ++h) {
        float w[8];
        step_weights<QT>(wd[u][h], lane, w);
#pragma unroll
        for (int t = 0; t < NT; ++t)
          if (t < ntok)
            acc[h][t] += w[0] * xa[t].x + w[1] * xa[t].y + w[2] * xa[t].z + w[3] * xa[t].w + w[4] * xb[t].x +
                         w[5] * xb[t].y + w[6] * xb[t].z + w[7] * xb[t].w;
      }
    }
  }
#pragma unroll
  for (int h = 0; h < kGemvRows; ++h)
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float v = acc[h][t];
#pragma unroll
      for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp][h][t] = v;
    }
  __syncthreads();
  // thread (row, token) adds the eight warps' partial sums
  const int tr = threadIdx.x / NT, tt = threadIdx.x % NT;
  if (tr < kGemvRows && tt < ntok && r0 + tr < rows) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kGemvWarps; ++w) v += red[w][tr][tt];
    y[tt * rows + r0 + tr] = v;
  }
}

template <int QT>
cudaError_t launch_gemv(const uint8_t *W, int64_t rows, int64_t k, const float *x, int ntok, float *y,
                        cudaStream_t s) {
  const unsigned blocks = (unsigned)((rows + kGemvRows - 1) / kGemvRows);
  if (ntok <= 1)
    gemv_proj_kernel<QT, 1><<<blocks, 32 * kGemvWarps, 0, s>>>(W, rows, k, x, ntok, y);
  else if (ntok <= 2)
    gemv_proj_kernel<QT, 2><<<blocks, 32 * kGemvWarps, 0, s>>>(W, rows, k, x, ntok, y);
  else if (ntok <= 4)
    gemv_proj_kernel<QT, 4><<<blocks, 32 * kGemvWarps, 0, s>>>(W, rows, k, x, ntok, y);
  else
    gemv_proj_kernel<QT, 8><<<blocks, 32 * kGemvWarps, 0, s>>>(W, rows, k, x, ntok, y);
  return cudaGetLastError();
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
  cudaStream_t s = (cudaStream_t)stream;
  const cudaError_t e = qtype == REDLITE_Q_Q8_0_STYLE
                            ? launch_gemv<3>((const uint8_t *)W, rows, k, x, n_tokens, y, s)
                            : launch_gemv<4>((const uint8_t *)W, rows, k, x, n_tokens, y, s);
  return e == cudaSuccess ? REDLITE_OK : REDLITE_ECUDA;
}
