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
#include "ptx.cuh"

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

// Exact small integers as floats without a conversion instruction: byte i
// of v, placed in the low mantissa byte of 2^23, minus 2^23 + bias (the
// result is an exact integer in fp32).
__device__ __forceinline__ float byte_f(uint32_t v, int i, float bias = 0.f) {
  return __uint_as_float(__byte_perm(v, 0x4B000000u, 0x7650u | (uint32_t)i)) - (8388608.f + bias);
}

// This lane's partial dot product of one row over one 256-input step, with
// the lane's 8 inputs xa, xb and their sum xs (the same for every row).
// Q8_0-style: d * sum(q x); Q4_K-style: d sc sum(q x) - dmin m sum(x),
// both per sub-block (the lane's 8 weights share one).  sh: the bit offset
// of the lane's 6-bit scale in the 96-bit scale field (6 j, j = lane / 4).
template <int QT>
__device__ __forceinline__ float step_dot(const uint32_t wd[5], int sh, float4 xa, float4 xb, float xs) {
  if constexpr (QT == 3) {
    // signed int8 q as unsigned q + 128 (xor 0x80 per byte); byte_f removes
    // the 128 again, so every q is exact before it multiplies x
    const uint32_t u01 = __byte_perm(__byte_perm(wd[1], wd[2], 0x0040u), __byte_perm(wd[3], wd[4], 0x0040u), 0x5410u) ^
                         0x80808080u;
    const uint32_t u23 = __byte_perm(__byte_perm(wd[1], wd[2], 0x0051u), __byte_perm(wd[3], wd[4], 0x0051u), 0x5410u) ^
                         0x80808080u;
    // weights 2i (u01 byte i) and 2i+1 (u23 byte i)
    float dot = byte_f(u01, 0, 128.f) * xa.x + byte_f(u23, 0, 128.f) * xa.y;
    dot += byte_f(u01, 1, 128.f) * xa.z + byte_f(u23, 1, 128.f) * xa.w;
    dot += byte_f(u01, 2, 128.f) * xb.x + byte_f(u23, 2, 128.f) * xb.y;
    dot += byte_f(u01, 3, 128.f) * xb.z + byte_f(u23, 3, 128.f) * xb.w;
    (void)xs;
    const float d = __half2float(__ushort_as_half((unsigned short)wd[0]));
    return d * dot;
  } else {
    const uint32_t lo = wd[4] & 0x0F0F0F0Fu, hi = (wd[4] >> 4) & 0x0F0F0F0Fu;  // weights 2i, 2i+1
    float dot = byte_f(lo, 0) * xa.x + byte_f(hi, 0) * xa.y;
    dot += byte_f(lo, 1) * xa.z + byte_f(hi, 1) * xa.w;
    dot += byte_f(lo, 2) * xb.x + byte_f(hi, 2) * xb.y;
    dot += byte_f(lo, 3) * xb.z + byte_f(hi, 3) * xb.w;
    const uint64_t f = (uint64_t)wd[1] | ((uint64_t)wd[2] << 32);
    const uint64_t g = (uint64_t)wd[2] | ((uint64_t)wd[3] << 32);
    const int sc = (int)((f >> sh) & 63u), mn = (int)((g >> (16 + sh)) & 63u);
    const float d = __half2float(__ushort_as_half((unsigned short)(wd[0] & 0xFFFFu)));
    const float dmin = __half2float(__ushort_as_half((unsigned short)(wd[0] >> 16)));
    return d * (float)sc * dot - dmin * (float)mn * xs;
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
  const int sh = 6 * (lane >> 2);  // this lane's sub-block (Q4_K-style scale field offset)
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
      float xs[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        xa[t] = xb[t] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < ntok) {
          const float4 *xp = reinterpret_cast<const float4 *>(x + t * k + 256 * s + 8 * lane);
          xa[t] = __ldg(xp), xb[t] = __ldg(xp + 1);
        }
        xs[t] = (xa[t].x + xa[t].y) + (xa[t].z + xa[t].w) + (xb[t].x + xb[t].y) + (xb[t].z + xb[t].w);
      }
#pragma unroll
      for (int h = 0; h < kGemvRows; ++h)
#pragma unroll
        for (int t = 0; t < NT; ++t)
          if (t < ntok) acc[h][t] += step_dot<QT>(wd[u][h], sh, xa[t], xb[t], xs[t]);
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

// The words of step_load for a row held in shared memory.
template <int QT>
__device__ __forceinline__ void step_load_smem(const uint8_t *row, int64_t s, int lane, uint32_t wd[5]) {
  if constexpr (QT == 3) {
    const uint8_t *blk = row + (8 * s + lane / 4) * 34;
    const unsigned short *qv = reinterpret_cast<const unsigned short *>(blk + 2 + 8 * (lane & 3));
    wd[0] = *reinterpret_cast<const unsigned short *>(blk);
#pragma unroll
    for (int i = 0; i < 4; ++i) wd[1 + i] = qv[i];
  } else {
    const uint8_t *blk = row + s * 144;
    const uint4 hd = *reinterpret_cast<const uint4 *>(blk);
    wd[0] = hd.x, wd[1] = hd.y, wd[2] = hd.z, wd[3] = hd.w;
    wd[4] = reinterpret_cast<const uint32_t *>(blk + 16)[lane];
  }
}

constexpr int kGsStages = 4;                 // row groups in flight per CTA, at most
constexpr int kGsPre = 2;                    // steps per warp whose inputs are held in registers
constexpr int kGsMaxStage = 24 * 1024;       // bytes of one row group (kGemvRows rows)

// Streaming form for matrices whose rows are 16-byte aligned: a persistent
// grid, each CTA walking row groups g = blockIdx.x, + gridDim.x, ...; a group
// (kGemvRows consecutive rows, contiguous in memory) arrives in a 4-stage
// shared-memory ring by one bulk copy, so every CTA keeps four groups of
// HBM reads in flight.  The 8 warps split each group's 256-input steps as in
// gemv_proj_kernel; one CTA barrier per group closes the reduction and frees
// the stage.  A bulk copy that does not land within the wait bound leaves NaN
// in that group's outputs.
template <int QT, int NT>
__global__ void __launch_bounds__(32 * kGemvWarps) gemv_stream_kernel(const uint8_t *__restrict__ W, int64_t rows,
                                                                     int64_t k, const float *__restrict__ x,
                                                                     int ntok, float *__restrict__ y,
                                                                     int64_t row_bytes, int n_groups, int nst) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ uint64_t full[kGsStages];
  __shared__ float red[2][kGemvWarps][kGemvRows][NT];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x, c = blockIdx.x;
  const int my_n = n_groups > c ? (n_groups - c + G - 1) / G : 0;
  const int64_t steps = k / 256;
  const size_t stage_bytes = (size_t)kGemvRows * row_bytes;
  if (tid == 0) {
    for (int i = 0; i < nst; ++i) ptx::mbar_init(&full[i], 1);
    ptx::mbar_fence_init();
  }
  __syncthreads();
  auto issue = [&](int i) {
    const int st = i % nst;
    const int64_t r0 = (int64_t)(c + (int64_t)i * G) * kGemvRows;
    const uint32_t bytes = (uint32_t)(min((int64_t)kGemvRows, rows - r0) * row_bytes);
    ptx::mbar_expect_tx(&full[st], bytes);
    ptx::bulk_g2s(ring + st * stage_bytes, W + r0 * row_bytes, bytes, &full[st]);
  };
  if (tid == 0)
    for (int i = 0; i < min(nst, my_n); ++i) issue(i);
  const int sh = 6 * (lane >> 2);  // this lane's sub-block (Q4_K-style scale field offset)
  // this lane's 8 inputs of a step (and their sum) for every token
  auto load_x = [&](int64_t s, float4 (&xa)[NT], float4 (&xb)[NT], float (&xs)[NT]) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      xa[t] = xb[t] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < ntok) {
        const float4 *xp = reinterpret_cast<const float4 *>(x + t * k + 256 * s + 8 * lane);
        xa[t] = __ldg(xp), xb[t] = __ldg(xp + 1);
      }
      xs[t] = (xa[t].x + xa[t].y) + (xa[t].z + xa[t].w) + (xb[t].x + xb[t].y) + (xb[t].z + xb[t].w);
    }
  };
  // a warp's steps are the same for every row group: for one or two tokens
  // and at most kGsPre steps per warp their inputs are loaded once, while
  // the first group's weights are still in flight
  constexpr int kPre = NT <= 2 ? kGsPre : 1;
  const bool pre = NT <= 2 && steps <= (int64_t)kGemvWarps * kPre;
  float4 pxa[kPre][NT], pxb[kPre][NT];
  float pxs[kPre][NT];
  if (pre) {
#pragma unroll
    for (int j = 0; j < kPre; ++j)
      if (warp + kGemvWarps * j < steps) load_x(warp + kGemvWarps * j, pxa[j], pxb[j], pxs[j]);
  }
  for (int i = 0; i < my_n; ++i) {
    const int st = i % nst;
    const int64_t r0 = (int64_t)(c + (int64_t)i * G) * kGemvRows;
    const bool landed = ptx::mbar_wait(&full[st], (uint32_t)((i / nst) & 1));
    const uint8_t *stage = ring + st * stage_bytes;
    float acc[kGemvRows][NT];
#pragma unroll
    for (int h = 0; h < kGemvRows; ++h)
#pragma unroll
      for (int t = 0; t < NT; ++t) acc[h][t] = 0.f;
    auto step_rows = [&](int64_t s, const float4 (&xa)[NT], const float4 (&xb)[NT], const float (&xs)[NT]) {
#pragma unroll
      for (int h = 0; h < kGemvRows; ++h) {
        if (r0 + h >= rows) break;
        uint32_t wd[5];
        step_load_smem<QT>(stage + h * row_bytes, s, lane, wd);
#pragma unroll
        for (int t = 0; t < NT; ++t)
          if (t < ntok) acc[h][t] += step_dot<QT>(wd, sh, xa[t], xb[t], xs[t]);
      }
    };
    if (pre) {
#pragma unroll
      for (int j = 0; j < kPre; ++j)
        if (warp + kGemvWarps * j < steps) step_rows(warp + kGemvWarps * j, pxa[j], pxb[j], pxs[j]);
    } else {
      for (int64_t s = warp; s < steps; s += kGemvWarps) {
        float4 xa[NT], xb[NT];
        float xs[NT];
        load_x(s, xa, xb, xs);
        step_rows(s, xa, xb, xs);
      }
    }
#pragma unroll
    for (int h = 0; h < kGemvRows; ++h)
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float v = acc[h][t];
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[i & 1][warp][h][t] = v;
      }
    __syncthreads();  // every warp is done with the stage and has stored its sums
    if (tid == 0 && i + nst < my_n) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(i + nst);
    }
    const int tr = tid / NT, tt = tid % NT;
    if (tr < kGemvRows && tt < ntok && r0 + tr < rows) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kGemvWarps; ++w) v += red[i & 1][w][tr][tt];
      y[tt * rows + r0 + tr] = landed ? v : __int_as_float(0x7fc00000);
    }
  }
}

template <int QT, int NT>
cudaError_t launch_stream(const uint8_t *W, int64_t rows, int64_t k, const float *x, int ntok, float *y,
                          int64_t row_bytes, cudaStream_t s) {
  const int n_groups = (int)((rows + kGemvRows - 1) / kGemvRows);
  // one row group per CTA up to eight CTAs per SM (every group's copy is in
  // flight from the start and no CTA works through two); beyond that a
  // persistent grid with a ring of up to kGsStages groups per CTA
  const int sms = device_sms();
  const int grid = min(n_groups, 8 * (sms > 0 ? sms : 148));
  const int nst = min(kGsStages, (n_groups + grid - 1) / grid);
  const size_t smem = (size_t)nst * kGemvRows * row_bytes;
  cudaError_t e = cudaFuncSetAttribute(gemv_stream_kernel<QT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  gemv_stream_kernel<QT, NT><<<grid, 32 * kGemvWarps, smem, s>>>(W, rows, k, x, ntok, y, row_bytes, n_groups, nst);
  return cudaGetLastError();
}

template <int QT>
cudaError_t launch_gemv(const uint8_t *W, int64_t rows, int64_t k, const float *x, int ntok, float *y,
                        cudaStream_t s) {
  const int64_t row_bytes = QT == 3 ? (k / 32) * 34 : (k / 256) * 144;
  if ((((uintptr_t)W) & 15) == 0 && row_bytes % 16 == 0 && kGemvRows * row_bytes <= kGsMaxStage) {
    if (ntok <= 1) return launch_stream<QT, 1>(W, rows, k, x, ntok, y, row_bytes, s);
    if (ntok <= 2) return launch_stream<QT, 2>(W, rows, k, x, ntok, y, row_bytes, s);
    if (ntok <= 4) return launch_stream<QT, 4>(W, rows, k, x, ntok, y, row_bytes, s);
    return launch_stream<QT, 8>(W, rows, k, x, ntok, y, row_bytes, s);
  }
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
