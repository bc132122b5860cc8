// tiles_simt.cu -- expert FFN tiles on the CUDA cores (fp32 FMA).
//
// "Red Metal dev8 -- resident routed top-k layer", steps 4-5: each selected
// expert runs gate, up, SiLU(gate)*up and down from its resident slot, and
// accumulator += router_weight * expert_output.  Work is expert-major: one
// CTA reads a tile of one expert's packed rows once and applies it to every
// token routed to that expert (NT tokens at a time).
//
// This is the general path (any supported shape, any tokens per expert);
// the fused decode kernel and the tensor-core grouped path are the fast
// paths for their regimes.
#include "internal.cuh"

namespace redlite {

constexpr int kSimtThreads = 256;
constexpr int kSimtNT = 4;           // tokens per pass
constexpr int kGateUpRowsPerCta = 32;
constexpr int kDownRowsPerCta = 64;

__device__ __forceinline__ void load_grids_smem(const uint8_t *grids, int8_t *g2, int8_t *g1) {
  const uint4 *s2 = reinterpret_cast<const uint4 *>(grids + kGridQ2Vals);
  const uint4 *s1 = reinterpret_cast<const uint4 *>(grids + kGridQ1Vals);
  for (int i = threadIdx.x; i < 512 * 8 / 16; i += blockDim.x) reinterpret_cast<uint4 *>(g2)[i] = s2[i];
  for (int i = threadIdx.x; i < 2048 * 8 / 16; i += blockDim.x) reinterpret_cast<uint4 *>(g1)[i] = s1[i];
}

// dot of one packed row (k inputs, groups G0..G0+k/8) with NT vectors in smem
template <int QT>
__device__ __forceinline__ void row_dot(const uint8_t *mat, int64_t G0, int k, bool tiled, const int8_t *grid,
                                        const float *vs, int vstride, int nt, float acc[kSimtNT]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < kSimtNT; ++j) acc[j] = 0.f;
  for (int gq = lane; gq < k / 8; gq += 32) {
    float w[8];
    decode_group_f32<QT>(mat, k, tiled, G0 + gq, grid, w);
#pragma unroll
    for (int j = 0; j < kSimtNT; ++j) {
      if (j < nt) {
        const float4 a = *reinterpret_cast<const float4 *>(vs + j * vstride + gq * 8);
        const float4 b = *reinterpret_cast<const float4 *>(vs + j * vstride + gq * 8 + 4);
        acc[j] += w[0] * a.x + w[1] * a.y + w[2] * a.z + w[3] * a.w + w[4] * b.x + w[5] * b.y + w[6] * b.z +
                  w[7] * b.w;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kSimtNT; ++j) acc[j] = warp_sum(acc[j]);
}

__device__ __forceinline__ const redlite_moe_expert &expert_of(const TileArgs &a, const ActiveEntry &e) {
  return e.expert >= 0 ? a.experts[e.expert] : a.shared;
}

__global__ void __launch_bounds__(kSimtThreads) gateup_simt_kernel(TileArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  int8_t *g2 = reinterpret_cast<int8_t *>(smem);
  int8_t *g1 = g2 + 512 * 8;
  float *xs = reinterpret_cast<float *>(g1 + 2048 * 8);  // [NT][hidden]
  __shared__ int s_tok[kSimtNT];

  const Ctrl *ctrl = reinterpret_cast<const Ctrl *>(a.ws + a.L.ctrl);
  if ((int)blockIdx.y >= ctrl->n_active) return;
  const ActiveEntry ae = reinterpret_cast<const ActiveEntry *>(a.ws + a.L.active)[blockIdx.y];
  if (ae.pair_count == 0) return;
  const redlite_moe_expert ex = expert_of(a, ae);
  const int F = ex.ffn, H = a.hidden;
  const int i0 = blockIdx.x * kGateUpRowsPerCta;
  if (i0 >= F) return;
  const Pair *pairs = reinterpret_cast<const Pair *>(a.ws + a.L.pairs) + ae.pair_start;
  float *hbuf = reinterpret_cast<float *>(a.ws + a.L.h);

  load_grids_smem(a.grids, g2, g1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int c0 = 0; c0 < ae.pair_count; c0 += kSimtNT) {
    const int nt = min(kSimtNT, ae.pair_count - c0);
    __syncthreads();
    if (threadIdx.x < nt) s_tok[threadIdx.x] = pairs[c0 + threadIdx.x].token;
    __syncthreads();
    for (int j = 0; j < nt; ++j) {
      const float4 *src = reinterpret_cast<const float4 *>(a.x + (size_t)s_tok[j] * H);
      for (int c = threadIdx.x; c < H / 4; c += blockDim.x) reinterpret_cast<float4 *>(xs + j * H)[c] = src[c];
    }
    __syncthreads();
    for (int r = warp; r < kGateUpRowsPerCta; r += kSimtThreads / 32) {
      const int i = i0 + r;
      if (i >= F) break;
      const int64_t G0 = (int64_t)i * H / 8;
      float gacc[kSimtNT], uacc[kSimtNT];
      const bool tiled = tiled_shape(F, H);
      if (ex.qtype == kQ2) {
        row_dot<kQ2>((const uint8_t *)ex.gate, G0, H, tiled, g2, xs, H, nt, gacc);
        row_dot<kQ2>((const uint8_t *)ex.up, G0, H, tiled, g2, xs, H, nt, uacc);
      } else {
        row_dot<kQ1>((const uint8_t *)ex.gate, G0, H, tiled, g1, xs, H, nt, gacc);
        row_dot<kQ1>((const uint8_t *)ex.up, G0, H, tiled, g1, xs, H, nt, uacc);
      }
#pragma unroll
      for (int j = 0; j < kSimtNT; ++j)
        if (lane == j && j < nt) hbuf[(size_t)(ae.pair_start + c0 + j) * a.max_ffn + i] = silu_mul(gacc[j], uacc[j]);
    }
  }
}

__global__ void __launch_bounds__(kSimtThreads) down_simt_kernel(TileArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  int8_t *g2 = reinterpret_cast<int8_t *>(smem);
  int8_t *g1 = g2 + 512 * 8;
  float *hs = reinterpret_cast<float *>(g1 + 2048 * 8);  // [NT][max_ffn]
  __shared__ Pair s_pair[kSimtNT];

  const Ctrl *ctrl = reinterpret_cast<const Ctrl *>(a.ws + a.L.ctrl);
  if ((int)blockIdx.y >= ctrl->n_active) return;
  const ActiveEntry ae = reinterpret_cast<const ActiveEntry *>(a.ws + a.L.active)[blockIdx.y];
  if (ae.pair_count == 0) return;
  const redlite_moe_expert ex = expert_of(a, ae);
  const int F = ex.ffn, H = a.hidden;
  const int r0 = blockIdx.x * kDownRowsPerCta;
  if (r0 >= H) return;
  const Pair *pairs = reinterpret_cast<const Pair *>(a.ws + a.L.pairs) + ae.pair_start;
  const float *hbuf = reinterpret_cast<const float *>(a.ws + a.L.h);

  load_grids_smem(a.grids, g2, g1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int c0 = 0; c0 < ae.pair_count; c0 += kSimtNT) {
    const int nt = min(kSimtNT, ae.pair_count - c0);
    __syncthreads();
    if (threadIdx.x < nt) s_pair[threadIdx.x] = pairs[c0 + threadIdx.x];
    for (int j = 0; j < nt; ++j) {
      const float4 *src = reinterpret_cast<const float4 *>(hbuf + (size_t)(ae.pair_start + c0 + j) * a.max_ffn);
      for (int c = threadIdx.x; c < F / 4; c += blockDim.x) reinterpret_cast<float4 *>(hs + j * F)[c] = src[c];
    }
    __syncthreads();
    for (int rr = warp; rr < kDownRowsPerCta; rr += kSimtThreads / 32) {
      const int r = r0 + rr;
      if (r >= H) break;
      const int64_t G0 = (int64_t)r * F / 8;
      float y[kSimtNT];
      const bool tiled = tiled_shape(H, F);
      if (ex.qtype == kQ2)
        row_dot<kQ2>((const uint8_t *)ex.down, G0, F, tiled, g2, hs, F, nt, y);
      else
        row_dot<kQ1>((const uint8_t *)ex.down, G0, F, tiled, g1, hs, F, nt, y);
#pragma unroll
      for (int j = 0; j < kSimtNT; ++j)
        if (lane == j && j < nt) atomicAdd(a.out + (size_t)s_pair[j].token * H + r, s_pair[j].weight * y[j]);
    }
  }
}

size_t simt_smem_bytes(int hidden, int max_ffn) {
  const size_t grids = 512 * 8 + 2048 * 8;
  const size_t v = sizeof(float) * kSimtNT * (size_t)(hidden > max_ffn ? hidden : max_ffn);
  return grids + v;
}

cudaError_t launch_simt_tiles(const TileArgs &a, int max_active, cudaStream_t stream) {
  const size_t smem = simt_smem_bytes(a.hidden, a.max_ffn);
  static int configured = 0;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gateup_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(down_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    configured = 1;
  }
  dim3 g1((a.max_ffn + kGateUpRowsPerCta - 1) / kGateUpRowsPerCta, max_active);
  gateup_simt_kernel<<<g1, kSimtThreads, smem, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2((a.hidden + kDownRowsPerCta - 1) / kDownRowsPerCta, max_active);
  down_simt_kernel<<<g2, kSimtThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace redlite
