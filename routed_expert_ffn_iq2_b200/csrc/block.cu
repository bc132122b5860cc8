// block.cu -- the post-attention block around the routed layer ("Red Lite
// dev16 -- complete full-attention parity", block composition paragraph:
// the attention residual, the post-attention RMSNorm, the full-width
// routed top-10 MoE plus shared expert, and the final residual):
//   xn  = RMSNorm(h) = gamma * h / sqrt(mean(h^2) + eps)
//   ids, w = router(W_r xn)          (softmax, top-k, renormalised)
//   out = h + layer(xn; ids, w)       (routed experts + shared expert)
// Three steps on the device: norm_router_kernel (the normalised state and
// the router logits), the router (router.cu), and the layer with out
// starting from h (the residual costs no extra pass).
#include "internal.cuh"

namespace redlite {

constexpr int kNrTok = 8;     // tokens per block (one warp each for the norm)
constexpr int kNrExp = 8;     // experts per block (one warp each for the logits)

cudaError_t launch_route_topk(const float *logits, int n_tokens, int n_experts, int top_k, int32_t *ids,
                              float *weights, cudaStream_t stream);

// Block (expert tile bx, token tile by): the tile's normalised states in
// shared memory (blocks with bx == 0 also write them out), then warp w's
// expert row dotted with each of them.  One pass over h per block; W_r rows
// are read once per token tile.
__global__ void __launch_bounds__(256) norm_router_kernel(const float *__restrict__ h, int n_tokens, int hidden,
                                                          const float *__restrict__ gamma, float eps,
                                                          const float *__restrict__ router_w, int n_experts,
                                                          float *__restrict__ xn, float *__restrict__ logits) {
  extern __shared__ float4 sx[];  // [kNrTok][hidden / 4]
  // the router kernel that follows may launch now; it waits for this grid
  // before it reads the logits
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.y * kNrTok, nt = min(kNrTok, n_tokens - t0);
  const int h4 = hidden / 4;
  // warp w normalises token t0 + w
  if (warp < nt) {
    const float4 *src = reinterpret_cast<const float4 *>(h + (size_t)(t0 + warp) * hidden);
    float ss = 0.f;
    for (int i = lane; i < h4; i += 32) {
      const float4 v = __ldg(src + i);
      sx[warp * h4 + i] = v;
      ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss / (float)hidden + eps);
    const float4 *g4 = reinterpret_cast<const float4 *>(gamma);
    float4 *dst = reinterpret_cast<float4 *>(xn + (size_t)(t0 + warp) * hidden);
    for (int i = lane; i < h4; i += 32) {
      const float4 g = __ldg(g4 + i), v = sx[warp * h4 + i];
      const float4 y = make_float4(g.x * v.x * inv, g.y * v.y * inv, g.z * v.z * inv, g.w * v.w * inv);
      sx[warp * h4 + i] = y;
      if (blockIdx.x == 0) dst[i] = y;
    }
  }
  __syncthreads();
  const int e = blockIdx.x * kNrExp + warp;
  if (e >= n_experts) return;
  const float4 *row = reinterpret_cast<const float4 *>(router_w + (size_t)e * hidden);
  float acc[kNrTok];
#pragma unroll
  for (int j = 0; j < kNrTok; ++j) acc[j] = 0.f;
  for (int i = lane; i < h4; i += 32) {
    const float4 r = __ldg(row + i);
#pragma unroll
    for (int j = 0; j < kNrTok; ++j)
      if (j < nt) {
        const float4 v = sx[j * h4 + i];
        acc[j] += r.x * v.x + r.y * v.y + r.z * v.z + r.w * v.w;
      }
  }
#pragma unroll
  for (int j = 0; j < kNrTok; ++j) {
    float v = acc[j];
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0 && j < nt) logits[(size_t)(t0 + j) * n_experts + e] = v;
  }
}

// Scratch regions of a block call: normalised states, logits, ids, weights.
struct BlockScratch {
  size_t xn, logits, ids, weights, total;
};
static BlockScratch block_scratch(int hidden, int n_experts, int max_tokens, int top_k) {
  BlockScratch b;
  size_t off = 0;
  b.xn = off;
  off = align256(off + sizeof(float) * (size_t)max_tokens * hidden);
  b.logits = off;
  off = align256(off + sizeof(float) * (size_t)max_tokens * n_experts);
  b.ids = off;
  off = align256(off + sizeof(int32_t) * (size_t)max_tokens * top_k);
  b.weights = off;
  off = align256(off + sizeof(float) * (size_t)max_tokens * top_k);
  b.total = off;
  return b;
}

}  // namespace redlite

using namespace redlite;

extern "C" size_t redlite_moe_block_scratch_bytes(int32_t hidden, int32_t n_experts, int32_t max_tokens,
                                                  int32_t top_k) {
  if (hidden <= 0 || n_experts <= 0 || max_tokens < 0 || top_k <= 0) return 0;
  return block_scratch(hidden, n_experts, max_tokens, top_k).total;
}

extern "C" int redlite_moe_block(const float *h, int32_t n_tokens, const float *norm_weight, float eps,
                                 const float *router_w, int32_t top_k, const redlite_moe_table *t,
                                 const redlite_moe_expert *shared, float *out, void *scratch, size_t scratch_bytes) {
  if (!t || n_tokens < 0 || n_tokens > t->max_tokens) return REDLITE_EINVAL;
  if (top_k < 1 || top_k > kMaxTopK || top_k > t->n_experts || t->n_experts > 1024) return REDLITE_EINVAL;
  if (t->hidden <= 0 || t->hidden % 4 || !(eps >= 0.f)) return REDLITE_EINVAL;
  if (n_tokens == 0) return REDLITE_OK;
  if (!h || !norm_weight || !router_w || !out || !scratch) return REDLITE_EINVAL;
  if ((((uintptr_t)h) | ((uintptr_t)norm_weight) | ((uintptr_t)router_w) | ((uintptr_t)out) |
       ((uintptr_t)scratch)) & 15)
    return REDLITE_EINVAL;
  const BlockScratch b = block_scratch(t->hidden, t->n_experts, t->max_tokens, top_k);
  if (b.total > scratch_bytes) return REDLITE_ENOMEM;
  const size_t smem = sizeof(float) * kNrTok * (size_t)t->hidden;
  if (smem > 200 * 1024) return REDLITE_EUNSUPPORTED;
  uint8_t *sc = (uint8_t *)scratch;
  float *xn = (float *)(sc + b.xn), *logits = (float *)(sc + b.logits), *w = (float *)(sc + b.weights);
  int32_t *ids = (int32_t *)(sc + b.ids);
  cudaStream_t s = (cudaStream_t)t->stream;
  if (cudaFuncSetAttribute(norm_router_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return REDLITE_ECUDA;
  const dim3 grid((unsigned)((t->n_experts + kNrExp - 1) / kNrExp), (unsigned)((n_tokens + kNrTok - 1) / kNrTok));
  norm_router_kernel<<<grid, 256, smem, s>>>(h, n_tokens, t->hidden, norm_weight, eps, router_w, t->n_experts, xn,
                                             logits);
  if (cudaGetLastError() != cudaSuccess) return REDLITE_ECUDA;
  if (launch_route_topk(logits, n_tokens, t->n_experts, top_k, ids, w, s) != cudaSuccess) return REDLITE_ECUDA;
  return layer_impl(xn, n_tokens, ids, w, top_k, t, shared, out, h);
}
