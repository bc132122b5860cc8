// router.cu -- the router step that feeds the layer: per token, softmax over
// the expert logits, the top-k experts by probability, and their
// probabilities renormalised to sum 1.  The pages name router integration
// as the milestone after the routed layer ("Red Metal dev8 -- resident
// routed top-k layer", section "Field validation"; "Red Lite dev10",
// section "What dev10 does not yet claim"); the arithmetic is the
// batched-decode recipe (softmax, top-k with ties to the lower id,
// renormalisation).
//
// One warp per token.  Lane l holds logits l, l + 32, ...  The selection
// ranks by logit (softmax is increasing, so this is the order by
// probability, and equal logits are equal probabilities): k rounds of a
// warp-wide arg-max with ties to the lower id.  The renormalised weight of
// a selected expert is exp(l - m) / sum over the selection of exp(l' - m),
// m the largest logit (the full softmax denominator cancels).
#include "internal.cuh"

namespace redlite {

constexpr int kRouterWarps = 8;           // tokens per 256-thread block
constexpr int kRouterPerLane = 32;        // logits a lane keeps in registers (n_experts <= 1024)

// (value, id) order of the selection: larger value first, equal values to
// the lower id.
__device__ __forceinline__ bool ranks_before(float v, int i, float w, int j) { return v > w || (v == w && i < j); }

template <int PER>
__global__ void __launch_bounds__(32 * kRouterWarps) route_topk_kernel(const float *__restrict__ logits, int n_tokens,
                                                                    int n_experts, int top_k, int32_t *__restrict__ ids,
                                                                    float *__restrict__ weights) {
  // launched as a programmatic dependent of the kernel that writes the
  // logits: wait for it, then let the layer kernel that follows start its
  // own prologue (it waits for this grid before it reads ids and weights)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
  if (t >= n_tokens) return;
  const float *lg = logits + (size_t)t * n_experts;
  float v[PER];
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < n_experts ? __ldg(lg + e) : -INFINITY;
    m = fmaxf(m, v[i]);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // selection: k rounds of arg-max over the values not yet taken; a taken
  // value becomes NaN, which ranks below everything (comparisons are false)
  float sel_v = 0.f;  // lane j < top_k keeps the j-th selected logit
  int sel_i = 0;
  for (int j = 0; j < top_k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      if (e < n_experts && !(v[i] != v[i]) && ranks_before(v[i], e, bv, bi)) bv = v[i], bi = e;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ranks_before(ov, oi, bv, bi)) bv = ov, bi = oi;
    }
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (lane + 32 * i == bi) v[i] = __int_as_float(0x7fc00000);  // taken
    if (lane == j) sel_v = bv, sel_i = bi;
  }
  const float p = lane < top_k ? expf(sel_v - m) : 0.f;
  float s = p;
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane < top_k) {
    ids[(size_t)t * top_k + lane] = sel_i;
    weights[(size_t)t * top_k + lane] = p / s;
  }
}

cudaError_t launch_route_topk(const float *logits, int n_tokens, int n_experts, int top_k, int32_t *ids,
                              float *weights, cudaStream_t stream) {
  const unsigned blocks = (unsigned)((n_tokens + kRouterWarps - 1) / kRouterWarps);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3(32 * kRouterWarps);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto launch = [&](cudaLaunchConfig_t &c) {
    return n_experts <= 32 * 16
               ? cudaLaunchKernelEx(&c, route_topk_kernel<16>, logits, n_tokens, n_experts, top_k, ids, weights)
               : cudaLaunchKernelEx(&c, route_topk_kernel<kRouterPerLane>, logits, n_tokens, n_experts, top_k, ids,
                                    weights);
  };
  cudaError_t e = launch(cfg);
  if (e != cudaSuccess) {  // without the dependent-launch attribute
    (void)cudaGetLastError();
    cfg.numAttrs = 0;
    e = launch(cfg);
  }
  return e;
}

}  // namespace redlite

using namespace redlite;

extern "C" int redlite_moe_route_topk(const float *logits, int32_t n_tokens, int32_t n_experts, int32_t top_k,
                                      int32_t *expert_ids, float *router_weights, void *stream) {
  if (n_tokens < 0 || n_experts <= 0 || n_experts > 32 * kRouterPerLane) return REDLITE_EINVAL;
  if (top_k < 1 || top_k > kMaxTopK || top_k > n_experts) return REDLITE_EINVAL;
  if (n_tokens == 0) return REDLITE_OK;
  if (!logits || !expert_ids || !router_weights) return REDLITE_EINVAL;
  return launch_route_topk(logits, n_tokens, n_experts, top_k, expert_ids, router_weights, (cudaStream_t)stream) ==
                 cudaSuccess
             ? REDLITE_OK
             : REDLITE_ECUDA;
}
