// route.cu -- token -> expert bucketing (counting sort of the (token, slot)
// pairs by expert id).
//
// Produces, in the workspace: the list of active experts in ascending id
// order (each with its first pair and pair count), the pairs sorted by
// expert, and the shared expert as a last active entry that owns every
// token with weight 1.  Invalid ids (outside [0, n_experts)) and selected
// slots without usable matrices are reported in the status word and their
// pairs are dropped ("the offending pair contributes nothing").
#include "internal.cuh"

namespace redlite {

__device__ bool expert_usable(const redlite_moe_expert &e, int hidden, int max_ffn) {
  if (!e.gate || !e.up || !e.down) return false;
  if (e.qtype != kQ2 && e.qtype != kQ1) return false;
  if (e.ffn <= 0 || e.ffn > max_ffn) return false;
  if (((uintptr_t)e.gate | (uintptr_t)e.up | (uintptr_t)e.down) & 15) return false;
  return shape_ok(e.ffn, hidden) && shape_ok(hidden, e.ffn);
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ int block_exclusive_scan(int v, int *smem32, int *total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) smem32[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = smem32[lane];
    int t = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    smem32[lane] = t - s;  // exclusive prefix of warp totals
    if (lane == 31) smem32[32] = t;
  }
  __syncthreads();
  const int r = smem32[wid] + x - v;
  *total = smem32[32];
  __syncthreads();
  return r;
}

// Single CTA of 1024 threads; n_experts <= kRouteMaxExperts.

__global__ void __launch_bounds__(1024) route_kernel(RouteArgs a) {
  extern __shared__ int sm[];
  int *cnt = sm;                      // [n_experts]
  int *cursor = sm + a.n_experts;     // [n_experts]
  __shared__ int scan_tmp[33];
  __shared__ int s_bad;
  const int E = a.n_experts;
  const int n = a.n_tokens * a.top_k;
  Ctrl *ctrl = reinterpret_cast<Ctrl *>(a.ws + a.L.ctrl);
  ActiveEntry *active = reinterpret_cast<ActiveEntry *>(a.ws + a.L.active);
  Pair *pairs = reinterpret_cast<Pair *>(a.ws + a.L.pairs);

  if (threadIdx.x == 0) s_bad = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  int bad = 0;
  for (int p = threadIdx.x; p < n; p += blockDim.x) {
    const int e = a.ids[p];
    if (e < 0 || e >= E) {
      bad |= REDLITE_STATUS_BAD_ID;
      continue;
    }
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  // drop experts whose slot is unusable
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    if (cnt[e] && !expert_usable(a.experts[e], a.hidden, a.max_ffn)) {
      cnt[e] = 0;
      bad |= REDLITE_STATUS_BAD_EXPERT;
    }
  }
  __syncthreads();
  // scan counts (each thread owns a contiguous run of experts)
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = threadIdx.x * per, e1 = min(E, e0 + per);
  int my_pairs = 0, my_active = 0;
  for (int e = e0; e < e1; ++e) {
    my_pairs += cnt[e];
    my_active += cnt[e] > 0;
  }
  int tot_pairs, tot_active;
  int pair_off = block_exclusive_scan(my_pairs, scan_tmp, &tot_pairs);
  int act_off = block_exclusive_scan(my_active, scan_tmp, &tot_active);
  for (int e = e0; e < e1; ++e) {
    cursor[e] = pair_off;
    if (cnt[e]) {
      active[act_off] = ActiveEntry{e, pair_off, cnt[e], 0, 0, 0, 0, 0};
      ++act_off;
    }
    pair_off += cnt[e];
  }
  __syncthreads();
  for (int p = threadIdx.x; p < n; p += blockDim.x) {
    const int e = a.ids[p];
    if (e < 0 || e >= E || cnt[e] == 0) continue;
    const int pos = atomicAdd(&cursor[e], 1);
    pairs[pos] = Pair{p / a.top_k, a.weights[p]};
  }
  int n_active = tot_active, n_pairs = tot_pairs;
  if (a.has_shared) {
    for (int t = threadIdx.x; t < a.n_tokens; t += blockDim.x) pairs[tot_pairs + t] = Pair{t, 1.0f};
    if (threadIdx.x == 0) active[tot_active] = ActiveEntry{-1, tot_pairs, a.n_tokens, 0, 0, 0, 0, 0};
    n_active += 1;
    n_pairs += a.n_tokens;
  }
  if (bad) atomicOr(&s_bad, bad);
  __syncthreads();
  // work units of the tensor-core path: per expert (width / 128 row tiles) x
  // (tokens / kTcTokens token tiles) for gate/up, (hidden / 128) x (same) for down
  {
    int carry_gu = 0, carry_dn = 0;
    for (int i0 = 0; i0 < n_active; i0 += blockDim.x) {
      const int i = i0 + threadIdx.x;
      int cgu = 0, cdn = 0;
      if (i < n_active) {
        ActiveEntry &ae = active[i];
        const bool sh = ae.expert < 0;
        ae.ffn = sh ? a.shared_ffn : a.experts[ae.expert].ffn;
        ae.qtype = sh ? a.shared_qtype : a.experts[ae.expert].qtype;
        const int nt = (ae.pair_count + kTcTokens - 1) / kTcTokens;
        cgu = (ae.ffn / 128) * nt;
        cdn = (a.hidden / 128) * nt;
      }
      int tg, td;
      const int og = block_exclusive_scan(cgu, scan_tmp, &tg);
      const int od = block_exclusive_scan(cdn, scan_tmp, &td);
      if (i < n_active) {
        active[i].gu_base = carry_gu + og;
        active[i].dn_base = carry_dn + od;
      }
      carry_gu += tg;
      carry_dn += td;
    }
    if (threadIdx.x == 0) {
      ctrl->n_active = n_active;
      ctrl->n_pairs = n_pairs;
      ctrl->n_gu_units = carry_gu;
      ctrl->n_dn_units = carry_dn;
      ctrl->ticket_gu = 0;
      ctrl->ticket_dn = 0;
      if (s_bad) atomicOr(a.status, s_bad);
    }
  }
}

cudaError_t launch_route(const RouteArgs &a, cudaStream_t stream) {
  const size_t smem = sizeof(int) * 2 * (size_t)a.n_experts;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  route_kernel<<<1, 1024, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace redlite
