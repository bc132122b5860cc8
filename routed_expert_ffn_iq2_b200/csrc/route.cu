// route.cu -- token -> expert bucketing (counting sort of the (token, slot)
// pairs by expert id), as three kernels:
//   route_count_kernel    nb blocks; block b counts the experts of its chunk
//                         of pairs into hist[e][b];
//   route_plan_kernel     one block; per expert the exclusive prefix of the
//                         block counts (hist[e][b] becomes block b's offset
//                         within expert e), the drop of unusable experts, the
//                         first pair of each kept expert, the active list and
//                         the tensor-core work-unit bases, the shared
//                         expert's pairs;
//   route_scatter_kernel  nb blocks; block b places its chunk's pairs.
//
// Produces, in the workspace: the list of active experts in ascending id
// order (each with its first pair and pair count), the pairs grouped by
// expert, and the shared expert as a last active entry that owns every
// token with weight 1.  Invalid ids (outside [0, n_experts)) and selected
// slots without usable matrices are reported in the status word and their
// pairs are dropped, so such a pair contributes nothing.  Within an
// expert the order of its pairs is not fixed.
#include <climits>

#include "internal.cuh"

namespace redlite {

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

constexpr int kRouteThreads = 512;  // count and scatter blocks
constexpr int kRouteUnroll = 4;     // pairs a thread loads before it counts or places them

__global__ void __launch_bounds__(kRouteThreads) route_count_kernel(RouteArgs a, int nb, int chunk) {
  extern __shared__ int cnt[];  // [n_experts]
  const int E = a.n_experts, n = a.n_tokens * a.top_k;
  const int b = blockIdx.x, p0 = b * chunk, p1 = min(n, p0 + chunk);
  int *hist = reinterpret_cast<int *>(a.ws + a.L.hist);
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int base = p0; base < p1; base += kRouteUnroll * kRouteThreads) {
    int ev[kRouteUnroll];
#pragma unroll
    for (int u = 0; u < kRouteUnroll; ++u) {
      const int p = base + u * kRouteThreads + (int)threadIdx.x;
      ev[u] = p < p1 ? __ldg(a.ids + p) : 0;
    }
#pragma unroll
    for (int u = 0; u < kRouteUnroll; ++u) {
      if (base + u * kRouteThreads + (int)threadIdx.x >= p1) continue;
      if (ev[u] < 0 || ev[u] >= E)
        bad = true;
      else
        atomicAdd(&cnt[ev[u]], 1);
    }
  }
  if (bad) atomicOr(a.status, REDLITE_STATUS_BAD_ID);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)e * nb + b] = cnt[e];
}

// One block of 1024 threads; nb <= 32 (one lane per counting block).
__global__ void __launch_bounds__(1024) route_plan_kernel(RouteArgs a, int nb) {
  extern __shared__ int cnt[];  // [n_experts]
  __shared__ int scan_tmp[33];
  __shared__ int s_bad;
  const int E = a.n_experts;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  Ctrl *ctrl = reinterpret_cast<Ctrl *>(a.ws + a.L.ctrl);
  ActiveEntry *active = reinterpret_cast<ActiveEntry *>(a.ws + a.L.active);
  Pair *pairs = reinterpret_cast<Pair *>(a.ws + a.L.pairs);
  int *hist = reinterpret_cast<int *>(a.ws + a.L.hist);
  int *estart = reinterpret_cast<int *>(a.ws + a.L.counts);

  if (threadIdx.x == 0) s_bad = 0;
  // per expert, a warp-wide scan over the counting blocks (lane = block);
  // eight experts per warp at a time so that their loads overlap
  for (int e0 = 8 * warp; e0 < E; e0 += 8 * nwarps) {
    int v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = (e0 + j < E && lane < nb) ? hist[(size_t)(e0 + j) * nb + lane] : 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      int x = v[j];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (e0 + j < E) {
        if (lane < nb) hist[(size_t)(e0 + j) * nb + lane] = x - v[j];
        if (lane == 31) cnt[e0 + j] = x;
      }
    }
  }
  __syncthreads();
  int bad = 0;
  // drop experts whose slot is unusable
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    if (cnt[e] && !expert_ok(a.experts[e], a.hidden, a.max_ffn, a.tiled_path)) {
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
    estart[e] = cnt[e] ? pair_off : -1;
    if (cnt[e]) {
      active[act_off] = ActiveEntry{e, pair_off, cnt[e], 0, 0, 0, 0, 0};
      ++act_off;
    }
    pair_off += cnt[e];
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

__global__ void __launch_bounds__(kRouteThreads) route_scatter_kernel(RouteArgs a, int nb, int chunk) {
  extern __shared__ int cursor[];  // [n_experts]; dropped experts start far below zero
  const int E = a.n_experts, n = a.n_tokens * a.top_k;
  const int b = blockIdx.x, p0 = b * chunk, p1 = min(n, p0 + chunk);
  const int *hist = reinterpret_cast<const int *>(a.ws + a.L.hist);
  const int *estart = reinterpret_cast<const int *>(a.ws + a.L.counts);
  Pair *pairs = reinterpret_cast<Pair *>(a.ws + a.L.pairs);
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int s = estart[e];
    cursor[e] = s < 0 ? INT_MIN / 2 : s + hist[(size_t)e * nb + b];
  }
  __syncthreads();
  for (int base = p0; base < p1; base += kRouteUnroll * kRouteThreads) {
    int ev[kRouteUnroll];
    float wv[kRouteUnroll];
#pragma unroll
    for (int u = 0; u < kRouteUnroll; ++u) {
      const int p = base + u * kRouteThreads + (int)threadIdx.x;
      ev[u] = p < p1 ? __ldg(a.ids + p) : -1;
      wv[u] = p < p1 ? __ldg(a.weights + p) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kRouteUnroll; ++u) {
      const int p = base + u * kRouteThreads + (int)threadIdx.x;
      if (ev[u] < 0 || ev[u] >= E) continue;
      const int pos = atomicAdd(&cursor[ev[u]], 1);
      if (pos >= 0) pairs[pos] = Pair{p / a.top_k, wv[u]};
    }
  }
}

cudaError_t launch_route(const RouteArgs &a, cudaStream_t stream) {
  const int n = a.n_tokens * a.top_k;
  const int nb = max(1, min(kRouteBlocks, (n + 255) / 256));
  const int chunk = (n + nb - 1) / nb;
  const size_t smem = sizeof(int) * (size_t)a.n_experts;
  route_count_kernel<<<nb, kRouteThreads, smem, stream>>>(a, nb, chunk);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_plan_kernel<<<1, 1024, smem, stream>>>(a, nb);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_scatter_kernel<<<nb, kRouteThreads, smem, stream>>>(a, nb, chunk);
  return cudaGetLastError();
}

}  // namespace redlite
