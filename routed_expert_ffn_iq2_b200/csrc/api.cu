// api.cu -- the C ABI declared in include/redlite_moe.h: argument checks on
// the host, then kernel launches on the caller's stream.
#include <string.h>

#include <vector>

#include "internal.cuh"


using namespace redlite;

static bool aligned16(const void *p) { return ((uintptr_t)p & 15) == 0; }

extern "C" {

size_t redlite_moe_grids_bytes(void) { return kGridBytes; }

int redlite_moe_expand_grids(const uint16_t *iq2_compact, const uint16_t *iq1_compact, void *grids_dev,
                             void *stream) {
  if (!iq2_compact || !iq1_compact || !grids_dev) return REDLITE_EINVAL;
  if ((uintptr_t)grids_dev & 255) return REDLITE_EINVAL;
  for (int e = 0; e < kQ2GridEntries; ++e)
    for (int j = 0; j < 8; ++j)
      if (((iq2_compact[e] >> (2 * j)) & 3) == 3) return REDLITE_EINVAL;
  for (int e = 0; e < kQ1GridEntries; ++e)
    for (int j = 0; j < 8; ++j)
      if (((iq1_compact[e] >> (2 * j)) & 3) == 3) return REDLITE_EINVAL;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t *g = (uint8_t *)grids_dev;
  if (cudaMemcpyAsync(g + kGridQ2Comp, iq2_compact, 2 * kQ2GridEntries, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return REDLITE_ECUDA;
  if (cudaMemcpyAsync(g + kGridQ1Comp, iq1_compact, 2 * kQ1GridEntries, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return REDLITE_ECUDA;
  if (launch_expand_grids((const uint16_t *)(g + kGridQ2Comp), (const uint16_t *)(g + kGridQ1Comp), g, s) !=
      cudaSuccess)
    return REDLITE_ECUDA;
  return cudaStreamSynchronize(s) == cudaSuccess ? REDLITE_OK : REDLITE_ECUDA;
}

size_t redlite_moe_matrix_bytes(int32_t qtype, int64_t rows, int64_t k) { return matrix_bytes(qtype, rows, k); }

size_t redlite_moe_workspace_bytes(int32_t hidden, int32_t n_experts, int32_t max_tokens, int32_t top_k,
                                   int32_t max_ffn) {
  if (hidden <= 0 || n_experts <= 0 || max_tokens < 0 || top_k <= 0 || max_ffn <= 0) return 0;
  return workspace_layout(hidden, n_experts, max_tokens, top_k, max_ffn).total;
}

static bool table_ok(const redlite_moe_table *t) {
  return t && t->hidden > 0 && t->hidden % 32 == 0 && t->n_experts > 0 && t->n_experts <= kRouteMaxExperts &&
         t->max_ffn > 0 && t->max_ffn % 32 == 0 && t->max_tokens >= 0 && t->experts && t->grids && t->workspace &&
         t->status && ((uintptr_t)t->workspace & 255) == 0;
}

int redlite_moe_workspace_reset(const redlite_moe_table *t) {
  if (!t || !t->workspace) return REDLITE_EINVAL;
  return cudaMemsetAsync(t->workspace, 0, t->workspace_bytes, (cudaStream_t)t->stream) == cudaSuccess
             ? REDLITE_OK
             : REDLITE_ECUDA;
}

}  // extern "C"

namespace redlite {

// The checks of a layer call that do not involve its data pointers:
// REDLITE_OK, or the error code the call returns before enqueuing anything.
static int layer_call_ok(int32_t n_tokens, int32_t top_k, const redlite_moe_table *t, const redlite_moe_expert *shared) {
  if (!table_ok(t)) return REDLITE_EINVAL;
  if (n_tokens < 0 || n_tokens > t->max_tokens) return REDLITE_EINVAL;
  if (top_k < 1 || top_k > kMaxTopK) return REDLITE_EINVAL;
  if (n_tokens == 0) return REDLITE_OK;  // the call enqueues nothing
  // min_ffn >= 256 declares every slot tiled: the fast kernels then run, and
  // the shared expert must be one they can read (selected slots are checked
  // on the device and reported in the status word)
  if (shared && !shared_ok(*shared, t, t->min_ffn >= 256)) return REDLITE_EINVAL;
  // the largest top_k this workspace can hold for the table's token limit
  if (workspace_layout(t->hidden, t->n_experts, t->max_tokens, top_k, t->max_ffn).total > t->workspace_bytes)
    return REDLITE_ENOMEM;
  return REDLITE_OK;
}

int layer_impl(const float *x, int32_t n_tokens, const int32_t *expert_ids, const float *router_weights, int32_t top_k,
               const redlite_moe_table *t, const redlite_moe_expert *shared, float *out, const float *residual) {
  const int ok = layer_call_ok(n_tokens, top_k, t, shared);
  if (ok != REDLITE_OK) return ok;
  if (n_tokens == 0) return REDLITE_OK;
  if (!x || !expert_ids || !router_weights || !out) return REDLITE_EINVAL;
  if (!aligned16(x) || !aligned16(out)) return REDLITE_EINVAL;
  const bool tiled = t->min_ffn >= 256;
  // region offsets are fixed by the table limits
  const WorkspaceLayout L = workspace_layout(t->hidden, t->n_experts, t->max_tokens, top_k, t->max_ffn);
  cudaStream_t s = (cudaStream_t)t->stream;
  uint8_t *ws = (uint8_t *)t->workspace;

  if (tiled && fused_supported(t->hidden, t->max_ffn, n_tokens, top_k, t->n_experts, shared != nullptr, device_sms())) {
    FusedArgs fa{};
    fa.x = x;
    fa.ids = expert_ids;
    fa.weights = router_weights;
    fa.out = out;
    fa.n_tokens = n_tokens;
    fa.top_k = top_k;
    fa.n_experts = t->n_experts;
    fa.hidden = t->hidden;
    fa.max_ffn = t->max_ffn;
    fa.experts = t->experts;
    if (shared) fa.shared = *shared;
    fa.has_shared = shared != nullptr;
    fa.grids = (const uint8_t *)t->grids;
    fa.ws = ws;
    fa.L = L;
    fa.status = t->status;
    fa.residual = residual;
    fa.wide = fused_wide_items(t->hidden, n_tokens * top_k, t->min_ffn, t->max_ffn, shared != nullptr,
                               shared ? shared->ffn : 0);
    return launch_fused(fa, s) == cudaSuccess ? REDLITE_OK : REDLITE_ECUDA;
  }
  const size_t out_bytes = sizeof(float) * (size_t)n_tokens * t->hidden;
  if (!residual) {
    if (cudaMemsetAsync(out, 0, out_bytes, s) != cudaSuccess) return REDLITE_ECUDA;
  } else if (residual != out) {
    if (cudaMemcpyAsync(out, residual, out_bytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess) return REDLITE_ECUDA;
  }
  const bool tc = tiled && tc_supported(t->hidden, t->max_ffn);
  RouteArgs ra{expert_ids, router_weights, n_tokens, top_k, t->n_experts, t->hidden, t->max_ffn,
               t->experts, shared != nullptr, shared ? shared->ffn : 0, shared ? shared->qtype : 0, tc, ws, L,
               t->status};
  if (launch_route(ra, s) != cudaSuccess) return REDLITE_ECUDA;
  TileArgs ta{};
  ta.x = x;
  ta.out = out;
  ta.n_tokens = n_tokens;
  ta.hidden = t->hidden;
  ta.max_ffn = t->max_ffn;
  ta.experts = t->experts;
  if (shared) ta.shared = *shared;
  ta.grids = (const uint8_t *)t->grids;
  ta.ws = ws;
  ta.L = L;
  ta.status = t->status;
  if (tc)
    return launch_tc(ta, s) == cudaSuccess ? REDLITE_OK : REDLITE_ECUDA;
  const int64_t routed = (int64_t)n_tokens * top_k;
  const int max_active = (int)((routed < t->n_experts ? routed : t->n_experts) + (shared ? 1 : 0));
  if (launch_simt_tiles(ta, max_active, s) != cudaSuccess) return REDLITE_ECUDA;
  return REDLITE_OK;
}

}  // namespace redlite

extern "C" {

int redlite_moe_layer(const float *x, int32_t n_tokens, const int32_t *expert_ids, const float *router_weights,
                      int32_t top_k, const redlite_moe_table *t, const redlite_moe_expert *shared, float *out) {
  return layer_impl(x, n_tokens, expert_ids, router_weights, top_k, t, shared, out, nullptr);
}

int redlite_moe_dequant(int32_t qtype, const void *packed, int64_t rows, int64_t k, const void *grids, float *out_f32,
                        uint16_t *out_bf16, void *stream) {
  if (!packed || !grids || (!out_f32 && !out_bf16)) return REDLITE_EINVAL;
  if (qtype != kQ2 && qtype != kQ1) return REDLITE_EINVAL;
  if (!shape_ok(rows, k)) return REDLITE_EUNSUPPORTED;
  if ((out_f32 && !aligned16(out_f32)) || (out_bf16 && !aligned16(out_bf16))) return REDLITE_EINVAL;
  return launch_dequant(qtype, packed, rows, k, grids, out_f32, out_bf16, (cudaStream_t)stream) == cudaSuccess
             ? REDLITE_OK
             : REDLITE_ECUDA;
}

int redlite_moe_upload_experts(int32_t hidden, const int32_t *ids, const redlite_moe_expert *host_experts, int32_t n,
                               void *pool, size_t pool_bytes, size_t pool_offset, redlite_moe_expert *table_dev,
                               int32_t n_experts, void *stream, redlite_moe_upload_counters *counters,
                               size_t *pool_end) {
  if (hidden <= 0 || n < 0 || (n > 0 && (!ids || !host_experts || !pool || !table_dev))) return REDLITE_EINVAL;
  if (!aligned16(pool)) return REDLITE_EINVAL;
  // plan the placement first: nothing is copied if anything is wrong
  std::vector<redlite_moe_expert> desc((size_t)n);
  std::vector<size_t> sizes((size_t)n * 3);
  size_t off = (pool_offset + 15) & ~size_t(15);
  int64_t bytes = 0;
  for (int i = 0; i < n; ++i) {
    const redlite_moe_expert &h = host_experts[i];
    if (ids[i] < 0 || ids[i] >= n_experts) return REDLITE_EINVAL;
    if ((h.qtype != kQ2 && h.qtype != kQ1) || h.ffn <= 0 || !h.gate || !h.up || !h.down) return REDLITE_EINVAL;
    const size_t gb = matrix_bytes(h.qtype, h.ffn, hidden), db = matrix_bytes(h.qtype, hidden, h.ffn);
    if (!gb || !db) return REDLITE_EUNSUPPORTED;
    const size_t s3[3] = {gb, gb, db};
    const void **dst[3] = {&desc[i].gate, &desc[i].up, &desc[i].down};
    desc[i].qtype = h.qtype;
    desc[i].ffn = h.ffn;
    for (int m = 0; m < 3; ++m) {
      *dst[m] = (const uint8_t *)pool + off;
      sizes[3 * i + m] = s3[m];
      off = (off + s3[m] + 15) & ~size_t(15);
      bytes += (int64_t)s3[m];
    }
  }
  if (off > pool_bytes) return REDLITE_ENOMEM;
  cudaStream_t s = (cudaStream_t)stream;
  // resident-layout copies stay alive until the stream is synchronised below
  std::vector<std::vector<uint8_t>> staged((size_t)n * 3);
  for (int i = 0; i < n; ++i) {
    const void *src[3] = {host_experts[i].gate, host_experts[i].up, host_experts[i].down};
    const void *dst[3] = {desc[i].gate, desc[i].up, desc[i].down};
    const int64_t shp[3][2] = {{host_experts[i].ffn, hidden}, {host_experts[i].ffn, hidden}, {hidden, host_experts[i].ffn}};
    for (int m = 0; m < 3; ++m) {
      std::vector<uint8_t> &buf = staged[3 * i + m];
      buf.resize(sizes[3 * i + m]);
      if (pack_matrix_host(host_experts[i].qtype, shp[m][0], shp[m][1], (const uint8_t *)src[m], buf.data()) !=
          REDLITE_OK)
        return REDLITE_EUNSUPPORTED;
      if (cudaMemcpyAsync((void *)dst[m], buf.data(), buf.size(), cudaMemcpyHostToDevice, s) != cudaSuccess)
        return REDLITE_ECUDA;
    }
    if (cudaMemcpyAsync(table_dev + ids[i], &desc[i], sizeof(redlite_moe_expert), cudaMemcpyHostToDevice, s) !=
        cudaSuccess)
      return REDLITE_ECUDA;
  }
  if (cudaStreamSynchronize(s) != cudaSuccess) return REDLITE_ECUDA;
  if (counters) {
    counters->loads += n;
    counters->copies += 3 * (int64_t)n;
    counters->bytes += bytes;
  }
  if (pool_end) *pool_end = off;
  return REDLITE_OK;
}

}  // extern "C"

extern "C" {

size_t redlite_moe_host_input_bytes(int32_t hidden, int32_t n_tokens, int32_t top_k) {
  if (hidden <= 0 || n_tokens <= 0 || top_k <= 0) return 0;
  return sizeof(float) * ((size_t)hidden + 2 * (size_t)top_k) * (size_t)n_tokens;
}

int redlite_moe_layer_host(const void *inputs_host, void *inputs_dev, int32_t n_tokens, int32_t top_k,
                           const redlite_moe_table *t, const redlite_moe_expert *shared, float *out_dev,
                           float *out_host) {
  const int ok = layer_call_ok(n_tokens, top_k, t, shared);
  if (ok != REDLITE_OK) return ok;
  if (n_tokens == 0) return REDLITE_OK;
  if (!inputs_host || !inputs_dev || !out_dev || !out_host) return REDLITE_EINVAL;
  if (!aligned16(inputs_dev) || !aligned16(out_dev)) return REDLITE_EINVAL;
  cudaStream_t s = (cudaStream_t)t->stream;
  const size_t nx = sizeof(float) * (size_t)n_tokens * (size_t)t->hidden;
  const size_t nk = sizeof(float) * (size_t)n_tokens * (size_t)top_k;
  if (cudaMemcpyAsync(inputs_dev, inputs_host, nx + 2 * nk, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return REDLITE_ECUDA;
  const uint8_t *in = (const uint8_t *)inputs_dev;
  const int rc = layer_impl((const float *)in, n_tokens, (const int32_t *)(in + nx), (const float *)(in + nx + nk),
                            top_k, t, shared, out_dev, nullptr);
  if (rc != REDLITE_OK) return rc;
  return cudaMemcpyAsync(out_host, out_dev, nx, cudaMemcpyDeviceToHost, s) == cudaSuccess ? REDLITE_OK
                                                                                          : REDLITE_ECUDA;
}

}  // extern "C"
