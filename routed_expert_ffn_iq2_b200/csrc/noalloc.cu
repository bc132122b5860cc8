// noalloc.cu -- the layer for callers that cannot allocate device memory.
//
// Same computation and the same fused decode kernel as redlite_moe_layer,
// but the kernel's scratch (control words, per-pair gate/up results,
// activation limbs) lives in one file-scope device array of fixed size
// instead of a caller-provided workspace.  Every GPU that loads this
// library holds that array until the process exits.
#include <mutex>

#include "internal.cuh"

namespace redlite {

// Scratch shared by every call on a device; 256-byte aligned, zero at load.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_setup_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device.  In host code the array's name is only a stand-in symbol, so
// the address must come from the runtime.  The first lookup also clears the
// control words on `stream` (the array is zero at load; this keeps the
// contract explicit).
int scratch_for_current_device(cudaStream_t stream, uint8_t **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return REDLITE_ECUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return REDLITE_ECUDA;
    if (cudaMemsetAsync(p, 0, sizeof(Ctrl), stream) != cudaSuccess) return REDLITE_ECUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = (uint8_t *)g_scratch_ptr[dev];
  return REDLITE_OK;
}

// Layout of the scratch for one call: only the regions the fused kernel uses.
WorkspaceLayout noalloc_layout(int hidden, int n_tokens, int top_k, int max_ffn) {
  WorkspaceLayout L{};
  const int64_t pairs = (int64_t)n_tokens * top_k + n_tokens;
  size_t off = 0;
  L.ctrl = off;
  off = align256(off + sizeof(Ctrl));
  L.slices = off;  // fixed place after the control block, as in the workspace layout
  off = align256(off + kSliceBytes);
  L.gu = off;
  off = align256(off + sizeof(float) * (size_t)pairs * (size_t)max_ffn);
  L.active = L.pairs = L.counts = L.hist = L.h = L.xb = off;
  L.total = off;
  L.max_pairs = (int)pairs;
  L.max_active = 0;
  return L;
}
}  // namespace

}  // namespace redlite

using namespace redlite;

extern "C" int redlite_moe_layer_noalloc(const float *x, int32_t n_tokens, const int32_t *expert_ids,
                                         const float *router_weights, int32_t top_k, const redlite_moe_table *t,
                                         const redlite_moe_expert *shared, float *out) {
  if (!t || t->hidden <= 0 || t->n_experts <= 0 || t->max_ffn <= 0 || !t->experts || !t->grids || !t->status)
    return REDLITE_EINVAL;
  if (n_tokens < 0 || top_k < 1 || top_k > kMaxTopK) return REDLITE_EINVAL;
  if (n_tokens == 0) return REDLITE_OK;
  if (!x || !expert_ids || !router_weights || !out) return REDLITE_EINVAL;
  if ((((uintptr_t)x) | ((uintptr_t)out)) & 15) return REDLITE_EINVAL;
  // the fused kernel reads the shared expert in the tiled layout: check it as
  // redlite_moe_layer does on that path
  if (shared && !shared_ok(*shared, t, true)) return REDLITE_EINVAL;
  // only the fused decode kernel runs here
  if (t->min_ffn < 256 || !fused_supported(t->hidden, t->max_ffn, n_tokens, top_k, t->n_experts, shared != nullptr, device_sms()))
    return REDLITE_EUNSUPPORTED;
  const WorkspaceLayout L = noalloc_layout(t->hidden, n_tokens, top_k, t->max_ffn);
  if (L.total > kNoAllocScratchBytes) return REDLITE_ENOMEM;
  cudaStream_t s = (cudaStream_t)t->stream;
  uint8_t *scratch = nullptr;
  const int rc = scratch_for_current_device(s, &scratch);
  if (rc != REDLITE_OK) return rc;
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
  fa.ws = scratch;
  fa.L = L;
  fa.status = t->status;
  fa.wide = fused_wide_items(t->hidden, n_tokens * top_k, t->min_ffn, t->max_ffn, shared != nullptr,
                             shared ? shared->ffn : 0);
  return launch_fused(fa, s) == cudaSuccess ? REDLITE_OK : REDLITE_ECUDA;
}
