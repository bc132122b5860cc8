// internal.cuh -- layouts and device helpers shared by the library's kernels.
//
// Format definitions follow the packed layouts documented in
// include/redlite_moe.h (IQ2_XS-style and IQ1_M-style blocks; the grids of
// "Red Lite dev10 -- standalone native Metal path", section "Quant grids").
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/redlite_moe.h"

namespace redlite {

constexpr int kQ2 = REDLITE_Q_IQ2XS_STYLE;
constexpr int kQ1 = REDLITE_Q_IQ1M_STYLE;
constexpr int kBlockWeights = 256;
constexpr int kQ2BlockBytes = 74;
constexpr int kQ1BlockBytes = 56;
constexpr int kQ2GridEntries = 512;
constexpr int kQ1GridEntries = 2048;

// ---------------------------------------------------------------- grid buffer
// Expanded once by redlite_moe_expand_grids; every offset is 256-aligned.
//   kGridQ2Vals : int8  [512][8]   IQ2 values 8/25/43
//   kGridQ1Vals : int8  [2048][8]  IQ1 values -1/0/+1
//   kGridQ2Bf16 : bf16  [512][8]   IQ2 values as bf16 (exact)
//   kGridQ1Bf16p: bf16  [2][2048][8] IQ1 (grid + delta) * 8 as bf16, delta
//                 +1/8 (plane 0) and -1/8 (plane 1): values -9,-7,-1,1,7,9
//   kGridQ2Comp : u16 [512], kGridQ1Comp : u16 [2048] (compact, as given)
constexpr size_t kGridQ2Vals = 0;
constexpr size_t kGridQ1Vals = kGridQ2Vals + 512 * 8;
constexpr size_t kGridQ2Bf16 = kGridQ1Vals + 2048 * 8;
constexpr size_t kGridQ1Bf16p = kGridQ2Bf16 + 512 * 8 * 2;
constexpr size_t kGridQ2Comp = kGridQ1Bf16p + 2 * 2048 * 8 * 2;
constexpr size_t kGridQ1Comp = kGridQ2Comp + 512 * 2;
constexpr size_t kGridBytes = kGridQ1Comp + 2048 * 2;

inline __host__ __device__ int block_bytes(int qtype) {
  return qtype == kQ2 ? kQ2BlockBytes : (qtype == kQ1 ? kQ1BlockBytes : 0);
}

// A rows x k matrix is supported when its weights form whole 256-weight
// blocks and no 32-weight run straddles two rows.
inline __host__ __device__ bool shape_ok(int64_t rows, int64_t k) {
  if (rows <= 0 || k <= 0) return false;
  if ((rows * k) % kBlockWeights) return false;
  if (k >= kBlockWeights) return k % kBlockWeights == 0;
  return (kBlockWeights % k == 0) && (k % 32 == 0);
}

inline __host__ __device__ size_t matrix_bytes(int qtype, int64_t rows, int64_t k) {
  if (!block_bytes(qtype) || !shape_ok(rows, k)) return 0;
  return (size_t)(rows * k / kBlockWeights) * block_bytes(qtype);
}

// ---------------------------------------------------------------- workspace
// Control words, the active-expert list, the token pairs sorted by expert
// and the per-pair hidden activations h.  Sizes depend on the table limits.
struct ActiveEntry {
  int expert;      // slot id, or -1 for the shared expert
  int pair_start;  // first pair of this expert in the sorted pair list
  int pair_count;  // tokens routed to it (0: skipped)
  int tile_base;   // first work ticket of this expert (fused scheduler)
};

struct Pair {
  int token;
  float weight;
};

// Control block: counters of the fused scheduler and the bucketing result.
struct Ctrl {
  int n_active;        // entries in the active list (incl. shared)
  int n_pairs;         // pairs in the sorted list
  int ticket;          // next work ticket
  int exit_count;      // CTAs that finished (the last one resets)
  int phase1_done;     // gate/up tickets completed
  int zero_done;       // output-zeroing tickets completed
  int pad[58];
};
static_assert(sizeof(Ctrl) == 256, "ctrl block is 256 bytes");

struct WorkspaceLayout {
  size_t ctrl, active, pairs, counts, done, h, total;
  int max_active, max_pairs;
};

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline WorkspaceLayout workspace_layout(int hidden, int n_experts, int max_tokens, int top_k, int max_ffn) {
  WorkspaceLayout L;
  (void)hidden;
  int64_t routed = (int64_t)max_tokens * top_k;
  L.max_pairs = (int)(routed + max_tokens);  // + shared expert pairs
  L.max_active = (int)((routed < n_experts ? routed : n_experts) + 1);
  size_t off = 0;
  L.ctrl = off;
  off = align256(off + sizeof(Ctrl));
  L.active = off;
  off = align256(off + sizeof(ActiveEntry) * (size_t)L.max_active);
  L.pairs = off;
  off = align256(off + sizeof(Pair) * (size_t)L.max_pairs);
  L.counts = off;
  off = align256(off + sizeof(int) * (size_t)(n_experts + 1));
  L.done = off;  // per-active-expert completion counters (fused scheduler)
  off = align256(off + sizeof(int) * (size_t)L.max_active);
  L.h = off;
  off = align256(off + sizeof(float) * (size_t)L.max_pairs * (size_t)max_ffn);
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- device helpers

__device__ __forceinline__ float fp16_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

__device__ __forceinline__ uint16_t ld_u16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

// Eight weights of group G (weights 8G..8G+7 of the matrix's row-major
// sequence), exact in fp32.  grid: expanded int8 values of the format.
template <int QT>
__device__ __forceinline__ void decode_group_f32(const uint8_t *__restrict__ mat, int64_t G,
                                                 const int8_t *__restrict__ grid, float w[8]) {
  const int64_t blk_i = G >> 5;
  const int g = (int)(G & 31);
  if constexpr (QT == kQ2) {
    const uint8_t *b = mat + blk_i * kQ2BlockBytes;
    const float d = fp16_bits_to_float(ld_u16(b));
    const int idx = b[6 + g] | (((b[38 + (g >> 3)] >> (g & 7)) & 1) << 8);
    const int sc = (b[2 + (g >> 3)] >> (4 * ((g >> 2) & 1))) & 15;
    const unsigned s = b[42 + g];
    const float scale = d * (float)(2 * sc + 1) * 0.125f;
    const int8_t *gv = grid + idx * 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float v = scale * (float)gv[j];
      w[j] = ((s >> j) & 1) ? -v : v;
    }
  } else {
    const uint8_t *b = mat + blk_i * kQ1BlockBytes;
    const float d = fp16_bits_to_float(ld_u16(b));
    const int nib = (b[34 + (g >> 1)] >> (4 * (g & 1))) & 15;
    const int idx = b[2 + g] | ((nib & 7) << 8);
    const float delta = (nib & 8) ? -0.125f : 0.125f;
    const int sub = g >> 1;
    const int bit = 3 * sub;
    // the 3-bit field may straddle two bytes of the 48-bit scales field
    const unsigned two = b[50 + (bit >> 3)] | ((bit >> 3) < 5 ? (unsigned)b[51 + (bit >> 3)] << 8 : 0u);
    const int sc = (two >> (bit & 7)) & 7;
    const float scale = d * (float)(2 * sc + 1);
    const int8_t *gv = grid + idx * 8;
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = scale * ((float)gv[j] + delta);
  }
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- launch arguments

struct RouteArgs {
  const int32_t *ids;
  const float *weights;
  int n_tokens, top_k, n_experts, hidden, max_ffn;
  const redlite_moe_expert *experts;
  bool has_shared;
  uint8_t *ws;
  WorkspaceLayout L;
  int32_t *status;
};

struct TileArgs {
  const float *x;
  float *out;
  int n_tokens, hidden, max_ffn;
  const redlite_moe_expert *experts;
  redlite_moe_expert shared;
  const uint8_t *grids;
  uint8_t *ws;
  WorkspaceLayout L;
};

constexpr int kRouteMaxExperts = 8192;
constexpr int kMaxTopK = 16;

cudaError_t launch_expand_grids(const uint16_t *comp2_dev, const uint16_t *comp1_dev, void *grids,
                                cudaStream_t stream);
cudaError_t launch_dequant(int qtype, const void *packed, int64_t rows, int64_t k, const void *grids, float *out_f32,
                           uint16_t *out_bf16, cudaStream_t stream);
cudaError_t launch_route(const RouteArgs &a, cudaStream_t stream);
cudaError_t launch_simt_tiles(const TileArgs &a, int max_active, cudaStream_t stream);

}  // namespace redlite
