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

#include <algorithm>

#include "../../include/redlite_moe.h"
#include "layout.cuh"

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
//   kGridQ2Sel  : u32 [512]   byte-permute selectors: nibble j = symbol j
//   kGridSign   : u32 [256]   nibble j bit 2 = sign bit j of a sign byte
//   kGridQ1Sel  : u32 [4096]  index e = idx | delta_bit << 11: nibble j =
//                 symbol j of grid entry idx | delta_bit << 2
//   kGridQ2Bsel : u64 [512], kGridQ1Bsel : u64 [2048]  bf16-pair selectors:
//                 bits 16w..16w+15 select weights 2w, 2w+1 as the byte pairs
//                 (2 s, 2 s + 1) of a table of three bf16 values indexed by
//                 the weights' symbols s
// A selector nibble picks one byte of a constant 8-byte table (see the
// decode kernels), so two byte-permutes turn a selector into eight signed
// int8 weights.
constexpr size_t kGridQ2Vals = 0;
constexpr size_t kGridQ1Vals = kGridQ2Vals + 512 * 8;
constexpr size_t kGridQ2Bf16 = kGridQ1Vals + 2048 * 8;
constexpr size_t kGridQ1Bf16p = kGridQ2Bf16 + 512 * 8 * 2;
constexpr size_t kGridQ2Comp = kGridQ1Bf16p + 2 * 2048 * 8 * 2;
constexpr size_t kGridQ1Comp = kGridQ2Comp + 512 * 2;
constexpr size_t kGridQ2Sel = kGridQ1Comp + 2048 * 2;
constexpr size_t kGridSign = kGridQ2Sel + 512 * 4;
constexpr size_t kGridQ1Sel = kGridSign + 256 * 4;
constexpr size_t kGridQ2Bsel = kGridQ1Sel + 4096 * 4;
constexpr size_t kGridQ1Bsel = kGridQ2Bsel + 512 * 8;
constexpr size_t kGridBytes = kGridQ1Bsel + 2048 * 8;

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

// Whether a slot descriptor can be used by a layer kernel: three non-null,
// 16-byte aligned matrices of a known format whose shapes the packed layout
// takes, 0 < ffn <= max_ffn.  The fast kernels (fused decode, tensor-core
// tiles) read every matrix in the tiled resident layout, so on their path the
// width must also be a multiple of 256.  Used on the host for the shared
// expert and on the device for every selected slot.
inline __host__ __device__ bool expert_ok(const redlite_moe_expert &e, int hidden, int max_ffn, bool tiled_path) {
  if (!e.gate || !e.up || !e.down) return false;
  if (e.qtype != kQ2 && e.qtype != kQ1) return false;
  if (e.ffn <= 0 || e.ffn > max_ffn) return false;
  if (((uintptr_t)e.gate | (uintptr_t)e.up | (uintptr_t)e.down) & 15) return false;
  if (tiled_path && (e.ffn % kBlockWeights || hidden % kBlockWeights)) return false;
  return shape_ok(e.ffn, hidden) && shape_ok(hidden, e.ffn);
}

// ---------------------------------------------------------------- workspace
// Control words, the active-expert list, the token pairs sorted by expert
// and the per-pair hidden activations h.  Sizes depend on the table limits.
struct ActiveEntry {
  int expert;      // slot id, or -1 for the shared expert
  int pair_start;  // first pair of this expert in the sorted pair list
  int pair_count;  // tokens routed to it (0: skipped)
  int gu_base;     // first gate/up work unit of this expert (tensor-core path)
  int dn_base;     // first down work unit of this expert (tensor-core path)
  int ffn;         // expert width
  int qtype;       // weight format
  int pad;
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
  int exit_count;      // fused decode kernel: CTAs that finished (the last one closes the call)
  int epoch;           // fused decode kernel: calls so far; its parity picks the counter set
  int out_ready[2];    // per parity: CTAs that initialised their part of out
  int slice_pairs[2];  // per parity: pairs whose slice counters that call used
  int n_gu_units;      // tensor-core path: gate/up work units
  int n_dn_units;      // tensor-core path: down work units
  int ticket_gu;       // next gate/up unit
  int ticket_dn;       // next down unit
  int pad[51];
};
static_assert(sizeof(Ctrl) == 256, "ctrl block is 256 bytes");

struct WorkspaceLayout {
  size_t ctrl, slices, active, pairs, counts, hist, h, xb, gu, total;
  int max_active, max_pairs;
};

// Fused decode kernel: h slices finished, per (first pair of a token chunk,
// 256-input slice of the expert width): counts of 16-row tiles written.  Two
// sets, picked by the parity of the call count: a call uses one and zeroes
// the part of the other that the previous call used.  They persist between
// calls, so they sit at a fixed offset, right after the control block,
// whatever the call's shape.
constexpr int kSlicesPerPair = 8;  // widths up to 2048
constexpr int kSliceStride = 32;   // ints between counters: one 128-byte line each

// Largest (token, slot) pair count the fused decode kernel takes.
constexpr int kRouteBlocks = 32;  // bucketing: blocks that count and place pairs
constexpr int kFusedMaxPairs = 640;
constexpr int kFusedMaxInst = kFusedMaxPairs + 2;  // selected experts + the shared expert, rounded up
constexpr int kSliceSetInts = (kFusedMaxPairs + 64) * kSlicesPerPair * kSliceStride;  // + shared pairs
constexpr size_t kSliceBytes = sizeof(int) * 2 * (size_t)kSliceSetInts;

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

inline WorkspaceLayout workspace_layout(int hidden, int n_experts, int max_tokens, int top_k, int max_ffn) {
  WorkspaceLayout L;
  int64_t routed = (int64_t)max_tokens * top_k;
  L.max_pairs = (int)(routed + max_tokens);  // + shared expert pairs
  L.max_active = (int)((routed < n_experts ? routed : n_experts) + 1);
  size_t off = 0;
  L.ctrl = off;
  off = align256(off + sizeof(Ctrl));
  L.slices = off;  // fixed place (see kSliceBytes)
  off = align256(off + kSliceBytes);
  L.active = off;
  off = align256(off + sizeof(ActiveEntry) * (size_t)L.max_active);
  L.pairs = off;
  off = align256(off + sizeof(Pair) * (size_t)L.max_pairs);
  L.counts = off;
  off = align256(off + sizeof(int) * (size_t)(n_experts + 1));
  L.hist = off;  // bucketing: per (expert, block) pair counts, then offsets
  off = align256(off + sizeof(int) * (size_t)kRouteBlocks * (size_t)n_experts);
  L.h = off;
  off = align256(off + sizeof(float) * (size_t)L.max_pairs * (size_t)max_ffn);
  L.xb = off;  // tensor-core path: the call's activations as bf16 [tokens][hidden]
  off = align256(off + 2 * (size_t)max_tokens * (size_t)hidden);
  // fused decode kernel: h per pair
  const int64_t ft = std::min<int64_t>(max_tokens, kFusedMaxPairs / (top_k > 0 ? top_k : 1));
  const int64_t fpairs = ft * top_k + ft;
  L.gu = off;
  off = align256(off + sizeof(float) * (size_t)fpairs * (size_t)max_ffn);
  L.total = off;
  return L;
}

// The shared expert of a layer call, checked on the host: a usable slot
// descriptor (expert_ok) whose width is at least the table's declared
// min_ffn; on the tiled path (min_ffn >= 256) a multiple of 256.
inline bool shared_ok(const redlite_moe_expert &e, const redlite_moe_table *t, bool tiled_path) {
  return expert_ok(e, t->hidden, t->max_ffn, tiled_path) && e.ffn >= t->min_ffn;
}

// ---------------------------------------------------------------- device helpers

__device__ __forceinline__ float fp16_bits_to_float(uint16_t h) { return __half2float(__ushort_as_half(h)); }

__device__ __forceinline__ uint16_t ld_u16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

// Eight weights of group G (weights 8G..8G+7 of the matrix's row-major
// sequence), exact in fp32, read from the resident layout of a rows x k
// matrix (tiled when tiled_shape(rows, k), else the interchange layout).
// grid: expanded int8 values of the format.
template <int QT>
__device__ __forceinline__ void decode_group_f32(const uint8_t *__restrict__ mat, int64_t k, bool tiled, int64_t G,
                                                 const int8_t *__restrict__ grid, float w[8]) {
  int idx, sc, nib = 0;
  unsigned s = 0;
  float d;
  if (tiled) {
    const int64_t n = 8 * G, r = n / k, kk = n % k;
    const int64_t kb = kk >> 8;
    const int g = (int)((kk & 255) >> 3), rr = (int)(r & 15);
    const uint8_t *tb = mat + tile_block_offset(QT, k, r, kb);
    if constexpr (QT == kQ2) {
      const Q2Loc o = q2_loc(rr, g);
      idx = tb[o.qs] | (((ld_u16(tb + o.qh_word) >> o.qh_bit) & 1) << 8);
      sc = (tb[o.scales + (g >> 3)] >> (4 * ((g >> 2) & 1))) & 15;
      const uint32_t sw = (uint32_t)tb[o.sign_word] | ((uint32_t)tb[o.sign_word + 1] << 8) |
                          ((uint32_t)tb[o.sign_word + 2] << 16) | ((uint32_t)tb[o.sign_word + 3] << 24);
#pragma unroll
      for (int j = 0; j < 8; ++j) s |= ((sw >> (4 * j + o.sign_shift)) & 1u) << j;
      d = fp16_bits_to_float(ld_u16(tb + o.d));
    } else {
      const Q1Loc o = q1_loc(rr, g);
      nib = (tb[o.nib_byte] >> o.nib_shift) & 15;
      idx = tb[o.qs] | ((nib & 7) << 8);
      const int bit = 3 * (g >> 1);
      const unsigned two = tb[o.scales + (bit >> 3)] | ((bit >> 3) < 5 ? (unsigned)tb[o.scales + (bit >> 3) + 1] << 8 : 0u);
      sc = (two >> (bit & 7)) & 7;
      d = fp16_bits_to_float(ld_u16(tb + o.d));
    }
  } else {
    const int64_t blk_i = G >> 5;
    const int g = (int)(G & 31);
    if constexpr (QT == kQ2) {
      const uint8_t *b = mat + blk_i * kQ2BlockBytes;
      d = fp16_bits_to_float(ld_u16(b));
      idx = b[6 + g] | (((b[38 + (g >> 3)] >> (g & 7)) & 1) << 8);
      sc = (b[2 + (g >> 3)] >> (4 * ((g >> 2) & 1))) & 15;
      s = b[42 + g];
    } else {
      const uint8_t *b = mat + blk_i * kQ1BlockBytes;
      d = fp16_bits_to_float(ld_u16(b));
      nib = (b[34 + (g >> 1)] >> (4 * (g & 1))) & 15;
      idx = b[2 + g] | ((nib & 7) << 8);
      const int bit = 3 * (g >> 1);
      // the 3-bit field may straddle two bytes of the 48-bit scales field
      const unsigned two = b[50 + (bit >> 3)] | ((bit >> 3) < 5 ? (unsigned)b[51 + (bit >> 3)] << 8 : 0u);
      sc = (two >> (bit & 7)) & 7;
    }
  }
  const int8_t *gv = grid + idx * 8;
  if constexpr (QT == kQ2) {
    const float scale = d * (float)(2 * sc + 1) * 0.125f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float v = scale * (float)gv[j];
      w[j] = ((s >> j) & 1) ? -v : v;
    }
  } else {
    const float scale = d * (float)(2 * sc + 1);
    const float delta = (nib & 8) ? -0.125f : 0.125f;
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = scale * ((float)gv[j] + delta);
  }
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }
// Same with the approximate divide (2 ulp; 0 once 1 + e^-g exceeds 2^126).
__device__ __forceinline__ float silu_mul_fast(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

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
  int shared_ffn, shared_qtype;
  bool tiled_path;  // the tensor-core kernels follow: slots must have the tiled layout
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
  int32_t *status;
};

constexpr int kRouteMaxExperts = 8192;
constexpr int kMaxTopK = 16;

cudaError_t launch_expand_grids(const uint16_t *comp2_dev, const uint16_t *comp1_dev, void *grids,
                                cudaStream_t stream);
cudaError_t launch_dequant(int qtype, const void *packed, int64_t rows, int64_t k, const void *grids, float *out_f32,
                           uint16_t *out_bf16, cudaStream_t stream);
cudaError_t launch_route(const RouteArgs &a, cudaStream_t stream);
cudaError_t launch_simt_tiles(const TileArgs &a, int max_active, cudaStream_t stream);
int pack_matrix_host(int qtype, int64_t rows, int64_t k, const uint8_t *src, uint8_t *dst);

struct FusedArgs {
  const float *x;
  const int32_t *ids;
  const float *weights;
  float *out;
  const float *residual;  // nullptr, or [n_tokens, hidden] added to out (out starts from it)
  int n_tokens, top_k, n_experts, hidden, max_ffn;
  const redlite_moe_expert *experts;
  redlite_moe_expert shared;
  int has_shared;
  const uint8_t *grids;
  uint8_t *ws;
  WorkspaceLayout L;
  int32_t *status;
  int wide;  // item shape: 0 one tile-block per warp and item, 1 two (fused_wide_items)
};
// Whether a fused call uses items of two tile-blocks per warp: hidden 2048,
// more than 32 (token, slot) pairs, one expert width, a multiple of 512
// (the kernel reports an expert of another width as BAD_EXPERT).
bool fused_wide_items(int hidden, int n_pairs, int min_ffn, int max_ffn, bool has_shared, int shared_ffn);
// Whether the fused decode kernel takes a call; sms: the device's SM count
// (0 if unknown: a B200's 148 is assumed).
bool fused_supported(int hidden, int max_ffn, int n_tokens, int top_k, int n_experts, bool has_shared, int sms);
int device_sms();

// Tensor-core (tcgen05) grouped path: tokens per work unit, and the launch.
constexpr int kTcTokens = 128;
bool tc_supported(int hidden, int max_ffn);
cudaError_t launch_tc(const TileArgs &a, cudaStream_t stream);
cudaError_t launch_fused(const FusedArgs &a, cudaStream_t stream);

// The layer with an optional residual: out = residual + layer(x) (out =
// layer(x) when residual is null).  Checks and path choice as
// redlite_moe_layer.
int layer_impl(const float *x, int32_t n_tokens, const int32_t *expert_ids, const float *router_weights, int32_t top_k,
               const redlite_moe_table *t, const redlite_moe_expert *shared, float *out, const float *residual);

}  // namespace redlite
