// decode_fused.cu -- one persistent kernel per decode-sized layer call.
//
// "Red Metal dev8 -- resident routed top-k layer", steps 4-6: every selected
// expert runs gate, up, SiLU(gate)*up and down from its resident slot and
// the layer accumulates out += router_weight * expert_output (plus the
// shared expert with weight 1, "Red Lite dev16", block composition).
//
// Structure (one CTA of 16 warps per SM, cooperative launch so all CTAs are
// resident):
//   prologue  every CTA copies the byte-permute selector tables into shared
//             memory and replicates them, buckets the (token, slot) pairs by
//             expert (identical in every CTA; one warp for calls of at most
//             32 pairs), reads the selected slots' descriptors, builds its
//             own item list and starts the first copies;
//   items     the work is a list of items of up to 16 warp units (a unit is
//             one tile-block, 16 rows x 256 inputs of a packed matrix, or
//             for large calls two adjacent ones) for a chunk of <= 2 tokens:
//             phase 1 items are gate and up tiles of the same rows (their
//             reduction yields h = SiLU(g) * u for those rows), phase 2
//             items are groups of down tiles (their reduction is added to
//             out with the router weight).  Gate/up items go to the CTAs in
//             contiguous ranges; down items in contiguous ranges, or, when
//             there are few, one or two consecutive ones to each CTA without
//             an extra gate/up item, or in time slots (see the item split);
//             warp w of a CTA handles unit w of each item;
//   streams   stage-major rings: a stage holds one item's units, filled by
//             one or two bulk copies (an item's tile-blocks are contiguous
//             in the resident layout); 4 stages, 2 for two-block units; the
//             last warp done with a stage refills it with the item a ring
//             ahead.  A warp converts its inputs to limbs when the item's
//             tokens or input block change, decodes its unit, writes its
//             partial sums to the item's reduction slot and moves on; the
//             item's reducer (warp item mod 16) adds the partials a few
//             items later;
//   slices    no grid barrier: the reducer of a gate/up item counts the
//             16-row tiles of h it wrote per (token chunk, 256-input slice)
//             with a release add; a warp about to decode a down tile-block
//             waits (acquire, bounded) until its slice of h is complete and
//             every CTA has initialised its part of out.  Down tiles stream
//             into the rings meanwhile.  Two counter sets alternate between
//             calls: a call zeroes the other set in its prologue, so the
//             call's end needs no reset pass.
//
// Arithmetic: weights are decoded to exact signed int8 values (IQ2: +-8,
// +-25, +-43; IQ1: 8*(grid + delta) in {+-1, +-7, +-9}) by two byte
// permutes per 8-weight group; activations are split into three signed
// 7-bit limbs of a 21-bit fixed-point value with a per-token power-of-two
// scale; the products run on the tensor cores (mma.sync s8, int32
// accumulation), the sub-block multiplier (2sc+1) is applied in int32 per
// sub-block and the block scale d in fp32 per 256 weights.  The only
// rounding is the activations' 2^-21 relative quantisation and fp32 sums.
#include <stdio.h>

#include "internal.cuh"

namespace redlite {

constexpr int kCWarps = 16;                // warps per CTA (all consume)
constexpr int kCThreads = 32 * kCWarps;    // 512
constexpr int kStageBytes = kQ2TileBlock;  // per tile-block slot of a stage: 1184 >= kQ1TileBlock
constexpr int kLimbPadW = 32;              // padding per limb plane (spreads shared-memory banks)
constexpr int kRedSlots = 6;               // reduction slots (items in flight)
constexpr int kRedLag = 2;                 // an item is reduced this many items after its own
constexpr int kMaxItems = 1536;            // items of one CTA (the host checks the bound)
constexpr int kRedFloats = 32;             // per warp and item: 16 rows x 2 token positions
constexpr int kTokChunk = 2;               // token positions per item

// Item shape.  W = 1: a warp decodes one tile-block per item (16 per item);
// W = 2 (calls with many items): two consecutive tile-blocks of the same 16
// rows (input blocks kb, kb + 1), accumulated together, so items, partial
// sums and reductions per tile-block halve.  W = 2 makes its room in shared
// memory with fewer selector-table replicas.
template <int W>
struct Shape {
  static constexpr int kRing = W == 1 ? 4 : 2;          // item stages in flight
  static constexpr int kStageTB = 16 * W;               // tile-block slots per stage
  static constexpr int kWPlane = 256 * W + kLimbPadW;  // bytes per limb plane of a warp's inputs
  static constexpr int kRep2 = W == 1 ? 16 : 8;         // replicas of the IQ2 selector table (bank spread)
  static constexpr int kRep1 = W == 1 ? 2 : 1;          // replicas of the IQ1 selector table
};
constexpr uint32_t kSpinLimit = 1u << 24;

// 8-byte tables the selector nibbles index: IQ2 +8,+25,+43,0,-8,-25,-43,0;
// IQ1 (delta +1/8) -7,1,9,0 and (delta -1/8) -9,-1,7,0, all scaled by 8.
constexpr uint32_t kQ2Pos = 0x002B1908u, kQ2Neg = 0x00D5E7F8u;
constexpr uint32_t kQ1Pos = 0x000901F9u, kQ1Neg = 0x0007FFF7u;

struct Inst {  // one selected expert (or the shared expert)
  const uint8_t *gate, *up, *down;
  int pair_start, count;
  int p1_base, p2_base;  // first work item of this instance in each phase
  int16_t qtype, ffn;
  int16_t ng1, ng2;  // items per token chunk in each phase
};
static_assert(sizeof(Inst) == 48, "instance records are 48 bytes");

// An item of a CTA's list, packed: instance (bits 0-9), token chunk (10-18),
// tile group (19-26), phase 2 (bit 27).
__device__ __forceinline__ uint32_t item_word(int inst, int chunk, int grp, int phase) {
  return (uint32_t)inst | ((uint32_t)chunk << 10) | ((uint32_t)grp << 19) | ((uint32_t)(phase - 1) << 27);
}
__device__ __forceinline__ int item_inst(uint32_t w) { return (int)(w & 1023u); }
__device__ __forceinline__ int item_chunk(uint32_t w) { return (int)((w >> 10) & 511u); }
__device__ __forceinline__ int item_grp(uint32_t w) { return (int)((w >> 19) & 255u); }
__device__ __forceinline__ int item_phase(uint32_t w) { return 1 + (int)(w >> 27); }
// tiles per phase-2 item for ffn / 256 = nkb (byte nkb - 1): 16 / nkb, at least 2
constexpr uint64_t kIt2Tab = 0x0202020304050810ull;
__device__ __forceinline__ int it2_of(int nkb) { return (int)((kIt2Tab >> (8 * (nkb - 1))) & 0xFFu); }

struct Smem {
  uint32_t *sel2, *sel1;
  uint32_t *items;  // [kMaxItems] this CTA's item list
  uint8_t *ring;   // [kRing][kStageTB][kStageBytes]: stage s holds item k = s mod kRing
  int *left;       // [kRing]: warps not yet done with the stage's item
  float *red;      // [kRedSlots][kCWarps][kRedFloats]
  uint8_t *wlimbs;  // [kCWarps][2 positions][3 limbs][kWPlane]: each warp's inputs
  Inst *inst;
  int *pair_tok;
  float *pair_w;
  uint64_t *full;    // [kRing]: stage landed
  uint64_t *rfull;   // [kRedSlots]: all warps' partials are in
  uint64_t *rfree;   // [kRedSlots]: the reducer is done with the slot
};

// Byte offsets of the shared-memory regions, each rounded up to 16 bytes
// (bulk-copy destinations need 16, mbarriers 8).
struct SmemPlan {
  size_t sel2, sel1, ring, red, wlimbs, inst, items, pair_tok, pair_w, full, left, rfull, rfree, total;
};
__host__ __device__ constexpr size_t r16(size_t v) { return (v + 15) & ~(size_t)15; }
template <int W>
__host__ __device__ constexpr SmemPlan smem_plan() {
  using Sh = Shape<W>;
  SmemPlan p{};
  size_t off = 0;
  p.sel2 = off, off = r16(off + 512 * Sh::kRep2 * 4);
  p.sel1 = off, off = r16(off + 4096 * Sh::kRep1 * 4);
  p.ring = off, off = r16(off + (size_t)Sh::kStageTB * Sh::kRing * kStageBytes);
  p.red = off, off = r16(off + sizeof(float) * kRedSlots * kCWarps * kRedFloats);
  p.wlimbs = off, off = r16(off + (size_t)kCWarps * kTokChunk * 3 * Sh::kWPlane);
  p.inst = off, off = r16(off + sizeof(Inst) * kFusedMaxInst);
  p.items = off, off = r16(off + sizeof(uint32_t) * kMaxItems);
  p.pair_tok = off, off = r16(off + sizeof(int) * (kFusedMaxPairs + 64));
  p.pair_w = off, off = r16(off + sizeof(float) * (kFusedMaxPairs + 64));
  p.full = off, off = r16(off + sizeof(uint64_t) * Sh::kRing);
  p.left = off, off = r16(off + sizeof(int) * Sh::kRing);
  p.rfull = off, off = r16(off + sizeof(uint64_t) * kRedSlots);
  p.rfree = off, off = r16(off + sizeof(uint64_t) * kRedSlots);
  p.total = off;
  return p;
}
template <int W>
constexpr bool plan_ok() {
  constexpr SmemPlan p = smem_plan<W>();
  return p.total + 64 <= 227 * 1024 && p.ring % 16 == 0 && p.full % 8 == 0 && p.rfull % 8 == 0 &&
         p.rfree % 8 == 0 && p.wlimbs % 16 == 0 && (kStageBytes % 16) == 0 && (kQ1TileBlock % 16) == 0;
}
static_assert(plan_ok<1>() && plan_ok<2>(), "shared memory size and alignment of the fused kernel");
// both shapes hold the same ring bytes (the bucketing scratch of large calls lives there)
static_assert(Shape<1>::kRing * Shape<1>::kStageTB == Shape<2>::kRing * Shape<2>::kStageTB, "ring bytes");

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory loads by 32-bit shared address.  The volatile forms read
// data that other threads or the bulk copies write (kept in program order);
// the plain form reads the selector tables, which nobody writes after setup.
__device__ __forceinline__ uint32_t lds_b32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds_table(uint32_t a) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds_b16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.b16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds_v2(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds_v4(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait on an mbarrier phase; false (and the TIMEOUT status bit) if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int32_t *status) {
  for (uint32_t it = 0; it < kSpinLimit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  atomicOr(status, REDLITE_STATUS_TIMEOUT);
  return false;
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ int ld_acquire(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

constexpr uint64_t kGridWaitNs = 1000000000ull;  // a grid-wide wait gives up after 1 s

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// counter += 1 with release semantics at GPU scope: every write that
// happens before it (this thread's, and through block barriers the block's)
// is visible to a thread that acquires the new value.
__device__ __forceinline__ void arrive_release(int *counter) {
  asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(counter) : "memory");
}

// Spin until *counter >= target; false (and the TIMEOUT status bit) if that
// takes longer than kGridWaitNs.  One thread per warp calls it; polls are
// spaced by a short sleep (many warps may wait on a few counters).
__device__ __noinline__ bool wait_count(const int *counter, int target, int32_t *status) {
  if (ld_acquire(counter) >= target) return true;
  const uint64_t t_end = global_ns() + kGridWaitNs;
  while (ld_acquire(counter) < target) {
    if (global_ns() > t_end) {
      atomicOr(status, REDLITE_STATUS_TIMEOUT);
      return false;
    }
    __nanosleep(64);
  }
  return true;  // the acquiring load orders what follows
}

// named barrier over all threads of the CTA (barrier 0 is __syncthreads)
__device__ __forceinline__ void all_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCThreads) : "memory"); }

__device__ __forceinline__ void mma_k32(int32_t d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

__device__ __forceinline__ void mma_k16(int32_t d[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%7,%7,%7,%7};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(b0), "r"(0));
}

__device__ __forceinline__ float half_bits(uint32_t h) { return __half2float(__ushort_as_half((unsigned short)h)); }

// Power-of-two exponent e with m < 2^e (m >= 0), clamped to [-106, 128] so
// that 2^(20-e) and 2^(e-20) are both normal floats.
__device__ __forceinline__ int pow2_above(float m) {
  const uint32_t E = __float_as_uint(m) >> 23;  // m >= 0: biased exponent
  int e = E ? (int)E - 126 : -126;
  return e < -106 ? -106 : e;
}
__device__ __forceinline__ float pow2f(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// limbs of one value scaled by 2^(20-e) (a power of two: exact)
__device__ __forceinline__ void to_limbs(float v, float scale, int &l0, int &l1, int &l2) {
  const int X = __float2int_rn(v * scale);
  l2 = ((X + 64) & 127) - 64;
  const int X1 = (X - l2) >> 7;
  l1 = ((X1 + 64) & 127) - 64;
  l0 = (X1 - l1) >> 7;
}

// Optional per-warp cycle counters and CTA timeline (build with
// -DREDLITE_TRACE): written to the 64 KB after the workspace layout's end.
#ifdef REDLITE_TRACE
#define TR_DECL long long tr_[10] = {0}; long long tr0_ = clock64()
#define TR(i) do { const long long t_ = clock64(); tr_[i] += t_ - tr0_; tr0_ = t_; } while (0)
#define TR_STAMP(i) do { if ((threadIdx.x & 31) == 0) { uint64_t g_; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(g_)); \
    reinterpret_cast<uint64_t *>(a.ws + a.L.total)[blockIdx.x * 32 + (i)] = g_; } } while (0)
#define TR_FLUSH() do { if (lane == 0) for (int i_ = 0; i_ < 10; ++i_) \
    reinterpret_cast<uint64_t *>(a.ws + a.L.total)[8192 + (blockIdx.x * 16 + warp) * 10 + i_] = tr_[i_]; } while (0)
#else
#define TR_DECL
#define TR(i)
#define TR_STAMP(i)
#define TR_FLUSH()
#endif

// ------------------------------------------------------------------ tile-block math
//
// Column n of the mma B operand (n = lane >> 2 of the lane holding it) is
// limb n % 3 of token position n / 3 of the item (n < 6); columns 6 and 7
// are zero.  bp: shared address of the limb plane the lane reads, at the
// tile-block's first input; bv: whether its column is used.
//
// IQ2_XS-style tile-block (16 rows x 256 inputs): acc[.] += partial dot
// products of the block's rows (mma C layout, limb columns).  Lane (q, t)
// decodes groups 4c + t of rows q and q+8 (fields i = 2c + h).  Per 8-weight
// group: the 9-bit index (one byte extract, one bit), one table load for
// the symbols' selector, the signs moved into bit 2 of each selector nibble
// by one shift and one mask of the group's sign word, two byte permutes.
template <int R2>
__device__ __forceinline__ void tb_q2(uint32_t tb, uint32_t g2, uint32_t bp, bool bv, float acc[4]) {
  static_assert(R2 == 16 || R2 == 8, "IQ2 table replicas");
  constexpr int kSh = R2 == 16 ? 14 : 13;  // byte offset of index bit 8: 256 entries x 4 R2 bytes
  const int lane = threadIdx.x & 31, q = lane >> 2, t = lane & 3;
  const uint32_t r4 = (uint32_t)(lane & (R2 - 1)) << 2;
  const uint4 qs = lds_v4(tb + 32 * lane);
  const uint4 sg = lds_v4(tb + 32 * lane + 16);
  const uint32_t qhs = lds_b16(tb + 1024 + 2 * lane) << kSh;
  const uint2 scw = lds_v2(tb + 1088 + 8 * q);
  const uint32_t dw = lds_b32(tb + 1152 + 4 * q);
  uint2 b[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) b[c] = bv ? lds_v2(bp + 32 * c + 8 * t) : make_uint2(0u, 0u);
  const uint32_t qsw[4] = {qs.x, qs.y, qs.z, qs.w};
  const uint32_t sgw[4] = {sg.x, sg.y, sg.z, sg.w};
  uint32_t sel[16];  // field i = 2c + h
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t qsb = __byte_perm(qsw[i >> 2], 0u, 0x4440u | (uint32_t)(i & 3));
    const uint32_t go = qsb * (4u * R2) + (((qhs >> i) & (1u << kSh)) | r4);  // index bit 8; R2 replicas
    const int m = i & 3;  // sign word i >> 2 holds this field's sign bit j at bit 4j + m
    const uint32_t sgn = (m <= 2 ? (sgw[i >> 2] << (2 - m)) : (sgw[i >> 2] >> 1)) & 0x44444444u;
    sel[i] = lds_table(g2 + go) | sgn;
  }
  // sub-block multipliers 2sc+1 as bytes: chunk c is byte c >> 1 of the even
  // (c even) or odd (c odd) nibble word of its row
  const uint32_t me0 = ((scw.x & 0x0F0F0F0Fu) << 1) | 0x01010101u, mo0 = ((scw.x >> 3) & 0x1E1E1E1Eu) | 0x01010101u;
  const uint32_t me1 = ((scw.y & 0x0F0F0F0Fu) << 1) | 0x01010101u, mo1 = ((scw.y >> 3) & 0x1E1E1E1Eu) | 0x01010101u;
  int32_t cb[4] = {0, 0, 0, 0};
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t a[4];
    a[0] = __byte_perm(kQ2Pos, kQ2Neg, sel[2 * c]);
    a[2] = __byte_perm(kQ2Pos, kQ2Neg, sel[2 * c] >> 16);
    a[1] = __byte_perm(kQ2Pos, kQ2Neg, sel[2 * c + 1]);
    a[3] = __byte_perm(kQ2Pos, kQ2Neg, sel[2 * c + 1] >> 16);
    const int m0 = (int)__byte_perm((c & 1) ? mo0 : me0, 0u, 0x4440u | (uint32_t)(c >> 1));
    const int m1 = (int)__byte_perm((c & 1) ? mo1 : me1, 0u, 0x4440u | (uint32_t)(c >> 1));
    int32_t d[4];
    mma_k32(d, a, b[c].x, b[c].y);
    cb[0] += m0 * d[0];
    cb[1] += m0 * d[1];
    cb[2] += m1 * d[2];
    cb[3] += m1 * d[3];
  }
  const float d0 = half_bits(dw & 0xFFFFu) * 0.125f, d1 = half_bits(dw >> 16) * 0.125f;
  acc[0] += d0 * (float)cb[0];
  acc[1] += d0 * (float)cb[1];
  acc[2] += d1 * (float)cb[2];
  acc[3] += d1 * (float)cb[3];
}

// IQ1_M-style tile-block: one k16 mma per 16-weight sub-block; lane t holds
// weights 4t..4t+3 of the sub-block (half of group 2s + (t >> 1)).
template <int R1>
__device__ __forceinline__ void tb_q1(uint32_t tb, uint32_t sel1, uint32_t bp, bool bv, float acc[4]) {
  const int lane = threadIdx.x & 31, q = lane >> 2, t = lane & 3, r = lane & (R1 - 1);
  const uint32_t pb = tb + 48 * (2 * q + (t >> 1));
  const uint4 qa = lds_v4(pb);
  const uint4 qb = lds_v4(pb + 16);
  const uint4 nb = lds_v4(pb + 32);
  const uint32_t s0 = lds_b32(tb + 768 + 12 * q), s1 = lds_b32(tb + 772 + 12 * q), s2 = lds_b32(tb + 776 + 12 * q);
  const uint64_t row0 = (uint64_t)s0 | ((uint64_t)(s1 & 0xFFFFu) << 32);
  const uint64_t row1 = (uint64_t)(s1 >> 16) | ((uint64_t)s2 << 16);
  const uint32_t dw = lds_b32(tb + 864 + 4 * q);
  uint32_t b[16];
#pragma unroll
  for (int s = 0; s < 16; ++s) b[s] = bv ? lds_b32(bp + 16 * s + 4 * t) : 0u;
  const int hshift = 16 * (t & 1);
  const uint32_t qsw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
  const uint32_t nbw[4] = {nb.x, nb.y, nb.z, nb.w};
  int32_t cb[4] = {0, 0, 0, 0};
#pragma unroll
  for (int s = 0; s < 16; ++s) {
    uint32_t sel[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = 2 * s + h;  // entry i = 2s + h
      const uint32_t qsb = (qsw[i >> 2] >> (8 * (i & 3))) & 0xFFu;
      const uint32_t nib = (nbw[i >> 3] >> (4 * (i & 7))) & 0xFu;
      sel[h] = lds_table(sel1 + 4 * ((qsb | (nib << 8)) * R1 + r)) >> hshift;
    }
    const uint32_t a0 = __byte_perm(kQ1Pos, kQ1Neg, sel[0]);
    const uint32_t a1 = __byte_perm(kQ1Pos, kQ1Neg, sel[1]);
    const int m0 = 2 * (int)((row0 >> (3 * s)) & 7u) + 1;
    const int m1 = 2 * (int)((row1 >> (3 * s)) & 7u) + 1;
    int32_t d[4];
    mma_k16(d, a0, a1, b[s]);
    cb[0] += m0 * d[0];
    cb[1] += m0 * d[1];
    cb[2] += m1 * d[2];
    cb[3] += m1 * d[3];
  }
  const float d0 = half_bits(dw & 0xFFFFu) * 0.125f, d1 = half_bits(dw >> 16) * 0.125f;
  acc[0] += d0 * (float)cb[0];
  acc[1] += d0 * (float)cb[1];
  acc[2] += d1 * (float)cb[2];
  acc[3] += d1 * (float)cb[3];
}

// Combine the limb columns of each token position: v = (row q, pos 0),
// (row q, pos 1), (row q+8, pos 0), (row q+8, pos 1), complete in lanes
// with t = lane & 3 = 0.
__device__ __forceinline__ void quad_rows(const float acc[4], float v[4]) {
  const int t = threadIdx.x & 3;
  const int n0 = 2 * t, n1 = 2 * t + 1;
  const float f0 = n0 < 6 ? (n0 % 3 == 0 ? 16384.f : (n0 % 3 == 1 ? 128.f : 1.f)) : 0.f;
  const float f1 = n1 < 6 ? (n1 % 3 == 0 ? 16384.f : (n1 % 3 == 1 ? 128.f : 1.f)) : 0.f;
  const int m0 = n0 / 3, m1 = n1 / 3;  // token position of the column (2 = none)
  v[0] = (m0 == 0 ? f0 * acc[0] : 0.f) + (m1 == 0 ? f1 * acc[1] : 0.f);
  v[1] = (m0 == 1 ? f0 * acc[0] : 0.f) + (m1 == 1 ? f1 * acc[1] : 0.f);
  v[2] = (m0 == 0 ? f0 * acc[2] : 0.f) + (m1 == 0 ? f1 * acc[3] : 0.f);
  v[3] = (m0 == 1 ? f0 * acc[2] : 0.f) + (m1 == 1 ? f1 * acc[3] : 0.f);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    v[j] += __shfl_xor_sync(0xffffffffu, v[j], 1);
    v[j] += __shfl_xor_sync(0xffffffffu, v[j], 2);
  }
}

// Store this warp's partial sums, scaled by the positions' limb scales sc0,
// sc1, to red[2 * row + position] (16 rows x 2 positions).
__device__ __forceinline__ void store_partials(const float acc[4], float sc0, float sc1, float *red) {
  const int lane = threadIdx.x & 31, q = lane >> 2, t = lane & 3;
  float v[4];
  quad_rows(acc, v);
  if (t == 0) {
    *reinterpret_cast<float2 *>(red + 2 * q) = make_float2(v[0] * sc0, v[1] * sc1);
    *reinterpret_cast<float2 *>(red + 2 * (q + 8)) = make_float2(v[2] * sc0, v[3] * sc1);
  }
}

// Limbs of the 256 W consecutive floats src[0 .. 256 W - 1] (the inputs of
// one token position that a warp's tile-blocks read): three planes of
// 256 W signed 7-bit limbs at dst, dst + kWPlane, dst + 2 kWPlane, with one
// scale for all of them.  Returns the scale 2^(e - 20), 2^e > max |src[i]|.
// Lane l converts inputs 8 W l .. 8 W l + 8 W - 1.  coherent: read through
// L2 only (data other CTAs wrote during this kernel).  Out of line: it runs
// once per token chunk.
template <int W>
__device__ __noinline__ float warp_slice_limbs(const float *src, bool coherent, uint8_t *dst) {
  constexpr int NV = 8 * W, kWPlane = Shape<W>::kWPlane;
  const int lane = threadIdx.x & 31;
  const float4 *s4 = reinterpret_cast<const float4 *>(src) + (NV / 4) * lane;
  float f[NV];
#pragma unroll
  for (int j = 0; j < NV / 4; ++j) {
    const float4 v = coherent ? __ldcg(s4 + j) : __ldg(s4 + j);
    f[4 * j] = v.x, f[4 * j + 1] = v.y, f[4 * j + 2] = v.z, f[4 * j + 3] = v.w;
  }
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) m = fmaxf(m, fabsf(f[i]));
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const int e = pow2_above(m);
  const float sc = pow2f(20 - e);
  uint32_t p[3][NV / 4];
#pragma unroll
  for (int l = 0; l < 3; ++l)
#pragma unroll
    for (int j = 0; j < NV / 4; ++j) p[l][j] = 0u;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    int l0, l1, l2;
    to_limbs(f[i], sc, l0, l1, l2);
    p[0][i >> 2] |= (uint32_t)(l0 & 0xFF) << (8 * (i & 3));
    p[1][i >> 2] |= (uint32_t)(l1 & 0xFF) << (8 * (i & 3));
    p[2][i >> 2] |= (uint32_t)(l2 & 0xFF) << (8 * (i & 3));
  }
#pragma unroll
  for (int l = 0; l < 3; ++l) {
    if constexpr (W == 1)
      *reinterpret_cast<uint2 *>(dst + l * kWPlane + 8 * lane) = make_uint2(p[l][0], p[l][1]);
    else
      *reinterpret_cast<uint4 *>(dst + l * kWPlane + 16 * lane) = make_uint4(p[l][0], p[l][1], p[l][2], p[l][3]);
  }
  __syncwarp();
  return pow2f(e - 20);
}

// Replicate the selector tables in place (word w of a table with r replicas
// holds source word w / r; replicas spread lanes over banks): warps 1..15
// (t = 0..479), named barrier 2.  Every source word is read before any is
// overwritten.  Out of line: it runs once per call.
template <int R2, int R1>
__device__ __noinline__ void replicate_tables(uint32_t *sel2, uint32_t *sel1, int t) {
  constexpr int NT = 480, BAR = 2;
  static_assert((R2 == 16 || R2 == 8) && (R1 == 2 || R1 == 1), "replication below assumes 16 or 8 / 2 or 1 replicas");
  constexpr int N2 = (512 + NT - 1) / NT, N1 = R1 == 2 ? (4096 + NT - 1) / NT : 0;
  uint32_t v2[N2], v1[N1 > 0 ? N1 : 1];
#pragma unroll
  for (int i = 0; i < N2; ++i) v2[i] = t + NT * i < 512 ? sel2[t + NT * i] : 0u;
#pragma unroll
  for (int i = 0; i < N1; ++i) v1[i] = t + NT * i < 4096 ? sel1[t + NT * i] : 0u;
  asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
  constexpr int Q = R2 / 4;  // 16-byte stores per entry
  const int rot = (t & 31) / (8 / Q > 0 ? 8 / Q : 1);  // lanes of one store wavefront cover distinct banks
#pragma unroll
  for (int r = 0; r < Q; ++r) {
    const int q = (r + rot) % Q;
#pragma unroll
    for (int i = 0; i < N2; ++i)
      if (t + NT * i < 512)
        reinterpret_cast<uint4 *>(sel2)[(t + NT * i) * Q + q] = make_uint4(v2[i], v2[i], v2[i], v2[i]);
  }
  if constexpr (R1 == 2) {
#pragma unroll
    for (int i = 0; i < N1; ++i)
      if (t + NT * i < 4096) reinterpret_cast<uint2 *>(sel1)[t + NT * i] = make_uint2(v1[i], v1[i]);
  }
  asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
}

// ------------------------------------------------------------------ the kernel

template <int W>
__global__ void __launch_bounds__(kCThreads, 1) decode_fused_kernel(FusedArgs a) {
  using Sh = Shape<W>;
  constexpr int kRing = Sh::kRing, kWPlane = Sh::kWPlane;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int H = a.hidden, T = a.n_tokens, K = a.top_k, E = a.n_experts;
  const int nkbH = H >> 8;
  // gate (and up) tiles per phase-1 item (W = 2 needs hidden 2048: two tiles
  // of 8 input blocks, each warp two blocks of one tile)
  const int it1 = W * max(1, 8 / nkbH);
  const int npairs = T * K;
  Ctrl *ctrl = reinterpret_cast<Ctrl *>(a.ws + a.L.ctrl);
  float *hbuf = reinterpret_cast<float *>(a.ws + a.L.gu);  // h per pair: [pairs][max_ffn]

  // ---- shared memory carve
  constexpr SmemPlan P = smem_plan<W>();
  Smem S;
  S.sel2 = reinterpret_cast<uint32_t *>(smem + P.sel2);
  S.sel1 = reinterpret_cast<uint32_t *>(smem + P.sel1);
  S.ring = smem + P.ring;
  S.red = reinterpret_cast<float *>(smem + P.red);
  S.wlimbs = smem + P.wlimbs;
  S.inst = reinterpret_cast<Inst *>(smem + P.inst);
  S.items = reinterpret_cast<uint32_t *>(smem + P.items);
  S.pair_tok = reinterpret_cast<int *>(smem + P.pair_tok);
  S.pair_w = reinterpret_cast<float *>(smem + P.pair_w);
  S.full = reinterpret_cast<uint64_t *>(smem + P.full);
  S.left = reinterpret_cast<int *>(smem + P.left);
  S.rfull = reinterpret_cast<uint64_t *>(smem + P.rfull);
  S.rfree = reinterpret_cast<uint64_t *>(smem + P.rfree);
  __shared__ int s_n_inst, s_n1, s_n2, s_bad, s_par, s_scan[33];
  __shared__ uint64_t s_lut_bar;
  TR_STAMP(0);
  // the next layer call may start its own table setup on SMs this grid frees
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- prologue part 1: barriers, then every independent global load.
  // One thread starts bulk copies of the two selector tables (unreplicated)
  // into the first bytes of their shared-memory regions; they are replicated
  // after the routing has been read.
  if (tid < kRing) {
    mbar_init(&S.full[tid], 1);
    S.left[tid] = kCWarps;
  }
  if (tid < kRedSlots) {
    mbar_init(&S.rfull[tid], kCWarps);
    mbar_init(&S.rfree[tid], 1);
  }
  if (tid == kCThreads - 1) {
    mbar_init(&s_lut_bar, 1);
    mbar_fence_init();
    s_bad = 0;
    // the expanded grids are set up once, before any layer call: they may be
    // read before the previous kernel of the stream has finished
    mbar_expect_tx(&s_lut_bar, (512 + 4096) * 4);
    bulk_g2s(S.sel2, a.grids + kGridQ2Sel, 512 * 4, &s_lut_bar);
    bulk_g2s(S.sel1, a.grids + kGridQ1Sel, 4096 * 4, &s_lut_bar);
  }
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  // Warm L2 with the call's small inputs and the whole slot table while the
  // previous kernel of the stream finishes: a prefetch reads nothing into
  // registers, and L2 stays coherent with writes that land after it.  One
  // 128-byte line per thread of the grid.
  {
    const unsigned g = (unsigned)cta * kCThreads + tid;
    const unsigned l_tab = (unsigned)(E * (int)sizeof(redlite_moe_expert) + 127) / 128u;
    const unsigned l_ids = (unsigned)(npairs * 4 + 127) / 128u;
    const unsigned l_x = (unsigned)(T * H * 4 + 127) / 128u;
    const char *p = nullptr;
    if (g < l_tab)
      p = reinterpret_cast<const char *>(a.experts) + 128 * g;
    else if (g < l_tab + l_ids)
      p = reinterpret_cast<const char *>(a.ids) + 128 * (g - l_tab);
    else if (g < l_tab + 2 * l_ids)
      p = reinterpret_cast<const char *>(a.weights) + 128 * (g - l_tab - l_ids);
    else if (g < l_tab + 2 * l_ids + l_x)
      p = reinterpret_cast<const char *>(a.x) + 128 * (g - l_tab - 2 * l_ids);
    else if (a.residual && g < l_tab + 2 * l_ids + 2 * l_x)
      p = reinterpret_cast<const char *>(a.residual) + 128 * (g - l_tab - 2 * l_ids - l_x);
    if (p) asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
  }
  __syncthreads();  // the mbarriers are initialised before anyone waits on them
  // the call's own inputs may come from the previous kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  TR_STAMP(7);

  int my_ids[2];
  float my_w[2];
  uint4 my_d[2][2];  // slot-table entry of each of this thread's pairs
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int p = tid + kCThreads * j;
    my_ids[j] = p < npairs ? __ldcg(a.ids + p) : -1;
    my_w[j] = p < npairs ? __ldcg(a.weights + p) : 0.f;
  }
  TR_STAMP(8);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int e = my_ids[j];
    if (e >= 0 && e < E) {
      const uint4 *d = reinterpret_cast<const uint4 *>(a.experts + e);
      my_d[j][0] = __ldg(d);
      my_d[j][1] = __ldg(d + 1);
    }
  }

  // work items per instance and their prefix sums (warp 0; n_inst is small)
  auto item_prefix = [&](int n_inst) {
    int base1 = 0, base2 = 0;
    for (int u0 = 0; u0 < n_inst; u0 += 32) {
      const int u = u0 + lane;
      int c1 = 0, c2 = 0;
      if (u < n_inst) {
        Inst &I = S.inst[u];
        const int nch = (I.count + kTokChunk - 1) / kTokChunk;
        const int it2 = W == 1 ? it2_of(I.ffn >> 8) : 32 / (I.ffn >> 8);  // down tiles per item
        const int ng1 = (I.ffn / 16 + it1 - 1) / it1, ng2 = (H / 16 + it2 - 1) / it2;
        I.ng1 = (int16_t)ng1, I.ng2 = (int16_t)ng2;
        c1 = nch * ng1;
        c2 = nch * ng2;
      }
      int i1 = c1, i2 = c2;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y1 = __shfl_up_sync(0xffffffffu, i1, o), y2 = __shfl_up_sync(0xffffffffu, i2, o);
        if (lane >= o) i1 += y1, i2 += y2;
      }
      if (u < n_inst) S.inst[u].p1_base = base1 + i1 - c1, S.inst[u].p2_base = base2 + i2 - c2;
      base1 += __shfl_sync(0xffffffffu, i1, 31);
      base2 += __shfl_sync(0xffffffffu, i2, 31);
    }
    if (lane == 0) {
      s_n_inst = n_inst, s_n1 = base1, s_n2 = base2;
      if (s_bad) atomicOr(a.status, s_bad);
    }
  };
  auto set_inst = [&](Inst &I, const redlite_moe_expert &d, int count, int pair_start, int &bad) {
    // (the W = 2 item shape pairs down input blocks: widths a multiple of 512)
    if (expert_ok(d, H, a.max_ffn, true) && (W == 1 || d.ffn % 512 == 0)) {
      I.gate = (const uint8_t *)d.gate, I.up = (const uint8_t *)d.up, I.down = (const uint8_t *)d.down;
      I.qtype = (int16_t)d.qtype, I.ffn = (int16_t)d.ffn, I.count = count;
    } else {
      bad |= REDLITE_STATUS_BAD_EXPERT;
      I.gate = I.up = I.down = nullptr;
      I.qtype = kQ2, I.ffn = 256, I.count = 0;
    }
    I.pair_start = pair_start;
  };
  if (npairs <= 32) {
    // ---- small call: warp 0 routes alone (lane p holds pair p)
    if (warp == 0) {
      const bool inrange = lane < npairs;
      const int e = inrange ? my_ids[0] : -1;
      const bool ok = e >= 0 && e < E;
      int bad = (inrange && !ok) ? REDLITE_STATUS_BAD_ID : 0;
      const unsigned lt = (1u << lane) - 1u;
      int n_inst, n_routed_pairs;
      redlite_moe_expert d;
      memcpy(reinterpret_cast<uint8_t *>(&d), &my_d[0][0], 16);
      memcpy(reinterpret_cast<uint8_t *>(&d) + 16, &my_d[0][1], 16);
      if (T == 1) {
        // one token: every valid pair is its own instance, in pair order (a
        // repeated id runs twice, each time with its own weight)
        const unsigned okm = __ballot_sync(0xffffffffu, ok);
        const int rank = __popc(okm & lt);
        if (ok) {
          S.pair_tok[rank] = 0;
          S.pair_w[rank] = my_w[0];
          set_inst(S.inst[rank], d, 1, rank, bad);
        }
        n_inst = n_routed_pairs = __popc(okm);
      } else {
        const int key = ok ? e : 0x7fffffff;
        int rank = 0;        // position of this pair in (expert, pair index) order
        unsigned less = 0u;  // lanes whose expert id is smaller
#pragma unroll 4
        for (int q = 0; q < 32; ++q) {
          const int kq = __shfl_sync(0xffffffffu, key, q);
          rank += (kq < key) || (kq == key && q < lane);
          less |= (unsigned)(kq < key) << q;
        }
        const unsigned same = __match_any_sync(0xffffffffu, key);
        const bool leader = ok && (same & lt) == 0;
        const unsigned leaders = __ballot_sync(0xffffffffu, leader);
        if (ok) {
          S.pair_tok[rank] = lane / K;
          S.pair_w[rank] = my_w[0];
        }
        if (leader) set_inst(S.inst[__popc(leaders & less)], d, __popc(same), rank, bad);
        n_inst = __popc(leaders);
        n_routed_pairs = __popc(__ballot_sync(0xffffffffu, ok));
      }
      TR_STAMP(17);
      if (a.has_shared) {
        if (lane == 0) set_inst(S.inst[n_inst], a.shared, T, n_routed_pairs, bad);
        if (lane < T) S.pair_tok[n_routed_pairs + lane] = lane, S.pair_w[n_routed_pairs + lane] = 1.f;
        n_inst += 1;
      }
      bad = __reduce_or_sync(0xffffffffu, bad);
      if (lane == 0) s_bad = bad;
      __syncwarp();
      TR_STAMP(18);
      item_prefix(n_inst);
      TR_STAMP(9);
    } else {
      // meanwhile the other warps replicate the selector tables
      mbar_wait(&s_lut_bar, 0, a.status);
      if (warp == 1) TR_STAMP(10);
      replicate_tables<Sh::kRep2, Sh::kRep1>(S.sel2, S.sel1, tid - 32);
      if (warp == 1) TR_STAMP(11);
    }
  } else {
    // ---- bucketing: counts per expert in the rings (scratch before any copy)
    uint4 *desc_s = reinterpret_cast<uint4 *>(S.ring);        // [npairs][2]: slot-table entries
    int *cnt = reinterpret_cast<int *>(desc_s + 2 * npairs);  // [E]
    int *first = cnt + E;                                     // [E]: lowest pair index
    int *ids_s = first + E;                                   // [npairs]
    float *w_s = reinterpret_cast<float *>(ids_s + npairs);
    for (int e = tid; e < E; e += kCThreads) cnt[e] = 0, first[e] = 0x7fffffff;
    __syncthreads();
    int bad = 0;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int p = tid + kCThreads * j;
      if (p >= npairs) continue;
      const int e = my_ids[j];
      ids_s[p] = e;
      w_s[p] = my_w[j];
      if (e < 0 || e >= E) {
        bad |= REDLITE_STATUS_BAD_ID;
        continue;
      }
      desc_s[2 * p] = my_d[j][0];
      desc_s[2 * p + 1] = my_d[j][1];
      atomicAdd(&cnt[e], 1);
      atomicMin(&first[e], p);
    }
    __syncthreads();
    // active experts in ascending id: exclusive scans of (count > 0) and counts
    int n_routed_pairs = 0;
    {
      const int per = (E + kCThreads - 1) / kCThreads;
      const int e0 = tid * per, e1 = min(E, e0 + per);
      int my_act = 0, my_pairs = 0;
      for (int e = e0; e < e1; ++e) {
        my_act += cnt[e] > 0;
        my_pairs += cnt[e];
      }
      int incl_a = my_act, incl_p = my_pairs;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, incl_a, o), yp = __shfl_up_sync(0xffffffffu, incl_p, o);
        if (lane >= o) incl_a += ya, incl_p += yp;
      }
      if (lane == 31) s_scan[warp] = incl_a, s_scan[16 + warp] = incl_p;
      __syncthreads();
      if (tid == 0) {
        int sa = 0, sp = 0;
        for (int w = 0; w < kCWarps; ++w) {
          const int ta = s_scan[w], tp = s_scan[16 + w];
          s_scan[w] = sa, s_scan[16 + w] = sp;
          sa += ta, sp += tp;
        }
        s_n_inst = sa;
        s_scan[32] = sp;
      }
      __syncthreads();
      int act = s_scan[warp] + incl_a - my_act, pst = s_scan[16 + warp] + incl_p - my_pairs;
      for (int e = e0; e < e1; ++e) {
        if (cnt[e] > 0) {
          redlite_moe_expert d;
          static_assert(sizeof(redlite_moe_expert) == 32, "slot-table entries are two 16-byte words");
          const uint4 d0 = desc_s[2 * first[e]], d1 = desc_s[2 * first[e] + 1];
          memcpy(reinterpret_cast<uint8_t *>(&d), &d0, 16);
          memcpy(reinterpret_cast<uint8_t *>(&d) + 16, &d1, 16);
          const int c = cnt[e];
          set_inst(S.inst[act], d, c, pst, bad);
          cnt[e] = pst;  // becomes the running cursor of the stable fill
          ++act;
          pst += c;
        }
      }
      __syncthreads();
      n_routed_pairs = s_scan[32];
    }
    int n_inst = s_n_inst;
    if (warp == kCWarps - 1) {
      // stable fill of the pair list (one warp, pairs in index order)
      for (int p0 = 0; p0 < npairs; p0 += 32) {
        const int p = p0 + lane;
        const int e = p < npairs ? ids_s[p] : -1;
        const bool ok = e >= 0 && e < E;
        const unsigned m = __match_any_sync(0xffffffffu, ok ? e : -1);
        if (ok) {
          const int rank = __popc(m & ((1u << lane) - 1u));
          const int pos = cnt[e] + rank;
          S.pair_tok[pos] = p / K;
          S.pair_w[pos] = w_s[p];
        }
        __syncwarp();
        if (ok && (m & ((1u << lane) - 1u)) == 0) cnt[e] += __popc(m);
        __syncwarp();
      }
    } else if (a.has_shared) {
      if (tid == 0) set_inst(S.inst[n_inst], a.shared, T, n_routed_pairs, bad);
      for (int t = tid; t < T; t += kCThreads - 32) S.pair_tok[n_routed_pairs + t] = t, S.pair_w[n_routed_pairs + t] = 1.f;
    }
    if (a.has_shared) n_inst += 1;
    if (bad) atomicOr(&s_bad, bad);
    __syncthreads();
    if (warp == 0) item_prefix(n_inst);
    // replicate the selector tables (the bucketing scratch in the rings is
    // not touched)
    if (warp > 0) {
      mbar_wait(&s_lut_bar, 0, a.status);
      replicate_tables<Sh::kRep2, Sh::kRep1>(S.sel2, S.sel1, tid - 32);
    }
  }
  TR_STAMP(16);

  // ---- the item split.  Gate/up items in contiguous ranges of N1 / G, the
  // first N1 mod G CTAs taking one more (so the h slices that complete last
  // are those of the first few experts).  Down items: many per CTA in
  // contiguous ranges; few (at most two per CTA without an extra gate/up
  // item) in ranges of one or two on those CTAs only; otherwise in time
  // slots: first one each for the CTAs without an extra gate/up item, then
  // one per CTA per round, in reverse item order, so the down items that need
  // the late slices come last.  (The host keeps every CTA's list within
  // kMaxItems; the clamps only guard the shared-memory list.)
  struct Split {
    int b1, my1, e1, first2, my2, b2;  // b2 >= 0: down items in one contiguous range
  };
  auto split = [&]() -> Split {
    Split p;
    const int N1 = s_n1, N2 = s_n2;
    const int r1 = N1 / G;
    p.e1 = N1 - r1 * G;
    p.b1 = cta < p.e1 ? (r1 + 1) * cta : (r1 + 1) * p.e1 + r1 * (cta - p.e1);
    p.my1 = min(r1 + (cta < p.e1), kMaxItems - 1);
    if (N2 >= 4 * G) {
      // many down items per CTA: contiguous ranges (consecutive items share
      // an expert's h slices and weights), in reverse CTA order
      const unsigned uG = (unsigned)G, uN2 = (unsigned)N2, rc = (unsigned)(G - 1 - cta);
      p.b2 = (int)(rc * uN2 / uG);
      p.my2 = (int)((rc + 1) * uN2 / uG) - p.b2;
      p.first2 = -1;
    } else if (N2 <= 2 * (G - p.e1)) {
      // few down items: only the CTAs without an extra gate/up item take
      // them, in contiguous ranges of one or two (two consecutive items of an
      // expert share its h slices and the warps' limbs), the single ones
      // first: the lowest items, whose h comes from the extra gate/up items
      // and so completes last, go to CTAs that have one down item
      const int nA = G - p.e1, q = N2 / nA, n_lo = nA - (N2 - q * nA), ia = cta - p.e1;
      p.b2 = ia < 0 ? 0 : ia < n_lo ? ia * q : n_lo * q + (ia - n_lo) * (q + 1);
      p.my2 = ia < 0 ? 0 : q + (ia >= n_lo);
      p.first2 = -1;
    } else {
      p.b2 = -1;
      p.first2 = (cta >= p.e1 && cta - p.e1 < N2) ? cta - p.e1 : -1;
      const int base = G - p.e1 + cta;  // this CTA's first round-robin slot
      p.my2 = (p.first2 >= 0) + (base < N2 ? (N2 - base + G - 1) / G : 0);
    }
    p.my2 = min(p.my2, kMaxItems - p.my1);
    return p;
  };
  // the global index of list entry k (gate/up entries first)
  auto item_index = [&](const Split &p, int k, int &phase) -> int {
    if (k < p.my1) {
      phase = 1;
      return p.b1 + k;
    }
    phase = 2;
    if (p.b2 >= 0) return p.b2 + (k - p.my1);
    int k2 = k - p.my1, slot;
    if (p.first2 >= 0 && k2 == 0) {
      slot = p.first2;
    } else {
      if (p.first2 >= 0) --k2;
      slot = G - p.e1 + cta + k2 * G;
    }
    return s_n2 - 1 - slot;
  };
  // warp wi's place in an item, packed: phase 1 (bits 0-3 tile offset,
  // 4-6 input block, 7 has a tile-block, 8 matrix: gate 0 / up 1); phase 2
  // items of an expert with ffn / 256 = nkb: byte nkb - 1 of p2 = tile
  // offset (bits 0-3), input block (4-6), has a tile-block (7)
  auto warp_place = [&](int wi, uint32_t &p1, uint64_t &p2) {
    const int r = wi & 7;
    p1 = (uint32_t)(r / nkbH) | ((uint32_t)(r % nkbH) << 4) | (r < it1 * nkbH ? 128u : 0u) | ((uint32_t)(wi >> 3) << 8);
    p2 = 0;
#pragma unroll
    for (int nkb = 1; nkb <= 8; ++nkb) {
      const uint64_t okb = wi < it2_of(nkb) * nkb ? 128u : 0u;
      p2 |= ((uint64_t)(wi / nkb) | ((uint64_t)(wi % nkb) << 4) | okb) << (8 * (nkb - 1));
    }
  };
  // a warp's tile-block of item word w: source, bytes (0: none), input
  // block and tile
  auto tile_of = [&](uint32_t p1, uint64_t p2, uint32_t w, const uint8_t *&src, int &kb, int &tile) -> uint32_t {
    const Inst &I = S.inst[item_inst(w)];
    const int tbb = tile_block_bytes(I.qtype);
    if constexpr (W == 2) {
      // phase 1: warp = matrix (bit 3), tile of the item (bit 2), input
      // blocks 2 (warp & 3) and + 1; phase 2: nkb / 2 warps per down tile,
      // each two consecutive input blocks
      if (item_phase(w) == 1) {
        tile = item_grp(w) * 2 + ((warp >> 2) & 1);
        kb = 2 * (warp & 3);
        if (tile >= I.ffn / 16) return 0;
        src = ((warp >> 3) ? I.up : I.gate) + (size_t)(tile * nkbH + kb) * tbb;
      } else {
        const int nkb = I.ffn >> 8, half = nkb >> 1;
        tile = item_grp(w) * (32 / nkb) + warp / half;
        kb = 2 * (warp % half);
        if (tile >= H / 16) return 0;
        src = I.down + (size_t)(tile * nkb + kb) * tbb;
      }
      return (uint32_t)tbb;
    }
    if (item_phase(w) == 1) {
      tile = item_grp(w) * it1 + (int)(p1 & 15u);
      kb = (int)((p1 >> 4) & 7u);
      if (!(p1 & 128u) || tile >= I.ffn / 16) return 0;
      src = ((p1 >> 8) ? I.up : I.gate) + (size_t)(tile * nkbH + kb) * tbb;
    } else {
      const int nkb = I.ffn >> 8;
      const uint32_t e = (uint32_t)(p2 >> (8 * (nkb - 1))) & 0xFFu;
      tile = item_grp(w) * it2_of(nkb) + (int)(e & 15u);
      kb = (int)((e >> 4) & 7u);
      if (!(e & 128u) || tile >= H / 16) return 0;
      src = I.down + (size_t)(tile * nkb + kb) * tbb;
    }
    return (uint32_t)tbb;
  };
  // copy item k into stage k % kRing: its gate and up tiles (phase 1,
  // tile-blocks of warps 0..7 and 8..15) or its down tiles (phase 2), each
  // contiguous in the resident layout; one thread
  auto issue = [&](int k) {
    const int s = k % kRing;
    const uint32_t w = S.items[k];
    const Inst &I = S.inst[item_inst(w)];
    const int tbb = tile_block_bytes(I.qtype);
    uint8_t *dst = S.ring + (size_t)s * Sh::kStageTB * kStageBytes;
    if (item_phase(w) == 1) {
      const int t0 = item_grp(w) * it1, nt = min(it1, I.ffn / 16 - t0);
      const uint32_t bytes = (uint32_t)(nt * nkbH * tbb);
      const size_t off0 = (size_t)t0 * nkbH * tbb;
      mbar_expect_tx(&S.full[s], 2 * bytes);
      bulk_g2s(dst, I.gate + off0, bytes, &S.full[s]);
      bulk_g2s(dst + 8 * W * kStageBytes, I.up + off0, bytes, &S.full[s]);
    } else {
      const int nkb = I.ffn >> 8, it = W == 1 ? it2_of(nkb) : 32 / nkb;
      const int t0 = item_grp(w) * it, nt = min(it, H / 16 - t0);
      const uint32_t bytes = (uint32_t)(nt * nkb * tbb);
      mbar_expect_tx(&S.full[s], bytes);
      bulk_g2s(dst, I.down + (size_t)t0 * nkb * tbb, bytes, &S.full[s]);
    }
  };

  if (warp == 0) {
    // ---- warp 0: this CTA's item list, then the first kRing copies of
    // every warp (the weights start streaming as soon as the routing is
    // known)
    __syncwarp();
    const Split sp = split();
    const int my1 = sp.my1, my2 = sp.my2;
    const int n_inst = s_n_inst;
    for (int k = lane; k < my1 + my2; k += 32) {
      int phase;
      const int j = item_index(sp, k, phase);
      int lo = 0, hi = n_inst - 1;  // last instance whose base <= j
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((phase == 1 ? S.inst[mid].p1_base : S.inst[mid].p2_base) <= j) lo = mid; else hi = mid - 1;
      }
      const Inst &I = S.inst[lo];
      const int ng = phase == 1 ? I.ng1 : I.ng2;
      const int loc = j - (phase == 1 ? I.p1_base : I.p2_base);
      S.items[k] = item_word(lo, loc / ng, loc % ng, phase);
    }
    __syncwarp();
    TR_STAMP(19);
    if (lane < min(kRing, my1 + my2)) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the rings were bucketing scratch
      issue(lane);
    }
    TR_STAMP(20);
  } else {
    if (warp == 1) {
      // this call's counter set (by the parity of the call count); the other
      // one, used by the previous call, is zeroed here, spread over the
      // grid's warps 1, for the next call
      const int par = ctrl->epoch & 1;
      int *other = reinterpret_cast<int *>(a.ws + a.L.slices) + (par ^ 1) * kSliceSetInts;
      const int n_old = min(ctrl->slice_pairs[par ^ 1], kFusedMaxPairs + 64) * kSlicesPerPair;
      for (int i = cta * 32 + lane; i < n_old; i += G * 32) other[i * kSliceStride] = 0;
      if (lane == 0) {
        s_par = par;
        if (cta == 0) {
          ctrl->out_ready[par ^ 1] = 0;
          ctrl->slice_pairs[par] = npairs + (a.has_shared ? T : 0);
        }
      }
    }
    // ---- the other warps zero this CTA's slice of out, or copy the
    // residual into it (the down items add into it once every CTA has;
    // out does not overlap the inputs)
    const unsigned total4 = (unsigned)(T * H / 4);
    const unsigned z0 = cta * total4 / (unsigned)G, z1 = (cta + 1) * total4 / (unsigned)G;
    for (unsigned i = z0 + tid - 32; i < z1; i += kCThreads - 32)
      reinterpret_cast<float4 *>(a.out)[i] =
          a.residual ? __ldg(reinterpret_cast<const float4 *>(a.residual) + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  uint32_t my_p1;
  uint64_t my_p2;
  warp_place(warp, my_p1, my_p2);
  __syncthreads();  // the item list and the replicated tables are visible
  const Split sp = split();
  const int my1 = sp.my1, my_items = sp.my1 + sp.my2;
  const int par = s_par;
  int *slices = reinterpret_cast<int *>(a.ws + a.L.slices) + par * kSliceSetInts;
  // this CTA's slice of out is initialised
  if (tid == 0) arrive_release(&ctrl->out_ready[par]);
  // slice counters, one per 128-byte line (many warps poll them)
  auto slice_ctr = [&](int pair, int slice) { return slices + (pair * kSlicesPerPair + slice) * kSliceStride; };
  bool out_ready = false;  // this warp has seen every CTA's part of out initialised
  TR_STAMP(1);
  TR_DECL;

  // The reducer of phase-1 item j (warp j mod 16) adds the item's partials
  // once all warps have stored them, writes h = SiLU(g) * u for its rows and
  // counts them for their slice of h.  Reductions run kRedLag items late, so
  // the reducer rarely waits for a slower warp; rj is the next item this warp
  // considers.
  int rj = 0;
  auto reduce_until = [&](int upto) {
    for (; rj < upto; ++rj) {
      if (rj % kCWarps != warp) continue;
      const uint32_t w = S.items[rj];
      const Inst &I = S.inst[item_inst(w)];
      const int chunk = item_chunk(w), grp = item_grp(w);
      const int ntok = min(kTokChunk, I.count - kTokChunk * chunk);
      const int pbase = I.pair_start + kTokChunk * chunk;
      const int r = rj % kRedSlots;
      const float *red = S.red + (size_t)r * kCWarps * kRedFloats;
      mbar_wait(&S.rfull[r], (uint32_t)((rj / kRedSlots) & 1), a.status);
      TR(8);
      const int pos = lane & 1;  // lane = 2 * row + position
      for (int ti = 0; ti < it1; ++ti) {
        const int tile = grp * it1 + ti;
        if (tile >= I.ffn / 16) break;
        float g = 0.f, u = 0.f;
        // the warps of tile ti: ti * (nkbH / W) + j (gate), 8 + that (up)
        for (int j = 0; j < nkbH / W; ++j) {
          g += red[(ti * (nkbH / W) + j) * kRedFloats + lane];
          u += red[(8 + ti * (nkbH / W) + j) * kRedFloats + lane];
        }
        if (pos < ntok)
          __stcg(hbuf + (size_t)(pbase + pos) * a.max_ffn + tile * 16 + (lane >> 1), silu_mul(g, u));
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&S.rfree[r]);
        // the item's tiles of h are written: count them for their 256-input
        // slice (it1 divides 16, so they lie in one)
        const int t0 = grp * it1, nt = min(it1, I.ffn / 16 - t0);
        if (nt > 0)
          asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(slice_ctr(pbase, t0 >> 4)), "r"(nt)
                       : "memory");
      }
      TR(9);
    }
  };

  // ---- main loop over this CTA's items
  TR_STAMP(2);
  // this warp's activation limbs: the input slice of its current tile-block
  // for the item's token positions (per-slice scales sc0, sc1)
  uint8_t *wl = S.wlimbs + (size_t)warp * kTokChunk * 3 * kWPlane;
  // what the limbs in wl hold: phase 1 (input block, the positions' tokens),
  // phase 2 (input block, first pair, positions) -- gate/up items of other
  // experts with the same tokens reuse them
  uint64_t lim_key = ~0ull;
  float sc0 = 0.f, sc1 = 0.f;
  const uint32_t g2 = smem_u32(S.sel2), g1 = smem_u32(S.sel1);
  const int ncol = lane >> 2, cpos = ncol / 3;  // this lane's B column: limb ncol % 3 of position cpos
  const uint32_t bp = smem_u32(wl) + (uint32_t)((cpos * 3 + ncol % 3) * kWPlane);
  for (int k = 0; k <= my_items; ++k) {
    if (k == my1) TR_STAMP(3);
    if (k == my_items) break;
    const int s = k % kRing;
    const uint32_t w = S.items[k];
    const Inst &I = S.inst[item_inst(w)];
    const int chunk = item_chunk(w), phase = item_phase(w);
    const int ntok = min(kTokChunk, I.count - kTokChunk * chunk);
    const int pbase = I.pair_start + kTokChunk * chunk;
    // ---- this warp's tile-block
    const uint8_t *src = nullptr;
    int kb = 0, tile = 0;
    const uint32_t bytes = tile_of(my_p1, my_p2, w, src, kb, tile);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    TR(0);
    if (bytes) {
      const uint64_t key =
          phase == 1 ? ((uint64_t)kb << 60) | ((uint64_t)(uint32_t)S.pair_tok[pbase] << 30) |
                           (uint32_t)(ntok > 1 ? S.pair_tok[pbase + 1] + 1 : 0)
                     : (1ull << 63) | ((uint64_t)kb << 60) | ((uint64_t)(uint32_t)pbase << 30) | (uint32_t)ntok;
      if (key != lim_key) {
        if (phase == 2) {
          // this slice of h is complete (16 tiles), and out is initialised
          // everywhere before the first down result is added into it
          if (lane == 0) {
            wait_count(slice_ctr(pbase, kb), 16, a.status);
            if (W == 2) wait_count(slice_ctr(pbase, kb + 1), 16, a.status);
            if (!out_ready) wait_count(&ctrl->out_ready[par], G, a.status);
          }
          out_ready = true;
          __syncwarp();
          TR(1);
        }
        // limbs of the item's token positions, this warp's 256 inputs
        lim_key = key;
        for (int j = 0; j < ntok; ++j) {
          const float *x = phase == 1 ? a.x + (size_t)S.pair_tok[pbase + j] * H + 256 * kb
                                      : hbuf + (size_t)(pbase + j) * a.max_ffn + 256 * kb;
          const float scj = warp_slice_limbs<W>(x, phase == 2, wl + j * 3 * kWPlane);
          if (j == 0) sc0 = scj; else sc1 = scj;
        }
        TR(2);
      }
    }
    // every warp waits for the stage, also one without a tile-block in it:
    // its refill must not start before all have seen this item's copy land
    mbar_wait(&S.full[s], (uint32_t)((k / kRing) & 1), a.status);
    if (bytes) {
      const bool bv = ncol < 6 && cpos < ntok;
      if (warp == 0 && k == 0) TR_STAMP(12);
      if (warp == 0 && k == my1) TR_STAMP(14);
      TR(3);
      // this warp's tile-block in the stage (phase 1: gate part, then up
      // part from slot 8; phase 2: down tiles from slot 0), tile-blocks at
      // their own size
      const int tbb = tile_block_bytes(I.qtype);
      uint32_t slot;  // this warp's first tile-block in the stage, in tile-blocks
      if constexpr (W == 1) {
        slot = phase == 1 ? (uint32_t)(warp & 7) : (uint32_t)warp;
      } else {
        const int nkb = I.ffn >> 8;
        slot = phase == 1 ? (uint32_t)(((warp >> 2) & 1) * 8 + 2 * (warp & 3))
                          : (uint32_t)((warp / (nkb >> 1)) * nkb + 2 * (warp % (nkb >> 1)));
      }
      const uint32_t tb = smem_u32(S.ring + (size_t)s * Sh::kStageTB * kStageBytes) +
                          (uint32_t)(phase == 1 ? (warp >> 3) * 8 * W * kStageBytes : 0) + slot * (uint32_t)tbb;
#pragma unroll
      for (int b = 0; b < W; ++b) {  // (W = 2: input blocks kb and kb + 1, limbs 256 bytes on)
        if (I.qtype == kQ2)
          tb_q2<Sh::kRep2>(tb + b * tbb, g2, bp + 256 * b, bv, acc);
        else
          tb_q1<Sh::kRep1>(tb + b * tbb, g1, bp + 256 * b, bv, acc);
      }
      if (warp == 0 && k == 0) TR_STAMP(13);
      if (warp == 0 && k == my1) TR_STAMP(15);
      TR(4);
    }
    // the last warp done with the stage refills it with item k + kRing
    __syncwarp();
    if (lane == 0 && atomicSub(&S.left[s], 1) == 1) {
      S.left[s] = kCWarps;
      if (k + kRing < my_items) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        issue(k + kRing);
      }
    }
    if (phase == 2) {
      // ---- down: this warp's rows go straight into out (fp32 atomics),
      // scaled by the router weight and the slice's limb scale
      if (bytes) {
        float v[4];
        quad_rows(acc, v);
        if ((lane & 3) == 0) {
          const int q = lane >> 2, row = tile * 16 + q;
          float *o0 = a.out + (size_t)S.pair_tok[pbase] * H + row;
          const float w0 = S.pair_w[pbase] * sc0;
          atomicAdd(o0, w0 * v[0]);
          atomicAdd(o0 + 8, w0 * v[2]);
          if (ntok > 1) {
            float *o1 = a.out + (size_t)S.pair_tok[pbase + 1] * H + row;
            const float w1 = S.pair_w[pbase + 1] * sc1;
            atomicAdd(o1, w1 * v[1]);
            atomicAdd(o1 + 8, w1 * v[3]);
          }
        }
      }
      TR(7);
      continue;
    }
    TR(5);
    // ---- gate/up: partial sums into the item's reduction slot
    const int r = k % kRedSlots;
    float *red = S.red + (size_t)r * kCWarps * kRedFloats;
    if (k >= kRedSlots) mbar_wait(&S.rfree[r], (uint32_t)(((k / kRedSlots) - 1) & 1), a.status);
    TR(6);
    if (bytes) store_partials(acc, sc0, sc1, red + warp * kRedFloats);
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.rfull[r]);
    TR(7);
    // ---- reductions of earlier items (all of them at the end of the phase)
    reduce_until(k + 1 == my1 ? my1 : k + 1 - kRedLag);
    TR(0);
  }
  TR_STAMP(22);
  TR_FLUSH();
  TR_STAMP(6);
  // ---- exit: the last CTA closes the call (the next call starts only once
  // this grid has completed, so plain stores do)
  TR_STAMP(23);
  __syncthreads();
  if (tid == 0 && atomicAdd(&ctrl->exit_count, 1) == G - 1) {
    ctrl->exit_count = 0;
    ctrl->epoch = ctrl->epoch + 1;
  }
}

size_t fused_smem_bytes(int w) { return (w == 2 ? smem_plan<2>().total : smem_plan<1>().total) + 64; }

bool fused_supported(int hidden, int max_ffn, int n_tokens, int top_k, int n_experts, bool has_shared, int sms) {
  if (hidden % 256 || hidden > 2048 || max_ffn % 256 || max_ffn > 2048) return false;
  if ((int64_t)n_tokens * top_k > kFusedMaxPairs) return false;
  if (has_shared && n_tokens > 64) return false;
  // every CTA's item list fits kMaxItems: at most (pairs + shared pairs) / 2
  // + instances token chunks, each with at most ffn / 16 / it1 phase-1 and
  // hidden / 16 / it2 phase-2 items
  {
    const int64_t pairs = (int64_t)n_tokens * top_k, sh = has_shared ? n_tokens : 0;
    const int64_t insts = (pairs < n_experts ? pairs : n_experts) + (has_shared ? 1 : 0);
    const int64_t chunks = (pairs + sh) / kTokChunk + insts;
    const int nkbH = hidden / 256, it1 = 8 / nkbH > 1 ? 8 / nkbH : 1;
    const int nkbF = max_ffn / 256, it2 = nkbF >= 6 ? 2 : (nkbF == 5 ? 3 : 16 / nkbF);
    const int64_t n1 = chunks * ((max_ffn / 16 + it1 - 1) / it1), n2 = chunks * ((hidden / 16 + it2 - 1) / it2);
    const int64_t g = sms > 0 ? sms : 148;
    if ((n1 + g - 1) / g + (n2 + g - 1) / g > kMaxItems) return false;
  }
  // bucketing scratch (slot-table entries, counts, first pairs, ids, weights) lives in the rings
  if ((size_t)n_experts * 8 + 40 * (size_t)kFusedMaxPairs >
      (size_t)Shape<1>::kStageTB * Shape<1>::kRing * kStageBytes)
    return false;
  return true;  // both item shapes fit shared memory (checked at compile time)
}

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  static int cached[64] = {};  // per device; a repeated store writes the same value
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < 64) cached[dev] = sms;
  return sms;
}

bool fused_wide_items(int hidden, int n_pairs, int min_ffn, int max_ffn, bool has_shared, int shared_ffn) {
  return hidden == 2048 && n_pairs > 32 && min_ffn == max_ffn && max_ffn % 512 == 0 &&
         (!has_shared || shared_ffn % 512 == 0);
}

template <int W>
static cudaError_t launch_shape(const FusedArgs &a, cudaStream_t stream, int sms) {
  const size_t smem = fused_smem_bytes(W);
  // the shared-memory limit is a per-device attribute of the kernel: set once per device
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static bool smem_set[64] = {};
  const bool cached = dev >= 0 && dev < 64 && smem_set[dev];
  if (!cached) {
    e = cudaFuncSetAttribute(decode_fused_kernel<W>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) smem_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(kCThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  static bool pdl_ok = true;  // dependent launch lets a call's table setup overlap the previous call
  cfg.numAttrs = pdl_ok ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, decode_fused_kernel<W>, a);
  if (e != cudaSuccess && cached) {
    // the device's context may have been reset since the attribute was set
    (void)cudaGetLastError();
    e = cudaFuncSetAttribute(decode_fused_kernel<W>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, decode_fused_kernel<W>, a);
  }
  if (e != cudaSuccess && pdl_ok) {
    (void)cudaGetLastError();
    pdl_ok = false;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_fused_kernel<W>, a);
  }
#ifdef REDLITE_DEBUG_LAUNCH
  if (e != cudaSuccess) fprintf(stderr, "decode_fused_kernel launch: %s\n", cudaGetErrorString(e));
#endif
  return e;
}

cudaError_t launch_fused(const FusedArgs &a, cudaStream_t stream) {
  const int sms = device_sms();
  if (sms <= 0) return cudaErrorNoDevice;
  return a.wide ? launch_shape<2>(a, stream, sms) : launch_shape<1>(a, stream, sms);
}

}  // namespace redlite
