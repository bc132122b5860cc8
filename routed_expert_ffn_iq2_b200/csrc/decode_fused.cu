// decode_fused.cu -- one persistent kernel per decode-sized layer call.
//
// "Red Metal dev8 -- resident routed top-k layer", steps 4-6: every selected
// expert runs gate, up, SiLU(gate)*up and down from its resident slot and
// the layer accumulates out += router_weight * expert_output (plus the
// shared expert with weight 1, "Red Lite dev16", block composition).
//
// Structure (one CTA per SM, cooperative launch so all CTAs are resident;
// 8 consumer warps + 1 producer warp per CTA):
//   prologue  every CTA copies the byte-permute selector tables into shared
//             memory, buckets the (token, slot) pairs by expert (stable,
//             identical in every CTA), reads the selected slots'
//             descriptors, enumerates the work items and converts the
//             activations to fixed-point limbs;
//   phase 1   16-row tiles of gate and of up of every selected expert, split
//             evenly over the CTAs; the producer warp streams each tile's
//             packed bytes by TMA bulk copy into a ring of shared-memory
//             stages; each consumer warp decodes one 16x256 tile-block and
//             the last warp to finish a tile reduces it and writes g or u to
//             the workspace; each CTA also zeroes a slice of `out`;
//   barrier   one grid-wide counter (bounded wait);
//   phase 2   groups of down tiles: h = SiLU(g) * u per token, y = W_down h,
//             out[token] += weight * y with fp32 atomics.  Down tiles are
//             prefetched into the ring while phase 1 finishes.
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

constexpr int kCWarps = 8;                 // consumer warps
constexpr int kCThreads = 32 * kCWarps;    // 256
constexpr int kFThreads = kCThreads + 32;  // + producer warp
constexpr int kRing = 6;
constexpr int kStageBytes = 8 * kQ2TileBlock;  // 9472 >= 8 * kQ1TileBlock
constexpr int kTokChunk = 4;
#ifndef REDLITE_REP2
#define REDLITE_REP2 16
#endif
constexpr int kRep2 = REDLITE_REP2;  // replicas of the IQ2 selector/sign tables (bank spread)
constexpr int kRep1 = 2;   // replicas of the IQ1 selector table
constexpr int kLimbPad = 32;  // padding per limb plane (spreads shared-memory banks)
constexpr uint32_t kSpinLimit = 1u << 24;


// 8-byte tables the selector nibbles index: IQ2 +8,+25,+43,0,-8,-25,-43,0;
// IQ1 (delta +1/8) -7,1,9,0 and (delta -1/8) -9,-1,7,0, all scaled by 8.
constexpr uint32_t kQ2Pos = 0x002B1908u, kQ2Neg = 0x00D5E7F8u;
constexpr uint32_t kQ1Pos = 0x000901F9u, kQ1Neg = 0x0007FFF7u;

struct Inst {  // one selected expert (or the shared expert)
  const uint8_t *gate, *up, *down;
  int qtype, ffn;
  int pair_start, count;
  int p1_base, p2_base;  // first work item of this instance in each phase
};

struct ItemInfo {
  int inst, chunk, sub, tile;  // phase 1: sub = 0 gate / 1 up; phase 2: tile group
  int phase;
};

struct Smem {
  uint32_t *sel2, *sgn2, *sel1;
  uint8_t *ring;
  float *red;  // [kRing][kCWarps][16 rows][4 tokens]
  uint8_t *limbs;
  Inst *inst;
  int *pair_tok;
  float *pair_w;
  uint64_t *full, *empty;
  uint64_t *pdone;  // per stage: all consumer warps' partials are in red (mbarrier, 8 arrivals)
  ItemInfo *info;
  float *tok_scale;  // per token slot: 2^(e - 20)
  float *wmax;       // [kCWarps][4] partial maxima
};

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Shared-memory loads by 32-bit shared address (never generic).  The
// volatile forms read data that other threads or the bulk copies write (kept
// in program order); the plain form reads the selector tables, which nobody
// writes after the setup.
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

// Bounded wait on an mbarrier phase; returns false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t it = 0; it < kSpinLimit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
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
// happens before it (this thread's, and through block barriers or warp syncs
// the block's) is visible to a thread that acquires the new value.
__device__ __forceinline__ void arrive_release(int *counter) {
  asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(counter) : "memory");
}

// Spin until *counter >= target; false (and the TIMEOUT status bit) if that
// takes longer than kGridWaitNs.  One thread per CTA calls it.
__device__ __noinline__ bool wait_count(const int *counter, int target, int32_t *status) {
  const uint64_t t_end = global_ns() + kGridWaitNs;
  while (ld_acquire(counter) < target) {
    if (global_ns() > t_end) {
      atomicOr(status, REDLITE_STATUS_TIMEOUT);
      return false;
    }
    __nanosleep(32);
  }
  return true;  // the acquiring load orders what follows
}

// named barrier over the consumer warps only
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCThreads) : "memory"); }

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

// Optional timeline (build with -DREDLITE_TRACE): CTA c writes %globaltimer
// stamps to the 32 words after the workspace layout's end, slot c * 32 + i.
#ifdef REDLITE_TRACE
#define TRACE(i)                                                                            \
  do {                                                                                      \
    if (threadIdx.x == 0) {                                                                 \
      uint64_t t_;                                                                          \
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                \
      reinterpret_cast<uint64_t *>(a.ws + a.L.total)[blockIdx.x * 32 + (i)] = t_;           \
      reinterpret_cast<uint64_t *>(a.ws + a.L.total)[148 * 48 + blockIdx.x * 32 + (i)] =    \
          (uint64_t)clock64();                                                              \
    }                                                                                       \
  } while (0)
#define TRACEC(i, v)                                                                                 \
  do {                                                                                               \
    if ((threadIdx.x & 31) == 0)                                                                     \
      reinterpret_cast<uint64_t *>(a.ws + a.L.total)[148 * 32 + (blockIdx.x * 16 + (i))] = (v);       \
  } while (0)
#define TRACE_DECL long long tr_acc_[12] = {0}; long long tr_t_ = 0
#define TRACE_T0() tr_t_ = clock64()
#define TRACE_ADD(c, i, j)            \
  do {                                \
    const long long d_ = clock64() - tr_t_; \
    if (c) tr_acc_[i] += d_;          \
    else tr_acc_[j] += d_;            \
  } while (0)
#define TRACE_CNT(c, i, j) \
  do {                     \
    if (c) tr_acc_[i] += 1; \
    else tr_acc_[j] += 1;   \
  } while (0)
#define TRACE_FLUSH()                                                                              \
  do {                                                                                             \
    if (threadIdx.x == 0)                                                                          \
      for (int i_ = 0; i_ < 12; ++i_)                                                              \
        reinterpret_cast<uint64_t *>(a.ws + a.L.total)[148 * 80 + blockIdx.x * 16 + i_] = tr_acc_[i_]; \
  } while (0)
#else
#define TRACE_DECL
#define TRACE_T0()
#define TRACE_ADD(c, i, j)
#define TRACE_CNT(c, i, j)
#define TRACE_FLUSH()
#define TRACE(i) \
  do {           \
  } while (0)
#define TRACEC(i, v) \
  do {               \
  } while (0)
#endif

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

// ------------------------------------------------------------------ tile-block math
//
// Column n of the mma B operand (n = lane >> 2 of the lane holding it) is
// limb n % 3 of token position 2p + n / 3 of the chunk (n < 6); columns 6
// and 7 are zero.  Each lane gets, per token pair p, the shared address of
// the limb plane it reads and whether its column is used.  Limb planes are
// int8 vectors.
template <int NP>
__device__ __forceinline__ void b_planes(uint32_t limbs, int lstride, int slot4, int ntok, uint32_t bp[NP],
                                         bool bv[NP]) {
  const int n = (threadIdx.x & 31) >> 2;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int pos = 2 * p + n / 3;
    const int slot = (slot4 >> (2 * pos)) & 3;
    bv[p] = n < 6 && pos < ntok;
    bp[p] = limbs + (uint32_t)((slot * 3 + n % 3) * lstride);
  }
}

// IQ2_XS-style tile-block (16 rows x 256 inputs): acc[p][.] += partial dot
// products of the block's rows with token pair p (mma C layout, limb
// columns).  Lane (q, t) decodes groups 4c + t of rows q and q+8.  All
// selector and activation loads are issued before the first mma so their
// latencies overlap.  Per 8-weight group: two byte extracts, the index bit,
// two multiply-adds for the table offsets (entry stride 64 bytes = 16
// replicas), two table loads, one OR, two byte permutes and one shift.
template <int NP>
__device__ __forceinline__ void tb_q2(uint32_t tb, uint32_t g2, uint32_t gs, const uint32_t bp[NP],
                                      const bool bv[NP], int kbase, float acc[NP][4]) {
  static_assert(kRep2 == 16, "table offsets below assume 16 replicas (64-byte entries)");
  const int lane = threadIdx.x & 31, q = lane >> 2, t = lane & 3;
  const uint32_t r4 = (uint32_t)(lane & 15) << 2;
  const uint4 qs = lds_v4(tb + 32 * lane);
  const uint4 sg = lds_v4(tb + 32 * lane + 16);
  const uint32_t qh14 = lds_b16(tb + 1024 + 2 * lane) << 14;
  const uint2 scw = lds_v2(tb + 1088 + 8 * q);
  const uint32_t dw = lds_b32(tb + 1152 + 4 * q);
  const uint32_t qsw[4] = {qs.x, qs.y, qs.z, qs.w};
  const uint32_t sgw[4] = {sg.x, sg.y, sg.z, sg.w};
  uint32_t sel[16];  // field i = 2c + h
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint32_t qsb = __byte_perm(qsw[i >> 2], 0u, 0x4440u | (uint32_t)(i & 3));
    const uint32_t sgb = __byte_perm(sgw[i >> 2], 0u, 0x4440u | (uint32_t)(i & 3));
    const uint32_t hi = ((qh14 >> i) & 0x4000u) | r4;  // index bit 8, times 64, plus replica
    const uint32_t go = qsb * 64u + hi;
    const uint32_t so = sgb * 64u + r4;
    sel[i] = lds_table(g2 + go) | lds_table(gs + so);
  }
  uint2 b[NP][8];
#pragma unroll
  for (int p = 0; p < NP; ++p)
#pragma unroll
    for (int c = 0; c < 8; ++c)
      b[p][c] = bv[p] ? lds_v2(bp[p] + kbase + 32 * c + 8 * t) : make_uint2(0u, 0u);
  // sub-block multipliers 2sc+1 as bytes: chunk c is byte c >> 1 of the even
  // (c even) or odd (c odd) nibble word of its row
  const uint32_t me0 = ((scw.x & 0x0F0F0F0Fu) << 1) | 0x01010101u, mo0 = ((scw.x >> 3) & 0x1E1E1E1Eu) | 0x01010101u;
  const uint32_t me1 = ((scw.y & 0x0F0F0F0Fu) << 1) | 0x01010101u, mo1 = ((scw.y >> 3) & 0x1E1E1E1Eu) | 0x01010101u;
  int32_t cb[NP][4];
#pragma unroll
  for (int p = 0; p < NP; ++p) cb[p][0] = cb[p][1] = cb[p][2] = cb[p][3] = 0;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t a[4];
    a[0] = __byte_perm(kQ2Pos, kQ2Neg, sel[2 * c]);
    a[2] = __byte_perm(kQ2Pos, kQ2Neg, sel[2 * c] >> 16);
    a[1] = __byte_perm(kQ2Pos, kQ2Neg, sel[2 * c + 1]);
    a[3] = __byte_perm(kQ2Pos, kQ2Neg, sel[2 * c + 1] >> 16);
    const int m0 = (int)__byte_perm((c & 1) ? mo0 : me0, 0u, 0x4440u | (uint32_t)(c >> 1));
    const int m1 = (int)__byte_perm((c & 1) ? mo1 : me1, 0u, 0x4440u | (uint32_t)(c >> 1));
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      int32_t d[4];
      mma_k32(d, a, b[p][c].x, b[p][c].y);
      cb[p][0] += m0 * d[0];
      cb[p][1] += m0 * d[1];
      cb[p][2] += m1 * d[2];
      cb[p][3] += m1 * d[3];
    }
  }
  const float d0 = half_bits(dw & 0xFFFFu) * 0.125f, d1 = half_bits(dw >> 16) * 0.125f;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    acc[p][0] += d0 * (float)cb[p][0];
    acc[p][1] += d0 * (float)cb[p][1];
    acc[p][2] += d1 * (float)cb[p][2];
    acc[p][3] += d1 * (float)cb[p][3];
  }
}

// IQ1_M-style tile-block: one k16 mma per 16-weight sub-block; lane t holds
// weights 4t..4t+3 of the sub-block (half of group 2s + (t >> 1)).
template <int NP>
__device__ __forceinline__ void tb_q1(uint32_t tb, uint32_t sel1, const uint32_t bp[NP], const bool bv[NP],
                                      int kbase, float acc[NP][4]) {
  const int lane = threadIdx.x & 31, q = lane >> 2, t = lane & 3, r = lane & (kRep1 - 1);
  const uint32_t pb = tb + 48 * (2 * q + (t >> 1));
  const uint4 qa = lds_v4(pb);
  const uint4 qb = lds_v4(pb + 16);
  const uint4 nb = lds_v4(pb + 32);
  const uint32_t s0 = lds_b32(tb + 768 + 12 * q), s1 = lds_b32(tb + 772 + 12 * q), s2 = lds_b32(tb + 776 + 12 * q);
  const uint64_t row0 = (uint64_t)s0 | ((uint64_t)(s1 & 0xFFFFu) << 32);
  const uint64_t row1 = (uint64_t)(s1 >> 16) | ((uint64_t)s2 << 16);
  const uint32_t dw = lds_b32(tb + 864 + 4 * q);
  const int hshift = 16 * (t & 1);
  const uint32_t qsw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
  const uint32_t nbw[4] = {nb.x, nb.y, nb.z, nb.w};
  uint32_t sel[32];  // entry i = 2s + h
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t qsb = (qsw[i >> 2] >> (8 * (i & 3))) & 0xFFu;
    const uint32_t nib = (nbw[i >> 3] >> (4 * (i & 7))) & 0xFu;
    sel[i] = lds_table(sel1 + 4 * ((qsb | (nib << 8)) * kRep1 + r)) >> hshift;
  }
  uint32_t b[NP][16];
#pragma unroll
  for (int p = 0; p < NP; ++p)
#pragma unroll
    for (int s = 0; s < 16; ++s) b[p][s] = bv[p] ? lds_b32(bp[p] + kbase + 16 * s + 4 * t) : 0u;
  int32_t cb[NP][4];
#pragma unroll
  for (int p = 0; p < NP; ++p) cb[p][0] = cb[p][1] = cb[p][2] = cb[p][3] = 0;
#pragma unroll
  for (int s = 0; s < 16; ++s) {
    const uint32_t a0 = __byte_perm(kQ1Pos, kQ1Neg, sel[2 * s]);
    const uint32_t a1 = __byte_perm(kQ1Pos, kQ1Neg, sel[2 * s + 1]);
    const int m0 = 2 * (int)((row0 >> (3 * s)) & 7u) + 1;
    const int m1 = 2 * (int)((row1 >> (3 * s)) & 7u) + 1;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      int32_t d[4];
      mma_k16(d, a0, a1, b[p][s]);
      cb[p][0] += m0 * d[0];
      cb[p][1] += m0 * d[1];
      cb[p][2] += m1 * d[2];
      cb[p][3] += m1 * d[3];
    }
  }
  const float d0 = half_bits(dw & 0xFFFFu) * 0.125f, d1 = half_bits(dw >> 16) * 0.125f;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    acc[p][0] += d0 * (float)cb[p][0];
    acc[p][1] += d0 * (float)cb[p][1];
    acc[p][2] += d1 * (float)cb[p][2];
    acc[p][3] += d1 * (float)cb[p][3];
  }
}

// Combine the limb columns of each token and store this warp's partial sums
// to red[row 0..15][token position 0..3].
template <int NP>
__device__ __forceinline__ void store_partials(const float acc[NP][4], float *red) {
  const int lane = threadIdx.x & 31, q = lane >> 2, t = lane & 3;
  const int n0 = 2 * t, n1 = 2 * t + 1;
  const float f0 = n0 < 6 ? (n0 % 3 == 0 ? 16384.f : (n0 % 3 == 1 ? 128.f : 1.f)) : 0.f;
  const float f1 = n1 < 6 ? (n1 % 3 == 0 ? 16384.f : (n1 % 3 == 1 ? 128.f : 1.f)) : 0.f;
  const int m0 = n0 / 3, m1 = n1 / 3;  // token within the pair (2 = none)
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    float v[4];  // (row q, tok 0), (row q, tok 1), (row q+8, tok 0), (row q+8, tok 1)
    v[0] = (m0 == 0 ? f0 * acc[p][0] : 0.f) + (m1 == 0 ? f1 * acc[p][1] : 0.f);
    v[1] = (m0 == 1 ? f0 * acc[p][0] : 0.f) + (m1 == 1 ? f1 * acc[p][1] : 0.f);
    v[2] = (m0 == 0 ? f0 * acc[p][2] : 0.f) + (m1 == 0 ? f1 * acc[p][3] : 0.f);
    v[3] = (m0 == 1 ? f0 * acc[p][2] : 0.f) + (m1 == 1 ? f1 * acc[p][3] : 0.f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[j] += __shfl_xor_sync(0xffffffffu, v[j], 1);
      v[j] += __shfl_xor_sync(0xffffffffu, v[j], 2);
    }
    if (t == 0) {
      red[q * 4 + 2 * p] = v[0];
      red[q * 4 + 2 * p + 1] = v[1];
      red[(q + 8) * 4 + 2 * p] = v[2];
      red[(q + 8) * 4 + 2 * p + 1] = v[3];
    }
  }
}

// One tile-block of either format for 1-2 (NP = 1) or 3-4 (NP = 2) token
// positions; the warp's partials go to red (16 x 4 floats).  Inlined at one
// call site.
__device__ __forceinline__ void warp_tile_block(int qtype, const uint8_t *tb_p, const Smem &S, const uint8_t *limbs_p,
                                                int lstride, int kbase, int slot4, int ntok, float *red) {
  const uint32_t tb = smem_u32(tb_p), limbs = smem_u32(limbs_p);
  if (qtype == kQ2) {
    const uint32_t g2 = smem_u32(S.sel2), gs = smem_u32(S.sgn2);
    if (ntok <= 2) {
      uint32_t bp[1];
      bool bv[1];
      b_planes<1>(limbs, lstride, slot4, ntok, bp, bv);
      float acc[1][4] = {{0.f, 0.f, 0.f, 0.f}};
      tb_q2<1>(tb, g2, gs, bp, bv, kbase, acc);
      store_partials<1>(acc, red);
    } else {
      uint32_t bp[2];
      bool bv[2];
      b_planes<2>(limbs, lstride, slot4, ntok, bp, bv);
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      tb_q2<2>(tb, g2, gs, bp, bv, kbase, acc);
      store_partials<2>(acc, red);
    }
  } else {
    const uint32_t g1 = smem_u32(S.sel1);
    if (ntok <= 2) {
      uint32_t bp[1];
      bool bv[1];
      b_planes<1>(limbs, lstride, slot4, ntok, bp, bv);
      float acc[1][4] = {{0.f, 0.f, 0.f, 0.f}};
      tb_q1<1>(tb, g1, bp, bv, kbase, acc);
      store_partials<1>(acc, red);
    } else {
      uint32_t bp[2];
      bool bv[2];
      b_planes<2>(limbs, lstride, slot4, ntok, bp, bv);
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      tb_q1<2>(tb, g1, bp, bv, kbase, acc);
      store_partials<2>(acc, red);
    }
  }
}

// Limbs of up to 4 vectors of n floats (n a multiple of 4, n <= 2048) read
// from global memory: vector j's limb planes go to dst + (3 j + limb) *
// lstride, scale_out[j] = 2^(e_j - 20) with 2^e_j > max |vector j|.  With
// up_off == 0 vector j is src + j * src_stride; otherwise it is SiLU(g) * u
// with g = src + j * src_stride and u = g + up_off.  Consumer thread tid
// holds float4 number t + nt * i (i < 3) of every vector.  Out of
// line and compact: it runs a few times per call, and the kernel's hot loop
// must stay in the instruction cache.  Threads t = 0..nt-1 (nt >= 176, a
// multiple of 32) take part, with two syncs on named barrier `bar`.
__device__ __noinline__ void limbs_from_global(int nvec, int n, const float *src, size_t src_stride, int up_off,
                                               uint8_t *dst, int lstride, float *wmax, float *scale_out, int t,
                                               int nt, int bar) {
  const int warp = t >> 5, lane = t & 31;
  const int per = n / 4;
  float4 v[4][3];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const int e4 = t + nt * i;
      v[j][i] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j < nvec && e4 < per) {
        const float *g = src + (size_t)j * src_stride;
        v[j][i] = __ldcg(reinterpret_cast<const float4 *>(g) + e4);
        if (up_off) {
          const float4 u = __ldcg(reinterpret_cast<const float4 *>(g + up_off) + e4);
          v[j][i] = make_float4(silu_mul_fast(v[j][i].x, u.x), silu_mul_fast(v[j][i].y, u.y),
                                silu_mul_fast(v[j][i].z, u.z), silu_mul_fast(v[j][i].w, u.w));
        }
      }
    }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v[j][i].x), fabsf(v[j][i].y)), fmaxf(fabsf(v[j][i].z), fabsf(v[j][i].w))));
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) wmax[warp * 4 + j] = m;
  }
  asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(nt) : "memory");
  const int nw = nt >> 5;
#pragma unroll 1
  for (int j = 0; j < nvec; ++j) {
    float mm = 0.f;
#pragma unroll
    for (int w = 0; w < kCWarps; ++w)
      if (w < nw) mm = fmaxf(mm, wmax[w * 4 + j]);
    const int e = pow2_above(mm);
    const float sc = pow2f(20 - e);
    if (t == 0) scale_out[j] = pow2f(e - 20);
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const int e4 = t + nt * i;
      if (e4 < per) {
        float4 f = v[0][i];
#pragma unroll
        for (int jj = 1; jj < 4; ++jj)
          if (jj == j) f = v[jj][i];
        const float fc[4] = {f.x, f.y, f.z, f.w};
        uint32_t p0 = 0, p1 = 0, p2 = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          int l0, l1, l2;
          to_limbs(fc[c], sc, l0, l1, l2);
          p0 |= (uint32_t)(l0 & 0xFF) << (8 * c);
          p1 |= (uint32_t)(l1 & 0xFF) << (8 * c);
          p2 |= (uint32_t)(l2 & 0xFF) << (8 * c);
        }
        uint8_t *d = dst + (size_t)j * 3 * lstride + 4 * e4;
        *reinterpret_cast<uint32_t *>(d) = p0;
        *reinterpret_cast<uint32_t *>(d + lstride) = p1;
        *reinterpret_cast<uint32_t *>(d + 2 * lstride) = p2;
      }
    }
  }
  asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(nt) : "memory");
}

// Replicate the selector tables in place (word w of a table with r replicas
// holds source word w / r; replicas spread lanes over banks): NT threads,
// t = 0..NT-1, named barrier BAR.  Every source word is read before any is
// overwritten.
template <int NT, int BAR>
__device__ __forceinline__ void replicate_tables(const Smem &S, int t) {
  static_assert(kRep2 == 16 && kRep1 == 2, "replication below assumes 16 / 2 replicas");
  constexpr int N2 = (512 + NT - 1) / NT, NS = (256 + NT - 1) / NT, N1 = (4096 + NT - 1) / NT;
  uint32_t v2[N2], vs[NS], v1[N1];
#pragma unroll
  for (int i = 0; i < N2; ++i) v2[i] = t + NT * i < 512 ? S.sel2[t + NT * i] : 0u;
#pragma unroll
  for (int i = 0; i < NS; ++i) vs[i] = t + NT * i < 256 ? S.sgn2[t + NT * i] : 0u;
#pragma unroll
  for (int i = 0; i < N1; ++i) v1[i] = t + NT * i < 4096 ? S.sel1[t + NT * i] : 0u;
  asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
  const int rot = (t & 31) >> 1;  // lanes of one store wavefront cover distinct banks
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int q = (r + rot) & 3;
#pragma unroll
    for (int i = 0; i < N2; ++i)
      if (t + NT * i < 512)
        reinterpret_cast<uint4 *>(S.sel2)[(t + NT * i) * 4 + q] = make_uint4(v2[i], v2[i], v2[i], v2[i]);
#pragma unroll
    for (int i = 0; i < NS; ++i)
      if (t + NT * i < 256)
        reinterpret_cast<uint4 *>(S.sgn2)[(t + NT * i) * 4 + q] = make_uint4(vs[i], vs[i], vs[i], vs[i]);
  }
#pragma unroll
  for (int i = 0; i < N1; ++i)
    if (t + NT * i < 4096) reinterpret_cast<uint2 *>(S.sel1)[t + NT * i] = make_uint2(v1[i], v1[i]);
  asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
}

// ------------------------------------------------------------------ the kernel

// The shared expert's instance (every token, weight 1), or an empty one with
// the BAD_EXPERT bit if its descriptor is not one this kernel can read.
__device__ void set_shared_inst(Inst &I, const FusedArgs &a, int pair_start, int &bad) {
  I.pair_start = pair_start;
  if (expert_ok(a.shared, a.hidden, a.max_ffn, true)) {
    I.gate = (const uint8_t *)a.shared.gate, I.up = (const uint8_t *)a.shared.up;
    I.down = (const uint8_t *)a.shared.down, I.qtype = a.shared.qtype, I.ffn = a.shared.ffn;
    I.count = a.n_tokens;
  } else {
    bad |= REDLITE_STATUS_BAD_EXPERT;
    I.gate = I.up = I.down = nullptr;
    I.qtype = kQ2, I.ffn = 256, I.count = 0;
  }
}

__device__ __forceinline__ int item_tiles_of(int ffn) {
  const int nkb = ffn >> 8;  // 8 / nkb tiles per item, nibble table for nkb = 1..7
  return nkb >= 8 ? 1 : (int)((0x1112248u >> (4 * (nkb - 1))) & 15u);
}

__global__ void __launch_bounds__(kFThreads, 1) decode_fused_kernel(FusedArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int H = a.hidden, T = a.n_tokens, K = a.top_k, E = a.n_experts;
  const int npairs = T * K;
  const int lstrideX = H + kLimbPad;
  const bool local_x = T <= kTokChunk;
  Ctrl *ctrl = reinterpret_cast<Ctrl *>(a.ws + a.L.ctrl);
  float *gu = reinterpret_cast<float *>(a.ws + a.L.gu);
  uint8_t *glimbs = a.ws + a.L.limbs;
  float *gscale = reinterpret_cast<float *>(a.ws + a.L.exps);

  // ---- shared memory carve
  Smem S;
  size_t off = 0;
  S.sel2 = reinterpret_cast<uint32_t *>(smem + off);
  off += 512 * kRep2 * 4;
  S.sgn2 = reinterpret_cast<uint32_t *>(smem + off);
  off += 256 * kRep2 * 4;
  S.sel1 = reinterpret_cast<uint32_t *>(smem + off);
  off += 4096 * kRep1 * 4;
  S.ring = smem + off;
  off += (size_t)kRing * kStageBytes;
  S.red = reinterpret_cast<float *>(smem + off);
  off += sizeof(float) * kRing * kCWarps * 64;
  S.limbs = smem + off;
  const int lmax = (H > a.max_ffn ? H : a.max_ffn) + kLimbPad;
  off += (size_t)kTokChunk * 3 * lmax;
  off = (off + 15) & ~size_t(15);
  S.inst = reinterpret_cast<Inst *>(smem + off);
  off += sizeof(Inst) * kFusedMaxInst;
  S.pair_tok = reinterpret_cast<int *>(smem + off);
  off += sizeof(int) * (kFusedMaxPairs + 64);
  S.pair_w = reinterpret_cast<float *>(smem + off);
  off += sizeof(float) * (kFusedMaxPairs + 64);
  S.full = reinterpret_cast<uint64_t *>(smem + off);
  off += sizeof(uint64_t) * kRing;
  S.empty = reinterpret_cast<uint64_t *>(smem + off);
  off += sizeof(uint64_t) * kRing;
  S.pdone = reinterpret_cast<uint64_t *>(smem + off);
  off += sizeof(uint64_t) * kRing;
  S.info = reinterpret_cast<ItemInfo *>(smem + off);
  off += sizeof(ItemInfo) * kRing;
  S.tok_scale = reinterpret_cast<float *>(smem + off);
  off += sizeof(float) * kTokChunk;
  S.wmax = reinterpret_cast<float *>(smem + off);
  off += sizeof(float) * kCWarps * 4;
  __shared__ int s_n_inst, s_n1, s_n2, s_bad, s_scan[33];
  TRACE(0);
  // the next layer call may start its own table setup on SMs this grid frees
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- prologue part 1: every independent global load first.  One thread
  // starts bulk copies of the three selector tables (unreplicated) into the
  // first bytes of their shared-memory regions; the consumers replicate them
  // after the routing, while the first weight copies are in flight.
  __shared__ uint64_t s_lut_bar;
  if (tid == kCThreads) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
      mbar_init(&S.pdone[s], kCWarps);
    }
    mbar_init(&s_lut_bar, 1);
    mbar_fence_init();
    s_bad = 0;
    // the expanded grids are set up once, before any layer call: they may be
    // read before the previous kernel of the stream has finished
    mbar_expect_tx(&s_lut_bar, (512 + 256 + 4096) * 4);
    bulk_g2s(S.sel2, a.grids + kGridQ2Sel, 512 * 4, &s_lut_bar);
    bulk_g2s(S.sgn2, a.grids + kGridSign, 256 * 4, &s_lut_bar);
    bulk_g2s(S.sel1, a.grids + kGridQ1Sel, 4096 * 4, &s_lut_bar);
  }
  __syncthreads();  // the mbarriers are initialised before anyone waits on them
  // the call's own inputs may come from the previous kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  int my_ids[3];
  float my_w[3];
  uint4 my_d[3][2];  // slot-table entry of each of this thread's pairs
  if (tid < kCThreads) {
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int p = tid + kCThreads * j;
      my_ids[j] = p < npairs ? __ldcg(a.ids + p) : -1;
      my_w[j] = p < npairs ? __ldcg(a.weights + p) : 0.f;
    }
    if (local_x)  // warm L2 for the conversion after the routing
      for (int i = tid; i < T * H / 32; i += kCThreads) asm volatile("prefetch.global.L2 [%0];" ::"l"(a.x + 32 * i));
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int e = my_ids[j];
      if (e >= 0 && e < E) {
        const uint4 *d = reinterpret_cast<const uint4 *>(a.experts + e);
        my_d[j][0] = __ldg(d);
        my_d[j][1] = __ldg(d + 1);
      }
    }
  }
  TRACE(1);

  // work items per instance and their prefix sums (warp 0; n_inst is small)
  auto item_prefix = [&](int n_inst) {
    int base1 = 0, base2 = 0;
    for (int u0 = 0; u0 < n_inst; u0 += 32) {
      const int u = u0 + lane;
      int c1 = 0, c2 = 0;
      if (u < n_inst) {
        const Inst &I = S.inst[u];
        const int nch = (I.count + kTokChunk - 1) / kTokChunk;
        const int it = item_tiles_of(I.ffn);
        c1 = nch * 2 * (I.ffn / 16);
        c2 = nch * ((H / 16 + it - 1) / it);
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
  if (npairs <= 32) {
    // ---- small call: warp 0 routes alone (lane p holds pair p), no block syncs
    if (warp == 0) {
      const bool inrange = lane < npairs;
      const int e = inrange ? my_ids[0] : -1;
      const bool ok = e >= 0 && e < E;
      int bad = (inrange && !ok) ? REDLITE_STATUS_BAD_ID : 0;
      const int key = ok ? e : 0x7fffffff;
      int rank = 0;          // position of this pair in (expert, pair index) order
      unsigned less = 0u;    // lanes whose expert id is smaller
#pragma unroll 4
      for (int q = 0; q < 32; ++q) {
        const int kq = __shfl_sync(0xffffffffu, key, q);
        rank += (kq < key) || (kq == key && q < lane);
        less |= (unsigned)(kq < key) << q;
      }
      const unsigned same = __match_any_sync(0xffffffffu, key), lt = (1u << lane) - 1u;
      const bool leader = ok && (same & lt) == 0;
      const unsigned leaders = __ballot_sync(0xffffffffu, leader);
      if (ok) {
        S.pair_tok[rank] = lane / K;
        S.pair_w[rank] = my_w[0];
      }
      if (leader) {
        Inst &I = S.inst[__popc(leaders & less)];
        redlite_moe_expert d;
        memcpy(reinterpret_cast<uint8_t *>(&d), &my_d[0][0], 16);
        memcpy(reinterpret_cast<uint8_t *>(&d) + 16, &my_d[0][1], 16);
        if (expert_ok(d, H, a.max_ffn, true)) {
          I.gate = (const uint8_t *)d.gate, I.up = (const uint8_t *)d.up, I.down = (const uint8_t *)d.down;
          I.qtype = d.qtype, I.ffn = d.ffn, I.count = __popc(same);
        } else {
          bad |= REDLITE_STATUS_BAD_EXPERT;
          I.gate = I.up = I.down = nullptr;
          I.qtype = kQ2, I.ffn = 256, I.count = 0;
        }
        I.pair_start = rank;
      }
      int n_inst = __popc(leaders);
      const int n_routed_pairs = __popc(__ballot_sync(0xffffffffu, ok));
      if (a.has_shared) {
        if (lane == 0) set_shared_inst(S.inst[n_inst], a, n_routed_pairs, bad);
        if (lane < T) S.pair_tok[n_routed_pairs + lane] = lane, S.pair_w[n_routed_pairs + lane] = 1.f;
        n_inst += 1;
      }
      bad = __reduce_or_sync(0xffffffffu, bad);
      if (lane == 0) s_bad = bad;
      __syncwarp();
      item_prefix(n_inst);
      TRACE(2);
      asm volatile("bar.arrive 3, %0;" ::"n"(64) : "memory");  // the routing is published to the producer
    } else if (warp < kCWarps) {
      // meanwhile the other consumer warps turn the (<= 4) tokens'
      // activations into limbs and then (the bulk copy has had time to land)
      // replicate the selector tables
      if (local_x)
        limbs_from_global(T, H, a.x, (size_t)H, 0, S.limbs, lstrideX, S.wmax, S.tok_scale, tid - 32, kCThreads - 32,
                          2);
      if (!mbar_wait(&s_lut_bar, 0) && lane == 0) atomicOr(a.status, REDLITE_STATUS_TIMEOUT);
      TRACE(13);
      replicate_tables<kCThreads - 32, 2>(S, tid - 32);
    } else {
      asm volatile("bar.sync 3, %0;" ::"n"(64) : "memory");  // the producer waits for the routing only
    }
  } else {
    // ---- bucketing: counts per expert in the ring (scratch before any copy)
    uint4 *desc_s = reinterpret_cast<uint4 *>(S.ring);  // [npairs][2]: slot-table entries
    int *cnt = reinterpret_cast<int *>(desc_s + 2 * npairs);  // [E]
    int *first = cnt + E;                                     // [E]: lowest pair index
    int *ids_s = first + E;                                   // [npairs]
    float *w_s = reinterpret_cast<float *>(ids_s + npairs);
    for (int e = tid; e < E; e += kFThreads) cnt[e] = 0, first[e] = 0x7fffffff;
    __syncthreads();
    int bad = 0;
    if (tid < kCThreads) {
#pragma unroll
      for (int j = 0; j < 3; ++j) {
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
    }
    __syncthreads();
    // active experts in ascending id: exclusive scans of (count > 0) and counts
    int n_routed_pairs = 0;
    {
      const int per = (E + kCThreads - 1) / kCThreads;
      const int e0 = tid < kCThreads ? tid * per : E, e1 = min(E, e0 + per);
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
      if (lane == 31 && warp < kCWarps) s_scan[warp] = incl_a, s_scan[16 + warp] = incl_p;
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
      if (tid < kCThreads) {
        int act = s_scan[warp] + incl_a - my_act, pst = s_scan[16 + warp] + incl_p - my_pairs;
        for (int e = e0; e < e1; ++e) {
          if (cnt[e] > 0) {
            Inst &I = S.inst[act];
            redlite_moe_expert d;
            static_assert(sizeof(redlite_moe_expert) == 32, "slot-table entries are two 16-byte words");
            const uint4 d0 = desc_s[2 * first[e]], d1 = desc_s[2 * first[e] + 1];
            memcpy(reinterpret_cast<uint8_t *>(&d), &d0, 16);
            memcpy(reinterpret_cast<uint8_t *>(&d) + 16, &d1, 16);
            const int c = cnt[e];
            if (expert_ok(d, H, a.max_ffn, true)) {
              I.gate = (const uint8_t *)d.gate, I.up = (const uint8_t *)d.up, I.down = (const uint8_t *)d.down;
              I.qtype = d.qtype, I.ffn = d.ffn, I.count = c;
            } else {
              bad |= REDLITE_STATUS_BAD_EXPERT;
              I.gate = I.up = I.down = nullptr;
              I.qtype = kQ2, I.ffn = 256, I.count = 0;
            }
            I.pair_start = pst;
            cnt[e] = pst;  // becomes the running cursor of the stable fill
            ++act;
            pst += c;
          }
        }
      }
      __syncthreads();
      n_routed_pairs = s_scan[32];
    }
    int n_inst = s_n_inst;
    if (warp == kCWarps) {
      // stable fill of the pair list (the producer warp, pairs in index order)
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
    } else {
      if (a.has_shared) {
        if (tid == 0) set_shared_inst(S.inst[n_inst], a, n_routed_pairs, bad);
        for (int t = tid; t < T; t += kCThreads) S.pair_tok[n_routed_pairs + t] = t, S.pair_w[n_routed_pairs + t] = 1.f;
      }
    }
    if (a.has_shared) n_inst += 1;
    if (bad) atomicOr(&s_bad, bad);
    __syncthreads();
    if (warp == 0) item_prefix(n_inst);
    // the ring's bucketing scratch is overwritten by bulk copies next
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    TRACE(2);
  }
  // gate/up items split evenly over the CTAs; down items in reverse CTA order
  // (a CTA with one more gate/up item tends to get one fewer down item).
  // Read once the routing is visible to the reading thread.
  const unsigned uG = (unsigned)G;
  int n_inst = 0, N1 = 0, N2 = 0, b1 = 0, b2 = 0, my1 = 0, my_items = 0;
  auto load_split = [&]() {
    n_inst = s_n_inst, N1 = s_n1, N2 = s_n2;
    const unsigned uN1 = (unsigned)N1, uN2 = (unsigned)N2;  // products < 2^31
    b1 = (int)(cta * uN1 / uG);
    const int e1i = (int)((cta + 1) * uN1 / uG), rc = G - 1 - cta;
    b2 = (int)(rc * uN2 / uG);
    const int e2i = (int)((rc + 1) * uN2 / uG);
    my1 = e1i - b1, my_items = my1 + (e2i - b2);
  };

  // ---- producer warp: streams this CTA's items through the ring
  if (warp == kCWarps) {
    load_split();
    if (lane == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes before bulk copies
      for (int k = 0; k < my_items; ++k) {
        const int s = k % kRing;
        if (k >= kRing && !mbar_wait(&S.empty[s], (uint32_t)(((k / kRing) - 1) & 1))) {
          atomicOr(a.status, REDLITE_STATUS_TIMEOUT);
          break;
        }
        ItemInfo inf;
        const uint8_t *src;
        uint32_t bytes;
        const bool p1 = k < my1;
        const int j = p1 ? b1 + k : b2 + (k - my1);
        int lo = 0, hi = n_inst - 1;  // last instance whose base <= j
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if ((p1 ? S.inst[mid].p1_base : S.inst[mid].p2_base) <= j) lo = mid; else hi = mid - 1;
        }
        const Inst &I = S.inst[lo];
        const int tbb = tile_block_bytes(I.qtype);
        inf.inst = lo;
        if (p1) {
          const int nt = I.ffn / 16, per = 2 * nt, loc = j - I.p1_base;
          inf.phase = 1, inf.chunk = loc / per, inf.sub = (loc % per) / nt, inf.tile = loc % nt;
          bytes = (uint32_t)((H / 256) * tbb);
          src = (inf.sub ? I.up : I.gate) + (size_t)inf.tile * bytes;
        } else {
          const int it = item_tiles_of(I.ffn), ngrp = (H / 16 + it - 1) / it, loc = j - I.p2_base;
          inf.phase = 2, inf.chunk = loc / ngrp, inf.tile = loc % ngrp, inf.sub = 0;
          const int tiles = min(it, H / 16 - inf.tile * it);
          const size_t tile_bytes = (size_t)(I.ffn / 256) * tbb;
          bytes = (uint32_t)(tiles * tile_bytes);
          src = I.down + (size_t)inf.tile * it * tile_bytes;
        }
        S.info[s] = inf;
        mbar_expect_tx(&S.full[s], bytes);
        bulk_g2s(S.ring + (size_t)s * kStageBytes, src, bytes, &S.full[s]);
      }
    }
  } else {
    // ---- consumers: zero this CTA's slice of out (the down items add into
    // it after the grid barrier; out does not overlap the inputs)
    {
      const unsigned total4 = (unsigned)(T * H / 4);
      const unsigned z0 = cta * total4 / uG, z1 = (cta + 1) * total4 / uG;
      for (unsigned i = z0 + tid; i < z1; i += kCThreads)
        reinterpret_cast<float4 *>(a.out)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    // ---- consumers: replicate the selector tables (small calls did it while
    // warp 0 routed)
    if (npairs > 32) {
      if (!mbar_wait(&s_lut_bar, 0) && lane == 0) atomicOr(a.status, REDLITE_STATUS_TIMEOUT);
      TRACE(13);
      replicate_tables<kCThreads, 1>(S, tid);
    }
    // ---- consumers: activations to limbs (locally, or phase 0 cooperative)
    if (local_x) {
      TRACE(12);
      if (npairs > 32)
        limbs_from_global(T, H, a.x, (size_t)H, 0, S.limbs, lstrideX, S.wmax, S.tok_scale, tid, kCThreads, 1);
    } else {
      for (int t = cta; t < T; t += G)
        limbs_from_global(1, H, a.x + (size_t)t * H, 0, 0, glimbs + (size_t)t * 3 * lstrideX, lstrideX, S.wmax,
                          gscale + t, tid, kCThreads, 1);
      consumers_sync();
      if (tid == 0) {
        arrive_release(&ctrl->phase0_done);
        wait_count(&ctrl->phase0_done, G, a.status);
      }
      consumers_sync();
    }
    consumers_sync();  // small calls: warp 0's routing and the other warps' limbs are done
    load_split();
    TRACE(3);

    // ---- main loop over this CTA's items
    int cur_inst = -1, cur_chunk = -1, cur_phase = 0;
    int ntok = 0;
    int slot4 = 0xE4;  // limb slot of token position j of the chunk: bits 2j, 2j + 1
    TRACE_DECL;
    for (int k = 0; k < my_items; ++k) {
      const int s = k % kRing;
      if (k == my1) {
        TRACE(4);
        // grid barrier: every CTA has written its g/u (it arrived when its
        // last gate/up item was reduced) and zeroed its slice of out
        if (my1 == 0) {
          consumers_sync();  // this CTA's zero stores precede the arrival
          if (tid == 0) {
            arrive_release(&ctrl->phase1_done);
          }
        }
        if (tid == 0) wait_count(&ctrl->phase1_done, G, a.status);
        consumers_sync();
        TRACE(5);
      }
      TRACE_T0();
      if (!mbar_wait(&S.full[s], (uint32_t)((k / kRing) & 1))) {
        if (lane == 0) atomicOr(a.status, REDLITE_STATUS_TIMEOUT);
      }
      const ItemInfo inf = S.info[s];
      TRACE_ADD(inf.phase == 1, 0, 1);
      TRACE_CNT(inf.phase == 1, 8, 9);
      TRACE_T0();
      const Inst &I = S.inst[inf.inst];
      const int qtype = I.qtype, F = I.ffn;
      const uint8_t *stage = S.ring + (size_t)s * kStageBytes;
      const int tbb = tile_block_bytes(qtype);
      const int pbase = I.pair_start + kTokChunk * inf.chunk;
      // (re)load the token chunk's limbs when the instance/chunk/phase changes
      if (inf.inst != cur_inst || inf.chunk != cur_chunk || inf.phase != cur_phase) {
        cur_inst = inf.inst, cur_chunk = inf.chunk, cur_phase = inf.phase;
        TRACE_CNT(inf.phase == 1, 10, 11);
        ntok = min(kTokChunk, I.count - kTokChunk * inf.chunk);
        slot4 = 0xE4;
        if (inf.phase == 1) {
          if (local_x) {
            slot4 = 0;  // limbs are indexed by token
            for (int j = 0; j < ntok; ++j) slot4 |= S.pair_tok[pbase + j] << (2 * j);
          } else {
            consumers_sync();  // every warp is done with the previous chunk's limbs
            const int nvec = 3 * lstrideX / 16;  // <= 390 for H <= 2048
            uint4 buf[kTokChunk][2];
#pragma unroll
            for (int j = 0; j < kTokChunk; ++j) {
              const int t = j < ntok ? S.pair_tok[pbase + j] : 0;
              const uint4 *src = reinterpret_cast<const uint4 *>(glimbs + (size_t)t * 3 * lstrideX);
#pragma unroll
              for (int h = 0; h < 2; ++h)
                if (j < ntok && tid + kCThreads * h < nvec) buf[j][h] = __ldcg(src + tid + kCThreads * h);
            }
#pragma unroll
            for (int j = 0; j < kTokChunk; ++j) {
              uint4 *dst = reinterpret_cast<uint4 *>(S.limbs + (size_t)j * 3 * lstrideX);
#pragma unroll
              for (int h = 0; h < 2; ++h)
                if (j < ntok && tid + kCThreads * h < nvec) dst[tid + kCThreads * h] = buf[j][h];
            }
            if (tid < ntok) S.tok_scale[tid] = __ldcg(gscale + S.pair_tok[pbase + tid]);
            consumers_sync();
          }
        } else {
          // h = SiLU(g) * u of the chunk's tokens, then its limbs
          consumers_sync();  // every warp is done with the previous limbs
          limbs_from_global(ntok, F, gu + (size_t)pbase * 2 * a.max_ffn, (size_t)2 * a.max_ffn, a.max_ffn, S.limbs,
                            F + kLimbPad, S.wmax, S.tok_scale, tid, kCThreads, 1);
        }
      }
      TRACE_ADD(inf.phase == 1, 2, 3);
      TRACE_T0();
      float *red = S.red + (size_t)s * kCWarps * 64;
      int nw, lst, kb;  // warps holding partials; limb stride and input offset of this warp
      if (inf.phase == 1) {
        nw = H / 256;  // <= 8: warp w takes input block w
        lst = lstrideX;
        kb = warp * 256;
      } else {
        const int nkb = F >> 8, it = item_tiles_of(F);
        const int tiles = min(it, H / 16 - inf.tile * it);
        nw = tiles * nkb;  // <= 8: warp w takes tile w / nkb, input block w % nkb
        lst = F + kLimbPad;
        kb = ((nkb & (nkb - 1)) == 0 ? (warp & (nkb - 1)) : warp % nkb) * 256;
      }
#ifdef REDLITE_TRACE
      const long long c0 = clock64();
#endif
      if (warp < nw) warp_tile_block(qtype, stage + warp * tbb, S, S.limbs, lst, kb, slot4, ntok, red + warp * 64);
#ifdef REDLITE_TRACE
      const long long tr_tb = clock64();
#endif
      TRACE_ADD(inf.phase == 1, 4, 5);
      TRACE_T0();
      // every warp announces its partials; warp k % 8 reduces the item once
      // all are in and frees the stage (the other warps move on at once)
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.pdone[s]);
      if (warp == k % kCWarps) {
        if (!mbar_wait(&S.pdone[s], (uint32_t)((k / kRing) & 1)) && lane == 0)
          atomicOr(a.status, REDLITE_STATUS_TIMEOUT);
        if (inf.phase == 1) {
          for (int j2 = lane; j2 < 16 * ntok; j2 += 32) {
            const int row = j2 & 15, j = j2 >> 4;
            float v = 0.f;
            for (int w = 0; w < nw; ++w) v += red[w * 64 + row * 4 + j];
            const float sc = S.tok_scale[(slot4 >> (2 * j)) & 3];
            gu[(size_t)(pbase + j) * 2 * a.max_ffn + (size_t)inf.sub * a.max_ffn + inf.tile * 16 + row] = v * sc;
          }
          if (k == my1 - 1) {
            // this CTA's last gate/up item: arrive at the grid barrier (the
            // release is cumulative over the warp's and, through the earlier
            // block barriers, the CTA's stores)
            __syncwarp();
            if (lane == 0) {
              arrive_release(&ctrl->phase1_done);
            }
          }
        } else {
          const int nkb = F >> 8, it = item_tiles_of(F);
          const int tiles = min(it, H / 16 - inf.tile * it);
          const int r0 = inf.tile * it * 16;
          for (int j = 0; j < ntok; ++j) {
            float *orow = a.out + (size_t)S.pair_tok[pbase + j] * H + r0;
            const float wj = S.pair_w[pbase + j] * S.tok_scale[(slot4 >> (2 * j)) & 3];
            for (int rt = lane; rt < tiles * 16; rt += 32) {  // rt = 16 tile + row
              const float *rp = red + (rt >> 4) * nkb * 64 + (rt & 15) * 4 + j;
              float v = 0.f;
              for (int kb = 0; kb < nkb; ++kb) v += rp[kb * 64];
              atomicAdd(orow + rt, wj * v);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[s]);
      }
      TRACE_ADD(inf.phase == 1, 6, 7);
#ifdef REDLITE_TRACE
      if (warp == 0 && k < 5) {  // tile-block start and end, item end (warp 0)
        TRACEC(k * 3, (uint64_t)c0);
        TRACEC(k * 3 + 1, (uint64_t)tr_tb);
        TRACEC(k * 3 + 2, (uint64_t)clock64());
      }
      if (warp == 0 && k == 0) TRACEC(15, (uint64_t)my1);
#endif
    }
    TRACE(9);
    TRACE_FLUSH();
    if (my_items == 0) {
      // no items at all: still count at the barrier (the zero stores first)
      consumers_sync();
      if (tid == 0) {
        arrive_release(&ctrl->phase1_done);
      }
    }
  }
  // ---- exit: the last CTA resets the counters for the next call
  __syncthreads();
  TRACE(6);
  if (tid == 0) {
    __threadfence();
    const int prev = atomicAdd(&ctrl->exit_count, 1);
    if (prev == G - 1) {
      ctrl->phase1_done = 0;
      ctrl->phase0_done = 0;
      __threadfence();
      ctrl->exit_count = 0;
    }
  }
}

size_t fused_smem_bytes(int hidden, int max_ffn) {
  size_t off = 512 * kRep2 * 4 + 256 * kRep2 * 4 + 4096 * kRep1 * 4;
  off += (size_t)kRing * kStageBytes;
  off += sizeof(float) * kRing * kCWarps * 64;
  const int lmax = (hidden > max_ffn ? hidden : max_ffn) + kLimbPad;
  off += (size_t)kTokChunk * 3 * lmax;
  off = (off + 15) & ~size_t(15);
  off += sizeof(Inst) * kFusedMaxInst;
  off += 2 * sizeof(int) * (kFusedMaxPairs + 64);
  off += 3 * sizeof(uint64_t) * kRing + sizeof(ItemInfo) * kRing;
  off += sizeof(float) * kTokChunk + sizeof(float) * kCWarps * 4;
  return off + 64;
}

bool fused_supported(int hidden, int max_ffn, int n_tokens, int top_k, int n_experts, bool has_shared) {
  if (hidden % 256 || hidden > 2048 || max_ffn % 256 || max_ffn > 2048) return false;
  if ((int64_t)n_tokens * top_k > kFusedMaxPairs) return false;
  if (has_shared && n_tokens > 64) return false;
  // bucketing scratch (slot-table entries, counts, first pairs, ids, weights) lives in the ring
  if ((size_t)n_experts * 8 + 40 * (size_t)kFusedMaxPairs > (size_t)kRing * kStageBytes) return false;
  return fused_smem_bytes(hidden, max_ffn) <= 227 * 1024;
}

cudaError_t launch_fused(const FusedArgs &a, cudaStream_t stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const size_t smem = fused_smem_bytes(a.hidden, a.max_ffn);
  e = cudaFuncSetAttribute(decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(kFThreads);
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
  e = cudaLaunchKernelEx(&cfg, decode_fused_kernel, a);
  if (e != cudaSuccess && pdl_ok) {
    (void)cudaGetLastError();
    pdl_ok = false;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_fused_kernel, a);
  }
#ifdef REDLITE_DEBUG_LAUNCH
  if (e != cudaSuccess) fprintf(stderr, "decode_fused_kernel launch: %s\n", cudaGetErrorString(e));
  {
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, decode_fused_kernel);
    int nb = -1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, decode_fused_kernel, kFThreads, smem);
    fprintf(stderr, "regs %d maxThreads %d static smem %zu dyn %zu blocks/SM %d\n", fa.numRegs,
            fa.maxThreadsPerBlock, fa.sharedSizeBytes, smem, nb);
  }
#endif
  return e;
}

}  // namespace redlite
