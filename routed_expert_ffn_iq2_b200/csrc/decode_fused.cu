// decode_fused.cu -- one persistent kernel per decode-sized layer call.
//
// "Red Metal dev8 -- resident routed top-k layer", steps 4-6: every selected
// expert runs gate, up, SiLU(gate)*up and down from its resident slot and
// the layer accumulates out += router_weight * expert_output (plus the
// shared expert with weight 1, "Red Lite dev16", block composition).
//
// Structure (one CTA per SM, cooperative launch so all CTAs are resident):
//   prologue  every CTA copies the byte-permute selector tables into shared
//             memory, buckets the (token, slot) pairs by expert (stable,
//             identical in every CTA), reads the selected slots'
//             descriptors and enumerates the work items;
//   phase 1   gate and up tiles (16 rows x hidden) of every selected expert,
//             split evenly over the CTAs; each tile's packed bytes arrive
//             by TMA bulk copy into a ring of shared-memory stages;
//             results g, u go to the workspace; each CTA also zeroes a
//             slice of `out`;
//   barrier   one grid-wide counter (bounded wait);
//   phase 2   down tiles: h = SiLU(g) * u per token, then y = W_down h and
//             out[token] += weight * y with fp32 atomics.
// Down tiles are prefetched into the ring while phase 1 finishes.
//
// Arithmetic: weights are decoded to exact signed int8 values (IQ2: +-8,
// +-25, +-43; IQ1: 8*(grid + delta) in {+-1, +-7, +-9}) by two byte
// permutes per 8-weight group; activations are split into three signed
// 7-bit limbs of a 21-bit fixed-point value with a per-token power-of-two
// scale; the products run on the tensor cores (mma.sync s8, int32
// accumulation), the sub-block multiplier (2sc+1) is applied in int32 per
// sub-block and the block scale d in fp32 per 256 weights.  The only
// rounding is the activations' 2^-21 relative quantisation and fp32 sums.
#include "internal.cuh"

namespace redlite {

constexpr int kFThreads = 256;
constexpr int kFWarps = kFThreads / 32;
constexpr int kRing = 6;
constexpr int kStageBytes = 8 * kQ2TileBlock;  // 9472 >= 8 * kQ1TileBlock
constexpr int kTokChunk = 4;
constexpr int kRep2 = 16;  // replicas of the IQ2 selector/sign tables (bank spread)
constexpr int kRep1 = 2;   // replicas of the IQ1 selector table
constexpr int kFusedMaxInst = kFusedMaxPairs + 2;
constexpr int kLimbPad = 32;  // padding per limb plane (spreads shared-memory banks)
constexpr uint32_t kSpinLimit = 1u << 24;

// 8-byte tables the selector nibbles index: IQ2 +8,+25,+43,0,-8,-25,-43,0;
// IQ1 (delta +1/8) -7,1,9,0 and (delta -1/8) -9,-1,7,0, all scaled by 8.
constexpr uint32_t kQ2Pos = 0x002B1908u, kQ2Neg = 0x00D5E7F8u;
constexpr uint32_t kQ1Pos = 0x000901F9u, kQ1Neg = 0x0007FFF7u;

struct Inst {          // one selected expert (or the shared expert)
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
  uint8_t *limbs;
  Inst *inst;
  int *pair_tok;
  float *pair_w;
  float *red;
  uint64_t *full;
  ItemInfo *info;
  int *tok_exp;
};

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
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

__device__ __forceinline__ void mma_k32(int32_t d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

__device__ __forceinline__ void mma_k16(int32_t d[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5}, {%6}, {%7,%7,%7,%7};"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(a0), "r"(a1), "r"(b0), "r"(0));
}

__device__ __forceinline__ float half_bits(uint32_t h) { return __half2float(__ushort_as_half((unsigned short)h)); }

// ------------------------------------------------------------------ tile-block math
//
// Column n of the mma B operand (n = lane >> 2 of the lane holding it) is
// limb n % 3 of token position 2p + n / 3 of the chunk (n < 6); columns 6
// and 7 are zero.  Each lane gets, per token pair p, a pointer to the limb
// plane it reads (nullptr: a zero column).  Limb planes are int8 vectors.
template <int NP>
__device__ __forceinline__ void b_planes(const uint8_t *limbs, int lstride, const int slots[4], int ntok,
                                         const uint8_t *bp[NP]) {
  const int n = (threadIdx.x & 31) >> 2;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int pos = 2 * p + n / 3;
    bp[p] = (n < 6 && pos < ntok) ? limbs + (size_t)(slots[pos] * 3 + n % 3) * lstride : nullptr;
  }
}

// IQ2_XS-style tile-block (16 rows x 256 inputs): acc[p][.] += partial dot
// products of the block's rows with token pair p (mma C layout, limb columns).
template <int NP>
__device__ __forceinline__ void tb_q2(const uint8_t *__restrict__ tb, const uint32_t *__restrict__ sel2,
                                      const uint32_t *__restrict__ sgn2, const uint8_t *const bp[NP], int kbase,
                                      float acc[NP][4]) {
  const int lane = threadIdx.x & 31, q = lane >> 2, t = lane & 3, r = lane & (kRep2 - 1);
  const uint4 qs = *reinterpret_cast<const uint4 *>(tb + 32 * lane);
  const uint4 sg = *reinterpret_cast<const uint4 *>(tb + 32 * lane + 16);
  const uint32_t qh = *reinterpret_cast<const uint16_t *>(tb + 1024 + 2 * lane);
  const uint2 scw = *reinterpret_cast<const uint2 *>(tb + 1088 + 8 * q);
  const uint32_t dw = *reinterpret_cast<const uint32_t *>(tb + 1152 + 4 * q);
  const uint32_t qsw[4] = {qs.x, qs.y, qs.z, qs.w};
  const uint32_t sgw[4] = {sg.x, sg.y, sg.z, sg.w};
  int32_t cb[NP][4];
#pragma unroll
  for (int p = 0; p < NP; ++p) cb[p][0] = cb[p][1] = cb[p][2] = cb[p][3] = 0;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t a[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = 2 * c + h;
      const uint32_t qsb = (qsw[i >> 2] >> (8 * (i & 3))) & 0xFFu;
      const uint32_t idx = qsb | (((qh >> i) & 1u) << 8);
      const uint32_t sgb = (sgw[i >> 2] >> (8 * (i & 3))) & 0xFFu;
      const uint32_t sel = sel2[idx * kRep2 + r] | sgn2[sgb * kRep2 + r];
      a[h] = __byte_perm(kQ2Pos, kQ2Neg, sel);
      a[2 + h] = __byte_perm(kQ2Pos, kQ2Neg, sel >> 16);
    }
    const int m0 = 2 * (int)((scw.x >> (4 * c)) & 15u) + 1;
    const int m1 = 2 * (int)((scw.y >> (4 * c)) & 15u) + 1;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const uint2 b = bp[p] ? *reinterpret_cast<const uint2 *>(bp[p] + kbase + 32 * c + 8 * t) : make_uint2(0u, 0u);
      int32_t d[4];
      mma_k32(d, a, b.x, b.y);
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
__device__ __forceinline__ void tb_q1(const uint8_t *__restrict__ tb, const uint32_t *__restrict__ sel1,
                                      const uint8_t *const bp[NP], int kbase, float acc[NP][4]) {
  const int lane = threadIdx.x & 31, q = lane >> 2, t = lane & 3, r = lane & (kRep1 - 1);
  const uint8_t *pb = tb + 48 * (2 * q + (t >> 1));
  const uint4 qa = *reinterpret_cast<const uint4 *>(pb);
  const uint4 qb = *reinterpret_cast<const uint4 *>(pb + 16);
  const uint4 nb = *reinterpret_cast<const uint4 *>(pb + 32);
  const uint32_t *scp = reinterpret_cast<const uint32_t *>(tb + 768 + 12 * q);
  const uint32_t s0 = scp[0], s1 = scp[1], s2 = scp[2];
  const uint64_t row0 = (uint64_t)s0 | ((uint64_t)(s1 & 0xFFFFu) << 32);
  const uint64_t row1 = (uint64_t)(s1 >> 16) | ((uint64_t)s2 << 16);
  const uint32_t dw = *reinterpret_cast<const uint32_t *>(tb + 864 + 4 * q);
  const uint32_t qsw[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
  const uint32_t nbw[4] = {nb.x, nb.y, nb.z, nb.w};
  const int hshift = 16 * (t & 1);
  int32_t cb[NP][4];
#pragma unroll
  for (int p = 0; p < NP; ++p) cb[p][0] = cb[p][1] = cb[p][2] = cb[p][3] = 0;
#pragma unroll
  for (int s = 0; s < 16; ++s) {
    uint32_t a[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = 2 * s + h;
      const uint32_t qsb = (qsw[i >> 2] >> (8 * (i & 3))) & 0xFFu;
      const uint32_t nib = (nbw[i >> 3] >> (4 * (i & 7))) & 0xFu;
      const uint32_t sel = sel1[(qsb | (nib << 8)) * kRep1 + r];
      a[h] = __byte_perm(kQ1Pos, kQ1Neg, sel >> hshift);
    }
    const int m0 = 2 * (int)((row0 >> (3 * s)) & 7u) + 1;
    const int m1 = 2 * (int)((row1 >> (3 * s)) & 7u) + 1;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const uint32_t b = bp[p] ? *reinterpret_cast<const uint32_t *>(bp[p] + kbase + 16 * s + 4 * t) : 0u;
      int32_t d[4];
      mma_k16(d, a[0], a[1], b);
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

// Combine the limb columns of each token and store the warp's partial sums:
// red[warp][row 0..15][token slot 0..3].
template <int NP>
__device__ __forceinline__ void store_partials(const float acc[NP][4], float *red) {
  const int lane = threadIdx.x & 31, q = lane >> 2, t = lane & 3, w = threadIdx.x >> 5;
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
      float *rw = red + w * 64;
      rw[q * 4 + 2 * p] = v[0];
      rw[q * 4 + 2 * p + 1] = v[1];
      rw[(q + 8) * 4 + 2 * p] = v[2];
      rw[(q + 8) * 4 + 2 * p + 1] = v[3];
    }
  }
}

// Run one tile-block of either format for up to 4 token positions and
// store this warp's partials.
__device__ __forceinline__ void warp_tile_block(int qtype, const uint8_t *tb, const Smem &S, const uint8_t *limbs,
                                                int lstride, int kbase, const int slots[4], int ntok) {
  if (ntok <= 2) {
    const uint8_t *bp[1];
    b_planes<1>(limbs, lstride, slots, ntok, bp);
    float acc[1][4] = {{0.f, 0.f, 0.f, 0.f}};
    if (qtype == kQ2)
      tb_q2<1>(tb, S.sel2, S.sgn2, bp, kbase, acc);
    else
      tb_q1<1>(tb, S.sel1, bp, kbase, acc);
    store_partials<1>(acc, S.red);
  } else {
    const uint8_t *bp[2];
    b_planes<2>(limbs, lstride, slots, ntok, bp);
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    if (qtype == kQ2)
      tb_q2<2>(tb, S.sel2, S.sgn2, bp, kbase, acc);
    else
      tb_q1<2>(tb, S.sel1, bp, kbase, acc);
    store_partials<2>(acc, S.red);
  }
}

// Fixed-point limbs of one vector v[0..n) (n a multiple of 32) by one warp:
// X = round(v * 2^(20-e)) with 2^e > max|v|, X = l0*2^14 + l1*2^7 + l2,
// each limb in [-64, 64].  Returns e.
__device__ int warp_limbs(const float *v, int n, uint8_t *dst, int lstride) {
  const int lane = threadIdx.x & 31;
  float m = 0.f;
  for (int i = lane; i < n; i += 32) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  int e = 0;
  if (m > 0.f) frexpf(m, &e);  // m < 2^e
  for (int i = lane; i < n; i += 32) {
    const int X = __float2int_rn(ldexpf(v[i], 20 - e));
    const int l2 = ((X + 64) & 127) - 64;
    const int X1 = (X - l2) >> 7;
    const int l1 = ((X1 + 64) & 127) - 64;
    const int l0 = (X1 - l1) >> 7;
    dst[i] = (uint8_t)(int8_t)l0;
    dst[lstride + i] = (uint8_t)(int8_t)l1;
    dst[2 * lstride + i] = (uint8_t)(int8_t)l2;
  }
  return e;
}

__device__ __forceinline__ float exp2i(int e) { return ldexpf(1.0f, e); }

// ------------------------------------------------------------------ the kernel

__device__ bool fused_expert_ok(const redlite_moe_expert &e, int hidden, int max_ffn) {
  if (!e.gate || !e.up || !e.down) return false;
  if (e.qtype != kQ2 && e.qtype != kQ1) return false;
  if (e.ffn <= 0 || e.ffn > max_ffn || e.ffn % 256) return false;
  if (((uintptr_t)e.gate | (uintptr_t)e.up | (uintptr_t)e.down) & 15) return false;
  return shape_ok(e.ffn, hidden) && shape_ok(hidden, e.ffn);
}

__device__ __forceinline__ int item_tiles_of(int ffn) {
  const int nkb = ffn / 256;
  return nkb >= 8 ? 1 : 8 / nkb;
}

__global__ void __launch_bounds__(kFThreads, 1) decode_fused_kernel(FusedArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int H = a.hidden, T = a.n_tokens, K = a.top_k, E = a.n_experts;
  const int npairs = T * K;
  const int lstrideX = H + kLimbPad;
  Ctrl *ctrl = reinterpret_cast<Ctrl *>(a.ws + a.L.ctrl);
  float *gu = reinterpret_cast<float *>(a.ws + a.L.gu);
  uint8_t *glimbs = a.ws + a.L.limbs;
  int *gexps = reinterpret_cast<int *>(a.ws + a.L.exps);

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
  S.red = reinterpret_cast<float *>(smem + off);
  off += sizeof(float) * kFWarps * 64;
  S.full = reinterpret_cast<uint64_t *>(smem + off);
  off += sizeof(uint64_t) * kRing;
  S.info = reinterpret_cast<ItemInfo *>(smem + off);
  off += sizeof(ItemInfo) * kRing;
  S.tok_exp = reinterpret_cast<int *>(smem + off);
  off += sizeof(int) * kTokChunk;
  __shared__ int s_n_inst, s_n1, s_n2, s_bad, s_scan[33];

  // ---- prologue: selector tables with replication, barriers
  {
    const uint32_t *g2 = reinterpret_cast<const uint32_t *>(a.grids + kGridQ2Sel);
    const uint32_t *gs = reinterpret_cast<const uint32_t *>(a.grids + kGridSign);
    const uint32_t *g1 = reinterpret_cast<const uint32_t *>(a.grids + kGridQ1Sel);
    for (int i = tid; i < 512 * kRep2; i += kFThreads) S.sel2[i] = g2[i / kRep2];
    for (int i = tid; i < 256 * kRep2; i += kFThreads) S.sgn2[i] = gs[i / kRep2];
    for (int i = tid; i < 4096 * kRep1; i += kFThreads) S.sel1[i] = g1[i / kRep1];
  }
  if (tid == 0) {
    for (int s = 0; s < kRing; ++s) mbar_init(&S.full[s], 1);
    mbar_fence_init();
    s_bad = 0;
  }

  // ---- bucketing: counts per expert in the ring (scratch before any copy)
  int *cnt = reinterpret_cast<int *>(S.ring);  // [E]
  int *ids_s = cnt + E;                        // [npairs]
  for (int e = tid; e < E; e += kFThreads) cnt[e] = 0;
  __syncthreads();
  int bad = 0;
  for (int p = tid; p < npairs; p += kFThreads) {
    const int e = a.ids[p];
    ids_s[p] = e;
    if (e < 0 || e >= E) {
      bad |= REDLITE_STATUS_BAD_ID;
      continue;
    }
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  // active experts in ascending id: exclusive scans of (count > 0) and counts
  {
    const int per = (E + kFThreads - 1) / kFThreads;
    const int e0 = tid * per, e1 = min(E, e0 + per);
    int my_act = 0, my_pairs = 0;
    for (int e = e0; e < e1; ++e) {
      my_act += cnt[e] > 0;
      my_pairs += cnt[e];
    }
    // two block scans (warp shuffles + one shared array)
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
      for (int w = 0; w < kFWarps; ++w) {
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
        Inst &I = S.inst[act];
        I.qtype = e;  // expert id for now; descriptor below
        I.pair_start = pst;
        I.count = cnt[e];
        cnt[e] = pst;  // becomes the running cursor of the stable fill
        ++act;
        pst += I.count;
      }
    }
  }
  __syncthreads();
  const int n_routed_pairs = s_scan[32];
  // stable fill of the pair list (one warp, pairs in index order)
  if (warp == 0) {
    for (int p0 = 0; p0 < npairs; p0 += 32) {
      const int p = p0 + lane;
      const int e = p < npairs ? ids_s[p] : -1;
      const bool ok = e >= 0 && e < E;
      const unsigned m = __match_any_sync(0xffffffffu, ok ? e : -1);
      if (ok) {
        const int rank = __popc(m & ((1u << lane) - 1u));
        const int pos = cnt[e] + rank;
        S.pair_tok[pos] = p / K;
        S.pair_w[pos] = a.weights[p];
      }
      __syncwarp();
      if (ok && (m & ((1u << lane) - 1u)) == 0) cnt[e] += __popc(m);
      __syncwarp();
    }
  }
  // descriptors; the shared expert is the last instance
  int n_inst = s_n_inst;
  for (int u = tid; u < n_inst; u += kFThreads) {
    Inst &I = S.inst[u];
    const redlite_moe_expert d = a.experts[I.qtype];
    if (fused_expert_ok(d, H, a.max_ffn)) {
      I.gate = (const uint8_t *)d.gate, I.up = (const uint8_t *)d.up, I.down = (const uint8_t *)d.down;
      I.qtype = d.qtype, I.ffn = d.ffn;
    } else {
      bad |= REDLITE_STATUS_BAD_EXPERT;
      I.gate = I.up = I.down = nullptr;
      I.qtype = kQ2, I.ffn = 256, I.count = 0;
    }
  }
  if (a.has_shared && tid == 0) {
    Inst &I = S.inst[n_inst];
    I.gate = (const uint8_t *)a.shared.gate, I.up = (const uint8_t *)a.shared.up;
    I.down = (const uint8_t *)a.shared.down, I.qtype = a.shared.qtype, I.ffn = a.shared.ffn;
    I.pair_start = n_routed_pairs, I.count = T;
  }
  if (a.has_shared)
    for (int t = tid; t < T; t += kFThreads) S.pair_tok[n_routed_pairs + t] = t, S.pair_w[n_routed_pairs + t] = 1.f;
  if (a.has_shared) n_inst += 1;
  if (bad) atomicOr(&s_bad, bad);
  __syncthreads();
  // work items per instance and their prefix sums (thread 0; n_inst is small)
  if (tid == 0) {
    int n1 = 0, n2 = 0;
    for (int u = 0; u < n_inst; ++u) {
      Inst &I = S.inst[u];
      const int nch = (I.count + kTokChunk - 1) / kTokChunk;
      const int it = item_tiles_of(I.ffn);
      const int ngrp = (H / 16 + it - 1) / it;
      I.p1_base = n1, I.p2_base = n2;
      n1 += nch * 2 * (I.ffn / 16);
      n2 += nch * ngrp;
    }
    s_n1 = n1, s_n2 = n2;
    if (s_bad) atomicOr(a.status, s_bad);
  }
  __syncthreads();
  const int N1 = s_n1, N2 = s_n2;
  const int b1 = (int)((int64_t)cta * N1 / G), e1i = (int)((int64_t)(cta + 1) * N1 / G);
  const int rc = G - 1 - cta;
  const int b2 = (int)((int64_t)rc * N2 / G), e2i = (int)((int64_t)(rc + 1) * N2 / G);
  const int my1 = e1i - b1, my2 = e2i - b2, my_items = my1 + my2;

  // ---- item lookup: instance of global phase item j (binary search on bases)
  auto find_inst = [&](int j, int phase) {
    int lo = 0, hi = n_inst - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      const int base = phase == 1 ? S.inst[mid].p1_base : S.inst[mid].p2_base;
      if (base <= j) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  // issue item k of this CTA into its ring stage (thread 0 only)
  auto issue = [&](int k) {
    const int s = k % kRing;
    ItemInfo inf;
    const uint8_t *src;
    uint32_t bytes;
    if (k < my1) {
      const int j = b1 + k, u = find_inst(j, 1);
      const Inst &I = S.inst[u];
      const int per = 2 * (I.ffn / 16), loc = j - I.p1_base;
      inf.phase = 1, inf.inst = u, inf.chunk = loc / per;
      const int rem = loc % per;
      inf.sub = rem / (I.ffn / 16), inf.tile = rem % (I.ffn / 16);
      const int tbb = tile_block_bytes(I.qtype);
      bytes = (uint32_t)((H / 256) * tbb);
      src = (inf.sub ? I.up : I.gate) + (size_t)inf.tile * bytes;
    } else {
      const int j = b2 + (k - my1), u = find_inst(j, 2);
      const Inst &I = S.inst[u];
      const int it = item_tiles_of(I.ffn), ngrp = (H / 16 + it - 1) / it, loc = j - I.p2_base;
      inf.phase = 2, inf.inst = u, inf.chunk = loc / ngrp, inf.tile = loc % ngrp, inf.sub = 0;
      const int tiles = min(it, H / 16 - inf.tile * it);
      const int tbb = tile_block_bytes(I.qtype);
      const size_t tile_bytes = (size_t)(I.ffn / 256) * tbb;
      bytes = (uint32_t)(tiles * tile_bytes);
      src = I.down + (size_t)inf.tile * it * tile_bytes;
    }
    S.info[s] = inf;
    mbar_expect_tx(&S.full[s], bytes);
    bulk_g2s(S.ring + (size_t)s * kStageBytes, src, bytes, &S.full[s]);
  };

  // ---- activations: T <= chunk: every CTA builds all limbs locally;
  // otherwise phase 0 converts tokens cooperatively into the workspace.
  const bool local_x = T <= kTokChunk;
  __syncthreads();  // the ring scratch (counts, ids) is dead from here on
  if (tid == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes before bulk copies
    for (int k = 0; k < min(kRing, my_items); ++k) issue(k);
  }
  if (local_x) {
    for (int t = warp; t < T; t += kFWarps) {
      const int e = warp_limbs(a.x + (size_t)t * H, H, S.limbs + (size_t)t * 3 * lstrideX, lstrideX);
      if (lane == 0) S.tok_exp[t] = e;
    }
  } else {
    for (int t = cta * kFWarps + warp; t < T; t += G * kFWarps) {
      const int e = warp_limbs(a.x + (size_t)t * H, H, glimbs + (size_t)t * 3 * lstrideX, lstrideX);
      if (lane == 0) gexps[t] = e;
    }
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      atomicAdd(&ctrl->phase0_done, 1);
      uint32_t it = 0;
      while (ld_acquire(&ctrl->phase0_done) < G) {
        if (++it > kSpinLimit) {
          atomicOr(a.status, REDLITE_STATUS_TIMEOUT);
          break;
        }
        __nanosleep(64);
      }
    }
  }
  __syncthreads();

  // ---- main loop over this CTA's items
  int cur_inst = -1, cur_chunk = -1, cur_phase = 0;
  int ntok = 0;
  int slots[kTokChunk] = {0, 0, 0, 0};  // limb slot of each token position of the chunk
  for (int k = 0; k < my_items; ++k) {
    const int s = k % kRing;
    if (k == my1) {
      // end of phase 1: zero a slice of out, then the grid barrier
      const size_t total4 = (size_t)T * H / 4;
      const size_t z0 = total4 * cta / G, z1 = total4 * (cta + 1) / G;
      for (size_t i = z0 + tid; i < z1; i += kFThreads) reinterpret_cast<float4 *>(a.out)[i] = make_float4(0, 0, 0, 0);
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        atomicAdd(&ctrl->phase1_done, 1);
        uint32_t it = 0;
        while (ld_acquire(&ctrl->phase1_done) < G) {
          if (++it > kSpinLimit) {
            atomicOr(a.status, REDLITE_STATUS_TIMEOUT);
            break;
          }
          __nanosleep(32);
        }
        __threadfence();
      }
      __syncthreads();
    }
    // wait for this stage's bytes (bounded)
    {
      uint32_t it = 0;
      const uint32_t parity = (uint32_t)((k / kRing) & 1);
      while (!mbar_try_wait(&S.full[s], parity)) {
        if (++it > kSpinLimit) {
          if (tid == 0) atomicOr(a.status, REDLITE_STATUS_TIMEOUT);
          break;
        }
      }
    }
    const ItemInfo inf = S.info[s];
    const Inst I = S.inst[inf.inst];
    const uint8_t *stage = S.ring + (size_t)s * kStageBytes;
    const int tbb = tile_block_bytes(I.qtype);
    const int pbase = I.pair_start + kTokChunk * inf.chunk;
    // (re)load the token chunk's limbs when the instance/chunk/phase changes
    if (inf.inst != cur_inst || inf.chunk != cur_chunk || inf.phase != cur_phase) {
      cur_inst = inf.inst, cur_chunk = inf.chunk, cur_phase = inf.phase;
      ntok = min(kTokChunk, I.count - kTokChunk * inf.chunk);
      for (int j = 0; j < kTokChunk; ++j) slots[j] = j;
      if (inf.phase == 1) {
        if (local_x) {
          for (int j = 0; j < ntok; ++j) slots[j] = S.pair_tok[pbase + j];  // limbs are indexed by token
        } else {
          const int nvec = 3 * lstrideX / 16;
          for (int j = 0; j < ntok; ++j) {
            const int t = S.pair_tok[pbase + j];
            const uint4 *src = reinterpret_cast<const uint4 *>(glimbs + (size_t)t * 3 * lstrideX);
            uint4 *dst = reinterpret_cast<uint4 *>(S.limbs + (size_t)j * 3 * lstrideX);
            for (int v = tid; v < nvec; v += kFThreads) dst[v] = __ldcg(src + v);
            if (tid == 0) S.tok_exp[j] = __ldcg(gexps + t);
          }
        }
      } else {
        // h = SiLU(g) * u for each token of the chunk, then its limbs
        const int F = I.ffn, lstrideH = F + kLimbPad;
        for (int j = warp; j < ntok; j += kFWarps) {
          const float *g = gu + (size_t)(pbase + j) * 2 * a.max_ffn;
          const float *u = g + a.max_ffn;
          float m = 0.f;
          for (int i = lane; i < F; i += 32) m = fmaxf(m, fabsf(silu_mul(__ldcg(g + i), __ldcg(u + i))));
#pragma unroll
          for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          int e = 0;
          if (m > 0.f) frexpf(m, &e);
          uint8_t *dst = S.limbs + (size_t)j * 3 * lstrideH;
          for (int i = lane; i < F; i += 32) {
            const int X = __float2int_rn(ldexpf(silu_mul(__ldcg(g + i), __ldcg(u + i)), 20 - e));
            const int l2 = ((X + 64) & 127) - 64;
            const int X1 = (X - l2) >> 7;
            const int l1 = ((X1 + 64) & 127) - 64;
            const int l0 = (X1 - l1) >> 7;
            dst[i] = (uint8_t)(int8_t)l0;
            dst[lstrideH + i] = (uint8_t)(int8_t)l1;
            dst[2 * lstrideH + i] = (uint8_t)(int8_t)l2;
          }
          if (lane == 0) S.tok_exp[j] = e;
        }
      }
      __syncthreads();
    }
    if (inf.phase == 1) {
      // one 16-row tile of gate or up: warp w takes input blocks w, w+8, ...
      const int nkb = H / 256;
      if (warp < nkb) {
        for (int kb = warp; kb < nkb; kb += kFWarps) {
          // warps with several input blocks accumulate through the partials
          // area: only H <= 2048 is routed here, so kb == warp
          warp_tile_block(I.qtype, stage + kb * tbb, S, S.limbs, lstrideX, kb * 256, slots, ntok);
        }
      }
      __syncthreads();
      if (tid < 16 * ntok) {
        const int row = tid & 15, j = tid >> 4;
        float v = 0.f;
        for (int w = 0; w < min(nkb, kFWarps); ++w) v += S.red[w * 64 + row * 4 + j];
        gu[(size_t)(pbase + j) * 2 * a.max_ffn + (size_t)inf.sub * a.max_ffn + inf.tile * 16 + row] =
            v * exp2i(S.tok_exp[slots[j]] - 20);
      }
    } else {
      // a group of down tiles: warp w takes tile-block w (tile w / nkb, input block w % nkb)
      const int F = I.ffn, nkb = F / 256, lstrideH = F + kLimbPad;
      const int it = item_tiles_of(F);
      const int tiles = min(it, H / 16 - inf.tile * it);
      const int ntb = tiles * nkb;  // <= 8
      if (warp < ntb) warp_tile_block(I.qtype, stage + warp * tbb, S, S.limbs, lstrideH, (warp % nkb) * 256, slots, ntok);
      __syncthreads();
      for (int j2 = tid; j2 < tiles * 16 * ntok; j2 += kFThreads) {
        const int j = j2 % ntok, rt = j2 / ntok;
        const int tile = rt / 16, row = rt % 16;
        float v = 0.f;
        for (int kb = 0; kb < nkb; ++kb) v += S.red[(tile * nkb + kb) * 64 + row * 4 + j];
        const int r = (inf.tile * it + tile) * 16 + row;
        const float y = v * exp2i(S.tok_exp[j] - 20);
        atomicAdd(a.out + (size_t)S.pair_tok[pbase + j] * H + r, S.pair_w[pbase + j] * y);
      }
    }
    __syncthreads();  // stage and partials consumed
    if (tid == 0 && k + kRing < my_items) issue(k + kRing);
  }
  if (my1 == my_items) {
    // no phase-2 items: still zero the slice and pass the barrier
    const size_t total4 = (size_t)T * H / 4;
    const size_t z0 = total4 * cta / G, z1 = total4 * (cta + 1) / G;
    for (size_t i = z0 + tid; i < z1; i += kFThreads) reinterpret_cast<float4 *>(a.out)[i] = make_float4(0, 0, 0, 0);
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      atomicAdd(&ctrl->phase1_done, 1);
    }
  }
  // ---- exit: the last CTA resets the counters for the next call
  __syncthreads();
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
  const int lmax = (hidden > max_ffn ? hidden : max_ffn) + kLimbPad;
  off += (size_t)kTokChunk * 3 * lmax;
  off = (off + 15) & ~size_t(15);
  off += sizeof(Inst) * kFusedMaxInst;
  off += 2 * sizeof(int) * (kFusedMaxPairs + 64);
  off += sizeof(float) * kFWarps * 64 * 2;
  off += sizeof(uint64_t) * kRing + sizeof(ItemInfo) * kRing + sizeof(int) * kTokChunk;
  return off + 64;
}

bool fused_supported(int hidden, int max_ffn, int n_tokens, int top_k, int n_experts, bool has_shared) {
  if (hidden % 256 || hidden > 2048 || max_ffn % 256 || max_ffn > 2048) return false;
  if ((int64_t)n_tokens * top_k > kFusedMaxPairs) return false;
  if (has_shared && n_tokens > 64) return false;
  if (n_experts > (kRing * kStageBytes) / 4 - kFusedMaxPairs) return false;
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
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_fused_kernel, a);
}

}  // namespace redlite
