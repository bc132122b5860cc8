// grouped_tc.cu -- the bucketed tensor-core path for calls with many tokens
// per expert (prefill).
//
// "Red Metal dev8 -- resident routed top-k layer", steps 4-6, for a batch of
// tokens: the (token, slot) pairs are bucketed by expert (route.cu), then
// every expert's gate/up and down projections run as dense contractions on
// the 5th-generation tensor cores (tcgen05.mma, bf16 operands, fp32
// accumulators in tensor memory).  Weights are decoded from the packed
// tile-blocks straight into tensor memory (each weight is exact in fp32 and
// rounded to bf16, nearest even), where the MMA reads its A operand; the
// activations (B) are rounded to bf16 the same way and staged in shared
// memory.  Accumulation is fp32.
//
// Work unit: (expert, 128 output rows, up to 128 of the expert's tokens).
//   gate/up  A = the rows of gate and of up, B = the tokens' activations;
//            D_gate, D_up in TMEM; epilogue h = SiLU(g) * u (bf16) per pair;
//   down     A = the rows of down, B = the pairs' h; epilogue out += w * D
//            with fp32 atomics.
// One persistent CTA per SM takes units cta, cta + grid, ...; its warps:
//   warp 0      one thread bulk-copies the packed tile-blocks of each
//               256-input column of a unit (8 per matrix) into a 2-deep ring;
//   warp 1      one thread issues the tcgen05.mma of every 64-input step and
//               commits them to the step's slot and, per unit, to an
//               accumulator buffer (one for gate/up, two for down);
//   warps 2-9   dequant warps: each decodes one tile-block (16 rows) of each
//               matrix, in the TMEM lane quarter its warp index may write,
//               into the A slots of a 4-step ring in tensor memory
//               (tcgen05.st), and fetches 16 rows of B with cp.async into the
//               matching shared-memory slot, a step ahead;
//   warps 10-13 the epilogue (TMEM -> registers -> h or out).
//
// Input order inside a 64-input step.  A thread of the 16-lane TMEM store
// holds four consecutive K positions of its two rows per 16-position chunk,
// and decodes 8-weight groups t and t + 4 of the step (t = lane % 4).  So
// TMEM position 32 c + 16 j + 4 t + i holds input 32 c + 8 t + 4 j + i of
// the step (c, j in {0, 1}, i < 4), and the bf16 copies of x and of h that
// B is loaded from are stored in that same order (perm64): the contraction
// over a step is a sum over all 64 inputs either way.
#include "internal.cuh"
#include "layout.cuh"
#include "ptx.cuh"

namespace redlite {
namespace {

constexpr int kDqWarps = 8;
constexpr int kEpWarps = 4;
constexpr int kTcWarps = 2 + kDqWarps + kEpWarps;
constexpr int kTcThreads = 32 * kTcWarps;  // 448
constexpr int kBTile = 128 * 64 * 2;       // 16 KB: up to 128 token rows x 64 bf16
constexpr int kPr = 2;                     // packed columns in flight
constexpr int kMaxUnits = 128;             // unit records per pass
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 256;         // accumulators in columns 0..255, A slots above

// Optional per-warp cycle counters (build with -DREDLITE_TC_TRACE): CTA c,
// warp w adds to 8 words at the end of the workspace layout, slot (c * 32 + w) * 8.
#ifdef REDLITE_TC_TRACE
#define TC_T0() const long long tc_t0_ = clock64()
#define TC_ADD(i) tc_acc_[i] += clock64() - tc_t0_
#define TC_DECL long long tc_acc_[8] = {0, 0, 0, 0, 0, 0, 0, 0}; const long long tc_start_ = clock64()
#define TC_FLUSH()                                                                                   \
  do {                                                                                               \
    tc_acc_[7] = clock64() - tc_start_;                                                              \
    if (lane == 0)                                                                                   \
      for (int i_ = 0; i_ < 8; ++i_)                                                                 \
        reinterpret_cast<long long *>(a.ws + a.L.total)[((size_t)(DOWN * 148 + blockIdx.x) * 32 + warp) * 8 + i_] += \
            tc_acc_[i_];                                                                             \
  } while (0)
#else
#define TC_T0()
#define TC_ADD(i)
#define TC_DECL
#define TC_FLUSH()
#endif

template <bool DOWN>
struct Cfg {
  static constexpr int kMats = DOWN ? 1 : 2;
  static constexpr int kAr = 4;                             // 64-input steps in flight
  static constexpr int kStep = kBTile;                      // shared memory per step: the B tile
  static constexpr int kPacked = kMats * 8 * kQ2TileBlock;  // one column, largest format
  static constexpr uint32_t kSlotCols = kMats * 32;         // TMEM columns of one step's A tiles
  static_assert(kAccCols + kAr * kSlotCols <= kTmemCols, "TMEM columns");
};

// Accumulator columns of a unit.  down: buffer b = unit count mod 2, columns
// 128 b ..  gate/up: two halves, half b = gate columns 64 b .. 64 b + 63 and
// up columns 128 + 64 b ..; a unit of at most 64 tokens takes the next half
// in turn, a larger one both (gate 0 .., up 128 ..).  The MMA thread and the
// epilogue warps replay the same sequence; mask: the halves the unit holds.
struct AccPlan {
  uint32_t gate, up;
  int mask;
};
template <bool DOWN>
__device__ __forceinline__ AccPlan acc_plan(int n_pad, uint32_t ucount, int &next) {
  AccPlan p;
  if (DOWN) {
    const int b = (int)(ucount & 1u);
    p.gate = 128u * b, p.up = 0u, p.mask = 1 << b;
  } else if (n_pad <= 64) {
    p.gate = 64u * next, p.up = 128u + 64u * next, p.mask = 1 << next;
    next ^= 1;
  } else {
    p.gate = 0u, p.up = 128u, p.mask = 3;
    next = 0;
  }
  return p;
}

// Position of input `in` of a 64-input step in the order the tensor-core
// kernels contract over (see the header): bit 2 moves to bit 4, bits 3-4 to bits 2-3.
__host__ __device__ __forceinline__ int perm64(int in) {
  return (in & ~31) | ((in & 4) << 2) | ((in & 24) >> 1) | (in & 3);
}

struct Unit {
  const uint8_t *mat0, *mat1;  // gate, up (or down, unused)
  int qtype, K, rt, p0, n_real, n_pad, pad0, pad1;
};
static_assert(sizeof(Unit) == 48, "unit records are 48 bytes");

struct Bars {
  uint64_t pfull[kPr], pempty[kPr], afull[8], aempty[8], accfull[2], accempty[2];
};

struct Smem {
  uint8_t *ring, *packed;
  const uint2 *sel2, *sel1;
  Unit *units;
  Bars *bars;
  uint32_t *taddr;
  float *stage;  // epilogue stages
};

constexpr int kEpStage = 2 * 16 * 128;  // epilogue: two 16-column x 128-row stages (fp32; bf16 for h)

template <bool DOWN>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)Cfg<DOWN>::kAr * Cfg<DOWN>::kStep + (size_t)kPr * Cfg<DOWN>::kPacked + 512 * 8 + 2048 * 8 +
         sizeof(Unit) * kMaxUnits + sizeof(Bars) + 16 + sizeof(float) * kEpStage;
}

template <bool DOWN>
__device__ __forceinline__ Smem carve(uint8_t *smem) {
  Smem S;
  uint8_t *p = reinterpret_cast<uint8_t *>(((uintptr_t)smem + 1023) & ~(uintptr_t)1023);  // swizzled tiles
  S.ring = p;
  p += (size_t)Cfg<DOWN>::kAr * Cfg<DOWN>::kStep;
  S.packed = p;
  p += (size_t)kPr * Cfg<DOWN>::kPacked;
  S.sel2 = reinterpret_cast<const uint2 *>(p);
  p += 512 * 8;
  S.sel1 = reinterpret_cast<const uint2 *>(p);
  p += 2048 * 8;
  S.units = reinterpret_cast<Unit *>(p);
  p += sizeof(Unit) * kMaxUnits;
  S.bars = reinterpret_cast<Bars *>(p);
  p += sizeof(Bars);
  S.taddr = reinterpret_cast<uint32_t *>(p);
  p += 16;
  S.stage = reinterpret_cast<float *>(p);
  return S;
}

// Work unit j of a phase: the last active entry whose first unit is <= j.
__device__ Unit make_unit(const TileArgs &a, const ActiveEntry *act, int n_active, int j, bool down) {
  int lo = 0, hi = n_active - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((down ? act[mid].dn_base : act[mid].gu_base) <= j) lo = mid; else hi = mid - 1;
  }
  const ActiveEntry e = act[lo];
  const redlite_moe_expert ex = e.expert >= 0 ? a.experts[e.expert] : a.shared;
  const int nrt = (down ? a.hidden : e.ffn) / 128;
  const int loc = j - (down ? e.dn_base : e.gu_base);
  const int tt = loc / nrt;
  Unit u;
  u.mat0 = (const uint8_t *)(down ? ex.down : ex.gate);
  u.mat1 = (const uint8_t *)(down ? nullptr : ex.up);
  u.qtype = e.qtype;
  u.K = down ? e.ffn : a.hidden;
  u.rt = loc % nrt;
  u.p0 = e.pair_start + kTcTokens * tt;
  u.n_real = min(kTcTokens, e.pair_count - kTcTokens * tt);
  u.n_pad = (u.n_real + 15) & ~15;
  u.pad0 = u.pad1 = 0;
  return u;
}

// (float)(2 n + 1) for 0 <= n < 2^22, exactly, without a conversion instruction.
__device__ __forceinline__ float odd_f(uint32_t n) { return __uint_as_float(0x4B000001u + 2 * n) - 8388608.f; }

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ptx::smem_u32(dst)), "l"(src) : "memory");
}

// --------------------------------------------------------------- dequant
//
// A lane builds the bf16 values of one (row, sub-block) as a table of three
// entries (the scaled grid values of symbols 0, 1, 2) in two registers; the
// byte-permute selectors of the weights' grid entry then pick a bf16 pair
// per instruction.  IQ2_XS-style signs are flipped with one XOR per pair.
// Lane (q, t) decodes rows q and q+8 of its tile-block, groups t and t + 4
// of each 64-input step, into the sixteen registers of one 16-lane TMEM
// store: group 4 c + t fills repetitions 2c (weights 0-3) and 2c+1
// (weights 4-7), row q in registers 0-1 of a repetition, row q+8 in 2-3.

__device__ __forceinline__ void put_group(uint32_t (&r)[16], int c, int h, uint4 v) {
  r[8 * c + 2 * h] = v.x;
  r[8 * c + 2 * h + 1] = v.y;
  r[8 * c + 4 + 2 * h] = v.z;
  r[8 * c + 4 + 2 * h + 1] = v.w;
}

// IQ2_XS-style tile-block fields of lane (q, t) (the resident layout's lane
// order: rows q and q+8, groups 4c + t, field i = 2c + h).
struct Q2Lane {
  uint32_t qs[4], sg[4], qh, sc0, sc1;
  float d0, d1;  // d / 8 of rows q and q+8
};

__device__ __forceinline__ Q2Lane load_q2(uint32_t tb, int lane) {
  Q2Lane r;
  const uint4 qs = ptx::lds128(tb + 32 * lane);
  const uint4 sg = ptx::lds128(tb + 32 * lane + 16);
  r.qs[0] = qs.x, r.qs[1] = qs.y, r.qs[2] = qs.z, r.qs[3] = qs.w;
  r.sg[0] = sg.x, r.sg[1] = sg.y, r.sg[2] = sg.z, r.sg[3] = sg.w;
  r.qh = ptx::lds16(tb + 1024 + 2 * lane);
  const int q = lane >> 2;
  const uint2 sc = ptx::lds64(tb + 1088 + 8 * q);
  r.sc0 = sc.x, r.sc1 = sc.y;
  const uint32_t dw = ptx::lds32(tb + 1152 + 4 * q);
  r.d0 = __half2float(__ushort_as_half((unsigned short)(dw & 0xFFFFu))) * 0.125f;
  r.d1 = __half2float(__ushort_as_half((unsigned short)(dw >> 16))) * 0.125f;
  return r;
}

// Step s (inputs 64s..64s+63 of the column) of one IQ2 tile-block: fields
// i = 4s + 2c + h (group 8s + 4c + t of row q+8h).
__device__ __forceinline__ void dequant_q2(const Q2Lane &L, int s, uint32_t sel2, uint32_t (&r)[16]) {
  const uint32_t qw = s == 0 ? L.qs[0] : s == 1 ? L.qs[1] : s == 2 ? L.qs[2] : L.qs[3];
  const uint32_t sw = s == 0 ? L.sg[0] : s == 1 ? L.sg[1] : s == 2 ? L.sg[2] : L.sg[3];
#pragma unroll
  for (int c2 = 0; c2 < 2; ++c2) {
    const int c = 2 * s + c2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int f = 2 * c2 + h;
      // sign word s holds bit j of field 4s + f at bit 4j + f
      const uint32_t qsb = (qw >> (8 * f)) & 0xFFu, sgz = (sw >> f) & 0x11111111u;
      const uint32_t idx = qsb | (((L.qh >> (4 * s + f)) & 1u) << 8);
      const uint2 sel = ptx::lds64_const(sel2 + 8 * idx);
      const uint32_t nib = ((h ? L.sc1 : L.sc0) >> (4 * c)) & 15u;
      const float sc = (h ? L.d1 : L.d0) * odd_f(nib);
      const uint32_t t0 = bf16x2(sc * 8.f, sc * 25.f), t1 = bf16x2(sc * 43.f, 0.f);
      // sign bits 2w, 2w+1 sit at bits 0 and 4 of byte w of sgz: that byte
      // times 2^15 + 2^27 puts them at bits 15 and 31 of pair w (masked; the
      // two shifted copies never overlap, so no carries)
      uint4 v;
      v.x = __byte_perm(t0, t1, sel.x) ^ ((__byte_perm(sgz, 0u, 0x4440u) * 0x08008000u) & 0x80008000u);
      v.y = __byte_perm(t0, t1, sel.x >> 16) ^ ((__byte_perm(sgz, 0u, 0x4441u) * 0x08008000u) & 0x80008000u);
      v.z = __byte_perm(t0, t1, sel.y) ^ ((__byte_perm(sgz, 0u, 0x4442u) * 0x08008000u) & 0x80008000u);
      v.w = __byte_perm(t0, t1, sel.y >> 16) ^ ((__byte_perm(sgz, 0u, 0x4443u) * 0x08008000u) & 0x80008000u);
      put_group(r, c2, h, v);
    }
  }
}

// IQ1_M-style tile-block fields of lane (q, t) for groups 8S + 4c + t (c =
// 0, 1) of every step S, rows q and q+8.  Group g sits in the record of
// pair p = g & 1 (here t & 1) as entry i = 2 (g >> 1) + h; with u = t >> 1
// the lane's entries of step S are bytes 2u, 2u+1 of qs words 2S and 2S+1,
// and its qh nibbles bytes u and 2+u of nibble word S.
struct Q1Lane {
  uint32_t qs[4], nb[4];
  uint64_t row0, row1;  // 3-bit sub-block scales of rows q and q+8, from sub-block u
  float d0, d1;
};

__device__ __forceinline__ Q1Lane load_q1(uint32_t tb, int lane) {
  Q1Lane r;
  const int q = lane >> 2, p = lane & 1, u = (lane >> 1) & 1;
  const uint32_t pb = tb + 48 * (2 * q + p);
  const uint4 qa = ptx::lds128(pb), qb = ptx::lds128(pb + 16);
  const uint4 nb = ptx::lds128(pb + 32);
  const uint32_t qsel = u ? 0x7632u : 0x5410u, nsel = u ? 0x4431u : 0x4420u;
  r.qs[0] = __byte_perm(qa.x, qa.y, qsel);
  r.qs[1] = __byte_perm(qa.z, qa.w, qsel);
  r.qs[2] = __byte_perm(qb.x, qb.y, qsel);
  r.qs[3] = __byte_perm(qb.z, qb.w, qsel);
  r.nb[0] = __byte_perm(nb.x, 0u, nsel);
  r.nb[1] = __byte_perm(nb.y, 0u, nsel);
  r.nb[2] = __byte_perm(nb.z, 0u, nsel);
  r.nb[3] = __byte_perm(nb.w, 0u, nsel);
  const uint32_t s0 = ptx::lds32(tb + 768 + 12 * q), s1 = ptx::lds32(tb + 772 + 12 * q),
                 s2 = ptx::lds32(tb + 776 + 12 * q);
  r.row0 = (uint64_t)s0 | ((uint64_t)(s1 & 0xFFFFu) << 32);
  r.row1 = (uint64_t)(s1 >> 16) | ((uint64_t)s2 << 16);
  r.row0 >>= 3 * u;  // sub-block of group 8S + 4c + t is 4S + 2c + u
  r.row1 >>= 3 * u;
  const uint32_t dw = ptx::lds32(tb + 864 + 4 * q);
  r.d0 = __half2float(__ushort_as_half((unsigned short)(dw & 0xFFFFu)));
  r.d1 = __half2float(__ushort_as_half((unsigned short)(dw >> 16)));
  return r;
}

__device__ __forceinline__ void dequant_q1(const Q1Lane &L, int S, uint32_t sel1, uint32_t (&r)[16]) {
  const uint32_t qw = S == 0 ? L.qs[0] : S == 1 ? L.qs[1] : S == 2 ? L.qs[2] : L.qs[3];
  const uint32_t nb16 = S == 0 ? L.nb[0] : S == 1 ? L.nb[1] : S == 2 ? L.nb[2] : L.nb[3];
#pragma unroll
  for (int c2 = 0; c2 < 2; ++c2) {
    const int sb = 4 * S + 2 * c2;  // sub-block, counted from the lane's first (u)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t qsb = (qw >> (16 * c2 + 8 * h)) & 0xFFu;
      const uint32_t nib = (nb16 >> (8 * c2 + 4 * h)) & 15u;
      const uint2 sel = ptx::lds64_const(sel1 + 8 * (qsb | ((nib & 7u) << 8)));
      const uint32_t sc3 = (uint32_t)(((h ? L.row1 : L.row0) >> (3 * sb)) & 7u);
      const float sc = (h ? L.d1 : L.d0) * odd_f(sc3);
      const float dl = (nib & 8u) ? -0.125f : 0.125f;
      const uint32_t t0 = bf16x2(sc * (dl - 1.f), sc * dl), t1 = bf16x2(sc * (dl + 1.f), 0.f);
      uint4 v;
      v.x = __byte_perm(t0, t1, sel.x);
      v.y = __byte_perm(t0, t1, sel.x >> 16);
      v.z = __byte_perm(t0, t1, sel.y);
      v.w = __byte_perm(t0, t1, sel.y >> 16);
      put_group(r, c2, h, v);
    }
  }
}

// --------------------------------------------------------------- the kernel

template <bool DOWN>
__global__ void __maxnreg__(128) grouped_tc_kernel(TileArgs a) {
  using C = Cfg<DOWN>;
  extern __shared__ uint8_t smem[];
  const Smem S = carve<DOWN>(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;
  const int H = a.hidden;
  Ctrl *ctrl = reinterpret_cast<Ctrl *>(a.ws + a.L.ctrl);
  const ActiveEntry *act = reinterpret_cast<const ActiveEntry *>(a.ws + a.L.active);
  const Pair *pairs = reinterpret_cast<const Pair *>(a.ws + a.L.pairs);
  __nv_bfloat16 *hbuf = reinterpret_cast<__nv_bfloat16 *>(a.ws + a.L.h);
  const __nv_bfloat16 *xb = reinterpret_cast<const __nv_bfloat16 *>(a.ws + a.L.xb);
  Bars &B = *S.bars;

  // selector tables, barriers, TMEM
  for (int i = tid; i < (512 + 2048) * 8 / 16; i += kTcThreads)
    reinterpret_cast<uint4 *>(const_cast<uint2 *>(S.sel2))[i] =
        __ldg(reinterpret_cast<const uint4 *>(a.grids + kGridQ2Bsel) + i);
  if (tid == 0) {
    for (int i = 0; i < kPr; ++i) ptx::mbar_init(&B.pfull[i], 1), ptx::mbar_init(&B.pempty[i], kDqWarps);
    for (int i = 0; i < C::kAr; ++i) ptx::mbar_init(&B.afull[i], kDqWarps), ptx::mbar_init(&B.aempty[i], 1);
    for (int i = 0; i < 2; ++i) ptx::mbar_init(&B.accfull[i], 1), ptx::mbar_init(&B.accempty[i], kEpWarps);
    ptx::mbar_fence_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(S.taddr, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *S.taddr;
  const int n_active = ctrl->n_active;
  const int n_units = DOWN ? ctrl->n_dn_units : ctrl->n_gu_units;
  const int my_total = n_units > cta ? (n_units - cta + G - 1) / G : 0;
  bool bad = false;
  TC_DECL;
  // per-role pipeline positions (they carry over between passes)
  uint32_t col = 0, step = 0, ucount = 0;
  uint32_t acc_use[2] = {0u, 0u};  // MMA thread / epilogue: uses of each accumulator buffer so far
  int acc_next = 0;

  for (int base = 0; base < my_total; base += kMaxUnits) {
    const int n_this = min(kMaxUnits, my_total - base);
    __syncthreads();  // every role is done with the previous pass's records
    for (int i = tid; i < n_this; i += kTcThreads) S.units[i] = make_unit(a, act, n_active, cta + (base + i) * G, DOWN);
    __syncthreads();

    if (warp == 0) {
      // ---- producer: packed tile-blocks, one 256-input column per ring slot
      if (lane == 0) {
        for (int u = 0; u < n_this; ++u) {
          const Unit U = S.units[u];
          const int tbb = tile_block_bytes(U.qtype), nkb = U.K / 256;
          for (int kb = 0; kb < nkb; ++kb, ++col) {
            const int ps = col % kPr;
            {
              TC_T0();
              if (col >= (uint32_t)kPr && !ptx::mbar_wait_suspend(&B.pempty[ps], ((col / kPr) - 1) & 1u))
                bad = true;
              TC_ADD(0);
            }
            ptx::mbar_expect_tx(&B.pfull[ps], (uint32_t)(C::kMats * 8 * tbb));
            uint8_t *dst = S.packed + (size_t)ps * C::kPacked;
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) {
              const uint8_t *mat = m ? U.mat1 : U.mat0;
              for (int i = 0; i < 8; ++i)
                ptx::bulk_g2s(dst + (m * 8 + i) * tbb, mat + ((size_t)(8 * U.rt + i) * nkb + kb) * tbb, tbb,
                              &B.pfull[ps]);
            }
          }
        }
      }
    } else if (warp == 1) {
      // ---- tensor-core issue (one thread)
      if (lane == 0) {
        for (int u = 0; u < n_this; ++u, ++ucount) {
          const Unit U = S.units[u];
          const AccPlan P = acc_plan<DOWN>(U.n_pad, ucount, acc_next);
          {
            TC_T0();
#pragma unroll
            for (int b = 0; b < 2; ++b)
              if ((P.mask >> b) & 1) {
                if (acc_use[b] >= 1 && !ptx::mbar_wait_suspend(&B.accempty[b], (acc_use[b] - 1) & 1u)) bad = true;
                ++acc_use[b];
              }
            TC_ADD(0);
          }
          ptx::tc_fence_after();
          const uint32_t d = tmem + P.gate, du = tmem + P.up;
          const uint32_t idesc = ptx::idesc_bf16_f32(128, U.n_pad);
          const int nsteps = U.K / 64;
          for (int k = 0; k < nsteps; ++k, ++step) {
            const int as = step % C::kAr;
            {
              TC_T0();
              if (!ptx::mbar_wait_suspend(&B.afull[as], (step / C::kAr) & 1u)) bad = true;
              TC_ADD(1);
            }
            ptx::tc_fence_after();
            // A: the step's slot in TMEM (gate, then up 32 columns on); B:
            // the step's shared-memory tile.  16 more inputs = 8 TMEM columns
            // = 32 bytes = 2 in the descriptor's start-address field.
            const uint32_t ag = tmem + kAccCols + (uint32_t)as * C::kSlotCols;
            const uint64_t db = ptx::sdesc_k_sw128(ptx::smem_u32(S.ring + (size_t)as * C::kStep));
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const bool acc = k > 0 || ks > 0;
              ptx::umma_bf16_ts(d, ag + 8 * ks, db + 2 * ks, idesc, acc);
              if (!DOWN) ptx::umma_bf16_ts(du, ag + 32 + 8 * ks, db + 2 * ks, idesc, acc);
            }
            ptx::umma_commit(&B.aempty[as]);  // the slot is free once these have read it
          }
#pragma unroll
          for (int b = 0; b < 2; ++b)
            if ((P.mask >> b) & 1) ptx::umma_commit(&B.accfull[b]);
        }
      }
    } else if (warp < 2 + kDqWarps) {
      // ---- dequant warps: one tile-block of each matrix into TMEM, 16 rows of B
      const int w = warp - 2;
      // the TMEM lanes this warp may write are 32 (warp % 4) .. + 31: its
      // tile-block (16 rows of the unit's 128) lies in that quarter
      const int tbi = 2 * (warp & 3) + (warp >= 6 ? 1 : 0);
      const uint32_t tlane = tmem + ((uint32_t)(16 * tbi) << 16);
      const uint32_t sel2a = ptx::smem_u32(S.sel2), sel1a = ptx::smem_u32(S.sel1);
      for (int u = 0; u < n_this; ++u) {
        const Unit U = S.units[u];
        const int nkb = U.K / 256;
        // B rows 16w + (lane >> 3) + 4i, 16-byte chunk lane & 7 of each step
        const __nv_bfloat16 *brow[4];
        int nb = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = 16 * w + (lane >> 3) + 4 * i;
          const int jj = min(j, U.n_real - 1);  // pad rows read a real row; their results are dropped
          if (j < U.n_pad) nb = i + 1;
          brow[i] = DOWN ? hbuf + (size_t)(U.p0 + jj) * a.max_ffn : xb + (size_t)pairs[U.p0 + jj].token * H;
        }
        const int tbb = tile_block_bytes(U.qtype), nsteps = 4 * nkb;
        // B rows of local step n into ring slot `as`, as one cp.async group;
        // issued a step ahead so the copies overlap the decode of the step
        // before.  Waiting for the slot's release also frees its A slot.
        auto fetch_b = [&](int n, uint32_t gstep) {
          const int as = gstep % C::kAr;
          {
            TC_T0();
            if (gstep >= (uint32_t)C::kAr && !ptx::mbar_wait_suspend(&B.aempty[as], ((gstep / C::kAr) - 1) & 1u))
              bad = true;
            TC_ADD(1);
          }
          uint8_t *bt = S.ring + (size_t)as * C::kStep;
          const int k0 = 64 * n + 8 * (lane & 7);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (i < nb) cp_async16(bt + ptx::sw128_offset(16 * w + (lane >> 3) + 4 * i, 8 * (lane & 7)), brow[i] + k0);
          asm volatile("cp.async.commit_group;" ::: "memory");
        };
        fetch_b(0, step);
        for (int kb = 0; kb < nkb; ++kb, ++col) {
          const int ps = col % kPr;
          {
            TC_T0();
            if (!ptx::mbar_wait_suspend(&B.pfull[ps], (col / kPr) & 1u)) bad = true;
            TC_ADD(0);
          }
          const uint32_t pk = ptx::smem_u32(S.packed) + ps * C::kPacked;
          Q2Lane l2[C::kMats];
          Q1Lane l1[C::kMats];
          if (U.qtype == kQ2) {
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) l2[m] = load_q2(pk + (m * 8 + tbi) * tbb, lane);
          } else {
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) l1[m] = load_q1(pk + (m * 8 + tbi) * tbb, lane);
          }
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&B.pempty[ps]);
#pragma unroll
          for (int s = 0; s < 4; ++s, ++step) {
            const int n = 4 * kb + s, as = step % C::kAr;
            const bool more = n + 1 < nsteps;
            if (more) fetch_b(n + 1, step + 1);
            // the slot's previous MMAs are done (waited for when its B rows were fetched)
            ptx::tc_fence_after();
            const uint32_t at = tlane + kAccCols + (uint32_t)as * C::kSlotCols;
            TC_T0();
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) {
              uint32_t r[16];
              if (U.qtype == kQ2)
                dequant_q2(l2[m], s, sel2a, r);
              else
                dequant_q1(l1[m], s, sel1a, r);
              ptx::tmem_st16x256_x4(at + 32 * m, r);
            }
            TC_ADD(2);
            ptx::tmem_wait_st();
            // this step's B rows landed (the next step's may still be in flight)
            if (more)
              asm volatile("cp.async.wait_group 1;" ::: "memory");
            else
              asm volatile("cp.async.wait_group 0;" ::: "memory");
            ptx::fence_proxy_async_smem();  // generic-proxy writes -> the tensor cores
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&B.afull[as]);
          }
        }
      }
    } else {
      // ---- epilogue: warp reads TMEM lanes 32 (warp % 4) .. + 31 (= tile rows)
      const int lq = warp & 3, row = 32 * lq + lane;
      const bool vec_out = ((uintptr_t)a.out & 15) == 0;  // 4-wide vector adds need 16-byte rows
      uint32_t ep_stage = 0;
      for (int u = 0; u < n_this; ++u, ++ucount) {
        const Unit U = S.units[u];
        const AccPlan P = acc_plan<DOWN>(U.n_pad, ucount, acc_next);
        {
          TC_T0();
#pragma unroll
          for (int b = 0; b < 2; ++b)
            if ((P.mask >> b) & 1) {
              if (!ptx::mbar_wait_suspend(&B.accfull[b], acc_use[b] & 1u)) bad = true;
              ++acc_use[b];
            }
          TC_ADD(0);
        }
        ptx::tc_fence_after();
        const uint32_t lq16 = (uint32_t)(32 * lq) << 16;
        const uint32_t d = tmem + P.gate + lq16, du = tmem + P.up + lq16;
        const int r = 128 * U.rt + row;
        // h is stored in the contraction order of the down kernel's steps
        const int rp = (r & ~63) | perm64(r & 63);
        Pair pl = {0, 0.f};  // down, scalar path: pair c0 - (c0 % 32) + lane of the unit, broadcast by shuffles
        // down, vector path: lane l holds the pair of column lq + 4 l (the
        // columns this warp adds), read once per unit
        Pair mine = {0, 0.f};
        if (DOWN && vec_out && lq + 4 * lane < U.n_real) mine = pairs[U.p0 + lq + 4 * lane];
        for (int c0 = 0; c0 < U.n_pad; c0 += 16) {
          uint32_t d0[16];
          ptx::tmem_ld16(d + (uint32_t)c0, d0);
          if (DOWN && vec_out) {
            // stage the 16 columns (tokens) x 128 rows, then warp lq adds
            // columns lq, lq + 4, .. into out, lane j taking rows 4j..4j+3:
            // one 4-wide vector add per lane, 512 contiguous bytes per column
            float *T = S.stage + (ep_stage & 1) * 16 * 128;
            ++ep_stage;
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) T[i * 128 + row] = __uint_as_float(d0[i]);
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpWarps) : "memory");
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int i = lq + 4 * k, col = c0 + i;
              const int tok = __shfl_sync(0xffffffffu, mine.token, (c0 >> 2) + k);
              const float wgt = __shfl_sync(0xffffffffu, mine.weight, (c0 >> 2) + k);
              if (col < U.n_real) {
                const float4 v = *reinterpret_cast<const float4 *>(T + i * 128 + 4 * lane);
                float *o = a.out + (size_t)tok * H + 128 * U.rt + 4 * lane;
                asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(o), "f"(wgt * v.x),
                             "f"(wgt * v.y), "f"(wgt * v.z), "f"(wgt * v.w)
                             : "memory");
              }
            }
          } else if (DOWN) {
            if ((c0 & 31) == 0) {
              const int jl = c0 + lane;
              if (jl < U.n_real) pl = pairs[U.p0 + jl];
            }
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int src = (c0 & 16) + i;
              const int tok = __shfl_sync(0xffffffffu, pl.token, src);
              const float wgt = __shfl_sync(0xffffffffu, pl.weight, src);
              if (c0 + i < U.n_real) atomicAdd(a.out + (size_t)tok * H + r, wgt * __uint_as_float(d0[i]));
            }
          } else {
            // h of 16 pairs x 128 rows staged as bf16 at the rows' permuted
            // places, then written as 16-byte pieces (pair i, piece g)
            uint32_t d1[16];
            ptx::tmem_ld16(du + (uint32_t)c0, d1);
            __nv_bfloat16 *T = reinterpret_cast<__nv_bfloat16 *>(S.stage) + (ep_stage & 1) * 16 * 128;
            ++ep_stage;
            ptx::tmem_wait_ld();
            const int prow = rp - 128 * U.rt;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              T[i * 128 + prow] = __float2bfloat16_rn(silu_mul_fast(__uint_as_float(d0[i]), __uint_as_float(d1[i])));
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpWarps) : "memory");
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int e = 32 * lq + lane + 128 * k, i = e >> 4, g = e & 15;
              if (c0 + i < U.n_real)
                *reinterpret_cast<uint4 *>(hbuf + (size_t)(U.p0 + c0 + i) * a.max_ffn + 128 * U.rt + 8 * g) =
                    *reinterpret_cast<const uint4 *>(T + i * 128 + 8 * g);
            }
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int b = 0; b < 2; ++b)
            if ((P.mask >> b) & 1) ptx::mbar_arrive(&B.accempty[b]);
        }
      }
    }
  }
  if (bad) atomicOr(a.status, REDLITE_STATUS_TIMEOUT);
  TC_FLUSH();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

// Activations to bf16 (round to nearest even), 8 per thread: inputs
// 8i..8i+7 (group G = i mod 8 of a 64-input step) go to positions perm64,
// two runs of four.
__global__ void to_bf16_kernel(const float *__restrict__ x, __nv_bfloat16 *__restrict__ xb, int64_t n8) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 v0 = __ldg(reinterpret_cast<const float4 *>(x) + 2 * i);
  const float4 v1 = __ldg(reinterpret_cast<const float4 *>(x) + 2 * i + 1);
  const int64_t base = (i >> 3) << 6;
  const int g = (int)(i & 7);
  const int p0 = perm64(8 * g), p1 = perm64(8 * g + 4);
  *reinterpret_cast<uint2 *>(xb + base + p0) = make_uint2(bf16x2(v0.x, v0.y), bf16x2(v0.z, v0.w));
  *reinterpret_cast<uint2 *>(xb + base + p1) = make_uint2(bf16x2(v1.x, v1.y), bf16x2(v1.z, v1.w));
}

}  // namespace

bool tc_supported(int hidden, int max_ffn) { return hidden % 256 == 0 && max_ffn % 256 == 0; }

cudaError_t launch_tc(const TileArgs &a, cudaStream_t stream) {
  static_assert(smem_bytes<false>() <= 227 * 1024 && smem_bytes<true>() <= 227 * 1024, "shared memory");
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(grouped_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_bytes<false>());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(grouped_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem_bytes<true>());
  if (e != cudaSuccess) return e;
  const int64_t n8 = (int64_t)a.n_tokens * a.hidden / 8;
  to_bf16_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, stream>>>(
      a.x, reinterpret_cast<__nv_bfloat16 *>(a.ws + a.L.xb), n8);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  grouped_tc_kernel<false><<<sms, kTcThreads, smem_bytes<false>(), stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  grouped_tc_kernel<true><<<sms, kTcThreads, smem_bytes<true>(), stream>>>(a);
  return cudaGetLastError();
}

}  // namespace redlite
