// grouped_tc.cu -- the bucketed tensor-core path for calls with many tokens
// per expert (prefill).
//
// "Red Metal dev8 -- resident routed top-k layer", steps 4-6, for a batch of
// tokens: the (token, slot) pairs are bucketed by expert (route.cu), then
// every expert's gate/up and down projections run as dense contractions on
// the 5th-generation tensor cores (tcgen05.mma, bf16 operands in shared
// memory, fp32 accumulators in tensor memory).  Weights are decoded from the
// packed tile-blocks into 128-byte-swizzled bf16 tiles (each weight is exact
// in fp32 and rounded to bf16, nearest even); activations are rounded to bf16
// the same way.  Accumulation is fp32.
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
//               commits them to the step's slot and, per unit, to one of two
//               accumulator buffers;
//   warps 2-9   dequant warp w decodes tile-block w (rows 16w..16w+15) of
//               each matrix into the A tiles of a ring of 64-input steps (3
//               deep for gate/up, 5 for down) and
//               fetches rows 16w..16w+15 of B with cp.async, a step ahead;
//   warps 10-13 the epilogue (TMEM -> registers -> h or out), overlapping
//               the next unit's contraction.
#include "internal.cuh"
#include "layout.cuh"
#include "ptx.cuh"

namespace redlite {
namespace {

constexpr int kDqWarps = 8;
constexpr int kEpWarps = 4;
constexpr int kTcWarps = 2 + kDqWarps + kEpWarps;
constexpr int kTcThreads = 32 * kTcWarps;  // 448
constexpr int kTile = 128 * 64 * 2;        // 16 KB: 128 rows x 64 bf16
constexpr int kPr = 2;                     // packed columns in flight
constexpr int kMaxUnits = 128;             // unit records per pass
constexpr uint32_t kTmemCols = 512;

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
  static constexpr int kAr = DOWN ? 5 : 3;                  // 64-input steps in flight
  static constexpr int kStep = (kMats + 1) * kTile;         // A tiles, then the B tile
  static constexpr int kPacked = kMats * 8 * kQ2TileBlock;  // one column, largest format
  static constexpr uint32_t kBufCols = DOWN ? 128 : 256;    // TMEM columns per accumulator buffer
};

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
};

template <bool DOWN>
constexpr size_t smem_bytes() {
  return 1024 + (size_t)Cfg<DOWN>::kAr * Cfg<DOWN>::kStep + (size_t)kPr * Cfg<DOWN>::kPacked + 512 * 8 + 2048 * 8 +
         sizeof(Unit) * kMaxUnits + sizeof(Bars) + 16;
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

// Step s (inputs 64s..64s+63 of the column) of one IQ2 tile-block into rows
// row0..row0+15 of the swizzled A tile: fields i = 4s + 2 c2 + h.  `lane` is
// the layout lane (q, t); the warp runs it on thread q + 8 t, so the eight
// threads of a quarter-warp store to eight different rows (conflict-free
// 128-bit stores in the swizzled tile) with a field order fixed at compile time.
__device__ __forceinline__ void dequant_q2(const Q2Lane &L, int s, uint32_t A, int row0, uint32_t sel2,
                                           int lane) {
  const int q = lane >> 2, t = lane & 3;
  const uint32_t qw = s == 0 ? L.qs[0] : s == 1 ? L.qs[1] : s == 2 ? L.qs[2] : L.qs[3];
  const uint32_t sw = s == 0 ? L.sg[0] : s == 1 ? L.sg[1] : s == 2 ? L.sg[2] : L.sg[3];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int c2 = j;
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
      ptx::sts128(A + ptx::sw128_offset(row0 + q + 8 * h, 32 * c2 + 8 * t), v);
    }
  }
}

// IQ1_M-style tile-block fields of lane (q, t): pair p = t >> 1 (groups
// 2 sb + p of rows q and q+8, field i = 2 sb + h); half = t & 1 takes
// sub-blocks 4S + 2 half + {0, 1} of step S.
struct Q1Lane {
  uint32_t qs[4], nb[4];
  uint64_t row0, row1;  // 3-bit sub-block scales of rows q and q+8, from sub-block 2 half
  float d0, d1;
};

__device__ __forceinline__ Q1Lane load_q1(uint32_t tb, int lane) {
  Q1Lane r;
  const int q = lane >> 2, p = (lane >> 1) & 1, half = lane & 1;
  const uint32_t pb = tb + 48 * (2 * q + p);
  const uint4 qa = ptx::lds128(pb), qb = ptx::lds128(pb + 16);
  const uint4 nb = ptx::lds128(pb + 32);
  // qs word 2S + half holds fields 8S + 4 half .. + 3 of step S
  r.qs[0] = half ? qa.y : qa.x;
  r.qs[1] = half ? qa.w : qa.z;
  r.qs[2] = half ? qb.y : qb.x;
  r.qs[3] = half ? qb.w : qb.z;
  // nibble word of step S: this lane's half of it
  r.nb[0] = half ? nb.x >> 16 : nb.x & 0xFFFFu;
  r.nb[1] = half ? nb.y >> 16 : nb.y & 0xFFFFu;
  r.nb[2] = half ? nb.z >> 16 : nb.z & 0xFFFFu;
  r.nb[3] = half ? nb.w >> 16 : nb.w & 0xFFFFu;
  const uint32_t s0 = ptx::lds32(tb + 768 + 12 * q), s1 = ptx::lds32(tb + 772 + 12 * q),
                 s2 = ptx::lds32(tb + 776 + 12 * q);
  r.row0 = (uint64_t)s0 | ((uint64_t)(s1 & 0xFFFFu) << 32);
  r.row1 = (uint64_t)(s1 >> 16) | ((uint64_t)s2 << 16);
  r.row0 >>= 6 * half;  // this lane's sub-blocks are 4 S + 2 half + {0, 1}
  r.row1 >>= 6 * half;
  const uint32_t dw = ptx::lds32(tb + 864 + 4 * q);
  r.d0 = __half2float(__ushort_as_half((unsigned short)(dw & 0xFFFFu)));
  r.d1 = __half2float(__ushort_as_half((unsigned short)(dw >> 16)));
  return r;
}

__device__ __forceinline__ void dequant_q1(const Q1Lane &L, int S, uint32_t A, int row0, uint32_t sel1,
                                           int lane) {
  const int q = lane >> 2, p = (lane >> 1) & 1, half = lane & 1;
  const uint32_t qw = S == 0 ? L.qs[0] : S == 1 ? L.qs[1] : S == 2 ? L.qs[2] : L.qs[3];
  const uint32_t nb16 = S == 0 ? L.nb[0] : S == 1 ? L.nb[1] : S == 2 ? L.nb[2] : L.nb[3];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int s2 = j;
    const int sb = 4 * S + s2;  // sub-block 4 S + 2 half + s2, counted from the lane's first
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int f = 2 * s2 + h;
      const uint32_t qsb = (qw >> (8 * f)) & 0xFFu;
      const uint32_t nib = (nb16 >> (4 * f)) & 15u;
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
      ptx::sts128(A + ptx::sw128_offset(row0 + q + 8 * h, 16 * (2 * half + s2) + 8 * p), v);
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
          const int buf = ucount & 1;
          {
            TC_T0();
            if (ucount >= 2 && !ptx::mbar_wait_suspend(&B.accempty[buf], ((ucount >> 1) - 1) & 1u)) bad = true;
            TC_ADD(0);
          }
          ptx::tc_fence_after();
          const uint32_t d = tmem + buf * C::kBufCols;
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
            const uint32_t a0 = ptx::smem_u32(S.ring + (size_t)as * C::kStep);
            // descriptors of the step's tiles; 16 more inputs = 32 bytes = 2 in the start-address field
            const uint64_t da = ptx::sdesc_k_sw128(a0), du = da + (kTile >> 4),
                           db = ptx::sdesc_k_sw128(a0 + C::kMats * kTile);
            if (k == 0) {
              ptx::umma_bf16(d, da, db, idesc, false);
              if (!DOWN) ptx::umma_bf16(d + 128, du, db, idesc, false);
            } else {
              ptx::umma_bf16_acc(d, da, db, idesc);
              if (!DOWN) ptx::umma_bf16_acc(d + 128, du, db, idesc);
            }
#pragma unroll
            for (int ks = 1; ks < 4; ++ks) {
              ptx::umma_bf16_acc(d, da + 2 * ks, db + 2 * ks, idesc);
              if (!DOWN) ptx::umma_bf16_acc(d + 128, du + 2 * ks, db + 2 * ks, idesc);
            }
            ptx::umma_commit(&B.aempty[as]);  // the slot is free once these have read it
          }
          ptx::umma_commit(&B.accfull[buf]);
        }
      }
    } else if (warp < 2 + kDqWarps) {
      // ---- dequant warps: A tiles (and this warp's 16 rows of B)
      const int w = warp - 2;
      const int ll = ((lane & 7) << 2) | (lane >> 3);  // the layout lane this thread decodes
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
        // issued a step ahead so the copies overlap the decode of the step before
        auto fetch_b = [&](int n, uint32_t gstep) {
          const int as = gstep % C::kAr;
          {
            TC_T0();
            if (gstep >= (uint32_t)C::kAr && !ptx::mbar_wait_suspend(&B.aempty[as], ((gstep / C::kAr) - 1) & 1u))
              bad = true;
            TC_ADD(1);
          }
          uint8_t *bt = S.ring + (size_t)as * C::kStep + C::kMats * kTile;
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
            for (int m = 0; m < C::kMats; ++m) l2[m] = load_q2(pk + (m * 8 + w) * tbb, ll);
          } else {
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) l1[m] = load_q1(pk + (m * 8 + w) * tbb, ll);
          }
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&B.pempty[ps]);
#pragma unroll
          for (int s = 0; s < 4; ++s, ++step) {
            const int n = 4 * kb + s, as = step % C::kAr;
            const bool more = n + 1 < nsteps;
            if (more) fetch_b(n + 1, step + 1);
            const uint32_t stg = ptx::smem_u32(S.ring) + as * C::kStep;
            TC_T0();
            if (U.qtype == kQ2) {
#pragma unroll
              for (int m = 0; m < C::kMats; ++m) dequant_q2(l2[m], s, stg + m * kTile, 16 * w, sel2a, ll);
            } else {
#pragma unroll
              for (int m = 0; m < C::kMats; ++m) dequant_q1(l1[m], s, stg + m * kTile, 16 * w, sel1a, ll);
            }
            TC_ADD(2);
            // this step's B rows landed (the next step's may still be in flight)
            if (more)
              asm volatile("cp.async.wait_group 1;" ::: "memory");
            else
              asm volatile("cp.async.wait_group 0;" ::: "memory");
            ptx::fence_proxy_async_smem();  // generic-proxy writes -> the tensor cores
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&B.afull[as]);
          }
        }
      }
    } else {
      // ---- epilogue: warp reads TMEM lanes 32 (warp % 4) .. + 31 (= tile rows)
      const int lq = warp & 3, row = 32 * lq + lane;
      for (int u = 0; u < n_this; ++u, ++ucount) {
        const Unit U = S.units[u];
        const int buf = ucount & 1;
        {
          TC_T0();
          if (!ptx::mbar_wait_suspend(&B.accfull[buf], (ucount >> 1) & 1u)) bad = true;
          TC_ADD(0);
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + buf * C::kBufCols + ((uint32_t)(32 * lq) << 16);
        const int r = 128 * U.rt + row;
        Pair pl = {0, 0.f};  // down: pair c0 - (c0 % 32) + lane of the unit, broadcast by shuffles
        for (int c0 = 0; c0 < U.n_pad; c0 += 16) {
          uint32_t d0[16];
          ptx::tmem_ld16(d + (uint32_t)c0, d0);
          if (DOWN) {
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
            uint32_t d1[16];
            ptx::tmem_ld16(d + 128 + (uint32_t)c0, d1);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int jj = c0 + i;
              if (jj < U.n_real)
                hbuf[(size_t)(U.p0 + jj) * a.max_ffn + r] =
                    __float2bfloat16_rn(silu_mul(__uint_as_float(d0[i]), __uint_as_float(d1[i])));
            }
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&B.accempty[buf]);
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

// Activations to bf16 (round to nearest even), 8 per thread.
__global__ void to_bf16_kernel(const float *__restrict__ x, __nv_bfloat16 *__restrict__ xb, int64_t n8) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 v0 = __ldg(reinterpret_cast<const float4 *>(x) + 2 * i);
  const float4 v1 = __ldg(reinterpret_cast<const float4 *>(x) + 2 * i + 1);
  reinterpret_cast<uint4 *>(xb)[i] =
      make_uint4(bf16x2(v0.x, v0.y), bf16x2(v0.z, v0.w), bf16x2(v1.x, v1.y), bf16x2(v1.z, v1.w));
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
