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
//   warps 2-9   dequant warps, two per TMEM lane quarter: thread i of a warp
//               whose lane quarter is qd owns row 32 qd + i of the unit's 128
//               rows (TMEM lane 32 qd + i) and writes, per step and matrix,
//               its 64 consecutive weights into 32 consecutive columns of the
//               step's A slot (tcgen05.st 32x32b).  Half kh of the quarter's
//               two warps takes steps 2 kh and 2 kh + 1 of every 256-input
//               column; the four warps of a half also fetch the 128 B rows of
//               their steps with cp.async into the step's shared-memory slot;
//   warps 10-13 the epilogue (TMEM -> registers -> h or out).
//
// A and B hold every step's 64 inputs in input order: TMEM column c of an A
// slot holds inputs 2c and 2c + 1 of its row, and a B row is the 64 inputs
// of the step as 128 contiguous bytes (before the hardware swizzle).
#include <type_traits>

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
  return 1024 + (size_t)Cfg<DOWN>::kAr * Cfg<DOWN>::kStep + (size_t)kPr * Cfg<DOWN>::kPacked + 512 * 8 + 4096 * 8 +
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
  p += 4096 * 8;
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
// A thread decodes the weights of one row: per 16-weight (IQ1_M-style) or
// 32-weight (IQ2_XS-style) sub-block it builds the bf16 values the row's
// grid symbols can take, scaled by d and the sub-scale, in two registers;
// the byte-permute selectors of a grid entry then pick one bf16 pair per
// instruction.  Every value is exact in fp32 before its one rounding to bf16
// (nearest even), so it equals redlite_moe_dequant's bf16 output.
//
// Row 32 qd + i of a unit lies in tile-block 2 qd + (i >> 4) of each column,
// at row rr = i & 15 of it (q = rr & 7, hh = rr >> 3 in the tiled layout).
// Half kh of a lane quarter reads the fields of its two steps (inputs 128 kh
// .. 128 kh + 127 of the column) once per column.

// IQ1_M-style fields of one row for half kh of a column.  Records p = 0, 1 of
// the tile-block (groups 2 s + p, s = 0..15) give, for the half's local
// sub-blocks s' = 0..7 (s = 8 kh + s'): qs word s' >> 1 (byte 2 (s' & 1) +
// hh), and nibble word s' >> 2 (byte s' & 3, shifted so the row's nibble is
// the byte's low nibble).
struct Q1Row {
  uint32_t qa[2][4], nb[2][2];
  uint32_t sc;  // 3-bit sub-scales of the local sub-blocks, s' at bit 3 s'
  float d8;     // d / 8
};

__device__ __forceinline__ Q1Row load_q1_row(uint32_t tb, int q, int hh, int kh) {
  Q1Row r;
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const uint32_t rec = tb + 48 * (2 * q + p);
    const uint4 a = ptx::lds128(rec + 16 * kh);
    const uint2 b = ptx::lds64(rec + 32 + 8 * kh);
    r.qa[p][0] = a.x, r.qa[p][1] = a.y, r.qa[p][2] = a.z, r.qa[p][3] = a.w;
    r.nb[p][0] = b.x >> (4 * hh), r.nb[p][1] = b.y >> (4 * hh);
  }
  // the 48-bit sub-scale fields of rows q and q + 8 are bytes 0-5 and 6-11
  const uint32_t s0 = ptx::lds32(tb + 768 + 12 * q), s1 = ptx::lds32(tb + 772 + 12 * q),
                 s2 = ptx::lds32(tb + 776 + 12 * q);
  const uint32_t lo = hh ? (s1 >> 16) | (s2 << 16) : s0, hi = hh ? s2 >> 16 : s1 & 0xFFFFu;
  r.sc = kh ? (lo >> 24) | (hi << 8) : lo & 0xFFFFFFu;
  const uint32_t dw = ptx::lds32(tb + 864 + 4 * q);
  r.d8 = __half2float(__ushort_as_half((unsigned short)(hh ? dw >> 16 : dw & 0xFFFFu))) * 0.125f;
  return r;
}

// Local step j (0, 1) of one IQ1 row into r[32]: group 2m + p of the step
// (sub-block s' = 4 j + m) fills registers 4 (2m + p) .. + 3.  The table
// sel1 has 4096 entries indexed by qs | nibble << 8 (the delta bit is index
// bit 11); its selectors pick from (X, Q) with X = P for delta +1/8 and
// X = R for delta -1/8, where P = (-7, 1), R = (-9, -1), Q = (9, 7) times
// d (2 sc + 1) / 8 -- the values 8 (grid + delta) of symbols 0, 1, 2 are
// slots 0, 1, 2 for +1/8 and 0, 1, 3 for -1/8.  selc[n]: the byte-permute
// that moves qs byte 2 (n & 1) + hh and nibble byte n into bytes 0 and 1.
__device__ __forceinline__ void dequant_q1_row(const Q1Row &R, int j, uint32_t sel1, const uint32_t (&selc)[4],
                                               uint32_t (&r)[32]) {
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int s = 4 * j + m;
    const uint32_t n2 = (s == 0 ? R.sc << 1 : R.sc >> (3 * s - 1)) & 14u;  // 2 * sub-scale
    const float sc8 = R.d8 * (__uint_as_float(0x4B000001u | n2) - 8388608.f);
    const uint32_t P = bf16x2(-7.f * sc8, sc8), Rv = bf16x2(-9.f * sc8, -sc8), Q = bf16x2(9.f * sc8, 7.f * sc8);
    const uint32_t RmP = Rv - P;
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const uint32_t idx = __byte_perm(R.qa[p][s >> 1], R.nb[p][s >> 2], selc[s & 3]) & 0xFFFu;
      const uint2 sel = ptx::lds64_const(sel1 + 8 * idx);
      const uint32_t X = (idx >> 11) * RmP + P;
      const int g = 2 * m + p;
      r[4 * g + 0] = __byte_perm(X, Q, sel.x);
      r[4 * g + 1] = __byte_perm(X, Q, sel.x >> 16);
      r[4 * g + 2] = __byte_perm(X, Q, sel.y);
      r[4 * g + 3] = __byte_perm(X, Q, sel.y >> 16);
    }
  }
}

// IQ2_XS-style fields of one row for half kh of a column.  Records t = 0..3
// of the tile-block (lanes 4q + t: groups 4c + t) give, for the local
// sub-blocks c' = c - 4 kh = 0..3: qs word c' >> 1 (byte 2 (c' & 1) after a
// shift by 8 hh), sign word c' >> 1 (bit 4 j' + 2 (c' & 1) = sign of weight
// j' after a shift by hh), and index bit 8 at bit 0 of byte t of vq[c'].
struct Q2Row {
  uint32_t qs[4][2], sg[4][2], vq[4];
  uint32_t sc;  // 4-bit sub-scales of the local sub-blocks, c' at bit 4 c'
  float d8;
};

__device__ __forceinline__ Q2Row load_q2_row(uint32_t tb, int q, int hh, int kh) {
  Q2Row r;
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t rec = tb + 32 * (4 * q + t);
    const uint2 a = ptx::lds64(rec + 8 * kh), b = ptx::lds64(rec + 16 + 8 * kh);
    r.qs[t][0] = a.x >> (8 * hh), r.qs[t][1] = a.y >> (8 * hh);
    r.sg[t][0] = b.x >> hh, r.sg[t][1] = b.y >> hh;
  }
  // index bit 8 of field i = 2c + hh is bit i of record t's u16
  const uint2 qh = ptx::lds64(tb + 1024 + 8 * q);
  const int sh = 8 * kh + hh;
  const uint32_t v = __byte_perm(__byte_perm(qh.x >> sh, qh.x >> (16 + sh), 0x0040u),
                                 __byte_perm(qh.y >> sh, qh.y >> (16 + sh), 0x0040u), 0x5410u);
#pragma unroll
  for (int c = 0; c < 4; ++c) r.vq[c] = v >> (2 * c);
  r.sc = ptx::lds32(tb + 1088 + 8 * q + 4 * hh) >> (16 * kh);
  const uint32_t dw = ptx::lds32(tb + 1152 + 4 * q);
  r.d8 = __half2float(__ushort_as_half((unsigned short)(hh ? dw >> 16 : dw & 0xFFFFu))) * 0.125f;
  return r;
}

// Local step j (0, 1) of one IQ2 row into r[32]: group 4 cc + t of the step
// (local sub-block c' = 2 j + cc) fills registers 4 (4 cc + t) .. + 3.  The
// value table is (8, 25 | 43, 0) times d (2 sc + 1) / 8; each pair's two
// sign bits become bits 15 and 31 of an XOR mask.
__device__ __forceinline__ void dequant_q2_row(const Q2Row &R, int j, uint32_t sel2, uint32_t (&r)[32]) {
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int c = 2 * j + cc;
    const uint32_t n2 = (c == 0 ? R.sc << 1 : R.sc >> (4 * c - 1)) & 30u;  // 2 * sub-scale
    const float sc8 = R.d8 * (__uint_as_float(0x4B000001u | n2) - 8388608.f);
    const uint32_t t0 = bf16x2(sc8 * 8.f, sc8 * 25.f), t1 = bf16x2(sc8 * 43.f, 0.f);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const uint32_t idx = __byte_perm(R.qs[t][j], R.vq[c], (uint32_t)(2 * cc) | ((4u + t) << 4)) & 0x1FFu;
      const uint2 sel = ptx::lds64_const(sel2 + 8 * idx);
      const uint32_t sgz = (R.sg[t][j] >> (2 * cc)) & 0x11111111u;
      const int g = 4 * cc + t;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t sw = w & 1 ? (w & 2 ? sel.y : sel.x) >> 16 : (w & 2 ? sel.y : sel.x);
        const uint32_t m = __byte_perm(sgz, 0u, 0x4440u + w) * 0x08008000u;
        r[4 * g + w] = __byte_perm(t0, t1, sw) ^ (m & 0x80008000u);
      }
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
  // (the IQ1 table gets a second half for delta -1/8: slot 2 -> 3, i.e.
  // selector nibbles 4, 5 -> 6, 7)
  {
    const uint4 *g = reinterpret_cast<const uint4 *>(a.grids + kGridQ2Bsel);
    uint4 *t2 = reinterpret_cast<uint4 *>(const_cast<uint2 *>(S.sel2));
    uint4 *t1 = reinterpret_cast<uint4 *>(const_cast<uint2 *>(S.sel1));
    for (int i = tid; i < 512 * 8 / 16; i += kTcThreads) t2[i] = __ldg(g + i);
    for (int i = tid; i < 2048 * 8 / 16; i += kTcThreads) {
      const uint4 v = __ldg(g + 512 * 8 / 16 + i);
      t1[i] = v;
      t1[i + 2048 * 8 / 16] = make_uint4(v.x + ((v.x & 0x44444444u) >> 1), v.y + ((v.y & 0x44444444u) >> 1),
                                         v.z + ((v.z & 0x44444444u) >> 1), v.w + ((v.w & 0x44444444u) >> 1));
    }
  }
  if (tid == 0) {
    for (int i = 0; i < kPr; ++i) ptx::mbar_init(&B.pfull[i], 1), ptx::mbar_init(&B.pempty[i], kDqWarps);
    for (int i = 0; i < C::kAr; ++i) ptx::mbar_init(&B.afull[i], kDqWarps / 2), ptx::mbar_init(&B.aempty[i], 1);
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
      // ---- dequant warps: rows 32 qd .. 32 qd + 31 of every matrix, steps
      // 2 kh and 2 kh + 1 of every column, and the B rows of those steps
      const int qd = warp & 3, kh = warp >= 6 ? 1 : 0;
      const int tbi = 2 * qd + (lane >> 4), rr = lane & 15, q = rr & 7, hh = rr >> 3;
      const uint32_t tlane = tmem + ((uint32_t)(32 * qd) << 16);
      const uint32_t sel2a = ptx::smem_u32(S.sel2), sel1a = ptx::smem_u32(S.sel1);
      uint32_t selc[4];
#pragma unroll
      for (int n = 0; n < 4; ++n) selc[n] = (uint32_t)(2 * (n & 1) + hh) | ((4u + n) << 4);
      for (int u = 0; u < n_this; ++u) {
        const Unit U = S.units[u];
        const int nkb = U.K / 256;
        // B rows 32 qd + (lane >> 3) + 4 i (i < 8), 16-byte chunk lane & 7:
        // the row of x (the pair's token) or of h (the pair) they copy
        int brow[8], nb = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int jr = 32 * qd + (lane >> 3) + 4 * i;
          const int jj = min(jr, U.n_real - 1);  // pad rows read a real row; their results are dropped
          if (jr < U.n_pad) nb = i + 1;
          brow[i] = DOWN ? U.p0 + jj : pairs[U.p0 + jj].token;
        }
        // B rows of local step n into ring slot gstep % kAr, as one cp.async
        // group; waiting for the slot's release also frees its A slot
        auto fetch_b = [&](int n, uint32_t gstep) {
          const int as = gstep % C::kAr;
          {
            TC_T0();
            if (gstep >= (uint32_t)C::kAr && !ptx::mbar_wait_suspend(&B.aempty[as], ((gstep / C::kAr) - 1) & 1u))
              bad = true;
            TC_ADD(1);
          }
          // the tensor cores read the slot's previous rows through the async
          // proxy; order those reads before these generic-proxy writes
          ptx::fence_proxy_async_smem();
          uint8_t *bt = S.ring + (size_t)as * C::kStep;
          const int k0 = 64 * n + 8 * (lane & 7);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (i < nb) {
              const __nv_bfloat16 *src = DOWN ? hbuf + (size_t)brow[i] * a.max_ffn : xb + (size_t)brow[i] * H;
              cp_async16(bt + ptx::sw128_offset(32 * qd + (lane >> 3) + 4 * i, 8 * (lane & 7)), src + k0);
            }
          asm volatile("cp.async.commit_group;" ::: "memory");
        };
        for (int kb = 0; kb < nkb; ++kb, ++col) {
          const uint32_t g0 = step + 4 * kb + 2 * kh;  // this half's first step of the column
          const int ps = col % kPr;
          {
            TC_T0();
            if (!ptx::mbar_wait_suspend(&B.pfull[ps], (col / kPr) & 1u)) bad = true;
            TC_ADD(0);
          }
          const uint32_t pk = ptx::smem_u32(S.packed) + ps * C::kPacked;
          // the column's fields of every matrix, then its two steps; one
          // instance per format so only one format's fields are live
          auto column = [&](auto fmt) {
            constexpr bool kIsQ2 = decltype(fmt)::value == kQ2;
            using Row = typename std::conditional<kIsQ2, Q2Row, Q1Row>::type;
            Row rows[C::kMats];
#pragma unroll
            for (int m = 0; m < C::kMats; ++m) {
              if constexpr (kIsQ2)
                rows[m] = load_q2_row(pk + (m * 8 + tbi) * kQ2TileBlock, q, hh, kh);
              else
                rows[m] = load_q1_row(pk + (m * 8 + tbi) * kQ1TileBlock, q, hh, kh);
            }
            // the fields were read through the generic proxy and the slot's
            // next bytes arrive through the async proxy (bulk copy): order
            // the reads before the release that lets the producer refill it
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&B.pempty[ps]);
            // the B rows of the two steps (after the fence, which would
            // otherwise wait for these copies too)
            fetch_b(4 * kb + 2 * kh, g0);
            fetch_b(4 * kb + 2 * kh + 1, g0 + 1);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int as = (int)((g0 + j) % C::kAr);
              // the slot's previous MMAs are done (waited for when its B rows were fetched)
              ptx::tc_fence_after();
              const uint32_t at = tlane + kAccCols + (uint32_t)as * C::kSlotCols;
              TC_T0();
#pragma unroll
              for (int m = 0; m < C::kMats; ++m) {
                uint32_t r[32];
                if constexpr (kIsQ2)
                  dequant_q2_row(rows[m], j, sel2a, r);
                else
                  dequant_q1_row(rows[m], j, sel1a, selc, r);
                ptx::tmem_st32x32b_x32(at + 32 * m, r);
              }
              TC_ADD(2);
              ptx::tmem_wait_st();
              // this step's B rows landed (the next step's may still be in flight)
              if (j == 0)
                asm volatile("cp.async.wait_group 1;" ::: "memory");
              else
                asm volatile("cp.async.wait_group 0;" ::: "memory");
              ptx::fence_proxy_async_smem();  // generic-proxy writes -> the tensor cores
              ptx::tc_fence_before();
              __syncwarp();
              if (lane == 0) ptx::mbar_arrive(&B.afull[as]);
            }
          };
          if (U.qtype == kQ2)
            column(std::integral_constant<int, kQ2>());
          else
            column(std::integral_constant<int, kQ1>());
        }
        step += 4 * nkb;
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
            // h of 16 pairs x 128 rows staged as bf16 in row order, then
            // written as 16-byte pieces (pair i, piece g)
            uint32_t d1[16];
            ptx::tmem_ld16(du + (uint32_t)c0, d1);
            __nv_bfloat16 *T = reinterpret_cast<__nv_bfloat16 *>(S.stage) + (ep_stage & 1) * 16 * 128;
            ++ep_stage;
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              T[i * 128 + row] = __float2bfloat16_rn(silu_mul_fast(__uint_as_float(d0[i]), __uint_as_float(d1[i])));
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
