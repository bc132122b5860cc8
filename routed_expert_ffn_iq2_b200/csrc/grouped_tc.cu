// grouped_tc.cu -- the bucketed tensor-core path for calls with many tokens
// per expert (prefill).
//
// "Red Metal dev8 -- resident routed top-k layer", steps 4-6, for a batch of
// tokens: the (token, slot) pairs are bucketed by expert (route.cu), then
// every expert's gate/up and down projections run as dense contractions on
// the 5th-generation tensor cores (tcgen05.mma, bf16 operands in shared
// memory, fp32 accumulators in tensor memory).  Weights are decoded from the
// packed blocks straight into 128-byte-swizzled bf16 tiles (each value is
// exact in fp32; bf16 rounds it to nearest even); activations are rounded to
// bf16 the same way.  Accumulation is fp32.
//
// Work unit (persistent CTAs, atomic tickets):
//   gate/up  expert e, 128 output rows of gate and of up, up to 256 tokens:
//            D_gate, D_up in TMEM [128 x N]; epilogue h = SiLU(g) * u (bf16)
//            to the workspace, one row per (token, expert) pair;
//   down     expert e, 128 output rows of down, up to 256 tokens: D in TMEM;
//            epilogue out[token] += weight * D with fp32 atomics.
// Inputs along K arrive in 64-wide chunks through two shared-memory stages:
// all threads fill one stage while the tensor cores consume the other.
#include "internal.cuh"
#include "ptx.cuh"

namespace redlite {

constexpr int kTcThreads = 256;
constexpr int kKc = 64;                        // K chunk: one 128-byte swizzle row of bf16
constexpr int kTileA = 128 * kKc * 2;          // 16 KB: 128 rows x 64 bf16
constexpr int kTileB = kTcTokens * kKc * 2;    // 32 KB: 256 tokens x 64 bf16

struct TcSmem {
  uint8_t *stage[2];  // gate/up: A_gate | A_up | B ; down: A | B
  int8_t *g2, *g1;    // expanded grids (int8)
  int *tok;           // tokens of the current unit
  float *wt;          // their router weights (down)
  uint64_t *mma_done; // [2]
  uint32_t *taddr;
  int *unit;
};

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&b);
}

// 8 weights of group G of a resident matrix -> 8 bf16 (exact fp32 values
// rounded to nearest even), read with the grid from shared memory.
template <int QT>
__device__ __forceinline__ uint4 group_bf16(const uint8_t *mat, int64_t k, int64_t G, const int8_t *grid) {
  float w[8];
  decode_group_f32<QT>(mat, k, true, G, grid, w);
  return make_uint4(bf16x2_bits(w[0], w[1]), bf16x2_bits(w[2], w[3]), bf16x2_bits(w[4], w[5]),
                    bf16x2_bits(w[6], w[7]));
}

// Decode rows [row0, row0+128) x inputs [k0, k0+64) of a matrix with k inputs
// into a swizzled bf16 tile (all threads; 1024 groups, 4 per thread).
template <int QT>
__device__ __forceinline__ void fill_weights(uint8_t *tile, const uint8_t *mat, int64_t k, int row0, int k0,
                                             const int8_t *grid) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int g = threadIdx.x + kTcThreads * i;  // 0..1023
    const int r = g >> 3, c8 = g & 7;
    const int64_t G = ((int64_t)(row0 + r) * k + k0 + 8 * c8) >> 3;
    *reinterpret_cast<uint4 *>(tile + ptx::sw128_offset(r, 8 * c8)) = group_bf16<QT>(mat, k, G, grid);
  }
}

__device__ __forceinline__ void fill_weights_any(int qtype, uint8_t *tile, const uint8_t *mat, int64_t k, int row0,
                                                 int k0, const TcSmem &S) {
  if (qtype == kQ2)
    fill_weights<kQ2>(tile, mat, k, row0, k0, S.g2);
  else
    fill_weights<kQ1>(tile, mat, k, row0, k0, S.g1);
}

// Token rows of B from fp32 activations (bf16-rounded); rows >= n_real are zero.
__device__ __forceinline__ void fill_tokens_f32(uint8_t *tile, const float *x, int64_t hidden, int k0, int n_real,
                                                int n_pad, const int *tok) {
  for (int g = threadIdx.x; g < n_pad * 8; g += kTcThreads) {
    const int j = g >> 3, c8 = g & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j < n_real) {
      const float4 *src = reinterpret_cast<const float4 *>(x + (size_t)tok[j] * hidden + k0 + 8 * c8);
      const float4 a = __ldg(src), b = __ldg(src + 1);
      v = make_uint4(bf16x2_bits(a.x, a.y), bf16x2_bits(a.z, a.w), bf16x2_bits(b.x, b.y), bf16x2_bits(b.z, b.w));
    }
    *reinterpret_cast<uint4 *>(tile + ptx::sw128_offset(j, 8 * c8)) = v;
  }
}

// Token rows of B from bf16 rows of h (row stride ld elements); rows >= n_real zero.
__device__ __forceinline__ void fill_tokens_bf16(uint8_t *tile, const __nv_bfloat16 *h, int64_t ld, int64_t row0,
                                                 int k0, int n_real, int n_pad) {
  for (int g = threadIdx.x; g < n_pad * 8; g += kTcThreads) {
    const int j = g >> 3, c8 = g & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (j < n_real) v = __ldcg(reinterpret_cast<const uint4 *>(h + (row0 + j) * ld + k0 + 8 * c8));
    *reinterpret_cast<uint4 *>(tile + ptx::sw128_offset(j, 8 * c8)) = v;
  }
}

struct UnitInfo {
  int inst, rt, n_real, n_pad, p0;
};

// Locate work unit j of one phase: the last active entry whose base <= j.
__device__ __forceinline__ UnitInfo find_unit(const ActiveEntry *act, int n_active, int j, bool down, int hidden) {
  int lo = 0, hi = n_active - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((down ? act[mid].dn_base : act[mid].gu_base) <= j) lo = mid; else hi = mid - 1;
  }
  const ActiveEntry &e = act[lo];
  const int nrt = (down ? hidden : e.ffn) / 128;
  const int loc = j - (down ? e.dn_base : e.gu_base);
  UnitInfo u;
  u.inst = lo;
  u.rt = loc % nrt;
  const int tt = loc / nrt;
  u.p0 = e.pair_start + kTcTokens * tt;
  u.n_real = min(kTcTokens, e.pair_count - kTcTokens * tt);
  u.n_pad = (u.n_real + 15) & ~15;
  return u;
}

__device__ __forceinline__ void carve(uint8_t *smem, TcSmem &S, int stage_bytes) {
  uintptr_t base = ((uintptr_t)smem + 1023) & ~(uintptr_t)1023;  // swizzled tiles need 1024-byte alignment
  uint8_t *p = reinterpret_cast<uint8_t *>(base);
  S.stage[0] = p;
  S.stage[1] = p + stage_bytes;
  p += 2 * stage_bytes;
  S.g2 = reinterpret_cast<int8_t *>(p);
  p += 512 * 8;
  S.g1 = reinterpret_cast<int8_t *>(p);
  p += 2048 * 8;
  S.tok = reinterpret_cast<int *>(p);
  p += sizeof(int) * kTcTokens;
  S.wt = reinterpret_cast<float *>(p);
  p += sizeof(float) * kTcTokens;
  S.mma_done = reinterpret_cast<uint64_t *>(p);
  p += 2 * sizeof(uint64_t);
  S.taddr = reinterpret_cast<uint32_t *>(p);
  p += 16;
  S.unit = reinterpret_cast<int *>(p);
}

__device__ __forceinline__ const redlite_moe_expert expert_desc(const TileArgs &a, const ActiveEntry &e) {
  return e.expert >= 0 ? a.experts[e.expert] : a.shared;
}

// One tensor-core kernel for both phases (DOWN selects the down projection).
template <bool DOWN>
__global__ void __launch_bounds__(kTcThreads, 1) grouped_tc_kernel(TileArgs a) {
  extern __shared__ uint8_t smem[];
  constexpr int kStageBytes = (DOWN ? 1 : 2) * kTileA + kTileB;
  constexpr uint32_t kCols = DOWN ? 256 : 512;  // TMEM columns: D (and D_up at +256)
  TcSmem S;
  carve(smem, S, kStageBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.hidden;
  Ctrl *ctrl = reinterpret_cast<Ctrl *>(a.ws + a.L.ctrl);
  const ActiveEntry *act = reinterpret_cast<const ActiveEntry *>(a.ws + a.L.active);
  const Pair *pairs = reinterpret_cast<const Pair *>(a.ws + a.L.pairs);
  __nv_bfloat16 *hbuf = reinterpret_cast<__nv_bfloat16 *>(a.ws + a.L.h);

  // expanded grids into shared memory
  for (int i = tid; i < (512 * 8 + 2048 * 8) / 16; i += kTcThreads)
    reinterpret_cast<uint4 *>(S.g2)[i] = __ldg(reinterpret_cast<const uint4 *>(a.grids + kGridQ2Vals) + i);
  if (warp == 0) {
    ptx::tmem_alloc(S.taddr, kCols);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::mbar_init(&S.mma_done[0], 1);
    ptx::mbar_init(&S.mma_done[1], 1);
    ptx::mbar_fence_init();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *S.taddr;
  const int n_active = ctrl->n_active;
  const int n_units = DOWN ? ctrl->n_dn_units : ctrl->n_gu_units;
  uint32_t waits[2] = {0u, 0u};  // completed phases consumed per stage
  bool timed_out = false;

  for (;;) {
    if (tid == 0) *S.unit = atomicAdd(DOWN ? &ctrl->ticket_dn : &ctrl->ticket_gu, 1);
    __syncthreads();
    const int j = *S.unit;
    if (j >= n_units || timed_out) break;
    const UnitInfo U = find_unit(act, n_active, j, DOWN, H);
    const ActiveEntry &E = act[U.inst];
    const redlite_moe_expert ex = expert_desc(a, E);
    for (int i = tid; i < U.n_real; i += kTcThreads) {
      const Pair pr = pairs[U.p0 + i];
      S.tok[i] = pr.token;
      S.wt[i] = pr.weight;
    }
    __syncthreads();
    const int K = DOWN ? E.ffn : H;
    const int nk = K / kKc;
    const uint32_t idesc = ptx::idesc_bf16_f32(128, U.n_pad);
    for (int kc = 0; kc < nk; ++kc) {
      const int st = kc & 1;
      if (kc >= 2) {  // the mma of chunk kc - 2 used this stage
        if (!ptx::mbar_wait(&S.mma_done[st], waits[st] & 1u)) timed_out = true;
        ++waits[st];
      }
      uint8_t *A0 = S.stage[st];
      if (DOWN) {
        fill_weights_any(E.qtype, A0, (const uint8_t *)ex.down, E.ffn, 128 * U.rt, kKc * kc, S);
        fill_tokens_bf16(A0 + kTileA, hbuf, a.max_ffn, U.p0, kKc * kc, U.n_real, U.n_pad);
      } else {
        fill_weights_any(E.qtype, A0, (const uint8_t *)ex.gate, H, 128 * U.rt, kKc * kc, S);
        fill_weights_any(E.qtype, A0 + kTileA, (const uint8_t *)ex.up, H, 128 * U.rt, kKc * kc, S);
        fill_tokens_f32(A0 + 2 * kTileA, a.x, H, kKc * kc, U.n_real, U.n_pad, S.tok);
      }
      ptx::fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        ptx::tc_fence_after();
        const uint32_t a0 = ptx::smem_u32(A0);
        const uint32_t b0 = a0 + (DOWN ? 1 : 2) * kTileA;
#pragma unroll
        for (int ks = 0; ks < kKc / 16; ++ks) {
          const bool acc = kc > 0 || ks > 0;
          ptx::umma_bf16(tmem, ptx::sdesc_k_sw128(a0 + 32 * ks), ptx::sdesc_k_sw128(b0 + 32 * ks), idesc, acc);
          if (!DOWN)
            ptx::umma_bf16(tmem + 256, ptx::sdesc_k_sw128(a0 + kTileA + 32 * ks), ptx::sdesc_k_sw128(b0 + 32 * ks),
                           idesc, acc);
        }
        ptx::umma_commit(&S.mma_done[st]);
      }
    }
    // drain the last two chunks' commits (they cover every mma of the unit)
    for (int kc = (nk >= 2 ? nk - 2 : 0); kc < nk; ++kc) {
      const int st = kc & 1;
      if (!ptx::mbar_wait(&S.mma_done[st], waits[st] & 1u)) timed_out = true;
      ++waits[st];
    }
    ptx::tc_fence_after();
    // epilogue: warp w reads TMEM lanes 32 (w % 4) .. (rows), column chunks of 16
    const int lg = warp & 3, half = warp >> 2;
    const int row = 32 * lg + lane;
    for (int c0 = 16 * half; c0 < U.n_pad; c0 += 32) {
      uint32_t d0[16];
      ptx::tmem_ld16(tmem + ((uint32_t)(32 * lg) << 16) + (uint32_t)c0, d0);
      if (DOWN) {
        ptx::tmem_wait_ld();
        const int r = 128 * U.rt + row;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int jj = c0 + i;
          if (jj < U.n_real) atomicAdd(a.out + (size_t)S.tok[jj] * H + r, S.wt[jj] * __uint_as_float(d0[i]));
        }
      } else {
        uint32_t d1[16];
        ptx::tmem_ld16(tmem + 256 + ((uint32_t)(32 * lg) << 16) + (uint32_t)c0, d1);
        ptx::tmem_wait_ld();
        const int col = 128 * U.rt + row;  // position within the expert's width
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int jj = c0 + i;
          if (jj < U.n_real)
            hbuf[(size_t)(U.p0 + jj) * a.max_ffn + col] =
                __float2bfloat16_rn(silu_mul(__uint_as_float(d0[i]), __uint_as_float(d1[i])));
        }
      }
    }
    ptx::tc_fence_before();
    timed_out = __syncthreads_or(timed_out);  // TMEM read and tokens consumed before the next unit
  }
  if (timed_out && lane == 0) atomicOr(a.status, REDLITE_STATUS_TIMEOUT);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 0) ptx::tmem_dealloc(tmem, kCols);
}

static size_t tc_smem_bytes(bool down) {
  const size_t stage = (down ? 1 : 2) * (size_t)kTileA + kTileB;
  return 1024 + 2 * stage + 512 * 8 + 2048 * 8 + 2 * sizeof(int) * kTcTokens + 2 * sizeof(uint64_t) + 16 + 16;
}

bool tc_supported(int hidden, int max_ffn) {
  return hidden % 256 == 0 && max_ffn % 256 == 0;
}

cudaError_t launch_tc(const TileArgs &a, cudaStream_t stream) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const size_t s_gu = tc_smem_bytes(false), s_dn = tc_smem_bytes(true);
  e = cudaFuncSetAttribute(grouped_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s_gu);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(grouped_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)s_dn);
  if (e != cudaSuccess) return e;
  grouped_tc_kernel<false><<<sms, kTcThreads, s_gu, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  grouped_tc_kernel<true><<<sms, kTcThreads, s_dn, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace redlite
