// grids.cu -- one-time codebook expansion and the dequantisation check kernel.
//
// "Red Lite dev10 -- standalone native Metal path", section "Quant grids":
// each grid entry is eight values kept as 2-bit symbols; IQ2_XS-style maps
// symbols to 0x08/0x19/0x2b, IQ1_M-style (2048-entry grid) to -1/0/+1.
// Value j of an entry is symbol (c >> 2j) & 3, symbols in ascending value
// order (the page leaves the order open).
#include "internal.cuh"

namespace redlite {

// One thread per (format, entry): writes the int8 values, the bf16 copies
// the tensor-core path reads, and keeps the compact entry.
// Byte-permute selectors that build weights 2w, 2w+1 of a grid entry (compact
// 2-bit symbols c) as bf16 pairs from a table of three bf16 values.
__device__ uint64_t bf16_pair_selectors(uint16_t c) {
  uint64_t sel = 0;
  for (int j = 0; j < 8; ++j) {
    const uint64_t s = (c >> (2 * j)) & 3;
    sel |= ((2 * s) | ((2 * s + 1) << 4)) << (8 * j);
  }
  return sel;
}

__global__ void expand_grids_kernel(const uint16_t *__restrict__ comp2, const uint16_t *__restrict__ comp1,
                                    uint8_t *__restrict__ grids) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < kQ2GridEntries) {
    const uint16_t c = comp2[t];
    int8_t *v = reinterpret_cast<int8_t *>(grids + kGridQ2Vals) + 8 * t;
    __nv_bfloat16 *vb = reinterpret_cast<__nv_bfloat16 *>(grids + kGridQ2Bf16) + 8 * t;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int s = (c >> (2 * j)) & 3;
      const int val = s == 0 ? 8 : (s == 1 ? 25 : 43);
      v[j] = (int8_t)val;
      vb[j] = __int2bfloat16_rn(val);
    }
    reinterpret_cast<uint16_t *>(grids + kGridQ2Comp)[t] = c;
    uint32_t sel = 0;
    for (int j = 0; j < 8; ++j) sel |= (uint32_t)((c >> (2 * j)) & 3) << (4 * j);
    reinterpret_cast<uint32_t *>(grids + kGridQ2Sel)[t] = sel;
    reinterpret_cast<uint64_t *>(grids + kGridQ2Bsel)[t] = bf16_pair_selectors(c);
    if (t < 256) {
      uint32_t sg = 0;
      for (int j = 0; j < 8; ++j) sg |= (uint32_t)((t >> j) & 1) << (4 * j + 2);
      reinterpret_cast<uint32_t *>(grids + kGridSign)[t] = sg;
    }
  } else if (t < kQ2GridEntries + kQ1GridEntries) {
    const int e = t - kQ2GridEntries;
    const uint16_t c = comp1[e];
    int8_t *v = reinterpret_cast<int8_t *>(grids + kGridQ1Vals) + 8 * e;
    __nv_bfloat16 *p0 = reinterpret_cast<__nv_bfloat16 *>(grids + kGridQ1Bf16p) + 8 * e;
    __nv_bfloat16 *p1 = p0 + 8 * kQ1GridEntries;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int s = (c >> (2 * j)) & 3;
      const int val = s - 1;
      v[j] = (int8_t)val;
      p0[j] = __int2bfloat16_rn(8 * val + 1);  // 8 * (val + 1/8)
      p1[j] = __int2bfloat16_rn(8 * val - 1);  // 8 * (val - 1/8)
    }
    reinterpret_cast<uint16_t *>(grids + kGridQ1Comp)[e] = c;
    uint32_t sel = 0;
    for (int j = 0; j < 8; ++j) sel |= (uint32_t)((c >> (2 * j)) & 3) << (4 * j);
    reinterpret_cast<uint32_t *>(grids + kGridQ1Sel)[e] = sel;
    reinterpret_cast<uint64_t *>(grids + kGridQ1Bsel)[e] = bf16_pair_selectors(c);
    reinterpret_cast<uint32_t *>(grids + kGridQ1Sel)[e + 2048] = sel | 0x44444444u;
  }
}

// Dequantise a packed matrix: one thread per 8-weight group.
template <int QT>
__global__ void dequant_kernel(const uint8_t *__restrict__ mat, int64_t n_groups, int64_t k, bool tiled,
                               const int8_t *__restrict__ grid, float *__restrict__ out_f32,
                               uint16_t *__restrict__ out_bf16) {
  for (int64_t G = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; G < n_groups;
       G += (int64_t)gridDim.x * blockDim.x) {
    float w[8];
    decode_group_f32<QT>(mat, k, tiled, G, grid, w);
    if (out_f32) {
      float4 *o = reinterpret_cast<float4 *>(out_f32 + 8 * G);
      o[0] = make_float4(w[0], w[1], w[2], w[3]);
      o[1] = make_float4(w[4], w[5], w[6], w[7]);
    }
    if (out_bf16) {
      uint32_t p[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        __nv_bfloat162 b = __floats2bfloat162_rn(w[2 * j], w[2 * j + 1]);
        p[j] = *reinterpret_cast<uint32_t *>(&b);
      }
      *reinterpret_cast<uint4 *>(out_bf16 + 8 * G) = make_uint4(p[0], p[1], p[2], p[3]);
    }
  }
}

cudaError_t launch_expand_grids(const uint16_t *comp2_dev, const uint16_t *comp1_dev, void *grids,
                                cudaStream_t stream) {
  const int n = kQ2GridEntries + kQ1GridEntries;
  expand_grids_kernel<<<(n + 255) / 256, 256, 0, stream>>>(comp2_dev, comp1_dev, (uint8_t *)grids);
  return cudaGetLastError();
}

cudaError_t launch_dequant(int qtype, const void *packed, int64_t rows, int64_t k, const void *grids, float *out_f32,
                           uint16_t *out_bf16, cudaStream_t stream) {
  const int64_t groups = rows * k / 8;
  const int threads = 256;
  int64_t blocks = (groups + threads - 1) / threads;
  if (blocks > 148 * 64) blocks = 148 * 64;
  const uint8_t *g = (const uint8_t *)grids;
  const bool tiled = tiled_shape(rows, k);
  if (qtype == kQ2)
    dequant_kernel<kQ2><<<(unsigned)blocks, threads, 0, stream>>>(
        (const uint8_t *)packed, groups, k, tiled, (const int8_t *)(g + kGridQ2Vals), out_f32, out_bf16);
  else
    dequant_kernel<kQ1><<<(unsigned)blocks, threads, 0, stream>>>(
        (const uint8_t *)packed, groups, k, tiled, (const int8_t *)(g + kGridQ1Vals), out_f32, out_bf16);
  return cudaGetLastError();
}

}  // namespace redlite
