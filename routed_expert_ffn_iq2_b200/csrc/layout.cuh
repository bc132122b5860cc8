// layout.cuh -- the resident ("tiled") byte layout of packed matrices.
//
// The slot builder stores each matrix whose rows are a multiple of 16 and
// whose inputs are a multiple of 256 in a tiled layout: the same bytes as
// the interchange layout (include/redlite_moe.h), regrouped per tile-block
// of 16 rows x 256 inputs so that every lane of a warp finds the fields of
// the weight groups it feeds into the tensor-core fragments in one or two
// 16-byte shared-memory loads.  Other shapes keep the interchange layout.
//
// Tile t covers rows 16t..16t+15; its k/256 tile-blocks follow each other in
// input order; tile-block (t, kb) starts at byte (t * k/256 + kb) * 16 * B,
// B = 74 (IQ2_XS-style) or 56 (IQ1_M-style).  Lane L of a warp has
// q = L >> 2 (rows q and q+8 of the tile) and t = L & 3.
//
// IQ2_XS-style tile-block (1184 bytes).  Lane L handles groups g = 4c + t
// (c = 0..7) of rows q (h = 0) and q+8 (h = 1); field index i = 2c + h.
//   [32L + i]        qs[g] of row q+8h
//   [32L + 16 + 4w]  u32 sign word w (w = 0..3): bit 4j + m = sign bit j of
//                    field i = 4w + m (bit j of signs[g] of row q+8h), so
//                    shifting word w left by 2 - m puts the sign of weight j
//                    at bit 4j + 2 of every nibble
//   [1024 + 2L]      u16: bit i = index bit 8 of that group
//   [1088 + 8q]      scales[0..3] of row q, then scales[0..3] of row q+8
//   [1152 + 4q]      d of row q, then d of row q+8
// IQ1_M-style tile-block (896 bytes).  Lanes L and L^1 (pair p = t >> 1)
// handle groups g = 2s + p (s = 0..15) of rows q and q+8, each lane half of
// every group (t & 1 selects weights 0-3 or 4-7); entry i = 2s + h.
//   [48(2q+p) + i]      qs[g] of row q+8h
//   [48(2q+p) + 32 + i/2] nibble (i & 1) = the qh nibble of that group
//   [768 + 12q]         scales[0..5] of row q, then of row q+8
//   [864 + 4q]          d of row q, then d of row q+8
#pragma once

#include <stdint.h>

namespace redlite {

constexpr int kTileRows = 16;
constexpr int kQ2TileBlock = 16 * 74;  // 1184
constexpr int kQ1TileBlock = 16 * 56;  // 896

inline __host__ __device__ bool tiled_shape(int64_t rows, int64_t k) {
  return rows > 0 && k > 0 && rows % kTileRows == 0 && k % 256 == 0;
}

inline __host__ __device__ int tile_block_bytes(int qtype) { return qtype == 1 ? kQ2TileBlock : kQ1TileBlock; }

// Byte offset of the tile-block holding row r, input block kb.
inline __host__ __device__ int64_t tile_block_offset(int qtype, int64_t k, int64_t r, int64_t kb) {
  return ((r / kTileRows) * (k / 256) + kb) * tile_block_bytes(qtype);
}

// Field offsets of (row-in-tile rr, group g) inside an IQ2 tile-block.
struct Q2Loc {
  int qs, sign_word, sign_shift, qh_word, qh_bit, scales, d;
};
inline __host__ __device__ Q2Loc q2_loc(int rr, int g) {
  const int q = rr & 7, h = rr >> 3, c = g >> 2, t = g & 3;
  const int L = 4 * q + t, i = 2 * c + h;
  Q2Loc o;
  o.qs = 32 * L + i;
  o.sign_word = 32 * L + 16 + 4 * (i >> 2);
  o.sign_shift = i & 3;
  o.qh_word = 1024 + 2 * L;
  o.qh_bit = i;
  o.scales = 1088 + 8 * q + 4 * h;
  o.d = 1152 + 4 * q + 2 * h;
  return o;
}

// Field offsets of (row-in-tile rr, group g) inside an IQ1 tile-block.
struct Q1Loc {
  int qs, nib_byte, nib_shift, scales, d;
};
inline __host__ __device__ Q1Loc q1_loc(int rr, int g) {
  const int q = rr & 7, h = rr >> 3, s = g >> 1, p = g & 1;
  const int base = 48 * (2 * q + p), i = 2 * s + h;
  Q1Loc o;
  o.qs = base + i;
  o.nib_byte = base + 32 + (i >> 1);
  o.nib_shift = 4 * (i & 1);
  o.scales = 768 + 12 * q + 6 * h;
  o.d = 864 + 4 * q + 2 * h;
  return o;
}

}  // namespace redlite
