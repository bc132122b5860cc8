// pack.cu -- host-side conversion of a packed matrix from the interchange
// layout (include/redlite_moe.h) to the resident tiled layout (layout.cuh).
// Same bytes, regrouped; shapes that are not tiled are copied unchanged.
#include <string.h>

#include "internal.cuh"

namespace redlite {

static void pack_tile_block_q2(const uint8_t *src, int64_t k, int64_t r0, int64_t kb, uint8_t *tb) {
  memset(tb, 0, kQ2TileBlock);
  for (int rr = 0; rr < 16; ++rr) {
    const uint8_t *b = src + ((r0 + rr) * (k / 256) + kb) * kQ2BlockBytes;
    for (int g = 0; g < 32; ++g) {
      const Q2Loc o = q2_loc(rr, g);
      tb[o.qs] = b[6 + g];
      for (int j = 0; j < 8; ++j) {  // sign bit j -> bit 4j + m of the field's sign word
        const int bit = 4 * j + o.sign_shift;
        tb[o.sign_word + (bit >> 3)] |= (uint8_t)(((b[42 + g] >> j) & 1) << (bit & 7));
      }
      const int hb = (b[38 + (g >> 3)] >> (g & 7)) & 1;
      uint16_t w = (uint16_t)(tb[o.qh_word] | (tb[o.qh_word + 1] << 8));
      w |= (uint16_t)(hb << o.qh_bit);
      tb[o.qh_word] = (uint8_t)(w & 0xFF);
      tb[o.qh_word + 1] = (uint8_t)(w >> 8);
    }
    const Q2Loc o = q2_loc(rr, 0);
    memcpy(tb + o.scales, b + 2, 4);
    memcpy(tb + o.d, b, 2);
  }
}

static void pack_tile_block_q1(const uint8_t *src, int64_t k, int64_t r0, int64_t kb, uint8_t *tb) {
  memset(tb, 0, kQ1TileBlock);
  for (int rr = 0; rr < 16; ++rr) {
    const uint8_t *b = src + ((r0 + rr) * (k / 256) + kb) * kQ1BlockBytes;
    for (int g = 0; g < 32; ++g) {
      const Q1Loc o = q1_loc(rr, g);
      tb[o.qs] = b[2 + g];
      const int nib = (b[34 + (g >> 1)] >> (4 * (g & 1))) & 15;
      tb[o.nib_byte] |= (uint8_t)(nib << o.nib_shift);
    }
    const Q1Loc o = q1_loc(rr, 0);
    memcpy(tb + o.scales, b + 50, 6);
    memcpy(tb + o.d, b, 2);
  }
}

int pack_matrix_host(int qtype, int64_t rows, int64_t k, const uint8_t *src, uint8_t *dst) {
  const size_t bytes = matrix_bytes(qtype, rows, k);
  if (!bytes) return REDLITE_EUNSUPPORTED;
  if (!tiled_shape(rows, k)) {
    memcpy(dst, src, bytes);
    return REDLITE_OK;
  }
  const int tbb = tile_block_bytes(qtype);
  for (int64_t t = 0; t < rows / 16; ++t)
    for (int64_t kb = 0; kb < k / 256; ++kb) {
      uint8_t *tb = dst + (t * (k / 256) + kb) * tbb;
      if (qtype == kQ2)
        pack_tile_block_q2(src, k, 16 * t, kb, tb);
      else
        pack_tile_block_q1(src, k, 16 * t, kb, tb);
    }
  return REDLITE_OK;
}

}  // namespace redlite

extern "C" int redlite_moe_pack_matrix(int32_t qtype, int64_t rows, int64_t k, const void *src, void *dst) {
  if (!src || !dst || src == dst) return REDLITE_EINVAL;
  if (qtype != redlite::kQ2 && qtype != redlite::kQ1) return REDLITE_EINVAL;
  return redlite::pack_matrix_host(qtype, rows, k, (const uint8_t *)src, (uint8_t *)dst);
}
