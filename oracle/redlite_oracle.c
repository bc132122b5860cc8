/*
 * redlite_oracle.c -- plain, slow, obviously correct CPU reference of the
 * routed top-k MoE layer over codebook-quantised experts.
 *
 * TEST INFRASTRUCTURE ONLY (see redlite_oracle.h).  No blocking, fusion or
 * reordering beyond the definitions below; fp64 accumulation throughout.
 */
#include "redlite_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ grids
 * "Red Lite dev10 -- standalone native Metal path", section "Quant grids":
 * each grid entry is eight values kept as compact 2-bit symbols; IQ2_XS maps
 * the symbols to 0x08/0x19/0x2b, IQ1_M (which reuses the 2048-entry IQ1_S
 * grid) maps them to -1/0/+1.  The page leaves the symbol order open.
 * Reading: value j of an entry is symbol (entry >> 2j) & 3, and symbols
 * 0,1,2 name the values in ascending order; symbol 3 names nothing. */
int oracle_expand_grid(int qtype, const uint16_t *compact, int n, int8_t *out) {
  static const int8_t iq2_vals[3] = {0x08, 0x19, 0x2b};
  static const int8_t iq1_vals[3] = {-1, 0, 1};
  const int8_t *vals;
  if (qtype == ORACLE_QTYPE_IQ2XS)
    vals = iq2_vals;
  else if (qtype == ORACLE_QTYPE_IQ1M)
    vals = iq1_vals;
  else
    return ORACLE_EINVAL;
  if (!compact || !out || n < 0) return ORACLE_EINVAL;
  for (int e = 0; e < n; ++e) {
    for (int j = 0; j < 8; ++j) {
      int sym = (compact[e] >> (2 * j)) & 3;
      if (sym == 3) return ORACLE_EINVAL;
      out[8 * e + j] = vals[sym];
    }
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------ scalars */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_fp16_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int expo = (h >> 10) & 31;
  int frac = h & 1023;
  double mag;
  if (expo == 0)
    mag = ldexp((double)frac, -24); /* zero or subnormal: frac * 2^-14 * 2^-10 */
  else if (expo == 31)
    mag = frac ? NAN : INFINITY;
  else
    mag = ldexp(1024.0 + frac, expo - 25); /* (1 + frac/1024) * 2^(expo-15) */
  return sign ? -mag : mag;
}

/* bfloat16 keeps the upper 16 bits of a binary32.  Rounding to nearest with
 * ties to even: look at the 16 dropped bits; above half rounds up, below
 * half rounds down, exactly half rounds to the even upper pattern. */
uint16_t oracle_float_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t upper = u >> 16, dropped = u & 0xffffu;
  if (dropped > 0x8000u || (dropped == 0x8000u && (upper & 1u))) upper += 1u;
  return (uint16_t)upper;
}

int oracle_block_bytes(int qtype) {
  if (qtype == ORACLE_QTYPE_IQ2XS) return 74;
  if (qtype == ORACLE_QTYPE_IQ1M) return 56;
  return -1;
}

/* A matrix of `rows` outputs and `k` inputs is its rows*k weights in row-major
 * order, cut into consecutive 256-weight blocks.  Reading (the pages do not
 * give block layouts): k is a multiple of 256, or a divisor of 256 that is a
 * multiple of 32 so that no 8-weight group or scale sub-block straddles rows. */
int oracle_shape_ok(int64_t rows, int64_t k) {
  if (rows <= 0 || k <= 0) return 0;
  if ((rows * k) % 256) return 0;
  if (k >= 256) return k % 256 == 0;
  return (256 % k == 0) && (k % 32 == 0);
}

/* ------------------------------------------------------------------ blocks */

static uint16_t load_u16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/* IQ2_XS-style block, 74 bytes per 256 weights (2.3125 bits per weight):
 *   bytes 0-1   d          fp16 block scale
 *   bytes 2-5   scales[4]  one 4-bit sub-scale per 32 weights, low nibble first
 *   bytes 6-37  qs[32]     low 8 bits of the 9-bit grid index of group g (8 weights)
 *   bytes 38-41 qh[4]      bit 8 of the index of group g: bit (g & 7) of qh[g >> 3]
 *   bytes 42-73 signs[32]  bit j of signs[g] set: weight 8g+j is negative
 * weight 8g+j = d * (2*sc+1)/8 * grid[idx][j] * (+1 or -1), sc of sub-block g>>2.
 * The odd-multiplier scale (2sc+1)/8 is this library's reading of the 4-bit
 * sub-scale (never zero).  Every such value is exact in fp32 and fp64. */
static double iq2_weight(const uint8_t *blk, int j, const int8_t *grid) {
  const uint8_t *scales = blk + 2, *qs = blk + 6, *qh = blk + 38, *signs = blk + 42;
  int g = j / 8, pos = j % 8;
  int idx = qs[g] | (((qh[g / 8] >> (g % 8)) & 1) << 8);
  int sub = g / 4;
  int sc = (scales[sub / 2] >> (4 * (sub % 2))) & 15;
  int neg = (signs[g] >> pos) & 1;
  double d = oracle_fp16_to_double(load_u16(blk));
  double v = d * (2.0 * sc + 1.0) / 8.0 * (double)grid[8 * idx + pos];
  return neg ? -v : v;
}

/* IQ1_M-style block, 56 bytes per 256 weights (1.75 bits per weight):
 *   bytes 0-1   d          fp16 block scale
 *   bytes 2-33  qs[32]     low 8 bits of the 11-bit grid index of group g
 *   bytes 34-49 qh[16]     one nibble per group (low nibble for even g):
 *                          bits 0-2 = index bits 8-10, bit 3 = delta sign
 *   bytes 50-55 scales[6]  sixteen 3-bit sub-scales (one per 16 weights),
 *                          sub-block b at bits 3b..3b+2 of the 48-bit
 *                          little-endian field
 * weight 8g+j = d * (2*sc+1) * (grid[idx][j] + delta), delta = -1/8 when the
 * nibble's bit 3 is set, else +1/8; sc of sub-block g>>1.  Exact in fp32. */
static double iq1_weight(const uint8_t *blk, int j, const int8_t *grid) {
  const uint8_t *qs = blk + 2, *qh = blk + 34, *scales = blk + 50;
  int g = j / 8, pos = j % 8;
  int nib = (qh[g / 2] >> (4 * (g % 2))) & 15;
  int idx = qs[g] | ((nib & 7) << 8);
  double delta = (nib & 8) ? -0.125 : 0.125;
  int sub = g / 2;
  uint64_t field = 0;
  for (int b = 0; b < 6; ++b) field |= (uint64_t)scales[b] << (8 * b);
  int sc = (int)((field >> (3 * sub)) & 7);
  double d = oracle_fp16_to_double(load_u16(blk));
  return d * (2.0 * sc + 1.0) * ((double)grid[8 * idx + pos] + delta);
}

/* Weights [start, start+count) of a packed matrix's row-major sequence. */
static void dequant_range(int qtype, const uint8_t *packed, int64_t start, int64_t count,
                          const int8_t *grid, double *out) {
  int bb = oracle_block_bytes(qtype);
  for (int64_t n = 0; n < count; ++n) {
    int64_t w = start + n;
    const uint8_t *blk = packed + (w / 256) * bb;
    int j = (int)(w % 256);
    out[n] = (qtype == ORACLE_QTYPE_IQ2XS) ? iq2_weight(blk, j, grid) : iq1_weight(blk, j, grid);
  }
}

int oracle_dequant_matrix(int qtype, const uint8_t *packed, int64_t rows, int64_t k,
                          const int8_t *grid, double *out) {
  if (oracle_block_bytes(qtype) < 0 || !packed || !grid || !out) return ORACLE_EINVAL;
  if (!oracle_shape_ok(rows, k)) return ORACLE_EINVAL;
  dequant_range(qtype, packed, 0, rows * k, grid, out);
  return ORACLE_OK;
}

/* ------------------------------------------------------------------ projection formats
 * The dense projections of the model the pages run use other GGUF formats
 * ("Red Lite dev15 -- DeltaNet projection bring-up", section
 * "Field-derived recurrent dimensions": ssm_ba Q8_0 (2048,64), ssm_out
 * Q4_K (4096,2048); "Red Lite dev16", section "Pinned full-attention graph":
 * attn_k / attn_v Q4_K (2048,512), attn_output Q4_K (4096,2048)).  The
 * pages print no bit layouts; the readings below are the plainest
 * packings of the named fields.
 *
 * Q8_0-style block, 34 bytes per 32 weights:
 *   bytes 0-1  d      fp16 block scale
 *   bytes 2-33 q[32]  signed 8-bit values
 * weight i = d * q[i].
 *
 * Q4_K-style super-block, 144 bytes per 256 weights (eight sub-blocks of 32):
 *   bytes 0-1   d       fp16 scale of the sub-block scales
 *   bytes 2-3   dmin    fp16 scale of the sub-block minima
 *   bytes 4-15  sm[12]  a 96-bit little-endian field: 6-bit scale of
 *                       sub-block j at bits 6j, 6-bit minimum of sub-block
 *                       j at bits 48 + 6j
 *   bytes 16-143 q[128] 4-bit values, weight i in byte i/2 (low nibble for
 *                       even i)
 * weight i = d * scale[i/32] * q_i - dmin * min[i/32]. */
int oracle_proj_block_weights(int qtype) {
  return qtype == ORACLE_QTYPE_Q8_0 ? 32 : (qtype == ORACLE_QTYPE_Q4_K ? 256 : -1);
}
int oracle_proj_block_bytes(int qtype) {
  return qtype == ORACLE_QTYPE_Q8_0 ? 34 : (qtype == ORACLE_QTYPE_Q4_K ? 144 : -1);
}

static double q8_0_weight(const uint8_t *blk, int i) {
  return oracle_fp16_to_double(load_u16(blk)) * (double)(int8_t)blk[2 + i];
}

static double q4_k_weight(const uint8_t *blk, int i) {
  const double d = oracle_fp16_to_double(load_u16(blk)), dmin = oracle_fp16_to_double(load_u16(blk + 2));
  const int j = i / 32;
  /* bits 6j.. and 48+6j.. of the 96-bit field bytes 4..15 */
  int sc = 0, mn = 0;
  for (int b = 0; b < 6; ++b) {
    const int bs = 6 * j + b, bm = 48 + 6 * j + b;
    sc |= ((blk[4 + bs / 8] >> (bs % 8)) & 1) << b;
    mn |= ((blk[4 + bm / 8] >> (bm % 8)) & 1) << b;
  }
  const int q = (blk[16 + i / 2] >> (4 * (i % 2))) & 15;
  return d * sc * q - dmin * mn;
}

/* Dequantise a rows x k matrix of a projection format (row-major weights
 * cut into consecutive blocks; k a multiple of the block size). */
int oracle_dequant_proj(int qtype, const uint8_t *packed, int64_t rows, int64_t k, double *out) {
  const int bw = oracle_proj_block_weights(qtype), bb = oracle_proj_block_bytes(qtype);
  if (bw < 0 || !packed || !out || rows <= 0 || k <= 0 || k % bw) return ORACLE_EINVAL;
  for (int64_t w = 0; w < rows * k; ++w) {
    const uint8_t *blk = packed + (w / bw) * bb;
    out[w] = qtype == ORACLE_QTYPE_Q8_0 ? q8_0_weight(blk, (int)(w % bw)) : q4_k_weight(blk, (int)(w % bw));
  }
  return ORACLE_OK;
}

/* y[t][r] = sum_c W[r][c] * x[t][c] for a projection-format matrix, in
 * double (c ascending).  x: [n_tokens, k] fp32; y: [n_tokens, rows]. */
int oracle_gemv_proj(int qtype, const uint8_t *packed, int64_t rows, int64_t k, const float *x, int n_tokens,
                     double *y) {
  if (n_tokens < 0 || !x || !y) return ORACLE_EINVAL;
  double *wd = (double *)malloc(sizeof(double) * (size_t)(rows * k));
  if (!wd) return ORACLE_EINVAL;
  int rc = oracle_dequant_proj(qtype, packed, rows, k, wd);
  if (rc == ORACLE_OK)
    for (int t = 0; t < n_tokens; ++t)
      for (int64_t r = 0; r < rows; ++r) {
        double s = 0.0;
        for (int64_t c = 0; c < k; ++c) s += wd[r * k + c] * (double)x[(int64_t)t * k + c];
        y[(int64_t)t * rows + r] = s;
      }
  free(wd);
  return rc;
}

/* ------------------------------------------------------------------ layer */

/* y[r] = sum_c W[r][c] * v[c] for r < rows, c < k, in double, c ascending.
 * Each row is dequantised 256 weights at a time into a small buffer. */
static void gemv(int qtype, const uint8_t *packed, int64_t rows, int64_t k, const int8_t *grid,
                 const double *v, double *y, int parallel_rows) {
#pragma omp parallel for schedule(static) if (parallel_rows)
  for (int64_t r = 0; r < rows; ++r) {
    double buf[256];
    double s = 0.0;
    for (int64_t c0 = 0; c0 < k; c0 += 256) {
      int64_t len = (k - c0 < 256) ? (k - c0) : 256;
      dequant_range(qtype, packed, r * k + c0, len, grid, buf);
      for (int64_t c = 0; c < len; ++c) s += buf[c] * v[c0 + c];
    }
    y[r] = s;
  }
}

static int expert_ok(const oracle_expert *ex, int hidden, const int8_t *g2, const int8_t *g1) {
  if (!ex || !ex->gate || !ex->up || !ex->down || ex->ffn <= 0) return 0;
  if (ex->qtype == ORACLE_QTYPE_IQ2XS && !g2) return 0;
  if (ex->qtype == ORACLE_QTYPE_IQ1M && !g1) return 0;
  if (oracle_block_bytes(ex->qtype) < 0) return 0;
  return oracle_shape_ok(ex->ffn, hidden) && oracle_shape_ok(hidden, ex->ffn);
}

/* "Red Metal dev8 -- resident routed top-k layer", step 4: each expert runs
 * gate, up, SiLU(gate)*up and down.  SiLU(z) = z / (1 + exp(-z)).
 * Step 5: accumulator += router_weight * expert_output.  The expert output
 * y is added with weight `omega` into acc. */
static void expert_ffn_accumulate(const oracle_expert *ex, int hidden, const double *xd,
                                  const int8_t *g2, const int8_t *g1, double omega, double *acc,
                                  int parallel_rows) {
  const int8_t *grid = (ex->qtype == ORACLE_QTYPE_IQ2XS) ? g2 : g1;
  int F = ex->ffn;
  double *g = (double *)malloc(sizeof(double) * F);
  double *u = (double *)malloc(sizeof(double) * F);
  double *h = (double *)malloc(sizeof(double) * F);
  double *y = (double *)malloc(sizeof(double) * hidden);
  gemv(ex->qtype, ex->gate, F, hidden, grid, xd, g, parallel_rows);
  gemv(ex->qtype, ex->up, F, hidden, grid, xd, u, parallel_rows);
  for (int i = 0; i < F; ++i) h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
  gemv(ex->qtype, ex->down, hidden, F, grid, h, y, parallel_rows);
  for (int r = 0; r < hidden; ++r) acc[r] += omega * y[r];
  free(g);
  free(u);
  free(h);
  free(y);
}

/* The layer, token by token (tokens are independent).  Router weights are
 * used as given: the layer does not renormalise them.  Duplicate ids in one
 * token each contribute.  The optional shared expert is added with weight 1
 * ("Red Lite dev16 -- complete full-attention parity": routed top-10 MoE plus
 * shared expert; no gate on the shared expert is named).  `out` is
 * overwritten; a residual add belongs to the caller. */
int oracle_moe_layer(const float *x, int n_tokens, int hidden, const int32_t *ids,
                     const float *weights, int top_k, int n_experts,
                     const oracle_expert *experts, const oracle_expert *shared,
                     const int8_t *grid_iq2, const int8_t *grid_iq1, double *out) {
  if (n_tokens < 0 || hidden <= 0 || top_k < 0 || n_experts < 0) return ORACLE_EINVAL;
  if (n_tokens == 0) return ORACLE_OK;
  if (!x || !out || (top_k > 0 && (!ids || !weights || !experts))) return ORACLE_EINVAL;
  if (shared && !expert_ok(shared, hidden, grid_iq2, grid_iq1)) return ORACLE_EINVAL;
  int skipped = 0;
  int par_tokens = n_tokens > 1;
#pragma omp parallel for schedule(dynamic, 1) if (par_tokens) reduction(| : skipped)
  for (int t = 0; t < n_tokens; ++t) {
    double *xd = (double *)malloc(sizeof(double) * hidden);
    double *acc = out + (int64_t)t * hidden;
    for (int c = 0; c < hidden; ++c) xd[c] = (double)x[(int64_t)t * hidden + c];
    for (int r = 0; r < hidden; ++r) acc[r] = 0.0;
    for (int s = 0; s < top_k; ++s) {
      int32_t e = ids[(int64_t)t * top_k + s];
      double omega = (double)weights[(int64_t)t * top_k + s];
      if (e < 0 || e >= n_experts || !expert_ok(&experts[e], hidden, grid_iq2, grid_iq1)) {
        skipped = 1;
        continue;
      }
      expert_ffn_accumulate(&experts[e], hidden, xd, grid_iq2, grid_iq1, omega, acc, !par_tokens);
    }
    if (shared) expert_ffn_accumulate(shared, hidden, xd, grid_iq2, grid_iq1, 1.0, acc, !par_tokens);
    free(xd);
  }
  return skipped ? ORACLE_SKIPPED_PAIRS : ORACLE_OK;
}

/* ------------------------------------------------------------------ router
 * The step that feeds the layer its expert ids and router weights.  The
 * pages name it as the milestone after the routed layer ("Red Metal dev8",
 * section "Field validation": router-network integration and real token
 * router outputs; "Red Lite dev10", section "What dev10 does not yet claim":
 * connect the actual router output to the top-k path) without stating its
 * arithmetic.  Reading (the router of the Qwen3-Next layers the pages run,
 * and the recipe of the batched-decode workload): per token,
 *   1. p = softmax(logits) over the n_experts logits (the largest logit is
 *      subtracted before exp; exp is libm's, in double);
 *   2. the top_k experts by p, in descending order of p, equal p going to
 *      the lower id first;
 *   3. their probabilities renormalised to sum 1: w_j = p_j / sum of the
 *      selected p. */
static void route_token(const double *lg, int n_experts, int top_k, double *p, char *taken, int32_t *ids,
                        double *w) {
  /* step 1: softmax */
  double m = lg[0];
  for (int e = 1; e < n_experts; ++e)
    if (lg[e] > m) m = lg[e];
  double sum = 0.0;
  for (int e = 0; e < n_experts; ++e) {
    p[e] = exp(lg[e] - m);
    sum += p[e];
  }
  for (int e = 0; e < n_experts; ++e) p[e] /= sum;
  /* step 2: top_k by probability, one at a time; only a strictly larger p
   * replaces the current choice, so equal p keep the lower id */
  memset(taken, 0, (size_t)n_experts);
  double sel = 0.0;
  for (int j = 0; j < top_k; ++j) {
    int best = -1;
    for (int e = 0; e < n_experts; ++e)
      if (!taken[e] && (best < 0 || p[e] > p[best])) best = e;
    taken[best] = 1;
    ids[j] = best;
    w[j] = p[best];
    sel += p[best];
  }
  /* step 3: renormalise over the selected experts */
  for (int j = 0; j < top_k; ++j) w[j] /= sel;
}

/* ids: [n_tokens, top_k]; weights: [n_tokens, top_k] doubles. */
int oracle_route_topk(const float *logits, int n_tokens, int n_experts, int top_k, int32_t *ids,
                      double *weights) {
  if (n_tokens < 0 || n_experts <= 0 || top_k <= 0 || top_k > n_experts) return ORACLE_EINVAL;
  if (n_tokens == 0) return ORACLE_OK;
  if (!logits || !ids || !weights) return ORACLE_EINVAL;
  double *lg = (double *)malloc(sizeof(double) * n_experts);
  double *p = (double *)malloc(sizeof(double) * n_experts);
  char *taken = (char *)malloc((size_t)n_experts);
  for (int t = 0; t < n_tokens; ++t) {
    for (int e = 0; e < n_experts; ++e) lg[e] = (double)logits[(int64_t)t * n_experts + e];
    route_token(lg, n_experts, top_k, p, taken, ids + (int64_t)t * top_k, weights + (int64_t)t * top_k);
  }
  free(lg);
  free(p);
  free(taken);
  return ORACLE_OK;
}

/* ------------------------------------------------------------------ block
 * The composition around the layer ("Red Lite dev16 -- complete
 * full-attention parity", block composition paragraph: the attention
 * residual, the post-attention RMSNorm, the routed top-10 MoE plus shared
 * expert, and the final residual).  For every token, h being the hidden
 * state after the attention residual:
 *   1. xn = RMSNorm(h): xn_i = gamma_i * h_i / sqrt(mean_j(h_j^2) + eps)
 *      (reading: the plain RMSNorm with a multiplicative weight);
 *   2. logits = W_r xn (router matrix [n_experts, hidden]);
 *   3. ids, weights = the router above applied to the logits;
 *   4. y = the routed layer of xn with those ids and weights, plus the
 *      shared expert with weight 1 (oracle_moe_layer's definition);
 *   5. out = h + y.
 * Every step is in double: xn and the logits are not rounded to float.
 * ids_out, weights_out (optional): the routing chosen in step 3. */
int oracle_moe_block(const float *h, int n_tokens, int hidden, const float *gamma, double eps,
                     const float *router_w, int n_experts, int top_k, const oracle_expert *experts,
                     const oracle_expert *shared, const int8_t *grid_iq2, const int8_t *grid_iq1, double *out,
                     int32_t *ids_out, double *weights_out) {
  if (n_tokens < 0 || hidden <= 0 || n_experts <= 0 || top_k <= 0 || top_k > n_experts || eps < 0.0)
    return ORACLE_EINVAL;
  if (n_tokens == 0) return ORACLE_OK;
  if (!h || !gamma || !router_w || !experts || !out) return ORACLE_EINVAL;
  if (shared && !expert_ok(shared, hidden, grid_iq2, grid_iq1)) return ORACLE_EINVAL;
  int skipped = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : skipped)
  for (int t = 0; t < n_tokens; ++t) {
    const float *ht = h + (int64_t)t * hidden;
    double *xn = (double *)malloc(sizeof(double) * hidden);
    double *lg = (double *)malloc(sizeof(double) * n_experts);
    double *p = (double *)malloc(sizeof(double) * n_experts);
    char *taken = (char *)malloc((size_t)n_experts);
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * top_k);
    double *w = (double *)malloc(sizeof(double) * top_k);
    double *acc = out + (int64_t)t * hidden;
    /* step 1 */
    double ss = 0.0;
    for (int i = 0; i < hidden; ++i) ss += (double)ht[i] * (double)ht[i];
    const double inv = 1.0 / sqrt(ss / hidden + eps);
    for (int i = 0; i < hidden; ++i) xn[i] = (double)gamma[i] * (double)ht[i] * inv;
    /* step 2 */
    for (int e = 0; e < n_experts; ++e) {
      double s = 0.0;
      for (int i = 0; i < hidden; ++i) s += (double)router_w[(int64_t)e * hidden + i] * xn[i];
      lg[e] = s;
    }
    /* step 3 */
    route_token(lg, n_experts, top_k, p, taken, ids, w);
    /* step 4 (as in oracle_moe_layer, with xn in double) */
    for (int r = 0; r < hidden; ++r) acc[r] = 0.0;
    for (int s = 0; s < top_k; ++s) {
      if (!expert_ok(&experts[ids[s]], hidden, grid_iq2, grid_iq1)) {
        skipped = 1;
        continue;
      }
      expert_ffn_accumulate(&experts[ids[s]], hidden, xn, grid_iq2, grid_iq1, w[s], acc, 0);
    }
    if (shared) expert_ffn_accumulate(shared, hidden, xn, grid_iq2, grid_iq1, 1.0, acc, 0);
    /* step 5 */
    for (int i = 0; i < hidden; ++i) acc[i] += (double)ht[i];
    for (int j = 0; j < top_k; ++j) {
      if (ids_out) ids_out[(int64_t)t * top_k + j] = ids[j];
      if (weights_out) weights_out[(int64_t)t * top_k + j] = w[j];
    }
    free(xn);
    free(lg);
    free(p);
    free(taken);
    free(ids);
    free(w);
  }
  return skipped ? ORACLE_SKIPPED_PAIRS : ORACLE_OK;
}

int oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}
