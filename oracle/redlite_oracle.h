/*
 * redlite_oracle.h -- plain CPU reference of the routed top-k MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA library never
 * includes, links or calls it, and it shares no code with the CUDA library.
 *
 * What it computes (fp64 accumulation, libm exp):
 *   - codebook expansion of the compact grids
 *       ("Red Lite dev10 -- standalone native Metal path", section "Quant grids");
 *   - dequantisation of the IQ2_XS-style and IQ1_M-style packed blocks
 *       (format readings stated at each function in redlite_oracle.c);
 *   - the routed layer: for every selected expert gate, up, SiLU(gate)*up,
 *     down, then accumulator += router_weight * expert_output, plus an
 *     optional shared expert with weight 1
 *       ("Red Metal dev8 -- resident routed top-k layer", steps 1-6;
 *        "Red Lite dev16 -- complete full-attention parity", the block
 *        composition paragraph: routed top-10 MoE plus shared expert);
 *   - the router that feeds the layer (softmax, top-k, renormalisation) and
 *     the block around it (RMSNorm, router, layer, residual), the steps the
 *     pages name as the next milestones.
 *
 * Parity status: every function here is pinned by tests that do not call
 * back into this library (hand-computed golden blocks, closed forms,
 * invariants, an independent numpy restatement).  See the test files.
 */
#ifndef REDLITE_ORACLE_H
#define REDLITE_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORACLE_QTYPE_IQ2XS 1
#define ORACLE_QTYPE_IQ1M 2
#define ORACLE_QTYPE_Q8_0 3 /* projection formats (see oracle_dequant_proj) */
#define ORACLE_QTYPE_Q4_K 4

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
/* returned (positive) by oracle_moe_layer when at least one (token, slot)
 * pair named an id outside [0, n_experts) or an expert without matrices;
 * such a pair contributes nothing. */
#define ORACLE_SKIPPED_PAIRS 1

typedef struct {
  int32_t qtype;
  int32_t ffn;
  const uint8_t *gate; /* packed, ffn rows x hidden */
  const uint8_t *up;   /* packed, ffn rows x hidden */
  const uint8_t *down; /* packed, hidden rows x ffn */
} oracle_expert;

/* Bytes of one 256-weight block (74 or 56), or -1 for an unknown qtype. */
int oracle_block_bytes(int qtype);

/* Expand n compact uint16 grid entries into n*8 int8 values.  IQ2: symbols
 * {0,1,2} -> {8,25,43}; IQ1: {0,1,2} -> {-1,0,+1}.  Symbol 3 -> ORACLE_EINVAL. */
int oracle_expand_grid(int qtype, const uint16_t *compact, int n, int8_t *out);

/* IEEE binary16 bit pattern -> double (normals, subnormals, zeros, inf, nan). */
double oracle_fp16_to_double(uint16_t h);

/* float -> bfloat16 bit pattern, round to nearest, ties to even. */
uint16_t oracle_float_to_bf16_rne(float f);

/* 1 if a matrix of `rows` outputs and `k` inputs has a valid packed layout. */
int oracle_shape_ok(int64_t rows, int64_t k);

/* Dequantise a whole packed matrix (rows x k, row-major weights) to double. */
int oracle_dequant_matrix(int qtype, const uint8_t *packed, int64_t rows, int64_t k,
                          const int8_t *grid, double *out);

/* The routed layer in fp64.  x: [n_tokens, hidden] fp32; ids, weights:
 * [n_tokens, top_k]; experts: host array [n_experts]; shared may be NULL.
 * grid_iq2: 512*8 expanded values, grid_iq1: 2048*8 (either may be NULL if
 * that format is unused).  out: [n_tokens, hidden] doubles, overwritten. */
int oracle_moe_layer(const float *x, int n_tokens, int hidden, const int32_t *ids,
                     const float *weights, int top_k, int n_experts,
                     const oracle_expert *experts, const oracle_expert *shared,
                     const int8_t *grid_iq2, const int8_t *grid_iq1, double *out);

/* The router: per token softmax over the n_experts float logits (fp64),
 * the top_k experts by probability in descending order (ties to the lower
 * id), their probabilities renormalised to sum 1.  ids, weights:
 * [n_tokens, top_k] (int32, double). */
int oracle_route_topk(const float *logits, int n_tokens, int n_experts, int top_k, int32_t *ids,
                      double *weights);

/* The post-attention block around the layer: out = h + layer(RMSNorm(h)),
 * RMSNorm with weight gamma [hidden] and eps, routed by the router above on
 * logits = router_w [n_experts, hidden] times the normalised state, plus
 * the optional shared expert; all in double.  ids_out / weights_out
 * ([n_tokens, top_k], optional) receive the routing. */
int oracle_moe_block(const float *h, int n_tokens, int hidden, const float *gamma, double eps,
                     const float *router_w, int n_experts, int top_k, const oracle_expert *experts,
                     const oracle_expert *shared, const int8_t *grid_iq2, const int8_t *grid_iq1, double *out,
                     int32_t *ids_out, double *weights_out);

/* Projection formats (Q8_0-style: 34 bytes / 32 weights; Q4_K-style: 144
 * bytes / 256 weights; layouts stated in redlite_oracle.c): weights and
 * bytes per block (-1 for another qtype), whole-matrix dequantisation and
 * the fp64 matrix-vector product y = W x for n_tokens vectors. */
int oracle_proj_block_weights(int qtype);
int oracle_proj_block_bytes(int qtype);
int oracle_dequant_proj(int qtype, const uint8_t *packed, int64_t rows, int64_t k, double *out);
int oracle_gemv_proj(int qtype, const uint8_t *packed, int64_t rows, int64_t k, const float *x, int n_tokens,
                     double *y);

/* Threads used by oracle_moe_layer (OpenMP build); returns the value in force. */
int oracle_set_threads(int n);

#ifdef __cplusplus
}
#endif
#endif
