/*
 * redlite_moe.h -- C ABI of the B200 (sm_100a) routed top-k MoE layer over
 * codebook-quantised experts.
 *
 * The layer ("Red Metal dev8 -- resident routed top-k layer", steps 1-6):
 * for every (token, slot) the selected expert runs gate, up, SiLU(gate)*up
 * and down from its resident slot, and the layer accumulates
 * out += router_weight * expert_output; an optional shared expert is added
 * with weight 1 ("Red Lite dev16 -- complete full-attention parity", block
 * composition: routed top-10 MoE plus shared expert).  Expert weights are
 * packed in one of two codebook formats whose grids are expanded once before
 * use ("Red Lite dev10 -- standalone native Metal path", section "Quant
 * grids").
 *
 * Conventions for every entry point:
 *   - Pointers documented "device" must be CUDA device (or managed) memory
 *     of the current device; "host" pointers are ordinary CPU memory.
 *   - The caller owns every buffer.  Entry points do not allocate device
 *     memory and do not keep pointers after they return (the kernels they
 *     enqueue read them until they complete).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously; nothing synchronises except
 *     where stated.
 *   - Return values: REDLITE_OK (0) or a negative REDLITE_E* code for errors
 *     found on the host (bad argument, unsupported shape, launch failure).
 *     Errors only visible on the device (an expert id out of range, an
 *     expert slot without matrices, a bounded wait that gave up) are ORed
 *     into the caller's device status word as REDLITE_STATUS_* bits; the
 *     offending (token, slot) pair contributes nothing.  No kernel traps.
 *
 * Packed matrix layout.  A matrix with `rows` outputs and `k` inputs is its
 * rows*k weights in row-major order cut into consecutive 256-weight blocks
 * (k a multiple of 256, or a divisor of 256 that is a multiple of 32).
 *   IQ2_XS-style block, 74 bytes / 256 weights:
 *     u16 d (fp16) | u8 scales[4] | u8 qs[32] | u8 qh[4] | u8 signs[32]
 *     group g (weights 8g..8g+7): idx = qs[g] | bit (g&7) of qh[g>>3] << 8,
 *     sc = nibble (g>>2)&1 of scales[g>>3],
 *     w = d * (2sc+1)/8 * grid2[idx][j] * (bit j of signs[g] ? -1 : +1)
 *   IQ1_M-style block, 56 bytes / 256 weights:
 *     u16 d (fp16) | u8 qs[32] | u8 qh[16] | u8 scales[6]
 *     nib = nibble (g&1) of qh[g>>1], idx = qs[g] | (nib&7) << 8,
 *     delta = (nib & 8) ? -1/8 : +1/8, sc = bits 3(g>>1).. of the 48-bit
 *     little-endian scales field,
 *     w = d * (2sc+1) * (grid1[idx][j] + delta)
 *   An expert is three matrices: gate [ffn x hidden], up [ffn x hidden],
 *   down [hidden x ffn], each 16-byte aligned.
 *
 * Resident layout.  Matrices held in a slot (and read by every kernel) are
 * in the library's resident layout: for rows a multiple of 16 and k a
 * multiple of 256 it is the same bytes regrouped per tile of 16 rows x 256
 * inputs so that each tensor-core lane reads its fields with wide loads
 * (redlite_moe_pack_matrix converts; redlite_moe_upload_experts does it
 * for you); for other shapes it is the interchange layout unchanged.  Both
 * layouts have the same size (redlite_moe_matrix_bytes).
 */
#ifndef REDLITE_MOE_H
#define REDLITE_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  REDLITE_Q_IQ2XS_STYLE = 1, /* expert formats (the layer) */
  REDLITE_Q_IQ1M_STYLE = 2,
  REDLITE_Q_Q8_0_STYLE = 3,  /* projection formats (redlite_proj_gemv) */
  REDLITE_Q_Q4_K_STYLE = 4
} redlite_qtype;

enum {
  REDLITE_OK = 0,
  REDLITE_EINVAL = -1,       /* null pointer, bad size, bad enum, bad grid symbol */
  REDLITE_EUNSUPPORTED = -2, /* shape outside what the kernels support */
  REDLITE_ENOMEM = -3,       /* caller-provided workspace or pool too small */
  REDLITE_ECUDA = -4,        /* a CUDA call or kernel launch failed */
  REDLITE_EAGAIN = -5        /* every slot the pool could evict is in flight: retry after work completes */
};

/* Bits ORed into the device status word. */
enum {
  REDLITE_STATUS_BAD_ID = 1,     /* an expert id outside [0, n_experts) */
  REDLITE_STATUS_BAD_EXPERT = 2, /* selected slot has null matrices, bad qtype or shape */
  REDLITE_STATUS_TIMEOUT = 4     /* a bounded in-kernel wait gave up */
};

/* One expert slot.  gate/up/down are device pointers to packed matrices. */
typedef struct {
  int32_t qtype; /* redlite_qtype */
  int32_t ffn;   /* F, rows of gate and up, inputs of down */
  const void *gate;
  const void *up;
  const void *down;
} redlite_moe_expert;

/* Everything a layer call needs besides its per-call tensors. */
typedef struct {
  int32_t hidden;    /* H */
  int32_t n_experts; /* entries of `experts` */
  int32_t max_ffn;   /* largest F of any expert (and of the shared expert) */
  int32_t max_tokens;/* largest n_tokens the workspace was sized for */
  int32_t min_ffn;   /* smallest F of any expert (incl. shared), 0 if unknown.
                      * Valid widths are 32, 64, 128 or multiples of 256, so
                      * min_ffn >= 256 tells the call that every expert has
                      * the tiled layout the fast paths need; otherwise the
                      * general path runs. */
  int32_t reserved;  /* 0 */
  const redlite_moe_expert *experts; /* device array [n_experts]: the slot table */
  const void *grids;                 /* device, redlite_moe_grids_bytes(), from expand_grids */
  void *workspace;                   /* device, caller-owned scratch */
  size_t workspace_bytes;            /* >= redlite_moe_workspace_bytes(...) */
  int32_t *status;                   /* device word; REDLITE_STATUS_* bits are ORed in */
  void *stream;                      /* cudaStream_t */
} redlite_moe_table;

/* Bytes of the expanded-grid buffer expand_grids writes.  (Library
 * convenience: no counterpart on the pages.) */
size_t redlite_moe_grids_bytes(void);

/* Grid expansion ("Red Lite dev10", section "Quant grids"; done once before
 * the pool is used).  iq2_compact: host [512] uint16, iq1_compact: host
 * [2048] uint16; entry value j is symbol (c >> 2j) & 3, symbols 0,1,2 map to
 * 8/25/43 (IQ2_XS-style) and -1/0/+1 (IQ1_M-style).  A symbol 3 anywhere
 * returns REDLITE_EINVAL before anything is enqueued.  grids_dev: device,
 * redlite_moe_grids_bytes() bytes, 256-byte aligned.  The host arrays may
 * be reused as soon as the call returns (they are staged synchronously). */
int redlite_moe_expand_grids(const uint16_t *iq2_compact, const uint16_t *iq1_compact, void *grids_dev,
                             void *stream);

/* Packed bytes of a rows x k matrix, or 0 if the shape is not supported.
 * (Library convenience: no counterpart on the pages.) */
size_t redlite_moe_matrix_bytes(int32_t qtype, int64_t rows, int64_t k);

/* Device scratch a layer call needs for these limits.  (Library
 * convenience: no counterpart on the pages.) */
size_t redlite_moe_workspace_bytes(int32_t hidden, int32_t n_experts, int32_t max_tokens, int32_t top_k,
                                   int32_t max_ffn);

/* (Library convenience: no counterpart on the pages.)
 * Zero the workspace (table->workspace_bytes): its control words and
 * completion counters.  Call once after allocating it; layer calls leave it
 * ready for the next call, a call that reported REDLITE_STATUS_TIMEOUT
 * included.  Enqueued on table->stream. */
int redlite_moe_workspace_reset(const redlite_moe_table *table);

/* The routed layer ("Red Metal dev8", steps 4-6).
 *   x              device [n_tokens, hidden] fp32, row-major
 *   n_tokens       0 .. table->max_tokens (0 returns REDLITE_OK, enqueues nothing)
 *   expert_ids     device [n_tokens, top_k] int32
 *   router_weights device [n_tokens, top_k] fp32, used as given (no renormalisation)
 *   top_k          1 .. 16
 *   expert_table   host struct (its device pointers are read by the kernels)
 *   shared_expert  host struct with device matrix pointers, or NULL
 *   out            device [n_tokens, hidden] fp32, overwritten (not accumulated into)
 * Enqueued on expert_table->stream; x, ids, weights and out must not be
 * written by other work until it completes, and out must not overlap x,
 * ids or weights.  Two calls that share a
 * workspace must be ordered on one stream.  Decode-sized calls run one
 * fused kernel; calls with many tokens per expert run the bucketed
 * tensor-core path (bf16 operands, fp32 accumulation). */
int redlite_moe_layer(const float *x, int32_t n_tokens, const int32_t *expert_ids, const float *router_weights,
                      int32_t top_k, const redlite_moe_table *expert_table, const redlite_moe_expert *shared_expert,
                      float *out);

/* The layer for inputs and output held in host memory (a library
 * convenience with no page counterpart; the arithmetic is
 * redlite_moe_layer's).  On expert_table->stream it copies the call's
 * packed inputs host -> device in one transfer, runs the layer on the
 * device copy and copies out back to the host:
 *   inputs_host  host buffer (page-locked for an asynchronous copy) of
 *                redlite_moe_host_input_bytes(hidden, n_tokens, top_k)
 *                bytes: x [n_tokens, hidden] fp32, then expert_ids
 *                [n_tokens, top_k] int32, then router_weights [n_tokens,
 *                top_k] fp32, contiguous
 *   inputs_dev   device buffer of the same size, 16-byte aligned: the
 *                staging copy the kernels read (caller-owned)
 *   out_dev      device [n_tokens, hidden] fp32, 16-byte aligned, written
 *   out_host     host [n_tokens, hidden] fp32 (page-locked for an
 *                asynchronous copy), written
 * n_tokens, top_k, expert_table and shared_expert as for redlite_moe_layer.
 * Asynchronous: the host buffers must stay valid, inputs_host unchanged and
 * out_host unread, until the stream has passed the call.  Errors: the
 * checks of redlite_moe_layer plus null or misaligned buffers, found on the
 * host before anything is enqueued; REDLITE_ECUDA if a copy or a launch
 * cannot be enqueued.  n_tokens = 0 returns REDLITE_OK and enqueues nothing. */
int redlite_moe_layer_host(const void *inputs_host, void *inputs_dev, int32_t n_tokens, int32_t top_k,
                           const redlite_moe_table *expert_table, const redlite_moe_expert *shared_expert,
                           float *out_dev, float *out_host);

/* Bytes of the packed host input buffer of redlite_moe_layer_host: 4
 * (hidden + 2 top_k) n_tokens; 0 for a negative or zero size. */
size_t redlite_moe_host_input_bytes(int32_t hidden, int32_t n_tokens, int32_t top_k);

/* The router that feeds the layer ("Red Metal dev8", section "Field
 * validation": router-network integration is the milestone after the
 * routed layer; "Red Lite dev10", section "What dev10 does not yet claim":
 * connect the router output to the top-k path).  Per token: softmax over
 * the n_experts logits, the top_k experts by probability (equal
 * probabilities: lower id first), their probabilities renormalised to sum
 * 1 -- the expert_ids / router_weights a layer call takes.
 *   logits          device [n_tokens, n_experts] fp32, finite
 *   n_tokens        >= 0 (0 returns REDLITE_OK and enqueues nothing)
 *   n_experts       1 .. 1024
 *   top_k           1 .. min(16, n_experts)
 *   expert_ids      device [n_tokens, top_k] int32, written in descending
 *                   order of probability
 *   router_weights  device [n_tokens, top_k] fp32, written
 * Ranks on the logits (the same order as the probabilities); the weights
 * are exp(l - max) / sum over the selection in fp32.  Enqueued on stream;
 * REDLITE_EINVAL for a size out of range or a null pointer. */
int redlite_moe_route_topk(const float *logits, int32_t n_tokens, int32_t n_experts, int32_t top_k,
                           int32_t *expert_ids, float *router_weights, void *stream);

/* The post-attention block around the layer ("Red Lite dev16 -- complete
 * full-attention parity", block composition paragraph: attention residual,
 * post-attention RMSNorm, routed top-10 MoE plus shared expert, final
 * residual).  Per token, h being the hidden state after the attention
 * residual:
 *   xn = norm_weight * h / sqrt(mean(h^2) + eps)      (RMSNorm)
 *   ids, weights = redlite_moe_route_topk(router_w xn, top_k)
 *   out = h + redlite_moe_layer(xn, ids, weights)       (incl. shared expert)
 *   h            device [n_tokens, hidden] fp32
 *   n_tokens     0 .. table->max_tokens
 *   norm_weight  device [hidden] fp32; eps >= 0
 *   router_w     device [n_experts, hidden] fp32 (the router's matrix)
 *   top_k        1 .. min(16, n_experts); n_experts <= 1024
 *   out          device [n_tokens, hidden] fp32; may be h itself (in place)
 *   scratch      device, >= redlite_moe_block_scratch_bytes(hidden,
 *                n_experts, table->max_tokens, top_k) bytes, caller-owned;
 *                holds the normalised state, logits, ids and weights
 * All pointers 16-byte aligned.  Enqueued on table->stream; the layer's
 * checks, paths and status word as redlite_moe_layer.  REDLITE_ENOMEM if
 * the scratch is too small. */
size_t redlite_moe_block_scratch_bytes(int32_t hidden, int32_t n_experts, int32_t max_tokens, int32_t top_k);
int redlite_moe_block(const float *h, int32_t n_tokens, const float *norm_weight, float eps, const float *router_w,
                      int32_t top_k, const redlite_moe_table *expert_table, const redlite_moe_expert *shared_expert,
                      float *out, void *scratch, size_t scratch_bytes);

/* The layer for callers that cannot allocate device memory.  Some callers
 * have no way to call cudaMalloc for the workspace: for example a plugin
 * running inside a host application that owns the whole device-memory
 * budget and hands out only the tensors it manages, or code with no
 * allocator at hand.  This entry point runs the same fused decode kernel as
 * redlite_moe_layer but keeps the kernel's scratch in a fixed 4 MiB array
 * that the library itself holds in device memory (every GPU that loads the
 * library keeps it until the process exits).  It allocates nothing.
 * There is no counterpart on the pages: it is an interface convenience.
 *   Arguments as redlite_moe_layer; table->workspace and
 *   table->workspace_bytes are ignored.
 *   Only decode-sized calls the fused kernel takes are accepted
 *   (n_tokens * top_k <= 640, hidden and every expert width multiples of
 *   256 up to 2048, table->min_ffn >= 256): otherwise REDLITE_EUNSUPPORTED.
 *   A call whose scratch (control block + 2 * 4 * max_ffn bytes per
 *   (token, slot) pair incl. the shared expert + about 3 * hidden bytes per
 *   token) exceeds 4 MiB returns REDLITE_ENOMEM before enqueuing anything.
 *   The first call on a device looks the array up (cudaGetSymbolAddress)
 *   and clears its control words on table->stream; make that first call
 *   before any stream capture.
 *   Every call on a device shares the one array, which keeps the last
 *   call's contents: calls that overlap on the GPU (different streams, or
 *   different host threads without ordering) race and must not be issued;
 *   order them on one stream. */
int redlite_moe_layer_noalloc(const float *x, int32_t n_tokens, const int32_t *expert_ids,
                              const float *router_weights, int32_t top_k, const redlite_moe_table *expert_table,
                              const redlite_moe_expert *shared_expert, float *out);

/* Host-side conversion of one matrix from the interchange layout to the
 * resident layout (library convenience: the resident layout is this
 * library's own; the pages keep the file's byte order).  src, dst: host buffers of redlite_moe_matrix_bytes()
 * bytes, not overlapping.  REDLITE_EUNSUPPORTED for shapes the kernels do
 * not take.  Pure host code: no device work. */
int redlite_moe_pack_matrix(int32_t qtype, int64_t rows, int64_t k, const void *src, void *dst);

/* Dequantise one matrix held in the resident layout (the bit-exactness
 * check of the decoders; library convenience, no counterpart on the pages).  packed: device; out_f32: device [rows*k] fp32 or
 * NULL; out_bf16: device [rows*k] bf16 bits (round to nearest even) or
 * NULL; outputs 16-byte aligned.  grids: expanded.  Enqueued on stream. */
int redlite_moe_dequant(int32_t qtype, const void *packed, int64_t rows, int64_t k, const void *grids, float *out_f32,
                        uint16_t *out_bf16, void *stream);

/* Slot-table builder: copies experts from host memory into a device pool
 * and writes their slot descriptors ("Red Metal dev8", steps 1-3: every
 * selected expert made resident, three positional reads per expert).
 * Matrices are converted to the resident layout on the way.
 *   hidden       H of the layer (sizes the matrices with each expert's ffn)
 *   ids          host [n] expert ids (slot index in table_dev)
 *   host_experts host [n]; gate/up/down are HOST pointers to packed bytes
 *                in the interchange layout
 *   pool         device, pool_bytes, 16-byte aligned; matrices are placed
 *                back to back at 16-byte aligned offsets from `pool_offset`
 *   table_dev    device [n_experts] slot table; entries ids[i] are written
 *   counters     host, optional: {loads, copies, bytes} are added to it
 *   pool_end     host, optional: receives the first free pool offset
 * Shapes are checked and placement is planned before anything is copied:
 * REDLITE_EUNSUPPORTED for a shape the kernels do not take, REDLITE_ENOMEM
 * if the pool is too small.  Three host->device copies per expert plus one
 * descriptor copy are enqueued on `stream`, then the call synchronises the
 * stream, so host buffers may be released when it returns. */
typedef struct {
  int64_t loads;  /* experts made resident */
  int64_t copies; /* host->device matrix copies (3 per expert) */
  int64_t bytes;  /* packed bytes copied */
} redlite_moe_upload_counters;

int redlite_moe_upload_experts(int32_t hidden, const int32_t *ids, const redlite_moe_expert *host_experts, int32_t n,
                               void *pool, size_t pool_bytes, size_t pool_offset, redlite_moe_expert *table_dev,
                               int32_t n_experts, void *stream, redlite_moe_upload_counters *counters,
                               size_t *pool_end);

/* ---------------------------------------------------------------- projections
 * The decode-GEMV for the other weight formats of the model the pages run
 * ("Red Lite dev15 -- DeltaNet projection bring-up", section "Field-derived
 * recurrent dimensions": ssm_ba Q8_0, ssm_out Q4_K; "Red Lite dev16",
 * section "Pinned full-attention graph": attn_k, attn_v, attn_output Q4_K).
 * The pages print no layouts; the library reads them as:
 *   Q8_0-style  34 bytes / 32 weights: u16 d (fp16) | int8 q[32];
 *               w = d * q
 *   Q4_K-style 144 bytes / 256 weights: u16 d | u16 dmin (fp16) | u8 sm[12]
 *               (96-bit little-endian field: 6-bit scale of sub-block j =
 *               weights 32j..32j+31 at bit 6j, 6-bit minimum at bit 48+6j)
 *               | u8 q[128] (weight i: nibble i & 1 of byte i / 2);
 *               w = d * scale * q - dmin * minimum
 * A rows x k matrix is its row-major weights cut into consecutive blocks. */

/* Packed bytes of a rows x k projection matrix (k a multiple of 256), or 0. */
size_t redlite_proj_matrix_bytes(int32_t qtype, int64_t rows, int64_t k);

/* y[t][r] = sum_c W[r][c] * x[t][c] for t < n_tokens (0..8), fp32.
 *   W  device, the packed matrix (2-byte aligned for Q8_0-style, 16-byte
 *      aligned for Q4_K-style); x device [n_tokens, k] fp32, 16-byte aligned;
 *   y  device [n_tokens, rows] fp32, overwritten.
 * REDLITE_EUNSUPPORTED if k is not a multiple of 256; enqueued on stream. */
int redlite_proj_gemv(int32_t qtype, const void *W, int64_t rows, int64_t k, const float *x, int32_t n_tokens,
                      float *y, void *stream);

/* ---------------------------------------------------------------- slot pool
 * The bounded, top-k-aware LRU pool of expert slots ("Red Metal dev8",
 * steps 1-3: the hard-bounded LRU makes every selected expert resident,
 * selected experts are protected from eviction while the remaining misses
 * are filled, every selected slot is pinned for the work that uses it;
 * "Red Lite dev9 -- native runtime foundation", section "Native selftest":
 * hard capacity enforcement, LRU hit/miss/eviction, protection of the
 * current top-k during acquire_many, in-flight slot protection).
 * The pool is a host object; it owns no device memory.  Not thread-safe:
 * one host thread drives a pool. */
typedef struct redlite_moe_pool redlite_moe_pool;

typedef struct {
  int64_t loads;     /* misses filled */
  int64_t hits;      /* selected experts already resident */
  int64_t evictions; /* resident experts replaced */
  int64_t copies;    /* host->device matrix copies (3 per load) */
  int64_t bytes;     /* packed bytes copied */
} redlite_moe_pool_counters;

/* A pool of `capacity` slots for experts 0..n_experts-1 (all empty).
 * NULL for a bad size or if host memory runs out. */
redlite_moe_pool *redlite_moe_pool_create(int32_t n_experts, int32_t capacity);
void redlite_moe_pool_destroy(redlite_moe_pool *pool);

/* The policy step (host only, no device work): make ids[0..n) resident.
 *   pass 1: every selected expert already resident is a hit: its slot is
 *           refreshed (most recently used) and protected;
 *   pass 2: each miss, in order, takes the lowest free slot, else the least
 *           recently used slot that is neither protected (selected in this
 *           call) nor pinned by a call still in flight; a repeated id shares
 *           its first occurrence's slot;
 *   then every selected slot is pinned under a new token.
 * Outputs per id: slot_of[i], miss[i] (1 if it must be filled), evicted[i]
 * (the expert whose slot it took, or -1).  REDLITE_ENOMEM if the distinct
 * ids exceed the capacity; REDLITE_EAGAIN if a miss finds no slot because
 * the others are in flight (nothing changes then); REDLITE_EINVAL for an id
 * outside [0, n_experts). */
int redlite_moe_pool_plan(redlite_moe_pool *pool, const int32_t *ids, int32_t n, int32_t *slot_of, int32_t *evicted,
                          uint8_t *miss, int64_t *token);

/* Unpin a token's slots now (the caller knows the work using them is done). */
int redlite_moe_pool_complete(redlite_moe_pool *pool, int64_t token);

/* Unpin a token's slots once the work enqueued on `stream` so far has
 * completed (a CUDA event, polled by later plans). */
int redlite_moe_pool_release(redlite_moe_pool *pool, int64_t token, void *stream);

/* Slot of a resident expert, or -1; pins of a slot, or -1 for a bad slot. */
int32_t redlite_moe_pool_slot_of(const redlite_moe_pool *pool, int32_t expert);
int32_t redlite_moe_pool_pins(const redlite_moe_pool *pool, int32_t slot);

/* The policy step plus the data movement: for every miss the expert's three
 * matrices are copied host -> device into its slot (slots_dev + slot *
 * slot_bytes: gate, up at the gate size rounded up to 16 bytes, down after),
 * then table_dev[id] is written and an evicted expert's entry cleared (a
 * stale id then reports BAD_EXPERT).  The copies run on the pool's own copy
 * streams (created on the current device at the first acquire with several
 * misses), forked from copy_stream and joined back into it, so they are
 * ordered after earlier work on copy_stream and before later work on it.
 * The work enqueued next on compute_stream waits for them, so a layer call
 * may follow at once; copies for the next selection overlap the current
 * layer kernel when copy_stream differs from compute_stream.
 *   host_experts  host [n_experts]; gate/up/down are HOST pointers to the
 *                 matrices already in the resident layout
 *                 (redlite_moe_pack_matrix); pinned host memory makes the
 *                 copies asynchronous; they must stay valid until the copies
 *                 complete
 *   slot_bytes    multiple of 16, >= 2 * round16(gate bytes) + down bytes of
 *                 every expert acquired (else REDLITE_ENOMEM)
 * After enqueuing the layer call, pass the token to redlite_moe_pool_release
 * with compute_stream. */
int redlite_moe_pool_acquire(redlite_moe_pool *pool, const int32_t *ids, int32_t n,
                             const redlite_moe_expert *host_experts, int32_t hidden, void *slots_dev,
                             size_t slot_bytes, redlite_moe_expert *table_dev, void *copy_stream,
                             void *compute_stream, redlite_moe_pool_counters *counters, int64_t *token);

#ifdef __cplusplus
}
#endif
#endif
