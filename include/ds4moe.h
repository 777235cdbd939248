/*
 * ds4moe.h -- C ABI of a B200 (sm_100a) routed mixture-of-experts FFN layer whose
 * routed experts are held in 2-bit Q2_K blocks and whose shared expert stays bf16.
 *
 * The layer is the routed MoE FFN of DeepSeek-V4-style models as run by the
 * DwarfStar (ds4) engine:
 *  - "antirez/ds4" README (molayo1419.me translation), paragraph on the 2-bit
 *    models: only the routed experts are quantised (down as Q2_K; the shared
 *    expert, projections and router keep their precision); acknowledgements:
 *    the GGUF quantisation layouts are llama.cpp's, so a routed weight block is
 *    the GGUF Q2_K super-block (84 bytes per 256 weights);
 *  - opensource-hub.com "antirez/ds4" FAQ, router-precision entry: the router
 *    score is sqrt(softplus(logit)), and the fp32 softplus must use an exact
 *    log1p series when exp(x) < 1/32 (the naive log(1 + exp(x)) fails a 3e-6
 *    check near x = -12).
 * Per token t with bf16 activations x_t (length H):
 *    logit_e = x_t . Wr_e (+ bias_e),  s_e = sqrt(softplus(logit_e)),
 *    the top_k experts by logit (ties to the lower index), w_j = s_j / sum s,
 *    y_t = sum_j w_j * down_j( silu(gate_j x_t) * up_j x_t ) + shared(x_t)   (fp32).
 *
 * Conventions shared by every call:
 *  - Every pointer named *_dev is a CUDA device pointer on the handle's device;
 *    every other pointer is host memory.  Host buffers are read (or written)
 *    during the call only and are never retained.
 *  - Device buffers passed in are owned by the caller; the handle owns its
 *    weights, its workspace and its CUDA graphs.
 *  - cuda_stream is a cudaStream_t (NULL = the legacy default stream).  Calls
 *    that take a stream only enqueue work and return; errors found on the
 *    device (a bounded wait that timed out, an out-of-range index) set a sticky
 *    status that ds4moe_sync_status() reports.
 *  - Every call returns a status; nothing aborts, throws or traps.  On an
 *    error ds4moe_last_error() holds a one-line reason.
 *  - A handle is not thread-safe: use one handle per host thread.
 *  - Test hook: the environment variable DS4MOE_FAULT injects a host-side failure without
 *    touching the GPU: "alloc" (ds4moe_create returns DS4MOE_ENOMEM), "h2d"
 *    (ds4moe_load_q2k_experts returns DS4MOE_ECUDA before its first copy), "launch"
 *    (ds4moe_route / ds4moe_route_static / ds4moe_forward return DS4MOE_ECUDA before their
 *    first launch).  It is read on every call.
 */
#ifndef DS4MOE_H
#define DS4MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ds4moe ds4moe; /* opaque handle, library-owned */

typedef enum {
    DS4MOE_OK = 0,
    DS4MOE_EINVAL = 1,   /* an argument is out of range, NULL or misaligned */
    DS4MOE_ENOMEM = 2,   /* a device or host allocation failed */
    DS4MOE_ECUDA = 3,    /* a CUDA runtime call failed (see ds4moe_last_error) */
    DS4MOE_ESTATE = 4,   /* the call needs state the handle lacks (e.g. no weights) */
    DS4MOE_ETIMEOUT = 5, /* a bounded device-side wait gave up */
    DS4MOE_EDEVICE = 6   /* a kernel found an invalid value on the device */
} ds4moe_status;

/* Force a forward path (flags of ds4moe_config). */
#define DS4MOE_FLAG_FORCE_DECODE  0x1u  /* batched-GEMV path (the default for T <= 32; no
                                           effect above 32 tokens, that path's limit) */
#define DS4MOE_FLAG_FORCE_PREFILL 0x2u  /* grouped tensor-core path for every T */
#define DS4MOE_FLAG_PROFILE       0x4u  /* record per-stage CUDA events in ds4moe_forward */
#define DS4MOE_FLAG_TRACE         0x8u  /* record a per-unit timeline of the batched-GEMV kernel */
#define DS4MOE_FLAG_TEST_TIMEOUT  0x10u /* test hook, one shot: in the first batched-GEMV forward
                                           of the handle, the first routed-down unit waits (about
                                           2 ms) for a count that is never reached, so that forward
                                           ends with DS4MOE_ETIMEOUT; later forwards run normally */

typedef struct {
    int32_t hidden;       /* H: multiple of 256, 256 .. 16384 */
    int32_t n_experts;    /* E: 1 .. 256 */
    int32_t top_k;        /* k: 1 .. min(E, 16) */
    int32_t inter;        /* I, routed expert intermediate: multiple of 256, 256 .. 16384 */
    int32_t shared_inter; /* I_s, shared expert intermediate: 0 (none) or a multiple of 256 */
    int32_t max_tokens;   /* largest T any later call passes: 1 .. 65536 */
    uint32_t flags;       /* DS4MOE_FLAG_* */
} ds4moe_config;

/* Per-handle counters (ds4moe_get_stats). */
typedef struct {
    int64_t router_fallback_tokens; /* tokens whose top-k was re-ranked with the fp64 sum */
    int32_t last_path;              /* 1 = decode (batched GEMV), 2 = prefill (grouped GEMM) */
    int32_t last_tokens;            /* T of the last forward */
    int32_t n_stages;               /* number of valid entries in stage_ms */
    float stage_ms[8];              /* per-stage device time of the last profiled forward */
} ds4moe_stats;

/* Create a handle on CUDA device `cuda_device` and allocate its workspace for
 * up to cfg->max_tokens tokens.  *out is set only on DS4MOE_OK. */
ds4moe_status ds4moe_create(const ds4moe_config *cfg, int cuda_device, ds4moe **out);

/* Free every device and host resource of the handle; NULL is ignored. */
void ds4moe_destroy(ds4moe *h);

/* Upload one layer's weights from host memory and repack them for the device.
 * Passage: the README translation's acknowledgements (the GGUF quantisation layouts are
 * llama.cpp's: a routed block is the GGUF Q2_K super-block) and its 2-bit paragraph (the
 * router and the shared expert keep their precision).
 *  gate_q2k, up_q2k: [E][I][H/256] Q2_K super-blocks of 84 bytes each
 *        (row r of expert e holds the H input weights of output r; blocks run
 *        along the input dimension).  down_q2k: [E][H][I/256] blocks likewise.
 *        Block layout (GGUF Q2_K): 16 scale bytes (low nibble = scale, high
 *        nibble = min), 64 bytes of 2-bit quants, fp16 d, fp16 dmin (LE);
 *        weight i of a block is d*scale*q - dmin*min with q at bit 2*((i%128)/32)
 *        of quant byte 32*(i/128) + i%32 and sub-block i/16.
 *  router_w_bf16: [E][H] bf16 bit patterns, row-major.
 *  router_bias:   [E] fp32 added to the logit before softplus, or NULL.
 *  shared_gate_bf16, shared_up_bf16: [I_s][H]; shared_down_bf16: [H][I_s]
 *        (bf16, row-major); all three NULL when shared_inter == 0.
 * Synchronous: returns once the weights are on the device.  May be called
 * again to replace the weights.  Host buffers need no particular alignment. */
ds4moe_status ds4moe_load_q2k_experts(ds4moe *h, const void *gate_q2k, const void *up_q2k,
                                      const void *down_q2k, const uint16_t *router_w_bf16,
                                      const float *router_bias, const uint16_t *shared_gate_bf16,
                                      const uint16_t *shared_up_bf16, const uint16_t *shared_down_bf16,
                                      void *cuda_stream);

/* Routing only: top-k, normalised weights and the token->expert permutation
 * for T tokens of x (bf16 [T][H], 16-byte aligned).
 * Passage: opensource-hub.com "antirez/ds4" FAQ, router-precision entry (score =
 * sqrt(softplus(logit)), the fp32 softplus by its log1p series); the top-k, the weight
 * normalisation and the permutation by expert are the routing of the workload definitions
 * (ties to the lower index).
 *  topk_idx_dev [T][k] int32 (slots by descending score), topk_w_dev [T][k] fp32;
 *  expert_offsets_dev [E+1] (exclusive scan of the per-expert pair counts),
 *  sorted_token_dev / sorted_slot_dev [T*k]: the (token, slot) pairs ordered by
 *  expert and, within an expert, by token; inv_pos_dev [T*k]: position of pair
 *  t*k + j in that order.  The last four may each be NULL.
 * The selected indices and the permutation are exactly those of an fp64
 * evaluation with sequential sums (near-ties are re-ranked in fp64). */
ds4moe_status ds4moe_route(ds4moe *h, const void *x_bf16_dev, int32_t T, int32_t *topk_idx_dev,
                           float *topk_w_dev, int32_t *expert_offsets_dev, int32_t *sorted_token_dev,
                           int32_t *sorted_slot_dev, int32_t *inv_pos_dev, void *cuda_stream);

/* Largest T that ds4moe_route_static accepts. */
#define DS4MOE_ROUTE_STATIC_MAX_TOKENS 256

/* ds4moe_route for up to DS4MOE_ROUTE_STATIC_MAX_TOKENS tokens without any allocation.
 * The pages have no counterpart: this is a service variant of the routing step for
 * callers that must not allocate device memory on the call path.  Outputs and results are
 * those of ds4moe_route (same layouts, same bit-exact indices and permutation), but every
 * output pointer is required (none may be NULL) and is written directly.
 *  Scratch: the router logits, error bounds, per-block expert counts and the active-expert
 *  list live in one file-scope __device__ array of the library (about 782 KiB per device,
 *  sized for 256 tokens x 256 experts).  No part of it has to start at zero: every word
 *  is written before it is read within one call.
 *  Set-up: the first call on each device, with that device current, resolves the array's
 *  address once (cudaGetSymbolAddress) and caches it per device number; make that first
 *  call before any stream capture begins.  Later calls make no runtime allocation of any
 *  kind.  The cache assumes the device's primary context for the life of the process:
 *  after cudaDeviceReset, or from a different context, the cached address is stale.
 *  Limits: T > DS4MOE_ROUTE_STATIC_MAX_TOKENS returns DS4MOE_EINVAL with a reason in
 *  ds4moe_last_error; T <= max_tokens of the handle as for ds4moe_route.
 *  Concurrency: all handles on a device share the one scratch array, so calls whose
 *  executions overlap on the device (different streams, or host threads) race on it and
 *  corrupt each other's results; order them on one stream or serialise them. */
ds4moe_status ds4moe_route_static(ds4moe *h, const void *x_bf16_dev, int32_t T, int32_t *topk_idx_dev,
                                  float *topk_w_dev, int32_t *expert_offsets_dev, int32_t *sorted_token_dev,
                                  int32_t *sorted_slot_dev, int32_t *inv_pos_dev, void *cuda_stream);

/* The whole layer for T tokens: x bf16 [T][H] (16-byte aligned) -> y fp32 [T][H]
 * (16-byte aligned).
 * Passages: molayo1419.me "antirez/ds4" README translation, paragraph on the 2-bit models
 * (routed experts in 2-bit GGUF blocks, shared expert and router at full precision) and
 * its acknowledgements (llama.cpp's Q2_K layout); the FAQ router-precision entry for the
 * score.  y_t = sum_j w_j down_j(silu(gate_j x_t) * up_j x_t) + shared(x_t).  T = 0 is a no-op.  Picks the batched-GEMV path for small T
 * and the grouped tensor-core path for large T unless a FORCE flag is set. */
ds4moe_status ds4moe_forward(ds4moe *h, const void *x_bf16_dev, int32_t T, float *y_f32_dev,
                             void *cuda_stream);

/* Same as ds4moe_forward with HOST buffers: copies x (bf16 [T][H]) to the device,
 * runs the layer and copies y (fp32 [T][H]) back, all on cuda_stream, and
 * returns after the copy back has finished.  Page-locked host buffers give
 * asynchronous copies; pageable ones work too.  On the batched-GEMV path (T <= 32) a
 * page-locked, device-mapped y (cudaHostAlloc / cudaHostRegister under unified
 * addressing) is written by the kernel directly, without a separate copy back. */
ds4moe_status ds4moe_forward_host(ds4moe *h, const uint16_t *x_bf16, int32_t T, float *y_f32,
                                  void *cuda_stream);

/* RMS renormalisation between chained layers (stateless; the 4-layer workload's
 * definition, not a passage of the pages):
 * x[t,i] = bf16_rne( y[t,i] / sqrt(mean_i y[t,i]^2 + 1e-6) ) for T tokens of width H. */
ds4moe_status ds4moe_rms_renorm(const float *y_f32_dev, int32_t T, int32_t H, uint16_t *x_bf16_dev,
                                void *cuda_stream);

/* Evaluate the router's fp32 score sqrt(softplus(l)) on n logits (diagnostic).
 * Passage: the FAQ router-precision entry (the naive form fails a 3e-6 check near -12).
 * variant 0 = the library's accurate form; 1 = the naive log(1 + exp(l)) form
 * that the router must not use (kept so tests can show the difference). */
ds4moe_status ds4moe_score_eval(const float *logits_dev, int32_t n, float *scores_dev, int32_t variant,
                                void *cuda_stream);

/* Copy one repacked weight matrix back into the host AoS Q2_K layout of
 * ds4moe_load_q2k_experts (which: 0 = gate, 1 = up, 2 = down) for expert e;
 * out must hold rows * K/256 * 84 bytes.  Synchronous.  For round-trip checks. */
ds4moe_status ds4moe_export_q2k(ds4moe *h, int32_t which, int32_t expert, void *out);

/* Synchronise the last stream used by the handle and return its sticky device
 * status (DS4MOE_OK, DS4MOE_ETIMEOUT or DS4MOE_EDEVICE); clears it. */
ds4moe_status ds4moe_sync_status(ds4moe *h);

/* Counters of the handle (see ds4moe_stats). Synchronises like ds4moe_sync_status. */
ds4moe_status ds4moe_get_stats(ds4moe *h, ds4moe_stats *out);

/* Timeline of the last batched-GEMV launch (handle created with DS4MOE_FLAG_TRACE).
 * That kernel hands out work units in four phases: shared gate/up; routed gate/up (per
 * expert group and 32 rows of I); shared down; routed down (per expert group and 64 rows
 * of H).  (The order can mix shared units into the routed phases; the current plan mixes
 * none.)  out receives up to max_records records of four int64, the device %globaltimer
 * in ns:
 *   unit records (unit_bounds[5] of them; unused ones are zero):
 *     unit | (ns from the consumers' start of the unit to their end of it) << 32, when
 *     its first copy was issued, when the consumers started it (its inputs ready), when
 *     its epilogue finished;
 *   then two records per CTA (unit_bounds[6] CTAs):
 *     start, when its own router rows were done, when every router row was done, when its
 *     top-k was done, when its routing table was ready, exit, 0, 0;
 *   then four records: the first unit of phases 2..4 and the end (words 0..3), and six
 *   timestamps of CTA 0's top-k of token 0 (words 8..13: start, logits loaded, selected,
 *   certified, re-ranked, weights written);
 *   then two more records per unit: when the consumers had written its partial sums
 *   (after waiting for a free partial buffer), when its epilogue started, the CTA that ran
 *   it | 1 << 16 if its pieces carried its inputs, when the consumers saw its pieces 0 and 1
 *   landed, when piece 1 was issued, when the consumers had computed piece 0, the SM cycles
 *   its epilogue took.
 * unit_bounds[0..4] receives the first unit of each phase and the end.  *n_records =
 * number of records written.
 * Synchronises. */
ds4moe_status ds4moe_get_trace(ds4moe *h, int64_t *out, int32_t max_records, int32_t *n_records,
                               int32_t *unit_bounds);

/* Static text for a status code. */
const char *ds4moe_status_string(ds4moe_status s);

/* One-line detail of the handle's last error, owned by the handle ("" if none). */
const char *ds4moe_last_error(const ds4moe *h);

#ifdef __cplusplus
}
#endif
#endif /* DS4MOE_H */
