/*
 * moe.h - quantized sparse Mixture-of-Experts feed-forward layer on one
 * NVIDIA B200 (sm_100a).  C ABI: plain pointers and sizes, no C++ or torch
 * types.  Every entry point returns a moe_status; nothing aborts or throws.
 *
 * The layer (per token t, per layer):
 *   router   logit_e = x_t . W_r[e] (+ b_e)                 e = 0..E-1
 *   route    p = softmax(logits); ids = the top_k experts by p (descending,
 *            equal p -> lower id); w_j = p_ids[j] / sum_j p_ids[j]
 *   experts  for each chosen expert and each shared expert:
 *            g = W_g x_t, u = W_u x_t, h = silu(g) * u, y_e = W_d h
 *   combine  y_t = bf16( sum_j w_j y_ids[j]  +  sum_s y_shared_s )
 * Source passages: "Qwen3.8-Flash-Next at 45 Tokens/sec on a 12GB GPU?"
 * (video transcript 1:37-2:16: 48 layers x 512 experts, a router per layer
 * picks 10 of them plus one always-on shared expert; 3:36-3:47: the partial
 * results of one token land on one output) and "Qwen3.8-Flash-Next on RTX
 * 5090 + 64GB", section "The 30-Second Overview" (10 routed + 1 shared per
 * token).  The pages do not define the expert network, the routing
 * normalisation or the quantised layouts; this library fixes them: SwiGLU
 * experts, softmax renormalised over the chosen k, and the block formats
 * below.
 *
 * Block formats (32 weights per block, blocks run along the reduction dim):
 *   MOE_Q4B32  16 bytes of int4 codes, two per byte (byte b: code 2b in the
 *              low nibble, code 2b+1 in the high nibble) + one fp16 scale s;
 *              w = s * (q - 8).                                   4.5 bit/w
 *   MOE_Q3B32  12 bytes: the 32 three-bit codes of one 96-bit little-endian
 *              integer (code j in bits 3j..3j+2) + one fp16 scale s;
 *              w = s * (q - 4).                                   3.5 bit/w
 *   MOE_Q2B32  8 bytes: the 32 two-bit codes of one 64-bit little-endian
 *              integer (code j in bits 2j..2j+1) + one fp16 scale s;
 *              w = s * (q - 2).                                   2.5 bit/w
 *              For the pages' fastest size Q2_0 ("Strata: Qwen3.8-Flash-Next
 *              (125B Moe) on a 8GB+ Nvidia GPU", tables "How fast?" and "The
 *              size").
 *
 * Canonical tensor layouts accepted by moe_load_layer (row-major, SoA: codes
 * and scales in separate arrays):
 *   gate, up   codes  [E][d_ff][d_model/32][B]   scales [E][d_ff][d_model/32]
 *   down       codes  [E][d_model][d_ff/32][B]   scales [E][d_model][d_ff/32]
 *   B = 16 (Q4B32), 12 (Q3B32) or 8 (Q2B32); scales are IEEE fp16 bit patterns.
 *   router_w   fp32 [E][d_model]; router_bias fp32 [E] or NULL.
 *   Shared experts: the same with n_shared in place of E and d_ff_shared.
 * The library copies them into its own device memory in a private tiled
 * order (same byte count); the caller's buffers are not referenced after
 * moe_load_layer returns.
 */
#ifndef QEFFN_MOE_H
#define QEFFN_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,     /* NULL pointer, bad size, bad layer index */
    MOE_ERR_OOM = -2,             /* device allocation failed or over the memory limit */
    MOE_ERR_CUDA = -3,            /* a CUDA runtime call failed; see moe_last_error() */
    MOE_ERR_NOT_LOADED = -4,      /* moe_forward on a layer never loaded */
    MOE_ERR_TOO_MANY_TOKENS = -5, /* T > max_tokens */
    MOE_ERR_DEVICE_TIMEOUT = -6,  /* a bounded device-side wait ran out */
    MOE_ERR_UNSUPPORTED = -7      /* a shape this build does not implement */
} moe_status;

typedef enum { MOE_Q4B32 = 1, MOE_Q3B32 = 2, MOE_Q2B32 = 3 } moe_qformat;

typedef struct {
    int d_model;        /* hidden size d; multiple of 256 */
    int n_experts;      /* routed experts E, 1..1024 */
    int d_ff;           /* routed expert intermediate size I; multiple of 64 */
    int top_k;          /* experts chosen per token, 1..min(E, 32) */
    int n_shared;       /* always-on shared experts, 0..4 */
    int d_ff_shared;    /* shared expert intermediate size; must equal d_ff */
    int n_layers;       /* layers the context can hold */
    int max_tokens;     /* largest T any call may pass */
    int fmt;            /* moe_qformat */
    long long device_mem_limit; /* bytes the context may allocate; 0 = no limit */
    int flags;          /* MOE_FLAG_* bits, 0 for normal use */
} moe_config;

/* moe_config.flags: test and diagnostic hooks, 0 in normal use (no page has a
 * counterpart).  The NO_* flags pin a call to one implementation (tests
 * compare the paths with each other); MOE_FLAG_SPLIT_DECODE selects an
 * alternative single-token kernel (measured slower on this shape, kept for
 * comparison); MOE_FLAG_TRACE records the decode
 * kernel's phase clocks; MOE_FLAG_TEST_WITHHOLD is a test hook for the
 * bounded device waits: in the context's first call of a decode kernel
 * (single-token, few-token or split) that kernel's CTA 0 withholds its router
 * logits, and in the context's first tensor-core gate/up GEMM CTA 0 never
 * signals its first accumulator as complete; every wait on them runs out
 * (about one second in the decode kernels, two in the GEMM), and the call
 * reports MOE_ERR_DEVICE_TIMEOUT through moe_get_device_error; later calls
 * run normally.  Both hooks are for tests only. */
#define MOE_FLAG_NO_DECODE_KERNEL 1   /* small T runs the general path, not the single-token kernel */
#define MOE_FLAG_NO_TENSOR_PREFILL 2  /* large T runs the CUDA-core expert path */
#define MOE_FLAG_NO_MULTI_DECODE 8    /* 2..32 tokens run the single-token kernel per token (up to 8) or the tensor-core path, not the few-token kernel */
#define MOE_FLAG_SPLIT_DECODE 16      /* with max_tokens == 1: the split single-token kernel (down projection by k chunk) */
#define MOE_FLAG_TEST_WITHHOLD 256    /* test hook described above */
#define MOE_FLAG_TRACE 4              /* record per-phase timestamps (moe_trace_read) */

typedef struct {
    const float *router_w;          /* [E][d] */
    const float *router_bias;       /* [E] or NULL (no bias) */
    const uint8_t *codes[3];        /* gate, up, down (canonical layouts above) */
    const uint16_t *scales[3];
    const uint8_t *sh_codes[3];     /* shared experts; ignored when n_shared == 0 */
    const uint16_t *sh_scales[3];
    int on_device;                  /* 1: all pointers are device memory of the
                                       context's device; 0: host memory */
} moe_layer_weights;

/* Per-layer records written by moe_forward_stack; any field may be NULL.
 * Only the token rows listed in rows[0..n_rows) are recorded (rows == NULL:
 * all T rows, in order).  Record r of layer l sits at [l][r][...]. */
typedef struct {
    uint16_t *x_bf16;   /* [n_layers][n_rec][d] bf16 input of each layer */
    uint16_t *y_bf16;   /* [n_layers][n_rec][d] bf16 output of each layer */
    float *y_f32;       /* [n_layers][n_rec][d] fp32 value that y_bf16 rounds */
    int32_t *ids;       /* [n_layers][n_rec][k] */
    float *w;           /* [n_layers][n_rec][k] */
    const int32_t *rows;/* device array of token indices, or NULL */
    int n_rows;         /* length of rows (ignored when rows == NULL) */
} moe_stack_record;

typedef struct moe_ctx moe_ctx;

/* A context owns one workspace (intermediates, the single-token kernel's
 * exchange buffers and counters).  Its forward calls must therefore run one
 * after another on the device: issue them on one stream, or order them with
 * events; calls that overlap on the GPU corrupt each other's results.  Use
 * one context per concurrent stream. */

/* Create a context on CUDA device `device` and allocate its workspace (sized
 * by max_tokens).  The context holds one stack of MoE layers of one shape (the
 * pages' model: 48 layers of 512 experts, 10 routed + 1 shared per token;
 * "Qwen3.8-Flash-Next at 45 Tokens/sec on a 12GB GPU?", video transcript
 * 1:37-2:16).  *out receives the handle.  Errors: INVALID_ARG (bad
 * config), UNSUPPORTED (shape outside the limits above), OOM, CUDA.
 * When the tensor-core path can run, the workspace also holds a decoded-weight
 * cache of min(experts, max_tokens * (top_k + n_shared) / 256) experts
 * (6 * d_model * d_ff bytes each) if it fits device_mem_limit; without it the
 * results are the same, only slower. */
MOE_API int moe_create(const moe_config *cfg, int device, moe_ctx **out);

/* Copy one layer's weights into the context (repacking them on the device)
 * and make the layer usable.  The weights are the block formats above (the
 * pages name their quantised types, e.g. IQ3_S or Q2_0, but give no layout:
 * "Running Qwen3.8-Flash-Next on a 4090 24GB", section "The engine rejects
 * Unsloth's embedding format"; this library's formats fix one).  Reloading a layer replaces it.  Work is queued
 * on `stream` (a cudaStream_t, NULL = default stream); the call returns after
 * the copies from caller memory have completed.  Errors: INVALID_ARG, OOM,
 * CUDA. */
MOE_API int moe_load_layer(moe_ctx *ctx, int layer, const moe_layer_weights *w, void *stream);

/* One layer on T tokens: router, softmax top-k, the chosen experts and the
 * shared expert, weighted combine ("Qwen3.8-Flash-Next at 45 Tokens/sec on a
 * 12GB GPU?", video transcript 1:50-2:16 and 3:36-3:47; "Qwen3.8-Flash-Next on
 * RTX 5090 + 64GB", section "The 30-Second Overview").  All pointers are
 * device memory:
 *   x_bf16 [T][d] input; y_bf16 [T][d] output; y_f32 [T][d] the fp32 value
 *   before the bf16 rounding, or NULL; ids [T][k] chosen experts (descending
 *   weight) and w [T][k] their weights, either may be NULL.
 * Asynchronous on `stream`; no host synchronisation and no allocation.
 * T == 0 is a no-op.  Errors: INVALID_ARG, NOT_LOADED, TOO_MANY_TOKENS, CUDA.
 * Implementation (not part of the contract): one token runs the persistent
 * single-token kernel, 2 to 32 tokens the persistent few-token kernel (one
 * launch per 8 tokens, reading the union of their experts once per layer;
 * shapes with n_experts <= 512, d_ff a multiple of 128 and d_model <= 3072),
 * 33 and more the tensor-core grouped GEMMs (from 1,024 tokens, experts
 * with at most 16 of them on a weight-streaming kernel); the CUDA-core grouped path runs
 * where none fits the shape (or under the MOE_FLAG_NO_* flags); each path
 * meets the same accuracy bound. */
MOE_API int moe_forward(moe_ctx *ctx, int layer, const uint16_t *x_bf16, int T,
                uint16_t *y_bf16, float *y_f32, int32_t *ids, float *w,
                void *stream);

/* Layers [layer0, layer0 + n_layers) stacked with a residual stream (the
 * pages' 48 stacked layers, video transcript 1:37-1:50 of "Qwen3.8-Flash-Next
 * at 45 Tokens/sec on a 12GB GPU?"; the normalisation between them is this
 * library's reading, below):
 *   r_0 = x (bf16 input, widened to fp32)
 *   x_l = bf16(rmsnorm(r_l)),  rmsnorm(r) = r / sqrt(mean(r^2) + 1e-6)
 *   r_{l+1} = r_l + float(moe_l(x_l))
 * and resid_out [T][d] fp32 = r_{layer0+n_layers}.  The pages only say the
 * layers are stacked; the normalisation without learned weight is this
 * library's reading.  x_bf16 and resid_out are device pointers; rec may be
 * NULL.  Asynchronous on `stream`, no allocation.  Errors as moe_forward. */
MOE_API int moe_forward_stack(moe_ctx *ctx, int layer0, int n_layers, const uint16_t *x_bf16,
                      int T, float *resid_out, const moe_stack_record *rec,
                      void *stream);

/* moe_forward_stack with HOST buffers: copies x_bf16 (host, pinned or
 * pageable) to the device, runs the stack and copies resid_out back to the
 * host; returns after the result is in host memory.  (The pages' engine takes
 * tokens from a host program; this is the same layer stack behind a call that
 * owns the copies.)  Errors as moe_forward_stack. */
MOE_API int moe_forward_stack_host(moe_ctx *ctx, int layer0, int n_layers,
                           const uint16_t *x_bf16_host, int T, float *resid_out_host,
                           void *stream);

/* Library plumbing without a counterpart in the pages: teardown, error
 * reporting, measurement and tracing.
 *
 * Free every device allocation of the context.  NULL is accepted.  A handle
 * must not be used after this call. */
MOE_API int moe_destroy(moe_ctx *ctx);

/* Read (and clear) the device error word that bounded device waits and
 * in-kernel checks set.  *code receives 0 or a MOE_ERR_* value.  Synchronises
 * the context's device.  When *code is nonzero the call also resets the
 * single-token kernel's cross-CTA arrival counters, which a kernel that gave
 * up part-way leaves mid-count: after a nonzero code, call this before the
 * next forward on the context. */
MOE_API int moe_get_device_error(moe_ctx *ctx, int *code);

/* L2 residency of the decode kernels' weight stream, the counterpart on one
 * GPU of the pages' expert cache, which keeps the experts in use in the
 * faster memory ("Qwen3.8-Flash-Next on RTX 5090 + 64GB", section 2 "Expert
 * Cache and CPU/GPU Split").  Here every expert already lives in HBM; the
 * shared experts are read by every token of every call, so in mode
 * MOE_L2_KEEP_SHARED their tiles are copied with the L2 eviction priority
 * evict_last and the routed experts' tiles and the router rows with
 * evict_first, which keeps the shared experts of all layers in the 126 MB L2
 * across calls when they fit; MOE_L2_STREAM (the default) copies everything
 * with the default priority.  The decode kernels are bound by the latency of
 * each layer's chain of steps, not by bandwidth, and keeping 83-106 MB of
 * shared experts measured no faster (one token, Q4: 1.2 % slower), hence the
 * default.  Applies to the single-token and few-token kernels; results do not
 * depend on it.  Errors: INVALID_ARG (NULL context, unknown mode). */
#define MOE_L2_STREAM 0
#define MOE_L2_KEEP_SHARED 1
MOE_API int moe_set_l2_policy(moe_ctx *ctx, int mode);

/* Measurement hook.  While enabled, each forward records a CUDA event pair on
 * the caller's stream around its dominant kernel (the kernel that streams the
 * expert weights).  moe_timing_read synchronises the device and returns, since
 * the previous read: the summed duration of the timed launches (ms), their
 * number, every kernel launch the library issued (timed or not), and the
 * name of the timed kernel (copied into name[0..name_len), NUL-terminated).
 * At most 65536 launches are timed between reads; later ones are counted but
 * not timed. */
MOE_API int moe_timing_enable(moe_ctx *ctx, int on);
MOE_API int moe_timing_read(moe_ctx *ctx, double *total_ms, long long *timed_launches,
                            long long *all_launches, char *name, int name_len);

/* Phase trace of the last persistent-kernel call (context created with
 * MOE_FLAG_TRACE).  Copies up to n_max records into out (host memory) and
 * returns their number in *n.  One record = 24 uint64: CTA index, layer,
 * then 22 slots of SM clock cycles since the start of that layer in that CTA
 * (phase ends and waits; the slot map is documented next to the kernel's
 * trace marks).  The caller's buffer must hold 24 * n_max values.
 * Synchronises the device. */
MOE_API int moe_trace_read(moe_ctx *ctx, unsigned long long *out, int n_max, int *n);

/* Routing without any device allocation.  The pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory (code
 * running inside another runtime's memory pool, services that forbid device
 * allocation after start-up, plain C hosts that only receive device
 * pointers).  It computes the router logits of T tokens and their softmax
 * top-k exactly as moe_forward does, from caller-owned device buffers:
 *   x_bf16 [T][d_model] bf16, router_w [n_experts][d_model] fp32 (16-byte
 *   aligned), router_bias [n_experts] fp32 or NULL; outputs ids [T][top_k]
 *   int32 and w [T][top_k] fp32 (descending weight, equal logits -> lower id;
 *   a NaN logit ranks as -inf).  Limits: d_model a multiple of 4 and at most
 *   16384, n_experts <= 1024, top_k <= min(n_experts, 32); anything else, or
 *   a misaligned router_w, returns MOE_ERR_INVALID_ARG before any work.
 * The logits live in a fixed array in device memory that the library holds
 * on every device that loads it, until the process exits:
 * T * n_experts must not exceed MOE_ROUTE_STATIC_MAX_LOGITS
 * (MOE_ERR_TOO_MANY_TOKENS otherwise, with a message in moe_last_error()).
 * The first call on a device looks up that array's device address (make it
 * before any stream capture on that device); the address is kept for the
 * process, so do not call this on a device after cudaDeviceReset on it.  Calls share the array: calls
 * that overlap on the GPU (other streams, other host threads) race; order
 * them on one stream.  Asynchronous on `stream`; calls no allocating routine.
 * Errors: INVALID_ARG, TOO_MANY_TOKENS, UNSUPPORTED (device index >= 64), CUDA. */
#define MOE_ROUTE_STATIC_MAX_LOGITS 65536
MOE_API int moe_route_static(const uint16_t *x_bf16, int T, int d_model, const float *router_w,
                             const float *router_bias, int n_experts, int top_k, int32_t *ids,
                             float *w, void *stream);

/* Static text for a status code. */
MOE_API const char *moe_status_string(int status);

/* Text of the most recent MOE_ERR_CUDA / MOE_ERR_OOM on this host thread. */
MOE_API const char *moe_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* QEFFN_MOE_H */
