/*
 * pae.h - C ABI of the pi0.5-style action-expert denoise loop on B200 (sm_100a).
 *
 * The operation: the flow-matching denoise loop of a pi0.5-style action expert,
 * as the PhyAI report describes its pi0.5 path ("PhyAI: Real-Time Physical AI
 * at the Edge", Sec. 5.1 "Follow one pi0.5 request through cache reuse and
 * graph replay" and Sec. 5.5 "Reuse only valid conditions"): the
 * vision-language prefix K/V is computed once per observation and cached, a
 * new observation invalidates it, timestep/modulation tables are precomputed
 * once, and a captured loop runs K Euler steps over the action tokens.  The
 * expert layer is a small transformer: adaptive RMSNorm modulated by the
 * timestep, GQA attention over [cached prefix | action tokens], a GeGLU MLP,
 * an input projection from actions and an output projection whose result v
 * advances the actions by x += dt * v.
 *
 * Conventions for every call:
 *  - One context per host thread; calls on one context are not thread-safe.
 *  - Device pointers are CUDA device memory on the device that was current at
 *    pae_create.  Host pointers are marked "host".
 *  - Matrices are row-major [out][in] (the "in" index contiguous).
 *  - Work is enqueued on the given stream and the call returns without waiting,
 *    except pae_create (synchronous) and pae_sync.
 *  - Argument and state errors are returned before anything is enqueued.
 *    CUDA failures return PAE_ERR_CUDA.  A device-side bounded wait that ran
 *    out sets an error word; the next call (or pae_sync) returns
 *    PAE_ERR_TIMEOUT.  No kernel traps.  pae_last_error() gives the message.
 *  - No call allocates device memory after pae_create, except the first
 *    pae_denoise for a new batch size, which instantiates a CUDA graph.
 */
#ifndef PAE_H
#define PAE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pae_ctx pae_ctx;
/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* pae_stream;

typedef enum {
  PAE_OK = 0,
  PAE_ERR_ARG = 1,         /* bad argument: null pointer, size out of range, bad grid  */
  PAE_ERR_STATE = 2,       /* call out of order: tables missing, prefix row never set  */
  PAE_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed                         */
  PAE_ERR_OOM = 4,         /* device allocation failed in pae_create                    */
  PAE_ERR_TIMEOUT = 5,     /* a device-side bounded wait ran out (error word set)       */
  PAE_ERR_UNSUPPORTED = 6  /* shape the kernels do not cover (see pae_create)           */
} pae_status;

typedef enum {
  PAE_FP32 = 0,   /* every tensor fp32 (CUDA-core kernels)                          */
  PAE_BF16 = 1,   /* bf16 weights and GEMM inputs, fp32 accumulation and residual   */
  PAE_W4A16 = 2   /* int4 projection weights (group-wise bf16 scales), bf16 inputs  */
} pae_dtype;

/*
 * Model shape.  L = layers, D = width, Hq/Hkv = query/KV heads, d = head_dim,
 * F = mlp_dim, A = action_dim, H = chunk (action tokens per request).
 * max_batch / max_prefix size the context's buffers.  group_size is the W4A16
 * quantisation group along K (must be 128; ignored otherwise).  rms_eps is the
 * epsilon of every adaptive RMSNorm.
 *
 * Supported (else PAE_ERR_UNSUPPORTED): Hq % Hkv == 0, Hq/Hkv <= 16, D % 32 == 0,
 * D <= 2048;
 * BF16/W4A16: D, Hq*d, F multiples of 128, d in {64, 128, 256}, H <= 256,
 * max_batch*H <= 4096.
 *
 * rope_base: 0 = no rotary position embedding (the default); > 0 = rotate
 * every query head and every action key at its position in the request's
 * joint [prefix | action] sequence, P_b + i for action token i of a request
 * with a P_b-token prefix (the cached prefix keys are taken as already
 * rotated at 0..P_b-1).  Rotate-half form: channel i < d/2 pairs with
 * i + d/2 and turns by pos * rope_base^(-2i/d).  The angles come from a
 * cos/sin table built once in float64 from the integer positions (the
 * vla.cpp abstract warns that positional-index precision changes actions).
 * prefix_width: 0 = no prefix production (the default); > 0 = the width of
 * the hidden states pae_set_prefix_hidden projects into the K/V slots (then
 * pae_weights.w_prefix_kv is required).
 */
typedef struct {
  int layers, width, n_q_heads, n_kv_heads, head_dim, mlp_dim, action_dim, chunk;
  int max_batch, max_prefix, group_size;
  int dtype;        /* pae_dtype */
  float rms_eps;
  float rope_base;  /* 0: off */
  int prefix_width; /* 0: no pae_set_prefix_hidden */
} pae_config;

/*
 * Parameters (device pointers; element type fp32 in PAE_FP32 mode, bf16
 * otherwise; int4 where noted).  pae_create copies and repacks everything, so
 * the caller may free its buffers when pae_create returns.
 *
 *   w_in  [D][A], b_in [D]        input projection  h = x W_in^T + b_in
 *   w_out [A][D], b_out [A]       output projection v = y W_out^T + b_out
 *   w_t1, w_t2 [D][D], b_t1, b_t2 [D]   time MLP  c = swish(W_t2 swish(W_t1 e + b_t1) + b_t2)
 *   w_mod [2L][3D][D], b_mod [2L][3D]   per layer l: index 2l = attention norm,
 *                                 2l+1 = MLP norm; rows ordered (scale, shift, gate)
 *   w_modf [2D][D], b_modf [2D]   final norm (scale, shift)
 *   w_qkv[l] [(Hq+2Hkv)d][D]      rows: Hq query heads, then Hkv keys, then Hkv values
 *   w_o[l] [D][Hq d], w_gate[l], w_up[l] [F][D], w_down[l] [D][F]
 * PAE_W4A16: w_qkv..w_down point to packed int4 [N][K/2] bytes (two's
 * complement codes in [-8, 7], low nibble = even k) and s_qkv..s_down to bf16
 * scales [N][K/group_size]; value = code * scale.  The s_* arrays are ignored in
 * the other modes.  Attention and MLP carry no biases.
 *   w_prefix_kv[l] [2 Hkv d][prefix_width]   prefix production (only when
 *                                 cfg.prefix_width > 0): layer l's key rows
 *                                 (Hkv heads) then value rows, fp32 in PAE_FP32
 *                                 mode, bf16 otherwise (also in PAE_W4A16).
 */
typedef struct {
  const void *w_in, *b_in, *w_out, *b_out;
  const void *w_t1, *b_t1, *w_t2, *b_t2;
  const void *w_mod, *b_mod, *w_modf, *b_modf;
  const void *const *w_qkv, *const *w_o, *const *w_gate, *const *w_up, *const *w_down;
  const void *const *s_qkv, *const *s_o, *const *s_gate, *const *s_up, *const *s_down;
  const void *const *w_prefix_kv;
} pae_weights;

/* Validate cfg, allocate the context's device buffers, copy and repack the
 * weights into the kernels' layouts, and synchronise once.  On failure *out
 * is NULL and nothing stays allocated.  Errors: PAE_ERR_ARG (null pointers,
 * non-positive sizes), PAE_ERR_UNSUPPORTED, PAE_ERR_OOM, PAE_ERR_CUDA. */
pae_status pae_create(const pae_config* cfg, const pae_weights* w, pae_ctx** out);

/* Cache the vision-language prefix of request `row` (report Sec. 5.1: the
 * prefix is computed once per observation and reused by every Euler step).
 * k_per_layer[l], v_per_layer[l] (host arrays of L device pointers) each point
 * to [len][Hkv][d] (fp32 in PAE_FP32 mode, bf16 otherwise).  The data are
 * copied into the context's slot for `row` on `stream`; the slot keeps a
 * fixed address, so captured graphs stay valid.  Each call replaces the row's
 * content and length: a new observation invalidates the old prefix.
 * 0 <= len <= max_prefix, 0 <= row < max_batch (else PAE_ERR_ARG). */
pae_status pae_set_prefix(pae_ctx* ctx, int row, const void* const* k_per_layer,
                          const void* const* v_per_layer, int len, pae_stream stream);

/* Produce and cache the prefix of request `row` from the prefix model's
 * per-layer hidden states (report Sec. 5.1: the vision-language prefix is
 * computed once per observation and its per-layer K/V cached): for every
 * layer l, y = h_l / sqrt(mean(h_l^2) + rms_eps) per token (a plain RMSNorm;
 * fold a learned gain into w_prefix_kv), [k | v] = y w_prefix_kv[l]^T, keys
 * rotated at positions 0..len-1 when rope_base > 0, written straight into the
 * row's K/V slot (no intermediate K/V buffer).  h_per_layer (host array of L
 * device pointers) each point to [len][prefix_width] (fp32 in PAE_FP32 mode,
 * bf16 otherwise).  Replaces the row's prefix like pae_set_prefix.
 * Errors: PAE_ERR_STATE if the context was created with prefix_width == 0;
 * PAE_ERR_ARG for a bad row, len outside [0, max_prefix] or NULL pointers. */
pae_status pae_set_prefix_hidden(pae_ctx* ctx, int row, const void* const* h_per_layer, int len,
                                 pae_stream stream);

/* Build the timestep conditioning once for a grid t[0..K] (host, float64,
 * strictly monotone, K >= 1, K <= 64): the sinusoidal embedding, the time MLP,
 * the per-step (scale, shift, gate) tables of every norm and dt_k =
 * t[k+1] - t[k] (report Sec. 5.1: precomputed timestep and modulation
 * tables).  A later call with the same K rewrites the tables in place and
 * keeps captured graphs; a different K drops them. */
pae_status pae_precompute_tables(pae_ctx* ctx, const double* t, int K, pae_stream stream);

/* Run the K Euler steps for rows 0..batch-1: x = noise; for k < K:
 * x += dt_k * v(x, t_k); out = x.  noise and out are device fp32
 * [batch][H][A]; out == noise is allowed.  Rows < batch must have a prefix
 * set and the tables must be built (else PAE_ERR_STATE).  batch == 0 is a
 * no-op.  The first call for a batch size captures the loop in a CUDA graph;
 * later calls replay it (report Sec. 5.1: CUDA Graph replay of the stable
 * loop).  0 <= batch <= max_batch. */
pae_status pae_denoise(pae_ctx* ctx, const float* noise, float* out, int batch,
                       pae_stream stream);

/* As pae_denoise, with noise and out in host memory (page-locked memory gives
 * asynchronous copies).  The host-to-device copy, the loop and the
 * device-to-host copy are all enqueued on `stream`; out is valid after the
 * stream is synchronised. */
pae_status pae_denoise_host(pae_ctx* ctx, const float* noise_host, float* out_host,
                            int batch, pae_stream stream);

/* Run only steps k_begin..k_end-1 of the tabled grid (0 <= k_begin < k_end <= K),
 * without graph capture: x = x_in; steps; x_out = x.  Splitting a trajectory
 * into consecutive ranges gives bitwise the same result as one call. */
pae_status pae_denoise_steps(pae_ctx* ctx, const float* x_in, float* x_out, int batch,
                             int k_begin, int k_end, pae_stream stream);

/* Options.  PAE_OPT_USE_GRAPH (default 1): 0 makes pae_denoise launch the
 * kernels directly.  PAE_OPT_WAIT_LIMIT_US (default 2000000): bound of every
 * device-side wait, in microseconds.  PAE_OPT_PDL (default 1, bf16 modes):
 * programmatic dependent launch between the loop's kernels, so a kernel's
 * weight loads overlap its predecessor's tail; 0 serialises the kernels.
 * PAE_OPT_MAX_SPLITK (default 8, range 1..16): largest split-K cluster the
 * projection planner may choose (a tuning knob; results stay within the
 * parity tolerance, bitwise identical only for the same setting).
 * PAE_OPT_PERSISTENT (default 0, bf16 mode): 1 runs all K steps of a call as
 * one persistent kernel (one CTA per SM, grid barriers between the phases of
 * each layer) instead of the graph of per-phase kernels, for batches with
 * batch * chunk <= 64.  The two paths round differently (both stay within
 * the parity tolerance); each is bitwise reproducible on its own, and
 * pae_denoise and pae_denoise_steps take the same path for the same batch.
 * PAE_OPT_FUSED_NORM (default 0, bf16 weights): 1 makes the QKV and gate/up
 * projections apply the adaRMSNorm to their fp32 input inside the kernel
 * (statistics from the residual projections' epilogues) instead of separate
 * norm kernels, for batches of at most one 64-token tile.  Both round within
 * the parity tolerance; each is bitwise reproducible.
 * PAE_OPT_FACTORED_NORM (default 0, bf16 / int4 weights; PAE_OPT_FUSED_NORM
 * takes precedence): 1 removes the separate norm kernels.  The O and down projections'
 * split-K epilogues write the next norm's operand bf16(h (1 + scale)) and
 * per-token sums of squares of h; QKV and gate/up multiply their accumulators
 * by 1/rms and add the shift projected through their weights (tables built by
 * pae_precompute_tables): the same value as projecting adaRMSNorm(h), rounded
 * differently (within the parity tolerance, bitwise reproducible).  Batches
 * whose O or down plan has no split-K keep the norm kernels.  Off by default:
 * at the pi0.5 shape the graph with the (cheap, shared-memory-free) norm
 * kernels overlaps better under programmatic dependent launch.
 * PAE_OPT_DATAFLOW (default 0, bf16 / int4 weights): batches with batch * chunk <= 64
 * run all K steps as one launch of thread-block clusters whose stages wait on
 * per-tile counters instead of kernel boundaries (no CUDA graph for these
 * batches; pae_denoise_steps takes the same path).  0 uses the captured graph
 * of per-stage kernels (the faster one at the pi0.5 shape so far).  The two paths round differently (the dataflow loop
 * applies each adaRMSNorm's 1/rms after the projection and its shift as a
 * precomputed projected term); both stay within the parity tolerance and each
 * is bitwise reproducible.  PAE_OPT_DATAFLOW_CLUSTER (default 0 = automatic):
 * force the cluster size (2, 4, 8 or 16) of the dataflow loop; a batch it
 * does not fit runs the graph. */
enum {
  PAE_OPT_USE_GRAPH = 1,
  PAE_OPT_WAIT_LIMIT_US = 2,
  PAE_OPT_PDL = 4,
  PAE_OPT_MAX_SPLITK = 5,
  PAE_OPT_PERSISTENT = 6,
  PAE_OPT_FUSED_NORM = 7,
  PAE_OPT_DATAFLOW = 8,
  PAE_OPT_DATAFLOW_CLUSTER = 9,
  PAE_OPT_FACTORED_NORM = 10
};
pae_status pae_set_option(pae_ctx* ctx, int option, long long value);

/* Kernel classes for profiling, as bit positions of PAE_OPT_PROFILE. */
enum {
  PAE_K_TRANSITION = 0, /* out_proj + Euler update + in_proj + first norm, per token */
  PAE_K_QKV = 1,        /* adaRMSNorm'd input x W_qkv -> q, k, v                      */
  PAE_K_ATTENTION = 2,  /* GQA over [cached prefix | action keys]                     */
  PAE_K_OPROJ = 3,      /* o W_o, gated residual                                      */
  PAE_K_NORM = 4,       /* adaRMSNorm of the residual stream                          */
  PAE_K_GATEUP = 5,     /* GeGLU gate/up projection                                   */
  PAE_K_DOWN = 6,       /* down projection, gated residual                            */
  PAE_K_PERSISTENT = 7, /* the whole loop as one persistent kernel (small batches)    */
  PAE_K_DATAFLOW = 8,   /* the whole loop as one launch of clusters (small batches)   */
  PAE_K_COUNT = 9
};
/* PAE_OPT_PROFILE (default 0): bit mask of PAE_K_* classes.  Launches of those
 * classes are bracketed by CUDA events on their stream (inside the captured
 * graph too).  After the stream is synchronised, pae_profile_read returns the
 * summed device time and the launch count of one class over the most recent
 * pae_denoise / pae_denoise_steps. */
enum { PAE_OPT_PROFILE = 3 };
pae_status pae_profile_read(pae_ctx* ctx, int kernel_class, double* total_ms, int* launches);

/* Queries.  PAE_Q_GRAPH_KERNELS: kernel nodes in the captured graph of
 * `batch` (0 if none captured yet).  PAE_Q_SPLITS: split-K factors of the four
 * projections for `batch`, packed as qkv | o<<8 | gateup<<16 | down<<24.
 * PAE_Q_TOKEN_TILE: MMA token tile for `batch`.  PAE_Q_ATTN_SPLITS: key splits
 * of the attention for `batch`.  PAE_Q_PERSISTENT: 1 if pae_denoise runs the
 * persistent kernel for `batch` (option on and the batch eligible), else 0.
 * PAE_Q_FUSED_NORM: how the graph for `batch` applies adaRMSNorm: 0 separate
 * norm kernels, 1 inside the projections from fp32 h (PAE_OPT_FUSED_NORM), 2
 * factored into the projections' epilogues (PAE_OPT_FACTORED_NORM).  PAE_Q_DATAFLOW: the
 * cluster size of the dataflow loop pae_denoise runs for `batch` (0: it runs
 * the graph or the persistent kernel).  PAE_Q_ATTN_CHUNK: keys per chunk of
 * the graph's attention kernel for `batch` (64 or 128). */
enum {
  PAE_Q_GRAPH_KERNELS = 1,
  PAE_Q_SPLITS = 2,
  PAE_Q_TOKEN_TILE = 3,
  PAE_Q_ATTN_SPLITS = 4,
  PAE_Q_PERSISTENT = 5,
  PAE_Q_FUSED_NORM = 6,
  PAE_Q_DATAFLOW = 7,
  PAE_Q_ATTN_CHUNK = 8
};
pae_status pae_query(pae_ctx* ctx, int what, int batch, long long* value);

/* The same launch-plan queries without a context or a device: what a context
 * created from `cfg`, with its options at their defaults, would use for
 * `batch` (PAE_Q_SPLITS, PAE_Q_TOKEN_TILE, PAE_Q_ATTN_SPLITS,
 * PAE_Q_ATTN_CHUNK or PAE_Q_FUSED_NORM; 0 in PAE_FP32 mode, which has no
 * tensor-core plan).
 * Host arithmetic only.  Errors: PAE_ERR_ARG for a NULL argument, a batch
 * outside [1, max_batch] or another query; the config is checked as by
 * pae_create (PAE_ERR_ARG / PAE_ERR_UNSUPPORTED). */
pae_status pae_plan_query(const pae_config* cfg, int what, int batch, long long* value);

/* Synchronise `stream` and report the device error word (PAE_ERR_TIMEOUT if a
 * bounded wait ran out since the last pae_clear_error).  pae_clear_error
 * resets it so the context can be used again, except after a failed drain
 * (the last bounded wait for copies or MMAs a kernel had already issued, whose
 * message says so): then copies may still be landing in the context's memory
 * and the error stays until the context is destroyed. */
pae_status pae_sync(pae_ctx* ctx, pae_stream stream);
void pae_clear_error(pae_ctx* ctx);

/* Message of the last failed call on ctx ("" if none).  With ctx == NULL, the
 * message of the last failed pae_create in this thread. */
const char* pae_last_error(const pae_ctx* ctx);

/* Copy an internal buffer to host memory for inspection (synchronous).
 * name: "x", "h", "y", "q", "o", "u", "kcache", "vcache", "tables", "dt",
 * "lens".  *bytes in: capacity of dst; out: bytes of the buffer (dst may be
 * NULL to query the size). */
pae_status pae_debug_copy(pae_ctx* ctx, const char* name, void* dst_host, size_t* bytes);

/* Timestep/modulation tables without a context and without allocating.
 * The pages have no counterpart: this entry point exists for callers that may
 * not allocate device memory while they run (a real-time control process past
 * its set-up, a host framework that owns all device memory in its own arena,
 * code that is capturing a stream into a CUDA graph).  They cannot call
 * pae_create, which allocates, but can build the same tables as
 * pae_precompute_tables into buffers they own.
 *   w: only w_t1, b_t1, w_t2, b_t2, w_mod, b_mod, w_modf, b_modf are read
 *      (device, layouts as in pae_create; fp32 if dtype is PAE_FP32, else bf16).
 *   t: host float64 grid t[0..K], strictly monotone.
 *   tables: device fp32 [K][(6*layers + 2)*width], the layout of the context's
 *      tables: per layer l and norm j (0 attention, 1 MLP) the rows
 *      (scale, shift, gate), then the final norm's (scale, shift).
 *   dt: device fp32 [K], dt_k = t[k+1] - t[k].
 * Limits: 1 <= K <= 64 and width <= 2048 (else PAE_ERR_ARG, message in
 * pae_last_error(NULL)).  Intermediates live in one fixed 1.5 MB device array
 * per device that every call shares: calls whose GPU work overlaps (streams
 * with no ordering between them) race and must be serialised by the caller.
 * The first call on a device looks the array up and sets kernel attributes;
 * make that first call before any stream capture.  That look-up is cached for
 * the life of the process: after cudaDeviceReset on a device, restart the
 * process before calling this entry point there again.  Devices with ordinals
 * of 64 and above give PAE_ERR_UNSUPPORTED.  A CUDA error already pending from
 * earlier work is reported as such (PAE_ERR_CUDA) before anything is
 * enqueued.  Asynchronous on `stream`. */
pae_status pae_precompute_tables_static(int layers, int width, int dtype, const pae_weights* w,
                                        const double* t, int K, float* tables, float* dt,
                                        pae_stream stream);

/* Free everything the context owns.  NULL is a no-op. */
void pae_destroy(pae_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* PAE_H */
