/*
 * wedlm.h -- C ABI of libwedlm, a B200 (sm_100a) implementation of WeDLM's
 * Streaming Parallel Decoding step.
 *
 * Method (hyper.ai summary of arXiv 2512.22737, section "Method"; sai.science
 * review "WeDLM: Reconciling Diffusion Language Models with Standard Causal
 * Attention for Fast Inference", sections Summary and Recommended Changes):
 * a sequence keeps a sliding window of W slots, each either filled (a
 * predicted token) or a mask.  One decode step
 *   1. refills the window with masks up to min(W, end - S) slots,
 *   2. reorders it so filled slots physically precede masks, each slot keeping
 *      its logical position S + offset (Topological Reordering),
 *   3. runs a causal forward over the reordered window against the persistent
 *      paged KV cache, with RoPE at logical positions,
 *   4. commits the leftmost contiguous run of slots that were filled when the
 *      step began: their K/V depend only on earlier tokens, so they join the
 *      cache and their tokens are emitted,
 *   5. fills masked slots by the distance-penalised entropy rule
 *      H~_j = H_j + lambda * j (j = slot offset): every slot with H~_j < tau,
 *      or the single argmin if none (one-by-one when tau_none is set), each
 *      with its argmax token (the mask id is never predicted),
 *   6. slides the window past the committed run.
 *
 * Conventions
 *   - All functions return a wedlm_status (0 = success, < 0 = error).  No
 *     function aborts the process or traps the GPU; device-side checks record a
 *     code in a device error word that the host reads after each call.
 *   - The library owns all device memory it allocates (weights, KV pages,
 *     scratch).  Host buffers passed in are owned by the caller and are only
 *     read or written during the call.
 *   - A context is bound to the CUDA device current at wedlm_create and to the
 *     stream given there (borrowed, not owned; NULL = legacy default stream).
 *     Calls are synchronous on return unless the name ends in _async.
 *   - A context is not thread-safe; use one context per host thread.
 *   - Sequence slots are integers in [0, max_batch).
 *   - KV pages hold WEDLM_PAGE_TOKENS tokens.  Pages for a sequence's whole
 *     length (prompt + max_new_tokens) are reserved at prefill; running out of
 *     pages returns WEDLM_ERR_OOM_PAGES and leaves the context unchanged.
 */
#ifndef WEDLM_H
#define WEDLM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t wedlm_status;

#define WEDLM_OK                  0
#define WEDLM_ERR_INVALID_ARG    -1  /* bad pointer, size, slot or tensor id */
#define WEDLM_ERR_OOM_PAGES      -2  /* KV page pool exhausted */
#define WEDLM_ERR_OOM_DEVICE     -3  /* cudaMalloc failed */
#define WEDLM_ERR_CUDA           -4  /* a CUDA runtime call failed */
#define WEDLM_ERR_DEVICE_ASSERT  -5  /* a kernel's own bounds check fired */
#define WEDLM_ERR_STATE          -6  /* call not valid in the current state */
#define WEDLM_ERR_UNSUPPORTED    -7  /* shape or dtype this build does not run */
#define WEDLM_ERR_TIMEOUT        -8  /* a bounded device wait gave up */
#define WEDLM_ERR_NONFINITE      -9  /* a masked slot's logits held a NaN or an infinity */

#define WEDLM_DTYPE_F32   0
#define WEDLM_DTYPE_BF16  1

#define WEDLM_MEM_HOST    0
#define WEDLM_MEM_DEVICE  1

#define WEDLM_PAGE_TOKENS 16

/* Model shape and capacity.  A causal decoder: token embedding, L blocks of
 * [RMSNorm -> GQA attention with RoPE -> residual, RMSNorm -> SwiGLU FFN ->
 * residual], final RMSNorm, untied LM head (the Qwen2.5-7B / Qwen3-8B
 * backbones the review names, without biases or QK-norm).
 * dtype selects the storage and arithmetic of weights, activations and KV:
 *   WEDLM_DTYPE_F32  fp32 everywhere (SIMT kernels; the exact-parity mode),
 *   WEDLM_DTYPE_BF16 bf16 storage, fp32 accumulation (tensor-core kernels).
 * Logits, the residual stream and all softmax/entropy arithmetic are fp32. */
typedef struct wedlm_model_cfg {
    int32_t n_layers;
    int32_t d_model;
    int32_t n_heads;        /* query heads */
    int32_t n_kv_heads;     /* KV heads; n_heads % n_kv_heads == 0 */
    int32_t head_dim;       /* even; bf16 mode requires 128 */
    int32_t ffn_dim;
    int32_t vocab;
    int32_t mask_id;        /* id of the mask token, in [0, vocab) */
    double  rope_theta;
    float   rms_eps;
    int32_t dtype;          /* WEDLM_DTYPE_* */
    int32_t max_batch;      /* sequence slots */
    int32_t max_window;     /* largest W any sequence may use (<= 64) */
    int32_t max_ctx;        /* largest prompt + max_new_tokens of a sequence */
    int32_t num_pages;      /* KV pool size in pages; 0 = max_batch * ceil(max_ctx / 16) */
    int32_t prefill_chunk;  /* prompt rows per prefill forward; 0 = 1024 */
} wedlm_model_cfg;

typedef struct wedlm_ctx wedlm_ctx;

/* Create a context on the current CUDA device.  Allocates weights storage
 * (uninitialised until wedlm_load_weights), the KV pool and scratch.
 * cuda_stream: a cudaStream_t (borrowed) or NULL. */
wedlm_status wedlm_create(const wedlm_model_cfg* cfg, void* cuda_stream, wedlm_ctx** out_ctx);

/* Free everything the context owns.  NULL is accepted. */
void wedlm_destroy(wedlm_ctx* ctx);

/* Static description of a status code. */
const char* wedlm_status_str(wedlm_status status);

/* Human-readable detail of the context's most recent error ("" if none).
 * The string is owned by the context and valid until its next call. */
const char* wedlm_last_error(const wedlm_ctx* ctx);

/* Weight tensors, all in nn.Linear layout [out_features][in_features],
 * row-major, contiguous:
 *   EMBED [vocab][d]       LM_HEAD [vocab][d]     FINAL_NORM [d]
 *   ATTN_NORM [d]          WQ [n_heads*head_dim][d]
 *   WK, WV [n_kv_heads*head_dim][d]               WO [d][n_heads*head_dim]
 *   FFN_NORM [d]           WG, WU [ffn][d]        WD [d][ffn]
 * (per-layer tensors take `layer` in [0, n_layers); others ignore it). */
#define WEDLM_T_EMBED       0
#define WEDLM_T_LM_HEAD     1
#define WEDLM_T_FINAL_NORM  2
#define WEDLM_T_ATTN_NORM   3
#define WEDLM_T_WQ          4
#define WEDLM_T_WK          5
#define WEDLM_T_WV          6
#define WEDLM_T_WO          7
#define WEDLM_T_FFN_NORM    8
#define WEDLM_T_WG          9
#define WEDLM_T_WU         10
#define WEDLM_T_WD         11

/* Copy one weight tensor into the context.  src points to host or device
 * memory (src_mem = WEDLM_MEM_*) holding the tensor in src_dtype.  Norm gains
 * must be WEDLM_DTYPE_F32.  Matrices must be in the context's dtype (no
 * conversion is performed).  The source is not retained.  Every tensor must be
 * loaded once before the first prefill. */
wedlm_status wedlm_load_weights(wedlm_ctx* ctx, int32_t tensor, int32_t layer,
                                const void* src, int32_t src_dtype, int32_t src_mem);

/* Admit a sequence into `slot`: reserve KV pages for prompt_len +
 * max_new_tokens positions, run the causal prefill forward over the prompt
 * (host int32 ids, caller-owned) and commit all of it to the cache.  The
 * sequence then decodes with a window of `window` slots (1 <= window <=
 * max_window).  The slot must be free (see wedlm_kv_reset).  The prefill
 * produces no logits: the first window is all masks. */
wedlm_status wedlm_prefill(wedlm_ctx* ctx, int32_t slot, const int32_t* prompt_ids,
                           int32_t prompt_len, int32_t max_new_tokens, int32_t window);

/* Release a slot's pages and window (slot = -1: every slot). */
wedlm_status wedlm_kv_reset(wedlm_ctx* ctx, int32_t slot);

/* Decode knobs (sai.science review, Recommended Changes: lambda = 0.10 and
 * tau in {0.3, 0.5, 0.9}; Reproducibility & code: a threshold of None gives
 * one-by-one decoding).  logit_scale multiplies the LM-head logits before
 * entropy and argmax (an inverse temperature; 1 = the model as loaded).
 *
 * blockwise selects the block-wise ("stop-and-wait") baseline the method is
 * compared against (hyper.ai summary, Method: block decoding must finalise the
 * whole block before any of it is cached): nothing is committed until every
 * slot of the window is filled, then the whole window is.
 *
 * temperature > 0 samples each fill token instead of taking the argmax (the
 * pages' evaluation decodes at T = 0.1, sai.science review, Reproducibility):
 * token = argmax_v (logit_scale * z_v / temperature + G_v) over v != mask_id
 * with Gumbel noise G_v = -log(-log(u_v)).  u_v comes from a counter-based
 * generator built on the SplitMix64 finaliser (Steele, Lea and Flood, "Fast
 * splittable pseudorandom number generators", 2014), mix(z): z += 0x9E3779B97F4A7C15;
 * z = (z ^ z >> 30) * 0xBF58476D1CE4E5B9; z = (z ^ z >> 27) * 0x94D049BB133111EB;
 * z ^= z >> 31.  With h = mix(mix(mix(mix(seed ^ slot) ^ step) ^ position) ^ v)
 * (slot = batch slot, step = that slot's decode steps so far, position = the
 * masked slot's logical position), u_v = ((h >> 40) + 0.5) / 2^24.  The
 * entropy that selects the slots is unchanged (temperature 1). */
typedef struct wedlm_step_params {
    float   lambda;       /* distance penalty per slot offset (nats) */
    float   tau;          /* fill threshold on H~ (nats), strict < */
    int32_t tau_none;     /* nonzero: fill exactly the argmin each step */
    float   logit_scale;  /* > 0 */
    int32_t blockwise;    /* nonzero: block-wise baseline (whole-window commits) */
    float   temperature;  /* 0: greedy fill; > 0: Gumbel-max sampling at this temperature */
    uint64_t seed;        /* sampling seed (ignored when temperature == 0) */
} wedlm_step_params;

/* Run one decode step for every active slot (a slot is active from prefill
 * until its committed length reaches prompt_len + max_new_tokens).
 * Outputs (host, caller-owned, may be NULL to skip):
 *   out_committed [max_batch * max_window]: the tokens committed by slot b this
 *                 step at out_committed[b * max_window + 0 .. count-1]
 *   out_counts    [max_batch]: tokens committed by each slot this step
 *   out_active    [1]: slots still decoding after this step
 * Synchronises the context's stream before returning.
 * Non-finite logits: a masked slot whose logits hold a NaN or an infinity
 * (a corrupted weight, an overflow) is never filled; its H~ reads as NaN and
 * its argmax as -1 in the debug items, the other slots are decided among
 * themselves (if none is valid, nothing is filled), the step's commit run is
 * committed as usual, and the call returns WEDLM_ERR_NONFINITE (after
 * wedlm_stream_step_async: the next call that reads the device error word). */
wedlm_status wedlm_stream_step(wedlm_ctx* ctx, const wedlm_step_params* params,
                               int32_t* out_committed, int32_t* out_counts, int32_t* out_active);

/* Enqueue `n_steps` decode steps on the context's stream and return without
 * waiting or copying results to the host.  Committed tokens accumulate on the
 * device (read them with wedlm_read_generated).  Slots that finish mid-way
 * stop decoding; their remaining steps are no-ops. */
wedlm_status wedlm_stream_step_async(wedlm_ctx* ctx, const wedlm_step_params* params, int32_t n_steps);

/* Copy every token committed so far after the prompt of `slot` (in position
 * order) to host `out_tokens` (capacity `cap`); *out_len receives the count.
 * Synchronises the stream. */
wedlm_status wedlm_read_generated(wedlm_ctx* ctx, int32_t slot, int32_t* out_tokens, int32_t cap,
                                  int32_t* out_len);

/* Per-slot counters (read from the device; synchronises the stream). */
typedef struct wedlm_seq_stats {
    int64_t steps;          /* decode steps run while active */
    int64_t forward_rows;   /* window rows forwarded by those steps */
    int64_t committed;      /* generated tokens committed */
    int64_t fills;          /* mask slots filled */
    int32_t committed_len;  /* S: prompt + committed tokens */
    int32_t end;            /* prompt_len + max_new_tokens */
    int32_t window;         /* W */
    int32_t active;         /* 1 while S < end */
} wedlm_seq_stats;

/* Copy the counters of `slot` into host `*out` (synchronises the stream).
 * WEDLM_ERR_INVALID_ARG for a slot outside [0, max_batch) or a NULL `out`. */
wedlm_status wedlm_get_stats(wedlm_ctx* ctx, int32_t slot, wedlm_seq_stats* out);

/* Number of kernels this context has launched since creation (each launch
 * counted once; a captured graph counts its kernels at every replay). */
wedlm_status wedlm_kernel_launches(const wedlm_ctx* ctx, int64_t* out);

/* Per-kernel timing.  While enabled, every launch the context makes is
 * bracketed by CUDA events on its stream (which adds a small gap between
 * kernels) and its duration is added to the kind's total.  Kinds: */
#define WEDLM_PROF_PREPARE       0   /* refill + reorder + embed + RMSNorm */
#define WEDLM_PROF_GEMM_QKV      1
#define WEDLM_PROF_QKV_ROPE      2   /* split-K sum + RoPE + K/V into pages */
#define WEDLM_PROF_ATTENTION     3
#define WEDLM_PROF_ATTN_COMBINE  4
#define WEDLM_PROF_GEMM_O        5
#define WEDLM_PROF_RESIDUAL_NORM 6
#define WEDLM_PROF_GEMM_GATE_UP  7
#define WEDLM_PROF_SWIGLU        8
#define WEDLM_PROF_GEMM_DOWN     9
#define WEDLM_PROF_GEMM_LM_HEAD 10
#define WEDLM_PROF_ENTROPY      11
#define WEDLM_PROF_SELECT       12
#define WEDLM_PROF_KINDS        13

/* bf16 GEMM launch shapes.  With autotuning on (the default), the first time a
 * projection kind (WEDLM_PROF_GEMM_*) runs at a given row count the context
 * times each candidate shape (activation rows per tile, K slices) on that
 * projection's weights with a plain store into scratch, on its own stream,
 * and keeps the fastest for the rest of its life; off, a fixed cost model
 * picks the shape.  Results depend on the shape only through fp32
 * accumulation order.  wedlm_autotune clears the recorded shapes. */
wedlm_status wedlm_autotune(wedlm_ctx* ctx, int32_t enable);

/* The shape recorded for (kind, rows): tile_w weight rows (128 or 256) by
 * tile_n activation rows per tile, k_splits slices of K, and the fastest timed
 * launch in microseconds (-1 when the shape came from the cost model).  Any
 * output pointer may be NULL.  WEDLM_ERR_STATE if none is recorded. */
wedlm_status wedlm_gemm_plan(wedlm_ctx* ctx, int32_t kind, int32_t rows, int32_t* tile_w, int32_t* tile_n,
                             int32_t* k_splits, float* us);

/* The schedule of the plan wedlm_gemm_plan reports, as a bit set: 1 CTA-pair
 * tiles, 2 hybrid K split (only the last partial round split), 4 cluster K
 * split (slices reduced through distributed shared memory), 8 K slices
 * reduced by the co-resident slices of a tile (otherwise, when split, by the
 * slice that finishes last), 16 two 128-row weight sub-tiles per CTA, 32
 * 32-deep k-blocks.  WEDLM_ERR_STATE if no plan is recorded. */
wedlm_status wedlm_gemm_schedule(wedlm_ctx* ctx, int32_t kind, int32_t rows, int32_t* schedule);

/* Test hook: record a GEMM launch shape for (kind, rows) as if the autotuner
 * had chosen it, so every epilogue can be checked under every schedule:
 * tile_n activation rows per tile (16..256), k_splits slices of K (1..16) and
 * `schedule` in the bits of wedlm_gemm_schedule (1 CTA pairs, 2 hybrid split,
 * 4 cluster split, 8 co-resident fixup, 16 two weight sub-tiles, 32 32-deep
 * k-blocks) plus 64 = the LM head's fused-entropy epilogue (kind LM_HEAD,
 * k_splits 1).  WEDLM_ERR_INVALID_ARG when the shape cannot be built as asked
 * or its K-split scratch does not fit the context.  Synchronises the stream;
 * the next step runs eagerly. */
wedlm_status wedlm_debug_set_plan(wedlm_ctx* ctx, int32_t kind, int32_t rows, int32_t tile_n, int32_t k_splits,
                                  int32_t schedule);

/* Enable (1) or disable (0) per-kernel timing; enabling clears the totals. */
wedlm_status wedlm_profile_enable(wedlm_ctx* ctx, int32_t on);

/* Synchronise and return the totals: ms[WEDLM_PROF_KINDS] (milliseconds) and
 * launches[WEDLM_PROF_KINDS] (either may be NULL). */
wedlm_status wedlm_profile_read(wedlm_ctx* ctx, double* ms, int64_t* launches);

/* ---------------------------------------------------------------------
 * Test hooks.  They expose intermediate state of the most recent step so the
 * tests can compare each stage with an independent CPU implementation.
 * ------------------------------------------------------------------- */

/* Items readable with wedlm_debug_read.  The last decode step ran `rows` =
 * (1 + highest active slot) * Ws physical rows, Ws = the largest window among
 * active slots; row b * Ws + r is physical row r of slot b. */
#define WEDLM_DBG_PERM     0  /* int32 [rows]: slot offset at each physical row (-1 = padding) */
#define WEDLM_DBG_POS      1  /* int32 [rows]: logical position at each row */
#define WEDLM_DBG_ROWTOK   2  /* int32 [rows]: token fed at each row */
#define WEDLM_DBG_LOGITS   3  /* float [rows][vocab]: unscaled LM-head logits per row */
#define WEDLM_DBG_HTILDE   4  /* float [max_batch][max_window]: H~ per slot offset (NaN if not masked) */
#define WEDLM_DBG_ARGMAX   5  /* int32 [max_batch][max_window]: argmax token per masked slot offset */
#define WEDLM_DBG_FILL     6  /* uint8 [max_batch][max_window]: 1 where the slot was filled this step */
#define WEDLM_DBG_KN       7  /* int32 [max_batch][3]: (k, rows n, filled count) of the step */
#define WEDLM_DBG_ROWSTRIDE 8 /* int32 [2]: (Ws, rows) of the last step */

/* Copy `bytes` of a debug item to host memory.  Synchronises the stream. */
wedlm_status wedlm_debug_read(wedlm_ctx* ctx, int32_t item, void* host_dst, int64_t bytes);

/* Read cached K and V of `slot`, `layer`, positions [pos0, pos0 + n), widened
 * to fp32, into host arrays of [n][n_kv_heads][head_dim] each. */
wedlm_status wedlm_debug_kv(wedlm_ctx* ctx, int32_t slot, int32_t layer, int32_t pos0, int32_t n,
                            float* host_k, float* host_v);

/* Greedy bf16 steps fuse the entropy pass into the LM head: the GEMM's
 * epilogue reduces each 32 vocabulary ids to (max, sum, weighted sum, argmax)
 * partials and logits are never written (sampled steps and fp32 mode keep the
 * two-pass path).  enable = 1 makes every step write logits and run the
 * separate entropy pass, so WEDLM_DBG_LOGITS is valid after greedy bf16 steps
 * too; enable = 2 makes every greedy bf16 step take the fused epilogue
 * (whatever the timing choice at its row count would be); 0 restores the
 * default (test hook; synchronises the stream). */
wedlm_status wedlm_debug_keep_logits(wedlm_ctx* ctx, int32_t enable);

/* Residual-stream capture for per-layer comparisons.  While enabled (1), every
 * decode step keeps x (fp32, the residual stream) entering each layer and
 * after the last one; wedlm_debug_residual copies layer `layer` (0..n_layers,
 * n_layers = after the last layer) for the first `rows` physical rows of the
 * most recent step, [rows][d_model], to host memory.  Enabling allocates
 * (n_layers + 1) * max_batch * max_window * d_model floats on the device and
 * turns CUDA-graph replay off; 0 frees it.  Both synchronise the stream. */
wedlm_status wedlm_debug_capture(wedlm_ctx* ctx, int32_t enable);
wedlm_status wedlm_debug_residual(wedlm_ctx* ctx, int32_t layer, float* host_dst, int32_t rows);

/* Read / replace a slot's window (host arrays of `n` entries; replacing is
 * used to drive both implementations from the same state). */
wedlm_status wedlm_debug_get_window(wedlm_ctx* ctx, int32_t slot, uint8_t* filled, int32_t* tokens,
                                    int32_t cap, int32_t* n);
wedlm_status wedlm_debug_set_window(wedlm_ctx* ctx, int32_t slot, const uint8_t* filled,
                                    const int32_t* tokens, int32_t n);

/* Copy the first `bytes` of a weight tensor's device storage to host memory,
 * as stored: WQ / WK / WV read the layer's fused [(hq + 2 hkv) * hd][d] block
 * and WG / WU the fused [2 ffn][d] block, in the row order the bf16 epilogues
 * use (RoPE partners / gate-up pairs in adjacent rows); other tensors as
 * loaded.  Synchronises the stream. */
wedlm_status wedlm_debug_read_weight(wedlm_ctx* ctx, int32_t tensor, int32_t layer, void* host_dst, int64_t bytes);

/* Fault injection on the host side: overwrite entry `index` of slot `slot`'s
 * device page table with `page`, unchecked (a value outside [0, num_pages)
 * makes the kernels' own bounds checks fire: the step skips those accesses
 * and returns WEDLM_ERR_DEVICE_ASSERT).  *old_page receives the previous
 * entry (may be NULL).  Synchronises the stream. */
wedlm_status wedlm_debug_set_page(wedlm_ctx* ctx, int32_t slot, int32_t index, int32_t page, int32_t* old_page);

/* Stand-alone launches of single stages on caller-provided DEVICE buffers
 * (no context; the caller owns all memory; stream may be NULL).
 *
 * Topological reordering (summary, section Method): for each of n_seq windows
 * of n[b] <= stride slots with flags filled[b*stride + j] (1 = filled):
 *   k[b]    = length of the leftmost run of filled slots,
 *   nf[b]   = number of filled slots,
 *   perm[b*stride + r] = slot offset at physical row r (filled slots in
 *             ascending order, then masks in ascending order; rows >= n[b]
 *             get -1),
 *   pos[b*stride + r]  = S[b] + perm (logical position; -1 past n[b]).
 * Bit-exact integer work. */
wedlm_status wedlm_reorder_window(const uint8_t* filled, const int32_t* n, const int32_t* S,
                                  int32_t n_seq, int32_t stride,
                                  int32_t* perm, int32_t* pos, int32_t* k, int32_t* nf, void* stream);

/* Distance-penalised entropy selection (summary, section Method; review,
 * Weaknesses: the functional form is not printed, read here as
 * H~ = H + lambda * offset).  For each of n_seq windows of n[b] <= stride slots:
 * logits[(b*stride + j) * vocab + v] (fp32, unscaled) are the logits of slot j;
 * only slots with filled == 0 are read.  For each such slot:
 *   H_j = entropy (nats) of softmax(logit_scale * logits) over ids != mask_id,
 *   argmax_j = lowest id attaining the max (never mask_id),
 *   htilde[b*stride+j] = H_j + lambda * j  (NaN for filled slots or j >= n[b]).
 * fill[b*stride+j] = 1 for slots chosen by the threshold / argmin rule, else 0;
 * argmax[b*stride+j] = argmax_j (or -1).  Device buffers, caller-owned.
 * A masked slot whose logits hold a NaN or an infinity is invalid: htilde NaN,
 * argmax -1, fill 0; the window's other slots are decided among themselves
 * (none valid: nothing filled) and the call returns WEDLM_ERR_NONFINITE with
 * every output written.  Synchronous; takes its scratch from cudaMallocAsync
 * on `stream`. */
wedlm_status wedlm_entropy_select(const float* logits, int32_t vocab, int32_t mask_id,
                                  const uint8_t* filled, const int32_t* n, int32_t n_seq, int32_t stride,
                                  const wedlm_step_params* params,
                                  float* htilde, int32_t* argmax, uint8_t* fill, void* stream);

/* Allocation-free wedlm_entropy_select.  (Not a step of the method: the
 * paper has no counterpart.)  It exists for callers that must not allocate
 * device memory: for example a runtime that has already reserved the device
 * for its own memory pool, where any further allocation fails or fragments
 * that pool, or a thread that must not take the allocator's locks or risk
 * the device-wide synchronisation an allocation may cause.  Same arguments,
 * outputs and device-pointer rules as wedlm_entropy_select; it allocates
 * nothing.  Like wedlm_entropy_select it is synchronous: it waits for
 * `stream` (only that stream, nothing device-wide) before returning.
 *
 * Its scratch is a fixed array inside the library image (about 1 MiB: room
 * for WEDLM_NOALLOC_MAX_ROWS rows), present on every GPU that loads the
 * library until the process exits.
 *   - n_seq * stride must be <= WEDLM_NOALLOC_MAX_ROWS; larger requests
 *     return WEDLM_ERR_INVALID_ARG without launching anything.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address once and keeps it for the life of the process;
 *     make that first call before any stream capture.  cudaDeviceReset
 *     destroys the context that address belongs to: after a reset in the
 *     same process, do not call this function again on that device.
 *   - Every call on a device shares the one array, and it keeps the previous
 *     call's contents (each call rewrites what it reads).  Calls whose work
 *     overlaps on the GPU (different streams or host threads without ordering
 *     between them) race on it and must be serialised by the caller. */
#define WEDLM_NOALLOC_MAX_ROWS 4096
/* (Non-finite logits: as for wedlm_entropy_select, WEDLM_ERR_NONFINITE.) */
wedlm_status wedlm_entropy_select_noalloc(const float* logits, int32_t vocab, int32_t mask_id,
                                          const uint8_t* filled, const int32_t* n, int32_t n_seq, int32_t stride,
                                          const wedlm_step_params* params,
                                          float* htilde, int32_t* argmax, uint8_t* fill, void* stream);

/* wedlm_entropy_select on caller-provided scratch, asynchronously: the call
 * enqueues its kernels on `stream` and returns; the outputs are valid once the
 * stream has been synchronised.  workspace: DEVICE memory, 256-byte aligned,
 * at least wedlm_entropy_select_workspace_bytes(n_seq, stride) bytes; its first
 * int32 is the call's device error word (cleared by the call itself; 3 = a
 * masked slot's logits held a NaN or an infinity, the slot treated as in
 * wedlm_entropy_select).  Nothing else in it needs initialising. */
wedlm_status wedlm_entropy_select_workspace_bytes(int32_t n_seq, int32_t stride, int64_t* bytes);
wedlm_status wedlm_entropy_select_async(const float* logits, int32_t vocab, int32_t mask_id,
                                        const uint8_t* filled, const int32_t* n, int32_t n_seq, int32_t stride,
                                        const wedlm_step_params* params, float* htilde, int32_t* argmax,
                                        uint8_t* fill, void* workspace, int64_t workspace_bytes, void* stream);

/* Reordered-causal GQA attention of window rows against a paged KV cache, on
 * the bf16 tensor-core path (summary, section Method: after Topological
 * Reordering the window runs a plain causal forward conditioned on the
 * persistent KV cache).  This is the kernel the decode step runs per layer.
 * All pointers are DEVICE memory owned by the caller, 256-byte aligned.
 *   q          bf16 [n_seq * stride][n_heads][128]: query rows after RoPE;
 *              row b * stride + r is physical window row r of sequence b.
 *   kv_pool    bf16 [num_pages][2 (K, V)][n_kv_heads][16 tokens][128]: one
 *              layer's page pool (K and V after RoPE for K).
 *   page_table int32 [n_seq][pages_per_seq]: page of each 16-token block.
 *   S, n       int32 [n_seq]: committed length and window rows of sequence b.
 *              Window row r's own K/V must already sit at cache position
 *              S[b] + r (the decode step's QKV epilogue writes them there).
 *   out        bf16 [n_seq * stride][n_heads][128]: softmax(q K^T / sqrt(128)) V
 *              of each row r < n[b] over cache positions 0 .. S[b] + r (rows
 *              r >= n[b] are not written).
 * max_ctx bounds S[b] + n[b] (it sizes the key chunks and the workspace);
 * n_heads % n_kv_heads == 0; stride <= 1024.
 * workspace: at least wedlm_attention_workspace_bytes(...) bytes; its first
 * int32 is a device error word (1: a page id outside [0, num_pages) or more
 * keys than max_ctx allows; 2: a bounded wait gave up), the rest holds the
 * key chunks' partial results.  The error word must be zero before a call
 * (zeroing the whole workspace once, e.g. with cudaMemsetAsync, is enough;
 * calls leave it as they found it while no error occurs).  Asynchronous: the
 * call enqueues the attention kernel (and, when a window's keys are split
 * into chunks, the kernel that combines them) on `stream` and returns; out
 * and the error word are valid once the stream has been synchronised.
 * WEDLM_ERR_INVALID_ARG for bad sizes, pointers or a too small workspace,
 * WEDLM_ERR_CUDA if the launch fails. */
wedlm_status wedlm_attention_workspace_bytes(int32_t n_seq, int32_t stride, int32_t n_heads, int32_t n_kv_heads,
                                             int32_t max_ctx, int64_t* bytes);
wedlm_status wedlm_attention_bf16(const void* q, const void* kv_pool, int32_t num_pages, int32_t n_heads,
                                  int32_t n_kv_heads, const int32_t* page_table, int32_t pages_per_seq,
                                  const int32_t* S, const int32_t* n, int32_t n_seq, int32_t stride,
                                  int32_t max_ctx, void* out, void* workspace, int64_t workspace_bytes,
                                  void* stream);

/* Dense projection on the bf16 tensor-core path: Y = X * W^T with X bf16
 * [M][K], W bf16 [N][K] (nn.Linear layout), Y fp32 [M][N], all DEVICE
 * pointers owned by the caller (16-byte aligned; K % 8 == 0).  This is the
 * kernel every QKV, O, gate/up, down and LM-head projection of the step runs
 * (split-K partial planes are summed before returning). */
wedlm_status wedlm_linear_bf16(const void* X, const void* W, float* Y, int32_t M, int32_t N, int32_t K,
                               void* stream);

/* wedlm_linear_bf16 with the launch shape pinned (tuning and test hook):
 * tile_n in {16, 32, 64, 128, 256} activation rows per tile (0 = automatic) and
 * k_splits in [1, 16] slices of K (0 = automatic; rounded to what K allows and
 * forced to 1 when N % 4 != 0).  Results agree with the automatic plan to fp32
 * accumulation order. */
wedlm_status wedlm_linear_bf16_plan(const void* X, const void* W, float* Y, int32_t M, int32_t N, int32_t K,
                                    int32_t tile_n, int32_t k_splits, void* stream);

/* wedlm_linear_bf16_plan with the schedule pinned as well; `schedule` is a bit
 * set (other bits: WEDLM_ERR_INVALID_ARG):
 *   1  CTA-pair tiles: two CTAs of a cluster compute a tile of 256 weight rows
 *      by tile_n activation rows with the two-CTA tensor-core MMA, each staging
 *      its own 128 weight rows and half of the activation rows; tile_n must be
 *      128 or 256 (WEDLM_ERR_INVALID_ARG otherwise);
 *   2  hybrid K split: the tiles that fill whole rounds of the persistent grid
 *      run over all of K, only the tiles of the last partial round are cut into
 *      k_splits slices (k_splits > 1), reduced by the slice that finishes last;
 *   4  cluster K split: the k_splits (2..4) slices of a tile are the CTAs of
 *      one thread-block cluster, one tile slice per CTA, and are reduced through
 *      distributed shared memory (not combinable with 1 or 2; tile_n 128 or 256;
 *      N % 4 == 0).
 * Results agree with wedlm_linear_bf16 to fp32 accumulation order. */
wedlm_status wedlm_linear_bf16_sched(const void* X, const void* W, float* Y, int32_t M, int32_t N, int32_t K,
                                     int32_t tile_n, int32_t k_splits, int32_t schedule, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* WEDLM_H */
