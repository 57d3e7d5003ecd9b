/*
 * flashcache.h — C ABI of the B200 (sm_100a) Flash-Cache step.
 *
 * One Flash-Cache step (Flash-dLLM; paper-digest page, Fig. 2 caption, and the
 * infernews post "Flash-dLLM: IO-aware KV caching and parallel decoding",
 * Flash-Cache paragraph): every sequence b of a batch brings a query of n_b
 * positions (the tracked positions plus the current masked window).  The step
 *   1. projects the query rows x_r to q, k, v with W_qkv (no bias),
 *   2. rotates q and k by RoPE at the rows' absolute positions,
 *   3. writes k and v into the sequence's KV cache at those positions,
 *   4. lets the query attend bidirectionally to the sequence's whole cache,
 *   5. sums the attention probabilities of every key over heads and query rows
 *      ("attention importance"),
 * and a separate call (fc_topk_tracked) reselects, per sequence, the k
 * candidate positions of highest importance as the next tracked set.
 *
 * Readings where the pages say nothing (the library follows them exactly):
 *   - RoPE pairs element i with i + d/2 (rotate-half), angle pos*theta^(-2i/d);
 *   - scores are q.k/sqrt(d); no biases; K/V heads = Q heads;
 *   - the cache rows are written before attending, so the query sees its own
 *     fresh K/V; every cache row of the sequence is attended (no mask);
 *   - importance of key j = sum over heads and query rows of P[row, j];
 *   - reselection ranks candidates by importance descending, then position
 *     ascending.
 *
 * Conventions for every entry point:
 *   - Pointers marked "dev" are CUDA device pointers on the handle's device;
 *     pointers marked "host" are host memory.  The caller owns all of them and
 *     keeps them alive until the work queued on the stream has finished.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Calls only enqueue work; none synchronises, except
 *     fc_get_error.
 *   - Integers are int32, floats IEEE binary32, bf16 values are raw 16-bit
 *     bfloat16 patterns.  Every array is dense, row-major, without padding.
 *   - A non-FC_OK status means nothing was enqueued, except FC_ERR_CUDA from a
 *     launch, after which the stream's state is whatever CUDA reports.
 *   - Problems only the device can see (a position outside its sequence, the
 *     same position twice in one sequence, inconsistent cu_seqlens, a bad
 *     candidate range, a barrier that timed out) set bits of a sticky device
 *     error word, read and cleared by fc_get_error.  The offending rows or
 *     sequences are skipped, no memory outside the documented arrays is
 *     touched, and the step's results are then undefined.
 */
#ifndef FLASHCACHE_H
#define FLASHCACHE_H

#include <stdint.h>

#if defined(__GNUC__)
#define FC_API __attribute__((visibility("default")))
#else
#define FC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fc_status {
  FC_OK = 0,
  FC_ERR_INVALID_ARG = -1,   /* a host-visible argument is wrong; nothing ran     */
  FC_ERR_UNSUPPORTED = -2,   /* valid request outside what this build supports    */
  FC_ERR_CUDA = -3,          /* a CUDA runtime/driver call failed                  */
  FC_ERR_OOM = -4,           /* device allocation of the workspace failed          */
  FC_ERR_DEVICE_CHECK = -5,  /* fc_get_error: the device error word is non-zero    */
  FC_ERR_TIMEOUT = -6        /* fc_get_error: a kernel gave up on a barrier wait   */
} fc_status;

/* Element type of x, W_qkv, the KV cache and `out`. */
enum { FC_DTYPE_BF16 = 0, FC_DTYPE_FP32 = 1 };

/* Bits of the device error word (fc_get_error). */
#define FC_DEVERR_POS_RANGE 0x01 /* q_pos[r] < 0 or >= its sequence's cache length */
#define FC_DEVERR_POS_DUP 0x02   /* a position appears twice in one sequence       */
#define FC_DEVERR_SEQLENS 0x04   /* cu_seqlens not monotone / totals disagree, or a
                                    sequence longer than the configured limits      */
#define FC_DEVERR_CAND 0x08      /* cand_lo/cand_hi/k_per_seq outside their ranges  */
#define FC_DEVERR_TIMEOUT 0x10   /* a kernel abandoned a bounded barrier wait       */

/* Model dimensions and capacity limits, fixed at fc_create. */
typedef struct fc_config {
  int hidden;        /* D: width of a query row x_r                                */
  int n_heads;       /* H: attention heads (K/V heads are the same H)             */
  int head_dim;      /* d: even; 128 selects the tensor-core path for bf16        */
  double rope_theta; /* RoPE base theta (> 1)                                     */
  int dtype;         /* FC_DTYPE_BF16 or FC_DTYPE_FP32                            */
  int max_batch;     /* largest B a step may pass (<= 4096)                       */
  int max_total_q;   /* largest T = sum n_b                                       */
  int max_total_k;   /* largest S = sum L_b                                       */
  int max_seqlen_q;  /* largest n_b                                               */
  int max_pos;       /* largest cache length L_b (L_b <= max_pos <= 262144)       */
  int max_topk;      /* largest k of fc_topk_tracked (<= 1024)                    */
} fc_config;

typedef struct fc_handle fc_handle;

/*
 * fc_create — validate `cfg`, bind the projection weights and allocate the
 * handle's workspace on the current CUDA device.
 *   cfg    host; copied.
 *   w_qkv  dev, [3*H*d, D] of cfg->dtype, row-major (each output row is K-major,
 *          i.e. contiguous along D).  Rows 0..H*d-1 are the Q heads, then the K
 *          heads, then the V heads; head h occupies rows h*d..h*d+d-1 of its
 *          block.  Kept by pointer: the caller keeps it alive and unchanged
 *          until fc_destroy.  16-byte aligned.
 *   out    host; receives the handle.
 * Returns FC_ERR_INVALID_ARG for a NULL pointer or an inconsistent config,
 * FC_ERR_UNSUPPORTED for a config this build cannot run, FC_ERR_OOM /
 * FC_ERR_CUDA if the workspace cannot be set up (no device, out of memory).
 * Synchronous (it uploads the RoPE table).
 */
FC_API fc_status fc_create(const fc_config* cfg, const void* w_qkv, fc_handle** out);

/*
 * fc_step — one Flash-Cache step on a packed, variable-length batch.
 *   batch         B >= 1, <= max_batch.
 *   x             dev, [T, D] of dtype: query rows of all sequences, sequence
 *                 b in rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1.
 *   q_pos         dev, int32 [T]: absolute position of every query row inside
 *                 its sequence, 0 <= q_pos[r] < L_b, distinct within a sequence.
 *   cu_seqlens_q  dev, int32 [B+1]: 0 = cu[0] <= cu[1] <= ... <= cu[B] = T.
 *   cu_seqlens_k  dev, int32 [B+1]: the same over cache rows, cu[B] = S;
 *                 L_b = cu_seqlens_k[b+1] - cu_seqlens_k[b] <= max_pos.
 *   total_q       T (host int), <= max_total_q.  With T = 0 nothing is
 *                 written except `importance` (zeroed when accumulate = 0).
 *   total_k       S (host int), <= max_total_k.
 *   k_cache       dev, [S, H, d] of dtype, updated in place: row
 *   v_cache       cu_seqlens_k[b] + q_pos[r] receives the rotated k (resp. v)
 *                 of query row r, rounded to nearest-even in dtype.  All other
 *                 rows are only read.  16-byte aligned.
 *   out           dev, [T, H, d] of dtype: attention output of every query row.
 *   importance    dev, float [S] or NULL (then not computed).  Per key j of
 *                 sequence b: sum over heads and query rows of b of the
 *                 normalised attention probability of j.  With accumulate = 0
 *                 it is overwritten, with accumulate = 1 the step's values are
 *                 added to what it holds (e.g. to sum over layers).
 * Host-detectable errors return FC_ERR_INVALID_ARG before anything is queued.
 * The same handle must not run two steps concurrently on different streams
 * (they share the workspace); consecutive calls on one stream are fine.
 */
FC_API fc_status fc_step(fc_handle* h, void* stream, int batch, const void* x, const int32_t* q_pos,
                  const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int total_q,
                  int total_k, void* k_cache, void* v_cache, void* out, float* importance,
                  int accumulate);

/*
 * fc_topk_tracked — reselect the tracked positions of every sequence.
 *   total_k       S (host int): length of `importance`, <= max_total_k.
 *   importance    dev, float [S] as written by fc_step.
 *   cu_seqlens_k  dev, int32 [B+1] (as for fc_step); a sequence whose range
 *                 leaves [0, S) sets FC_DEVERR_CAND and gets a row of -1.
 *   cand_lo/hi    dev, int32 [B]: sequence b's candidates are the positions
 *                 cand_lo[b] <= j < cand_hi[b] (0 <= lo <= hi <= L_b), normally
 *                 its decoded positions.
 *   k_per_seq     dev, int32 [B] or NULL: number kept for sequence b
 *                 (0 <= k_b <= k); NULL keeps k for every sequence.
 *   k             row width of `tracked`, 0 <= k <= max_topk.
 *   tracked       dev, int32 [B, k]: row b lists the kept positions ordered by
 *                 importance descending, equal scores by position ascending;
 *                 entries past min(k_b, number of candidates) are -1.
 * Exact and deterministic: the same inputs give the same output bits.
 */
FC_API fc_status fc_topk_tracked(fc_handle* h, void* stream, int batch, int total_k,
                          const float* importance,
                          const int32_t* cu_seqlens_k, const int32_t* cand_lo,
                          const int32_t* cand_hi, const int32_t* k_per_seq, int k,
                          int32_t* tracked);

/*
 * fc_step_host — fc_step followed by fc_topk_tracked with the per-step inputs
 * and outputs in host memory: the serving form of a step, in which the
 * weights and the KV cache stay resident on the device, a step's query rows,
 * positions and lengths come in and its attention output and tracked
 * positions go out.
 *   x, q_pos, cu_seqlens_q, cu_seqlens_k, total_q, total_k
 *                 as for fc_step, but x, q_pos and both cu_seqlens in HOST
 *                 memory.
 *   k_cache, v_cache  dev, as for fc_step (updated in place).
 *   cand_lo, cand_hi, k_per_seq (or NULL), k
 *                 as for fc_topk_tracked, arrays in HOST memory.
 *   out           HOST, [T, H, d] of dtype.
 *   tracked       HOST, int32 [B, k] (may be NULL when k = 0).
 * The importance of the step is computed into a handle-owned device buffer
 * (fc_step gives access to it).
 * The call returns once the work is queued; it does not wait for the GPU.
 * Two handle-owned copy streams and two sets of device staging buffers let
 * the input copy of one call and the output copy of the previous call run
 * while the kernels of the current call run on `stream`.  q_pos, the two
 * cu_seqlens, cand_lo, cand_hi and k_per_seq are read during the call
 * (gathered into a handle-owned pinned block that is copied as one; the call
 * waits on the host if that block's copy from two calls earlier is still
 * running); x must stay unchanged, and out / tracked must not be read, until
 * the caller has called fc_host_sync(h, stream) and `stream` has reached that
 * point (e.g. cudaStreamSynchronize).  Page-locked host memory makes the copies
 * asynchronous; pageable memory is accepted but serialises the copies with
 * the host.  The first call allocates the staging buffers (two copies of x,
 * the small arrays, out and tracked, sized from the config) and the copy
 * streams; FC_ERR_OOM / FC_ERR_CUDA if that fails.  Argument errors return
 * FC_ERR_INVALID_ARG before anything is queued.  One handle: one stream.
 */
FC_API fc_status fc_step_host(fc_handle* h, void* stream, int batch, const void* x,
                              const int32_t* q_pos, const int32_t* cu_seqlens_q,
                              const int32_t* cu_seqlens_k, int total_q, int total_k,
                              void* k_cache, void* v_cache, const int32_t* cand_lo,
                              const int32_t* cand_hi, const int32_t* k_per_seq, int k, void* out,
                              int32_t* tracked);

/*
 * fc_host_sync — make `stream` wait (on the device, without blocking the
 * host) until every copy queued by earlier fc_step_host calls has completed.
 * After cudaStreamSynchronize(stream) the host outputs of all those calls are
 * complete and their host inputs are no longer read.
 */
FC_API fc_status fc_host_sync(fc_handle* h, void* stream);

/*
 * fc_get_error — wait for the stream of the handle's last call, copy the
 * device error word to *device_error_word (host) and clear it.
 * Returns FC_OK when the word was 0, FC_ERR_TIMEOUT when it holds
 * FC_DEVERR_TIMEOUT, otherwise FC_ERR_DEVICE_CHECK; FC_ERR_CUDA if the wait
 * or the copy failed.
 */
FC_API fc_status fc_get_error(fc_handle* h, int32_t* device_error_word);

/*
 * fc_selftest_wait_timeout — exercise the failure path of the bounded barrier
 * waits.  Enqueues one CTA that waits on an mbarrier nothing arrives at, using
 * the same bounded wait as the tensor-core kernels but a limit of `limit_us`
 * microseconds (1 .. 2,000,000).  When the limit passes it sets
 * FC_DEVERR_TIMEOUT in the handle's error word and returns; fc_get_error then
 * reports FC_ERR_TIMEOUT and the CUDA context remains usable.
 */
FC_API fc_status fc_selftest_wait_timeout(fc_handle* h, void* stream, int limit_us);

/*
 * fc_last_step_work — how the attention work of the handle's last fc_step was
 * split (waits for the stream of the last call):
 *   items           work items, one per (sequence, head, query tile), or, in
 *                   a small-batch step split over the SMs (FC_OPT_ATTN_SPLIT),
 *                   one per work entry (an item's run of key tiles);
 *   two_pass_items  items given to the two-pass attention kernel from the
 *                   start: all of them when the step asked for importance (it
 *                   needs every row's final normaliser before the column sums,
 *                   so that kernel scans K twice) or was split, none otherwise
 *                   (bf16 tensor-core path; 0 on the CUDA-core path);
 *   handed_over     items of a step without importance that the one-pass
 *                   kernel handed to the two-pass kernel because a score
 *                   exceeded its row's reference (the maximum over the item's
 *                   first key tile) by more than 64 in log2 units.
 * Host pointers.  For tests and measurement tools.
 */
FC_API fc_status fc_last_step_work(fc_handle* h, int32_t* items, int32_t* two_pass_items,
                                   int32_t* handed_over);

/*
 * fc_last_cuda_error — text of the last CUDA failure behind an FC_ERR_CUDA of
 * fc_step on this handle: the kernel being launched and CUDA's error name and
 * string ("no CUDA error recorded" if none).  The pointer stays valid until
 * the calling thread's next call.
 */
FC_API const char* fc_last_cuda_error(const fc_handle* h);

/*
 * fc_set_option — select among equivalent implementations (results agree
 * within the parity bar; for tests and measurement).
 *   FC_OPT_QKV_KERNEL: the projection kernel of the bf16 tensor-core path:
 *     0 (default) and 1: the CTA-pair kernel (256-row tiles, the whole
 *       reduction per pair); 2: the split-K kernel (128-row tiles, the
 *       reduction split over a thread-block cluster).  The split-K kernel
 *       was measured no faster than the pair kernel on any shape tried, so
 *       the default does not choose it.
 *   FC_OPT_QKV_SPLIT: CTAs per cluster of the split-K kernel, 1..8, or 0
 *     (default) to choose by occupancy.  The reduction over the hidden size is
 *     cut into that many nearly equal runs of 64-wide steps; a value above
 *     hidden / 64 leaves some CTAs without a step and is rejected at fc_step
 *     with FC_ERR_INVALID_ARG.
 *   FC_OPT_ATTN_SPLIT: small-batch attention on the tensor-core path.  0
 *     (default): when H * (ceil(total_q / 128) + batch - 1) is at most the
 *     SM count and either the step has no importance or the caches hold 1280
 *     rows or more on average (total_k >= 1280 * batch), every (sequence,
 *     head, 128-row query tile)
 *     item is split into min(SMs / items, 8, its 128-key tiles) entries (at
 *     least one) over runs of key tiles; a first launch stores each entry's row
 *     maxima and normalisers, a second combines them into the rows'
 *     log-sum-exp, computes P, P V and the column sums over its own keys, and
 *     the item's last entry adds the parts of O in entry order (so results do
 *     not depend on timing).  1: never split.  2: split whenever the batch is
 *     small enough, whatever the cache length (for tests and measurement).
 * FC_ERR_INVALID_ARG for an unknown option or value.
 */
#define FC_OPT_QKV_KERNEL 1
#define FC_OPT_QKV_SPLIT 2
#define FC_OPT_ATTN_SPLIT 3
FC_API fc_status fc_set_option(fc_handle* h, int option, int value);

/*
 * fc_qkv_plan — the projection kernel fc_step launches for total_q query rows
 * under the current options (host only, no GPU work).
 *   *kernel: 0 the CUDA-core path (shapes outside the tensor-core kernels),
 *            1 the CTA-pair kernel (256-row tiles, whole reduction per pair),
 *            2 the split-K kernel (128-row tiles, the reduction split over a
 *              thread-block cluster of *split CTAs, partial sums added through
 *              distributed shared memory).
 *   *split: CTAs per cluster for kernel 2, else 0.
 *   *max_clusters (may be NULL): clusters of that size the GPU holds at once
 *     (when the plan is not kernel 2: of the largest split it considered);
 *     a negative value is the CUDA error code of the occupancy query, negated.
 * With kernel 2 forced and no split forced, the split is the largest (at most
 * 8 and hidden / 64) whose clusters all fit on the GPU at once.
 * FC_ERR_INVALID_ARG for a null handle or output, total_q < 0.
 */
FC_API fc_status fc_qkv_plan(const fc_handle* h, int total_q, int* kernel, int* split,
                             int* max_clusters);

/* Number of kernels the last fc_step / fc_topk_tracked call enqueued (host). */
FC_API int fc_last_launch_count(const fc_handle* h);

/*
 * Per-kernel timing for measurement tools.  fc_profile(h, 1) makes every later
 * fc_step / fc_topk_tracked / fc_step_host record a CUDA event pair on its
 * stream around each kernel it launches, and fc_step_host also around its
 * input copies and its output copies on its copy streams (up to 4096 records);
 * fc_profile(h, 0) stops recording.
 * fc_profile_read waits for the recorded work, writes for each slot
 * (0 prep, 1 qkv_rope_scatter, 2 attention (the two-pass attention kernel
 * of the tensor-core path: every item of a step with importance, the items
 * handed over in a step without; in a small-batch step whose items are split
 * over the SMs, its second launch: pass 2 and the combine of the parts),
 * 3 importance_finalize, 4 topk, 5 attention_one_pass (the one-pass kernel of
 * a tensor-core step without importance), 6 h2d_copy and 7 d2h_copy (the copy
 * blocks of fc_step_host), 8 attention_split_pass1 (the first launch of a
 * split small-batch step: every entry's row statistics))
 * the summed milliseconds to ms[slot] and the record count to launches[slot]
 * (host arrays of FC_PROFILE_SLOTS entries), and clears the records.
 * fc_profile_timeline (call it before fc_profile_read) waits for the recorded
 * work and writes, for the first min(max_records, count) records in recording
 * order, the slot and the start and end times in milliseconds after the first
 * record's start (host arrays); *n receives the number written.
 */
#define FC_PROFILE_SLOTS 9
FC_API fc_status fc_profile(fc_handle* h, int enable);
FC_API fc_status fc_profile_timeline(fc_handle* h, int max_records, int32_t* slot, float* start_ms,
                                     float* end_ms, int* n);
FC_API fc_status fc_profile_read(fc_handle* h, float* ms, int* launches);

/*
 * fc_attention_noalloc — attention and importance without any device
 * allocation.  The paper has no counterpart to this entry point: it exists for
 * callers that cannot call cudaMalloc (a runtime or host application that owns
 * all device memory, a plug-in running inside another process's context, a
 * pool handed over to a caching allocator) and so cannot create a handle,
 * whose workspace fc_create allocates.
 *
 * For query rows that are already projected and rotated, it computes what
 * fc_step computes after its projection: out[r] = softmax(q_r K_b^T/sqrt(d)) V_b
 * over every row of sequence b's cache, and importance[j] = sum over heads and
 * query rows of the probability of key j (overwritten, no accumulate).
 *   dtype          FC_DTYPE_BF16 or FC_DTYPE_FP32 (q, caches and out)
 *   q              dev, [T, H, d]: rotated queries, not scaled
 *   cu_seqlens_q/k dev, int32 [B+1], as for fc_step (sequences with ranges
 *                  outside [0, T) / [0, S) are skipped)
 *   k_cache, v_cache dev, [S, H, d], only read
 *   out            dev, [T, H, d];  importance  dev, float [S].  Rows of a
 *                  sequence whose cache is empty (L_b = 0) get zeros: they
 *                  have no key to attend.
 * Limits: S <= FC_NOALLOC_MAX_KEYS, d <= 256, B and H <= 65535, and
 * H * T < 2^23 (a key's importance, at most H * T, is summed in signed 2^-40
 * fixed point); larger sizes return FC_ERR_UNSUPPORTED before anything is
 * queued.
 * Its scratch (a fixed-point accumulator of FC_NOALLOC_MAX_KEYS + 32 int64,
 * 512 KiB) is a static array in the library's device image: every GPU that
 * loads the library holds it until the process exits, and every call shares
 * it.  Each call clears the part it uses on `stream` first; calls whose work
 * overlaps on the GPU (two streams, or two threads) race on it.  The first
 * call in a CUDA context looks up the array's device address in that context
 * (once per context: the device's primary context, or each context the
 * caller makes current); make that first call before any stream capture.  Do
 * not keep using the library in a process across cudaDeviceReset.
 */
#define FC_NOALLOC_MAX_KEYS 65536
FC_API fc_status fc_attention_noalloc(void* stream, int dtype, int batch, int n_heads,
                                      int head_dim, const void* q, const int32_t* cu_seqlens_q,
                                      const int32_t* cu_seqlens_k, int total_q, int total_k,
                                      const void* k_cache, const void* v_cache, void* out,
                                      float* importance);

/* Release the workspace and the handle (NULL is a no-op).  Waits for all work
 * on the handle's device first (cudaDeviceSynchronize). */
FC_API void fc_destroy(fc_handle* h);

/* ==========================================================================
 * Model step: the decoder stack around the Flash-Cache layer.
 *
 * The Flash-dLLM pages evaluate LLaDA-8B (paper-digest page, evaluation;
 * forum post, configuration table).  One model step runs the query rows of
 * every sequence (tracked positions + masked window) through n_layers
 * LLaMA-style decoder layers, each attending through the Flash-Cache step of
 * fc_step (its own K/V cache per layer), then scores the rows the caller names
 * with the LM head: per row the top token, its softmax probability (the
 * confidence) and the Flash-Verify acceptance confidence >= threshold
 * (paper-digest page, Flash-Verify; threshold 0.9 in the configuration).
 * Layer (no biases; rms_norm(x) = x / sqrt(mean(x^2) + eps)):
 *   h += Wo . attn(rms_norm(h) * g_attn)
 *   h += Wd . (silu(Wg . m) * (Wu . m)),  m = rms_norm(h) * g_mlp
 * and the LM head reads rms_norm(h) * g_final.  Every activation between
 * kernels is bf16; each kernel accumulates in fp32.
 * ========================================================================== */
typedef struct fc_model_config {
  fc_config layer;      /* attention layer: dtype FC_DTYPE_BF16, head_dim 128,
                           n_heads even, hidden a multiple of 256; the max_*
                           limits bound every step as for fc_create */
  int n_layers;         /* >= 1 */
  int intermediate;     /* SwiGLU width I, a multiple of 128 */
  int vocab;            /* V >= 1 */
  int max_head_rows;    /* rows the LM head may score per step, >= 1 */
  float rms_eps;        /* e.g. 1e-5 */
  float threshold;      /* acceptance threshold on the confidence, e.g. 0.9 */
} fc_model_config;

/* One decoder layer's weights: device pointers, bf16, row-major, 16-byte
 * aligned, kept by pointer until fc_model_destroy. */
typedef struct fc_layer_weights {
  const void* attn_norm;  /* [D] */
  const void* w_qkv;      /* [3*H*d, D], as for fc_create */
  const void* w_o;        /* [D, H*d] */
  const void* mlp_norm;   /* [D] */
  const void* w_gate;     /* [I, D] */
  const void* w_up;       /* [I, D] */
  const void* w_down;     /* [D, I] */
} fc_layer_weights;

typedef struct fc_model fc_model;

/*
 * fc_model_create — validate `cfg`, bind the weights (`layers`: host array of
 * n_layers entries; final_norm dev [D]; lm_head dev [V, D]) and allocate the
 * workspace (one Flash-Cache handle for the attention of every layer, the
 * bf16 activations h, a [max_total_q, D], o [max_total_q, H*d],
 * s [max_total_q, I], the LM-head rows [max_head_rows, D] and statistics).
 * FC_ERR_UNSUPPORTED for shapes outside the tensor-core path,
 * FC_ERR_INVALID_ARG for NULL or misaligned pointers, FC_ERR_OOM / FC_ERR_CUDA.
 */
FC_API fc_status fc_model_create(const fc_model_config* cfg, const fc_layer_weights* layers,
                                 const void* final_norm, const void* lm_head, fc_model** out);

/*
 * fc_model_step — one model step on a packed, variable-length batch.
 *   batch, q_pos, cu_seqlens_q, cu_seqlens_k, total_q (>= 1), total_k
 *                 as for fc_step (dev).
 *   x             dev, [T, D] bf16: the input embeddings of the query rows.
 *   k_caches, v_caches  host arrays of n_layers dev pointers, [S, H, d] bf16
 *                 each, updated in place as by fc_step for every layer.
 *   head_rows     dev, int32 [n_head_rows]: packed query rows (0 <= r < T) the
 *                 LM head scores; n_head_rows 0 skips the head.
 *   importance    dev, float [S] or NULL: the attention importance summed over
 *                 every layer (overwritten).
 *   token         dev, int32 [n_head_rows]: index of the largest logit (the
 *                 lowest index on ties).
 *   confidence    dev, float [n_head_rows]: its softmax probability.
 *   accept        dev, uint8 [n_head_rows]: confidence >= threshold.
 *   h_out         dev, [T, D] bf16 or NULL: the residual stream after the
 *                 last layer.
 * Enqueued on `stream`; device-side checks and timeouts go to the error word
 * of the model's layer handle (fc_model_layer_handle + fc_get_error).
 */
FC_API fc_status fc_model_step(fc_model* m, void* stream, int batch, const void* x,
                               const int32_t* q_pos, const int32_t* cu_seqlens_q,
                               const int32_t* cu_seqlens_k, int total_q, int total_k,
                               void* const* k_caches, void* const* v_caches,
                               const int32_t* head_rows, int n_head_rows, float* importance,
                               int32_t* token, float* confidence, uint8_t* accept, void* h_out);

/* The Flash-Cache handle the model runs its attention through (owned by the
 * model): for fc_topk_tracked on the model's importance, fc_get_error,
 * fc_profile and fc_last_launch_count (which then counts the model step's
 * kernels). */
FC_API fc_handle* fc_model_layer_handle(fc_model* m);

/*
 * fc_decode_iteration — one draft-and-verify decode iteration of every
 * sequence (Flash-Verify: the model is its own drafter and verifier; draft and
 * [MASK] tokens are checked through two views; every prediction that meets
 * the confidence threshold is accepted in the same iteration; the tracked
 * positions are reselected by importance).  All on the device, on `stream`:
 *  1. query of sequence b = its K tracked positions, then the W positions of
 *     its window [window_start[b], window_start[b] + W);
 *  2. [MASK] view: undecided window rows read embed[mask_id]; draft view: they
 *     read embed[draft] (embed[mask_id] with no draft); decided rows read
 *     embed[token] in both; one fc_model_step per view, the LM head on the
 *     window rows, the draft view's importance summed over layers;
 *  3. an undecided window position is accepted when the [MASK] view's
 *     confidence >= threshold (its token), or when the draft view predicts the
 *     position's draft with confidence >= threshold; if nothing in a window is
 *     accepted, its undecided position with the highest [MASK]-view confidence
 *     is (lowest position on ties); undecided positions get the [MASK] view's
 *     prediction as their next draft; a fully decided window advances by W
 *     when the next window still ends inside the span (window_start + 2W <=
 *     gen_end);
 *  4. tracked := the top-K positions of [0, window_start) by the draft view's
 *     importance, window_start as advanced in step 3.
 *   cu_seqlens_k, total_k      dev, as for fc_step; k_caches/v_caches as for
 *                              fc_model_step (the caches keep the draft view's
 *                              rows: both views write the same rows and the
 *                              draft view runs second).
 *   embed          dev, [V, D] bf16 (V = the model's vocab).
 *   mask_id        0 <= mask_id < V.
 *   n_tracked (K)  <= max_topk; window (W) >= 1; B * (K + W) <= max_total_q and
 *                  B * W <= max_head_rows of the model's config.
 *   tracked        dev, int32 [B, K], in/out: positions, each in [0, ws) (so
 *                  window_start >= K); entries past the candidates are -1.
 *   window_start   dev, int32 [B], in/out.   gen_end  dev, int32 [B]: end of
 *                  the generated span (window_start + W <= gen_end <= L_b).
 *   tokens, draft  dev, int32 [S] (one entry per cache row, -1 = none), in/out.
 *   n_accepted     dev, int32 [B], out: tokens accepted this iteration.
 *   importance     dev, float [S] or NULL: when given, receives the draft
 *                  view's importance summed over layers, the scores the
 *                  reselection of step 4 ranked (a handle-owned buffer is used
 *                  otherwise).
 * Device-side checks (positions, ids) set the layer handle's error word.
 */
FC_API fc_status fc_decode_iteration(fc_model* m, void* stream, int batch,
                                     const int32_t* cu_seqlens_k, int total_k,
                                     void* const* k_caches, void* const* v_caches,
                                     const void* embed, int mask_id, int n_tracked, int window,
                                     int32_t* tracked, int32_t* window_start,
                                     const int32_t* gen_end, int32_t* tokens, int32_t* draft,
                                     int32_t* n_accepted, float* importance);

/*
 * fc_model_lm_head — the last stage of fc_model_step on rows the caller
 * supplies: the LM head over rows that are already final-normed
 * (rms_norm(h) * g_final), then per row the top token, its softmax
 * probability (the confidence) and the Flash-Verify acceptance
 * confidence >= threshold (paper-digest page, Flash-Verify).  The logits are
 * never written: the kernel keeps per 256-column tile the maximum, its index
 * and the sum of exp(logit - maximum), and a second kernel merges the tiles.
 *   rows           dev, [n_rows, D] bf16, 16-byte aligned.
 *   n_rows         1 <= n_rows <= max_head_rows of the model's config.
 *   token, confidence, accept   dev, as for fc_model_step.
 * Uses the model's LM-head statistics buffer: not concurrent with another
 * call on the same model.
 */
FC_API fc_status fc_model_lm_head(fc_model* m, void* stream, const void* rows, int n_rows,
                                  int32_t* token, float* confidence, uint8_t* accept);

/* Release the model, its layer handle and workspace (NULL is a no-op). */
FC_API void fc_model_destroy(fc_model* m);

/* Static, human-readable name of a status. */
FC_API const char* fc_status_str(fc_status s);

#ifdef __cplusplus
}
#endif

#endif /* FLASHCACHE_H */
