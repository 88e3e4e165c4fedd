/*
 * h2o.h -- C ABI of the B200 (sm_100a) chunked H2O sparse-attention step.
 *
 * The operation is the heavy-hitter (H2O) KV-cache step of "Learning how to
 * Forget: Fine-tuning for Long-Context Sparse Attention" (arXiv 2608.19920):
 *   - paper page, section "Kernel Support Needs": attention kernels should
 *     return, beside the SDPA output, the summed attention weights
 *     sum_i w[b,h,i,j] of every key slot j, under the positional mask
 *     (b,h,i,j) -> -inf * I[P + i < t(b,h,j)];
 *   - paper page, section "Improvements to Heavy-Hitter Oracle (H2O)": a
 *     slot's H2O score accumulates those sums, and new content overwrites the
 *     slots with the smallest scores.
 * One call of h2o_step processes one chunk of T new tokens per sequence:
 *   1. SDPA of the chunk's queries against the C-slot cache plus the chunk
 *      itself (cache fully visible, causal inside the chunk, diagonal
 *      included), softmax scale 1/sqrt(d), GQA: query head h reads KV head
 *      h / (Hq / Hkv);
 *   2. per KV head, the weight every candidate key received, summed over the
 *      chunk's rows and over the Hq/Hkv query heads of the group, is added to
 *      its score (cache slots: old score + sum; chunk tokens: the sum);
 *   3. per (sequence, KV head), of the n valid slots plus T chunk tokens the C
 *      with the largest score survive (equal scores: the larger position
 *      survives); kept cache entries stay in their slots, and the kept chunk
 *      tokens, in position order, fill the free slots in ascending slot order.
 * That is the default policy; h2o_set_policy selects the normalized ranking
 * or the insert-always order instead (enum h2o_policy).
 *
 * Conventions for every entry point:
 *   - Every call returns a status (H2O_OK or a negative H2O_ERR_*); none
 *     aborts the process. h2o_last_error() describes the last failure.
 *   - Pointers named "device" are CUDA device pointers of the context's
 *     device; "host" pointers are host memory. The caller owns every buffer it
 *     passes; the library owns the cache and its workspace.
 *   - "stream" is a cudaStream_t (NULL = the legacy default stream). Calls are
 *     asynchronous and stream-ordered unless stated otherwise; buffers passed
 *     to a call must stay valid until the stream reaches it.
 *   - Layouts are dense row-major (C order), element type H2O_BF16
 *     (bfloat16) or H2O_FP32 (float) as chosen at creation:
 *       q, out [B, Hq,  T, d]      k, v [B, Hkv, T, d]
 *       cache  [B, Hkv, C, d]      scores (float) / positions (int32) [B, Hkv, C]
 *     q, k, v, out must be 16-byte aligned.
 *   - Supported shapes: d in {64, 128}; Hq % Hkv == 0; C >= 1; T >= 1;
 *     positions stay below 2^31. All sequences of the batch advance together:
 *     the chunk of a call holds positions P .. P+T-1 of every sequence.
 *   - The valid cache slots of every (sequence, KV head) are always the
 *     prefix 0 .. n-1, with n = min(C, tokens processed); every state the
 *     library produces has this form and h2o_set_state() rejects others.
 *   - A kernel that waits longer than its bound (H2O_WAIT_TIMEOUT_MS below)
 *     stops, records the fact in a device-visible error word and returns;
 *     the next call on that context reports H2O_ERR_TIMEOUT and the context
 *     is poisoned (every later call returns H2O_ERR_POISONED).
 */
#ifndef H2O_H_
#define H2O_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct h2o_ctx h2o_ctx;

enum h2o_status {
    H2O_OK = 0,
    H2O_ERR_ARG = -1,         /* bad argument, shape or state */
    H2O_ERR_ALIGN = -2,       /* a pointer is not 16-byte aligned */
    H2O_ERR_OOM = -3,         /* device or host allocation failed */
    H2O_ERR_CUDA = -4,        /* a CUDA runtime/driver call failed */
    H2O_ERR_TIMEOUT = -5,     /* a device-side wait ran out of its bound */
    H2O_ERR_POISONED = -6,    /* an earlier device error: context unusable */
    H2O_ERR_UNSUPPORTED = -7  /* shape outside the supported set */
};

enum h2o_dtype { H2O_BF16 = 0, H2O_FP32 = 1 };

/* Eviction ranking ("Learning how to Forget", paper page, section
 * "Improvements to Heavy-Hitter Oracle (H2O)"): candidates are ranked by
 *   H2O_POLICY_SUM         their H2O score phi (the default), or
 *   H2O_POLICY_NORMALIZED  phi / (t - t_j): the score over the candidate's age,
 *                          with t = P + T the token count after the step and
 *                          t_j the candidate's position (every age >= 1).
 * Ties go to the larger position under both. The stored scores are phi
 * under both policies; only the ranking key differs.
 *   H2O_POLICY_INSERT_ALWAYS  the order the same section describes, new
 *                          content overwriting the lowest-scoring slots:
 *                          before the chunk attends, the n + T - C valid
 *                          slots with the lowest scores so far are evicted
 *                          (the older position first among equal scores);
 *                          the T chunk tokens, in position order, take the
 *                          empty and evicted slots in ascending order; then
 *                          the rows attend to the buffer under the position
 *                          mask of section "Kernel Support Needs" and every
 *                          slot's score grows by its weights. Every chunk
 *                          token enters, so a step needs T <= C
 *                          (H2O_ERR_UNSUPPORTED otherwise). */
enum h2o_policy { H2O_POLICY_SUM = 0, H2O_POLICY_NORMALIZED = 1, H2O_POLICY_INSERT_ALWAYS = 2 };

/* Create a bf16 context on the current CUDA device: an empty cache of C slots
 * per (sequence, KV head), P = 0. Allocates all device memory it will need for
 * chunks of up to T = C tokens (larger chunks grow the workspace once).
 * *out receives the handle, NULL on failure. */
int h2o_create(int B, int Hq, int Hkv, int d, int C, h2o_ctx **out);

/* As h2o_create, with the element type (enum h2o_dtype) and the largest
 * chunk length to size the workspace for (max_T >= 1). */
int h2o_create_ex(int B, int Hq, int Hkv, int d, int C, int dtype, int max_T, h2o_ctx **out);

/* Free every resource of the context (synchronises its device first).
 * NULL is accepted. */
int h2o_destroy(h2o_ctx *ctx);

/* Select the eviction policy (enum h2o_policy) for the following steps; the
 * default is H2O_POLICY_SUM. Takes effect from the next h2o_step; call it
 * between steps (it is not stream-ordered). The first selection of
 * H2O_POLICY_INSERT_ALWAYS allocates that variant's workspace (a compact copy
 * of the cache and per-slot arrays; H2O_ERR_CUDA / H2O_ERR_OOM if that
 * fails, in which case nothing stays allocated and the policy is unchanged).
 * H2O_ERR_ARG for an unknown policy. */
int h2o_set_policy(h2o_ctx *ctx, int policy);

/* One H2O step on the chunk (q, k, v) of T tokens (device pointers, layouts
 * above); writes the attention output to out (device). Updates the cache,
 * scores and positions; P advances by T. Asynchronous on `stream`. */
int h2o_step(h2o_ctx *ctx, const void *q, const void *k, const void *v, void *out,
             int T, void *stream);

/* nchunks consecutive H2O steps of T tokens each, the same results as that
 * many h2o_step calls: chunk i is read at q + i * B*Hq*T*d elements (k, v:
 * + i * B*Hkv*T*d) and its output written at out + i * B*Hq*T*d (device
 * pointers, layouts as h2o_step, the context's element type). Because every
 * chunk was written before the call, each step after the first may begin its
 * attention to the chunk's own tokens while the previous step's eviction is
 * still running (tensor-core path, H2O_POLICY_SUM and H2O_POLICY_NORMALIZED;
 * the others run the steps one after another). Stops at the first failing
 * step and returns its status (the steps before it have been enqueued).
 * Asynchronous on `stream`. */
int h2o_prefill(h2o_ctx *ctx, const void *q, const void *k, const void *v, void *out,
                int T, int nchunks, void *stream);

/* Backward of one step's chunk SDPA with the step's key set held fixed
 * ("Learning how to Forget", paper page, section "Gradient Computation
 * Strategy for Sparse Attention": training through the sparse cache replays
 * the logged eviction decisions, so each step's attention is differentiated
 * for the keys it actually attended to; the eviction carries no gradient).
 * The context's current cache (K, V and the n valid slots, as h2o_set_state
 * left it) is taken as the step's pre-step cache and is not modified; q, k,
 * v are the step's chunk (device, layouts above, context dtype), lse its
 * natural-log LSE (device float [B, Hq, T], as h2o_lse returned after the
 * step) and dout = dL/dout [B, Hq, T, d] (context dtype). Writes, as device
 * float (fp32) arrays,
 *   dq [B, Hq, T, d], dK, dV [B, Hkv, C, d] (the cache slots; zero in empty
 *   slots), dk, dv [B, Hkv, T, d] (the chunk),
 * with the key / value gradients of a KV head summed over the query heads of
 * its group. The row term sum_j p_j dp_j (= dout . out) is recomputed from
 * the attention weights, so the step's output is not an input. Every pointer
 * must be 16-byte aligned. The first call (and one with a longer chunk than
 * before) allocates the backward's row workspace. Asynchronous on `stream`. */
int h2o_backward(h2o_ctx *ctx, const void *q, const void *k, const void *v, const float *lse,
                 const void *dout, int T, float *dq, float *dK, float *dV, float *dk, float *dv,
                 void *stream);

/* h2o_step with HOST buffers: copies q, k, v to library-owned device staging
 * buffers, runs the step and copies the output back into out (host). Page-
 * locked host memory gives asynchronous copies; pageable memory works too.
 * Returns after the output has arrived in out (synchronises `stream`). */
int h2o_step_host(h2o_ctx *ctx, const void *q, const void *k, const void *v, void *out,
                  int T, void *stream);

/* Pipelined form of h2o_step_host for a run of chunks: enqueues the upload of
 * (q, k, v) from HOST memory into one of two library-owned device staging
 * slots (on an internal upload stream), the step (on `stream`) and the
 * download of the output into out (HOST, on an internal download stream), and
 * returns without waiting. Successive calls alternate the slots, so the
 * upload of chunk c+1 and the download of chunk c-1 overlap the step of chunk
 * c; events order each slot's reuse. Use page-locked host memory: pageable
 * memory is correct but serialises the copies. q, k, v must stay unchanged
 * and out must not be read until h2o_host_sync returns; chunks must be
 * submitted in sequence order on one stream, and the other calls that touch
 * the context (h2o_reset, h2o_get_state, ...) only after h2o_host_sync.
 * Same shapes and errors as h2o_step; the first call creates the two streams
 * and three events per slot, and a larger T than before grows both slots once
 * (synchronising). The paper has no counterpart of this host interface. */
int h2o_step_host_async(h2o_ctx *ctx, const void *q, const void *k, const void *v, void *out,
                        int T, void *stream);

/* Waits until every upload and download enqueued by h2o_step_host_async has
 * finished (the outputs are in host memory), then reports any device error
 * as h2o_sync_check does. The caller's `stream` is not synchronised. */
int h2o_host_sync(h2o_ctx *ctx);

/* Current H2O scores, float [B, Hkv, C] (device dst); 0 in empty slots. */
int h2o_scores(h2o_ctx *ctx, float *dst, void *stream);

/* Current slot positions, int32 [B, Hkv, C] (device dst); -1 = empty. */
int h2o_positions(h2o_ctx *ctx, int32_t *dst, void *stream);

/* Host-side counters: *P = tokens processed per sequence, *n = valid slots
 * per (sequence, KV head). Either pointer may be NULL. No synchronisation. */
int h2o_counters(const h2o_ctx *ctx, int64_t *P, int64_t *n);

/* Description of the last failure on this context (ctx = NULL: the last
 * failure of this thread that had no context, e.g. in h2o_create). */
const char *h2o_last_error(const h2o_ctx *ctx);

/* ---- inspection, checkpoint and test hooks ---------------------------- */

/* Candidates of the last step, for each (sequence, KV head): index c < n_prev
 * is cache slot c, index n_prev + t is chunk token t, with n_prev the valid
 * slot count before that step. scores: updated score (old + weight sum);
 * pos: position; kept: 1 if it survived. Device arrays of [B, Hkv, ncand]
 * with ncand = n_prev + T_last (query it with h2o_last_step_info). Under
 * H2O_POLICY_INSERT_ALWAYS the cache candidates are the entries kept before
 * the attention, in slot order (n_prev counts them), and every candidate is
 * kept. Any of the three pointers may be NULL. */
int h2o_candidates(h2o_ctx *ctx, float *scores, int32_t *pos, uint8_t *kept, void *stream);

/* Slot each chunk token of the last step was written to, -1 if dropped:
 * device int32 [B, Hkv, T_last]. */
int h2o_token_slots(h2o_ctx *ctx, int32_t *dst, void *stream);

/* Natural-log softmax normaliser (log-sum-exp of the scaled logits) of every
 * query row of the last step: device float [B, Hq, T_last]. */
int h2o_lse(h2o_ctx *ctx, float *dst, void *stream);

/* T and the pre-step valid count n_prev of the last step (host ints). */
int h2o_last_step_info(const h2o_ctx *ctx, int *T_last, int *n_prev);

/* Export the cache: K, V [B, Hkv, C, d] (context dtype), scores float and
 * positions int32 [B, Hkv, C] (device pointers, any may be NULL), and the
 * counters P and n (host int64, may be NULL). */
int h2o_get_state(h2o_ctx *ctx, void *K, void *V, float *scores, int32_t *positions,
                  int64_t *P, int64_t *n, void *stream);

/* Import a cache exported by h2o_get_state (or built by the caller). Checks,
 * on the host after copying positions back (synchronises `stream`): for every
 * (sequence, KV head) positions[0..n-1] are distinct values in [0, P) and
 * positions[n..C-1] are -1; 0 <= n <= min(C, P). On success the next step
 * processes positions P .. P+T-1. Device pointers; P, n by value. */
int h2o_set_state(h2o_ctx *ctx, const void *K, const void *V, const float *scores,
                  const int32_t *positions, int64_t P, int64_t n, void *stream);

/* Empty the cache and set P = 0 (asynchronous on `stream`). */
int h2o_reset(h2o_ctx *ctx, void *stream);

/* Check the context's device error word after synchronising `stream`;
 * returns H2O_OK, or H2O_ERR_TIMEOUT (and poisons the context). */
int h2o_sync_check(h2o_ctx *ctx, void *stream);

/* Self-test of the bounded device wait: launches one block that waits on a
 * shared-memory barrier nothing will complete, giving up after timeout_ms
 * milliseconds, synchronises `stream` and returns what the context's error
 * word reports (H2O_ERR_TIMEOUT when the bound works). No memory traffic is
 * in flight during the wait. Poisons the context, as any timeout does. */
int h2o_selftest_wait(h2o_ctx *ctx, int timeout_ms, void *stream);

/* Per-kernel timing (tracing). h2o_profile_begin allocates CUDA events for
 * up to max_steps steps and makes every following h2o_step record an event
 * on its stream before its first kernel and after each kernel. h2o_profile_end
 * synchronises those events, stops recording and reports, per kernel name
 * (in launch order of a step), the summed device time in milliseconds and the
 * number of launches. names/total_ms/launches are host arrays of max_kernels
 * entries; returns the number of kernel names (>= 0) or an error. */
int h2o_profile_begin(h2o_ctx *ctx, int max_steps);
int h2o_profile_end(h2o_ctx *ctx, int max_kernels, const char **names, double *total_ms,
                    int *launches);

/* Eviction alone, without any device allocation. The paper has no
 * counterpart of this entry point; it exists for callers that cannot call
 * cudaMalloc -- plugin hosts and serving runtimes that only hand out buffers
 * they pre-allocated under a fixed memory budget, and latency-critical paths
 * where an allocation would synchronise the device.
 * Given, for `groups` (sequence, KV head) groups, the updated candidate scores
 * and positions of one step (device float / int32 [groups, n+T]: cache slots
 * 0..n-1, then the T chunk tokens at positions P..P+T-1), it computes what
 * h2o_step's eviction computes under H2O_POLICY_SUM (it ranks by the scores
 * as given): kept flags (device uint8 [groups, n+T]), the
 * slot of each chunk token or -1 (device int32 [groups, T]), and updates the
 * slot scores and positions (device float / int32 [groups, C], in/out: kept
 * cache slots take their new score, kept chunk tokens fill the free slots in
 * ascending order, leftover free slots become empty). The caller owns every
 * buffer. Scratch (the free-slot lists) lives in a static device array of
 * 262144 int32 (1 MiB) that every GPU loading the library holds until exit;
 * groups * C above that returns H2O_ERR_UNSUPPORTED. The first call on a
 * device looks up that array's device address (once per device, and again
 * when the device's CUDA context has changed, as after cudaDeviceReset); make
 * that first call before any stream capture. Each device has its own copy of the
 * array and every call on that device shares it, keeping whatever the last
 * call left there: calls that overlap on the GPU (for example on two streams)
 * race, so serialise them. Nothing in it needs clearing between calls. Asynchronous on `stream`; errors are
 * described by h2o_last_error(NULL). */
int h2o_select_noalloc(int groups, int C, int n, int T, int64_t P, const float *cand_score,
                       const int32_t *cand_pos, float *scores, int32_t *positions, uint8_t *kept,
                       int32_t *token_slot, void *stream);

/* Self-test of the exponentials the tensor-core kernels use: for device
 * float x[0..n), writes the FMA-pipe polynomial 2^x of degree 3 (y_poly3)
 * and degree 4 (y_poly4), and the hardware approximation ex2.approx.ftz
 * (y_mufu), all device float [n]. Asynchronous on `stream`. */
int h2o_selftest_exp2(const float *x, float *y_poly3, float *y_poly4, float *y_mufu, int n,
                      void *stream);

/* Library build identifier (static string). */
const char *h2o_version(void);

/* Per-step kernel launches issued by h2o_step for this context (host int);
 * fills names (static strings) up to max_names. */
int h2o_kernel_plan(const h2o_ctx *ctx, int T, const char **names, int max_names);

#ifdef __cplusplus
}
#endif

/* Environment knobs (read at h2o_create):
 *   H2O_WAIT_TIMEOUT_MS  how long a kernel polls an mbarrier before it gives
 *                        up (default 2000 ms); values < 1 are ignored.
 */
#endif /* H2O_H_ */
