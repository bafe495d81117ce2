/*
 * h2o.h -- C ABI of the H2O chunk-step library (libh2o.so, sm_100a).
 *
 * Method: H2O (heavy-hitter oracle) sparse attention over a fixed-capacity KV
 * cache, processed chunk by chunk, as described in "Learning how to Forget:
 * Fine-tuning for Long-Context Sparse Attention":
 *   - Abstract: an implementation of H2O sparse attention with a dedicated
 *     scaled dot product attention (SDPA) kernel;
 *   - §1 Introduction ¶1: KV information is held in a fixed-size cache whose
 *     slots are evicted once it is full;
 *   - §1 Introduction ¶3: combinable with grouped query attention (GQA);
 *   - FAQ answer 3: the SDPA kernel also returns the summed attention weights;
 *   - Figure 1(a): a prefill chunk of full length, then chunks of S tokens.
 *
 * One chunk step, per (batch b, KV head h), with t0 = tokens already seen:
 *   1. attend:  each query row (g, i) of h's group (query head g uses KV head
 *               g / (Hq/Hkv)) sees every valid cache slot plus the chunk keys
 *               j <= i; p = softmax(q.k / sqrt(d)); out = p . V.
 *   2. summed weights: c_j = sum over the group's query heads and the chunk's
 *               queries of p_ij, for each cache slot and each chunk key.
 *   3. accumulate: score[slot] += c_slot for every valid slot (running sum).
 *   4. evict:   need = max(0, S - empty slots); among valid slots whose token
 *               position is older than the recent window (pos < t0 - R), the
 *               `need` smallest by (score, pos) are evicted.
 *   5. scatter: freed = ascending(evicted slots, then the first S - need empty
 *               slots); chunk token i goes to freed[i]: its K and V rows,
 *               pos = t0 + i, score = c of chunk key i.
 * A prefill is the same step on an empty cache (it evicts nothing).
 *
 * Layouts (row-major, contiguous, element type = the handle's dtype):
 *   q, out        [B, Hq,  S, d]
 *   k, v          [B, Hkv, S, d]
 *   cache K, V    [B, Hkv, M, d]   (library-owned)
 *   scores        [B, Hkv, M]  float32;  positions [B, Hkv, M] int32 (-1 = empty)
 *
 * Pointers: q/k/v/out and every read-back buffer may be device memory or host
 * memory (pinned or pageable); host buffers are staged through library-owned
 * device buffers with stream-ordered copies.  The caller owns all of them.
 * Host inputs of a step are copied on a stream of the handle's own into one of
 * two staging sets, so that they overlap the previous step's kernels; the
 * step's kernels wait for them.  A grouped step (h2o_step_layers) of at least
 * eight layers with host outputs runs its layers in sub-groups of four and
 * copies each sub-group's outputs to the host on a stream of its own while the
 * later sub-groups compute.  Like device buffers, host buffers may be reused
 * (inputs) or read (out) once `stream` has passed the step (e.g. after
 * cudaStreamSynchronize(stream)): the step's last work on `stream` waits for
 * every output copy.  With pageable memory the CUDA runtime may make the
 * copies synchronous.
 * Streams: `stream` is a cudaStream_t (NULL = the legacy default stream); every
 * call only enqueues work on it, except where stated.  A handle is not
 * thread-safe.
 *
 * Errors: every call returns an h2o_status; nothing aborts or throws across the
 * ABI.  h2o_last_error() gives the message of the last failing call.  A device
 * error raised inside a step's kernels (a bounded wait that timed out, too few
 * evictable slots found on the device) is written to the handle's device error
 * word and reported by a LATER call on the handle, as H2O_ETIMEOUT, H2O_ESHAPE
 * or H2O_ECUDA: the first call that finds the step's work finished (steps do
 * not wait for the GPU, so that may be several steps later).  Such a report
 * does not name the step that failed, and every step enqueued since the last
 * point at which the handle was known to be clean (a call that returned after
 * waiting for the GPU: a read-back into host memory, or any step while the
 * environment sets H2O_SYNC_CHECK=1) has then run on a cache whose contents
 * are unspecified: destroy the handle.  With
 * H2O_SYNC_CHECK=1 every step waits for its own kernels and reports its own
 * device error.
 */
#ifndef H2O_H_
#define H2O_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct h2o_ctx* h2o_t;

typedef enum {
  H2O_OK = 0,
  H2O_EINVAL = -1,   /* bad argument (null pointer, dtype, d, Hq % Hkv, R >= M) */
  H2O_ESHAPE = -2,   /* shape cannot be served: P > M, S > M, fewer evictable slots than needed,
                        or a stream past 2^31 - 1 tokens (positions are int32) */
  H2O_ESTATE = -3,   /* step before prefill, prefill twice */
  H2O_ENOMEM = -4,   /* a device or pinned allocation failed */
  H2O_ECUDA = -5,    /* a CUDA runtime call or kernel launch failed */
  H2O_ETIMEOUT = -6  /* a bounded in-kernel wait ran out; the step's results are invalid */
} h2o_status;

typedef enum { H2O_F32 = 0, H2O_BF16 = 1 } h2o_dtype;

/* Eviction policy of a handle.
 *   H2O_POLICY_H2O  the heavy-hitter policy described at the top: evict the
 *                   `need` eligible slots with the smallest (score, pos).
 *   H2O_POLICY_LR   recency only: evict the `need` eligible slots holding the
 *                   oldest tokens (smallest pos), so the cache holds the most
 *                   recent tokens.  The page "Learning how to Forget: Fine-
 *                   tuning for Long-Context Sparse Attention" names an `lr`
 *                   policy beside `h2o` (Tables 1 and 6) without defining
 *                   it; this is the plainest reading of the name.  Attention,
 *                   summed weights and scores are computed as for H2O (the
 *                   scores are kept but do not decide evictions).            */
typedef enum { H2O_POLICY_H2O = 0, H2O_POLICY_LR = 1 } h2o_policy;

/* Create a handle for one layer's caches.
 *   M    cache capacity (slots) per (batch, KV head), M >= 1
 *   R    protected recent window in tokens, 0 <= R < M
 *   Hq   query heads; Hkv KV heads; Hq % Hkv == 0
 *   d    head dimension, 64 or 128
 *   dtype H2O_F32 or H2O_BF16 (q/k/v/out/cache element type)
 * No device memory is allocated until the prefill (the batch size is known
 * then).  The scale is fixed at 1/sqrt(d); natural-base softmax.
 * Returns H2O_OK and *out, or H2O_EINVAL.                                     */
int h2o_create(int64_t M, int64_t R, int Hq, int Hkv, int d, int dtype, h2o_t* out);

/* h2o_create with an eviction policy (h2o_policy); h2o_create is
 * h2o_create_policy(..., H2O_POLICY_H2O, out).  H2O_EINVAL for an unknown
 * policy.                                                                     */
int h2o_create_policy(int64_t M, int64_t R, int Hq, int Hkv, int d, int dtype, int policy,
                      h2o_t* out);

/* Prefill: the first chunk, P tokens (1 <= P <= M), causal attention among
 * themselves with an empty cache.  Token t goes to slot t with score = its
 * summed attention weight.  Allocates the cache (zero-filled), scores,
 * positions and scratch on the current device.  `out` may be NULL (outputs
 * are then not written).  Errors: H2O_ESTATE if already prefilled, H2O_ESHAPE
 * if P > M, H2O_ENOMEM.                                                       */
int h2o_prefill(h2o_t h, const void* q, const void* k, const void* v, void* out,
                int B, int64_t P, void* stream);

/* One chunk step of S tokens (1 <= S <= M) at t0 = tokens seen so far, on the
 * batch size fixed at prefill: attend, accumulate, evict, scatter (see top).
 * The new K/V rows are copied into the cache inside the step, so the caller
 * may reuse q/k/v once the stream has passed the step.
 * Errors: H2O_ESTATE before prefill; H2O_ESHAPE if fewer than `need` slots are
 * evictable (valid slots minus the min(R, t0) protected ones).                */
int h2o_step(h2o_t h, const void* q, const void* k, const void* v, void* out,
             int64_t S, void* stream);

/* One chunk step of S tokens on each of n handles (the layers of a model, or
 * any caches that take a chunk together): the same result as calling
 * h2o_step(hs[l], q[l], k[l], v[l], out ? out[l] : NULL, S, stream) for
 * l = 0 .. n-1.  When the handles have identical sizes and state (M, R, Hq,
 * Hkv, d, dtype, B, tokens seen) and the chunk takes the one-kernel
 * tensor-core path (bf16, d = 128), all layers share one attention launch and
 * one score/select/scatter launch (per group of up to 32 layers), so a partial
 * last wave of thread blocks is paid once per group and not once per layer
 * (Table 6 of "Learning how to Forget: Fine-tuning for Long-Context Sparse
 * Attention": the policy's cost must stay a small share of a training step);
 * otherwise each layer runs its own launches.  The handles must be distinct;
 * `out` may be NULL (no outputs) or hold n pointers (each may be NULL).
 * Profiling (h2o_set_profiling) is read from hs[0]: its timings then cover the
 * attention and the tail launches of all n layers.
 * Errors: as h2o_step, for the first handle that fails; H2O_EINVAL for a NULL
 * or repeated handle.  A failure before any launch leaves every handle as it
 * was.                                                                        */
int h2o_step_layers(h2o_t* hs, int n, const void* const* q, const void* const* k,
                    const void* const* v, void* const* out, int64_t S, void* stream);

/* Copy the state out (each pointer may be NULL to skip it):
 *   slots      [B, Hkv, S_last] int32: the slots the last step (or prefill)
 *              filled, ascending; these are its evicted slots followed by the
 *              previously empty slots it used
 *   scores     [B, Hkv, M] float32 (0 for empty slots)
 *   positions  [B, Hkv, M] int32, -1 for empty slots
 * Errors: H2O_ESTATE before prefill.                                          */
int h2o_read_state(h2o_t h, int32_t* slots, float* scores, int32_t* positions, void* stream);

/* The last step's buffer delta ("Learning how to Forget: Fine-tuning for
 * Long-Context Sparse Attention", Figure 1(c): per chunk, the slots written
 * and the tokens they received), each pointer may be NULL to skip it:
 *   slots              [B, Hkv, S_last] int32: the slots the step filled,
 *                      ascending (as h2o_read_state returns them); chunk
 *                      token i (its K/V rows are the step's own inputs) went
 *                      to slots[.., i]
 *   evicted_positions  [B, Hkv, S_last] int32: the token position slots[.., i]
 *                      held before the step, -1 if it was empty.
 * Together with the chunk's K/V these rebuild each step's cache from the
 * previous one.  Errors: H2O_ESTATE before prefill.                           */
int h2o_read_delta(h2o_t h, int32_t* slots, int32_t* evicted_positions, void* stream);

/* Copy the cache contents out: k_cache, v_cache [B, Hkv, M, d] of the handle's
 * dtype (NULL skips).  Rows of empty slots are zero.                          */
int h2o_read_kv(h2o_t h, void* k_cache, void* v_cache, void* stream);

/* Counters of the handle: out[0] = B, out[1] = t0 (tokens seen), out[2] =
 * valid slots per (batch, KV head), out[3] = S of the last step, out[4] =
 * device kernels launched by the last step (or prefill).                      */
int h2o_info(h2o_t h, int64_t out[5]);

/* Per-kernel timing.  on = 1 turns it on and restarts the count of profiled
 * steps, on = 2 turns it on and keeps the count, on = 0 turns it off (the
 * default).  While on, each step records CUDA events around its kernels on the
 * caller's stream, into a ring that holds the last 64 profiled steps, so steps
 * can be enqueued back to back and read afterwards.  The events sit between
 * the step's kernels and so keep the next kernel from starting while the
 * previous one drains (programmatic dependent launch).  h2o_step_timings()
 * waits for the events of the profiled step `age` profiled steps before the
 * last (age 0 = the last) and writes up to n
 * durations in milliseconds:
 *   ms[0] attention + summed weights, ms[1] the tail: score accumulate,
 *   select and scatter (one fused launch, or three kernels when the fused one
 *   cannot run for these sizes or H2O_SPLIT_TAIL=1 is set in the environment).
 *   Returns the number written (>= 0) or a negative status
 *   (H2O_ESTATE if no such profiled step).  h2o_last_timings(h, ms, n) is
 *   h2o_step_timings(h, 0, ms, n).                                            */
int h2o_set_profiling(h2o_t h, int on);
int h2o_step_timings(h2o_t h, int age, float* ms, int n);
int h2o_last_timings(h2o_t h, float* ms, int n);

/* Free every resource of the handle (synchronises the device first).  NULL is
 * accepted.                                                                   */
int h2o_destroy(h2o_t h);

/* Message of the last failing call on h (or of the last failing h2o_create /
 * standalone call on this thread when h is NULL).  Never NULL.                */
const char* h2o_last_error(h2o_t h);

/* Standalone selection step (step 4 above) on caller-owned device arrays, for
 * n_heads independent caches of M slots each:
 *   scores [n_heads, M] float32, positions [n_heads, M] int32 (-1 = empty)
 *   evicted [n_heads, need] int32 (output): the `need` smallest (score, pos)
 *   among slots with 0 <= pos < t0 - R, ascending by slot.
 * Errors: H2O_EINVAL on bad sizes; H2O_ESHAPE if a cache has fewer than `need`
 * eligible slots (checked on the device; reported by this call, which then
 * synchronises the stream).                                                   */
int h2o_select(const float* scores, const int32_t* positions, int n_heads, int64_t M,
               int64_t t0, int64_t R, int64_t need, int32_t* evicted, void* stream);

/* Allocation-free attention with summed attention weights.  The paper has no
 * counterpart to this call: it exists for callers that cannot call cudaMalloc
 * -- a serving engine that reserves nearly all device memory for its own pool
 * up front, or latency-critical code that cannot afford cudaMalloc's implicit
 * device synchronisation.  It allocates nothing: the caller passes every input
 * and output, and the only scratch (the fixed-point accumulator rows of the
 * summed weights and an error word) is a fixed 16 MiB array in the library's
 * static device memory, which every GPU that loads the library holds until the
 * process exits.
 *
 * Computes steps 1-2 above (attend, summed weights) for one chunk against a
 * caller-owned cache, without touching any handle state:
 *   q, out [B, Hq, S, d]; k, v [B, Hkv, S, d]; k_cache, v_cache [B, Hkv, M, d]
 *   (only slots [0, n_valid) are read; may be NULL when n_valid == 0), all
 *   device pointers of `dtype`;
 *   colsum [B, Hkv, M + S] float32 (device): colsum[.., c] for c < M is slot
 *   c's summed weight (0 for c >= n_valid), colsum[.., M + j] chunk key j's.
 * Limit: B * Hkv * W <= 2 * 2^20 (64-bit words), with W = M + S rounded up to
 * a multiple of 4; larger problems return H2O_ESHAPE.  Each call clears the
 * words it uses (stream-ordered memsets, no allocation) before its kernels.
 * Set-up: the first call on a device looks up the device address of the
 * scratch array with that device current; make that first call before any
 * stream capture on the device.
 * Sharing: every call on a device uses the same scratch, which keeps the last
 * call's contents; calls whose GPU work overlaps (different streams, or
 * different host threads, without ordering between them) race on it and give
 * wrong results.  Order them on one stream or with events.
 * Errors: H2O_EINVAL (NULL pointer, bad sizes), H2O_ESHAPE (above the limit),
 * H2O_ECUDA; the message is read with h2o_last_error(NULL).  A bounded
 * in-kernel wait that runs out is not reported by this call (its outputs are
 * then invalid); the handle API reports it.                                   */
int h2o_attend_noalloc(const void* q, const void* k, const void* v, const void* k_cache,
                       const void* v_cache, int B, int Hq, int Hkv, int d, int dtype, int64_t M,
                       int64_t n_valid, int64_t S, void* out, float* colsum, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* H2O_H_ */
