/*
 * lf_decode.h — C ABI of the B200 (sm_100a) LongFlow fused decode step.
 *
 * One decode step over a fixed-budget KV cache, in ONE kernel launch:
 *   1. single-query GQA attention of the current token over every filled
 *      cache slot plus the new token itself;
 *   2. a per-slot importance score taken from that same softmax, with no
 *      history: the probability of the current query averaged over the G
 *      query heads of the slot's KV group;
 *   3. when the cache is full, eviction of the lowest-scoring slot that is
 *      not protected (the first `sink` slots and the last `window`
 *      positions are protected; ties go to the lowest slot index), and an
 *      in-place overwrite of that slot with the new token's K/V/position.
 *      While a slot is still free (position -1), the new token goes to the
 *      lowest free slot and nothing is evicted.
 *
 * Sources: "LongFlow: Efficient KV Cache Compression for Reasoning Models"
 * (gist.science summary) §2A "Principios de Diseño" (zero-history,
 * zero-cost importance estimation), §2B "Derivación de la Métrica de
 * Importancia" (evict the token whose removal least changes the attention
 * output, scored from its attention weight), §2C "Implementación de Alto
 * Rendimiento" (static pre-allocated KV cache; one fused kernel doing
 * attention, importance estimation and eviction); and the blog page
 * "Долгая память: Оптимизация кэша для сложных рассуждений", sections
 * "Оптимизированная Реализация с Объединенными Ядрами" (O and the score
 * produced in one pass over KV blocks and a mask moved between HBM and
 * on-chip memory) and "Ограничения Памяти при Моделировании Длинных
 * Последовательностей" (one token evicted after every attention step).
 * The exact score, the sink/window protection and the tie-break are fixed
 * by this library's specification, not by the pages.
 *
 * Conventions shared by every call
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Every tensor pointer is a DEVICE pointer owned by the caller; the
 *     library never frees, keeps or reallocates it.  Layouts are dense,
 *     row-major, with no padding:
 *        q       [B, Hq, D]          bf16
 *        k_new   [B, Hkv, D]         bf16      v_new  [B, Hkv, D]    bf16
 *        kcache  [B, Hkv, budget, D] bf16      vcache [B, Hkv, budget, D]
 *        pos     [B, Hkv, budget]    int32, the token position held by each
 *                                    slot, -1 = free slot
 *        out     [B, Hq, D]          fp32
 *        evicted [B, Hkv]            int32
 *     Query head h reads KV head h / G, G = Hq / Hkv.
 *   - q, k_new, v_new, kcache, vcache and out must be 16-byte aligned, pos
 *     and evicted 4-byte aligned.
 *   - Calls are asynchronous on the stream given to lf_init (or
 *     lf_set_stream); arguments are checked on the host before anything is
 *     enqueued.  A failed check enqueues nothing.
 *   - A handle is not thread-safe: it caches launch plans and holds the
 *     status word, so calls on one handle come from one thread at a time.
 *     Separate handles are independent.
 *   - A handle belongs to the device that was current at lf_init.  Calls
 *     that plan or enqueue work with it (prefill, decode, lf_get_split)
 *     return LF_EINVAL, enqueueing nothing, when another device is
 *     current.  Every tensor must be memory of that device; this is not
 *     checked (the pointer's device is not queried on the hot path).
 *   - Return codes (never exceptions): LF_OK, or one of the negative
 *     LF_E* codes below; lf_strerror names them.
 */
#ifndef LF_DECODE_H
#define LF_DECODE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LF_OK 0
#define LF_EINVAL (-1)       /* bad argument: null/misaligned pointer, shape, budget, sink, window */
#define LF_ENOTINIT (-2)     /* null or destroyed handle */
#define LF_ECUDA (-3)        /* a CUDA runtime call or kernel launch failed */
#define LF_EDEVICE (-4)      /* the kernel flagged an error (see lf_status_bits) */
#define LF_EUNSUPPORTED (-5) /* the current device is not sm_100 or lacks a needed feature */

/* device status bits, as set by the kernels and returned by lf_status_bits */
#define LF_STATUS_WAIT_TIMEOUT 1  /* a bounded wait on a shared-memory barrier gave up */
#define LF_STATUS_NO_CANDIDATE 2  /* full cache but no unprotected slot (corrupt pos table) */
#define LF_STATUS_BAD_SEQ_BUDGET 4 /* a per-sequence budget outside 1 .. budget (ragged calls) */

/* Eviction scores (lf_set_score) */
#define LF_SCORE_MEAN_PROB 0  /* probability averaged over the group's query heads (default) */
#define LF_SCORE_ALPHA_L1V 1  /* that average times the L1 norm of the slot's value vector */

#if defined(__GNUC__)
#define LF_API __attribute__((visibility("default")))
#else
#define LF_API
#endif

typedef struct lf_ctx* lf_handle;

/* Create a handle for one attention layer shape on the CURRENT device.
 *   B, Hq, Hkv, D: batch, query heads, KV heads (Hq % Hkv == 0, Hq/Hkv <= 8),
 *   head dimension (64 or 128).  max_budget: largest budget later calls may
 *   pass.  cuda_stream: a cudaStream_t (NULL = legacy default stream).
 * Allocates one small device status word (cudaMalloc) and nothing else;
 * later calls never allocate.  On failure *h is set to NULL. */
LF_API int lf_init(lf_handle* h, int B, int Hq, int Hkv, int D, int max_budget, void* cuda_stream);

/* Change the stream later calls are enqueued on. */
LF_API int lf_set_stream(lf_handle h, void* cuda_stream);

/* Write a prompt into an empty cache (the statically pre-allocated cache of
 * "Implementación de Alto Rendimiento"): k, v [B, Hkv, n, D] go to slots
 * 0..n-1 of kcache/vcache [B, Hkv, budget, D]; pos[j] = j for j < n and -1
 * after.  0 <= n <= budget <= max_budget, else LF_EINVAL: compressing a
 * prompt longer than the budget is outside the method, which targets the
 * decode phase (summary page §5, "Limitaciones").  k and v may be NULL when
 * n == 0. */
LF_API int lf_prefill_cache(lf_handle h, const uint16_t* k, const uint16_t* v, int n,
                     uint16_t* kcache, uint16_t* vcache, int32_t* pos, int budget);

/* THE fused decode step (one kernel launch).  For every row (b, g):
 *   t = 1 + max(pos) over filled slots (0 for an empty cache);
 *   out[b, h] = softmax over {filled slots, new token} of
 *               (q[b,h] . k) / sqrt(D), applied to the matching v;
 *   if some slot is free: e = lowest free slot, evicted[b,g] = -1;
 *   else: score_j = mean over the group's heads of the probability of slot
 *         j, candidates = { j >= sink and pos[j] < t - window },
 *         e = candidate of lowest score (lowest j on ties), evicted[b,g] = e;
 *   then kcache/vcache slot e <- k_new/v_new and pos[e] <- t.
 * Eviction happens after the attention, so it never changes this step's
 * out.  Requires 1 <= budget <= max_budget, sink >= 0, window >= 1 and
 * budget > sink + window (so a full cache with distinct positions always
 * has a candidate).  Positions in pos must be distinct; the kernel flags
 * LF_STATUS_NO_CANDIDATE, writes evicted = -2 and leaves the row's cache
 * unchanged when a full row has no candidate.
 * A budget too large for one thread-block cluster of at most 16 CTAs to
 * hold the row's logits in shared memory is rejected with LF_EINVAL, before
 * anything is enqueued.  Measured on a B200: budgets up to 65,536 slots plan
 * for groups of up to 4 heads (98,304 do not), and up to 49,152 for 5 to 8
 * heads (65,536 do not); lf_get_split answers the question for a budget.
 * Near ties: scores are computed in fp32; when the two lowest candidate
 * scores of a row are within a relative 1e-4 of each other, the kernel
 * rescores those candidates in fp64 before choosing. */
LF_API int lf_decode_step(lf_handle h,
                   const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                   uint16_t* kcache, uint16_t* vcache, int32_t* pos,
                   int budget, int sink, int window,
                   float* out, int32_t* evicted_idx);

/* Plain decode attention over filled slots + the new token: the same
 * kernel with scoring and eviction compiled out.  Nothing is written but
 * out.  This is the no-eviction control the fused step is timed against. */
LF_API int lf_decode_attention(lf_handle h,
                        const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                        const uint16_t* kcache, const uint16_t* vcache, const int32_t* pos,
                        int budget, float* out);

/* Ragged batch: lf_decode_step with a budget per sequence.
 * seq_budget: DEVICE int32 [B], 4-byte aligned, owned by the caller and
 * read by the kernel; batch entry b (all its KV heads) then has the cache
 * of slots 0 .. seq_budget[b] - 1 alone.  The slots beyond are neither
 * read (not even for t) nor written, so they may hold anything.  Each
 * sequence appends while one of its slots is free and evicts once its own
 * budget is full, exactly as lf_decode_step does for a budget of
 * seq_budget[b]; rows at different positions and fill levels may share a
 * batch.  `budget` is still the allocated slots per row (the cache stride)
 * and bounds every seq_budget[b].
 * A row's slots are split evenly over the CTAs of its cluster, and the
 * clusters take rows from a counter in the handle's device memory as they
 * finish the previous ones (a dynamic schedule: work per row follows
 * seq_budget[b]).  Calls on one handle must therefore not run concurrently.
 * Device-side checks: a seq_budget[b] outside 1 .. budget sets
 * LF_STATUS_BAD_SEQ_BUDGET; its rows get out computed over the clamped
 * budget, evicted = -2, and no cache write.  A full sequence with
 * seq_budget[b] <= sink + window has no candidate (LF_STATUS_NO_CANDIDATE,
 * evicted = -2).  Host checks as lf_decode_step, plus seq_budget non-null
 * and aligned (else LF_EINVAL).  Follows the handle's score (lf_set_score).
 * The pages do not treat ragged batches; this is the serving-batch form of
 * the same per-row step. */
LF_API int lf_decode_step_ragged(lf_handle h,
                   const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                   uint16_t* kcache, uint16_t* vcache, int32_t* pos,
                   int budget, const int32_t* seq_budget, int sink, int window,
                   float* out, int32_t* evicted_idx);

/* lf_decode_attention with a budget per sequence (seq_budget as in
 * lf_decode_step_ragged): attention over each sequence's filled slots
 * among 0 .. seq_budget[b] - 1 plus the new token; only out is written. */
LF_API int lf_decode_attention_ragged(lf_handle h,
                        const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                        const uint16_t* kcache, const uint16_t* vcache, const int32_t* pos,
                        int budget, const int32_t* seq_budget, float* out);

/* FP8 KV storage.  kcache / vcache hold one byte per element: OCP E4M3
 * codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities; S.1111.111 is NaN; largest finite magnitude 448), with one
 * positive, finite fp32 scale per cache tensor: code c stands for
 * E4M3(c) * k_scale in kcache and E4M3(c) * v_scale in vcache.  Layouts are
 * those of the bf16 cache with uint8_t elements: [B, Hkv, budget, D],
 * 16-byte aligned.  Writing a value x (the prompt in lf_prefill_cache_fp8,
 * the new token in the step) stores the code of x / scale, the quotient
 * taken in fp32 (IEEE, correctly rounded) and rounded to the nearest E4M3
 * value, ties to even; finite quotients beyond +-448 saturate to +-448.
 * The step is lf_decode_step (or lf_decode_step_ragged when seq_budget is
 * non-null) on the dequantised cache, decoding in the K and V loops; the
 * new token takes part in its own step with its exact bf16 k_new / v_new,
 * and only its stored copy is quantised.  It follows the handle's score.
 * The pages name 8-bit floats only for another method's medium-importance
 * tokens (ARKV summary, "Fase de Decodificación": tokens held in low
 * precision such as FP8 and dequantised on the fly); applying the format to
 * the whole LongFlow cache is this library's extension.  Returns LF_EINVAL
 * for a scale that is not positive and finite, or as lf_decode_step. */
LF_API int lf_prefill_cache_fp8(lf_handle h, const uint16_t* k, const uint16_t* v, int n,
                         uint8_t* kcache, uint8_t* vcache, int32_t* pos, int budget,
                         float k_scale, float v_scale);

LF_API int lf_decode_step_fp8(lf_handle h,
                   const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                   uint8_t* kcache, uint8_t* vcache, int32_t* pos,
                   int budget, const int32_t* seq_budget, int sink, int window,
                   float k_scale, float v_scale,
                   float* out, int32_t* evicted_idx);

/* Attention only over an E4M3 cache (nothing scored or written but out);
 * seq_budget may be null. */
LF_API int lf_decode_attention_fp8(lf_handle h,
                        const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                        const uint8_t* kcache, const uint8_t* vcache, const int32_t* pos,
                        int budget, const int32_t* seq_budget, float k_scale, float v_scale,
                        float* out);

/* Eviction score used by later lf_decode_step calls on this handle.
 *   LF_SCORE_MEAN_PROB (default): score_j as documented for lf_decode_step.
 *   LF_SCORE_ALPHA_L1V: the LongFlow summary page's own form (§2B
 *     "Derivación de la Métrica de Importancia"): the token's attention
 *     weight times the L1 norm of its value vector, sum_l |v_j[l]|.  The
 *     page states it for one head; for a KV group the weight is the
 *     probability averaged over the group's query heads, so
 *     score_j = mean_i p_ij * ||v_j||_1.  The norm is taken in the same pass
 *     from the V tile already in shared memory; near ties are rescored in
 *     fp64 with the norm recomputed in fp64.  Candidates, tie-break and
 *     output are unchanged.
 * Returns LF_EINVAL for any other value (the handle keeps its score). */
LF_API int lf_set_score(lf_handle h, int score);

/* The handle's eviction score (LF_SCORE_*), or a negative LF_E* code. */
LF_API int lf_get_score(lf_handle h);

/* Tuning: number of CTAs (a thread-block cluster) that split one row's
 * slots; 0 = automatic.  Must be 0 or a power of two <= 16. */
LF_API int lf_set_split(lf_handle h, int split);

/* The split the next call with this budget would use (after lf_set_split). */
LF_API int lf_get_split(lf_handle h, int budget);

/* Synchronise the handle's stream, then read and clear the device status
 * word.  Returns LF_OK if no kernel flagged an error since the last call,
 * LF_EDEVICE otherwise (the bits are then available from lf_status_bits),
 * or LF_ECUDA if the stream reported an error. */
LF_API int lf_get_status(lf_handle h);

/* Status bits captured by the last lf_get_status (LF_STATUS_* above). */
LF_API int lf_status_bits(lf_handle h);

/* Free the status word and the handle.  Synchronises the stream first. */
LF_API int lf_destroy(lf_handle h);

/* Static, NUL-terminated name of a return code. */
LF_API const char* lf_strerror(int code);

/* Library ABI version, (major << 16) | minor. */
LF_API int lf_version(void);

/* lf_decode_step for callers that cannot allocate device memory.
 *
 * The LongFlow pages have no counterpart to this call; it exists for users
 * of this library.  lf_init allocates the device status word the fused
 * kernel writes its error bits into, and some callers cannot make that
 * cudaMalloc: runtimes that reserve the device memory up front in a pool of
 * their own and forbid allocations outside it, or hosts that hand a kernel
 * only its buffers and a stream.  This entry point takes no handle and
 * allocates nothing.  Its scratch, the status word, lives in a fixed
 * 256-byte array in the library's device memory (a file-scope __device__
 * array), which every GPU that loads the library holds until the process
 * exits.  The kernel needs one 4-byte word of it, whatever the sizes; a call
 * whose scratch would not fit is rejected with LF_EINVAL.
 *
 * Arguments, layouts, alignment and results are those of lf_decode_step,
 * with the shape (B, Hq, Hkv, D) and the stream passed directly (budget is
 * capped at 1 << 22).  The status word is cleared on the stream before the
 * launch.  Device-side errors are not reported through lf_get_status: a row
 * the kernel could not evict shows evicted_idx = -2 and an unchanged cache.
 *
 * The first call on a device sets up that device (with it current): it
 * looks up the device address of the scratch array and the device's limits.
 * Make that first call before any stream capture.  All calls share the one
 * scratch array, so calls that overlap on the GPU (on different streams)
 * race on the status word; results in out, evicted_idx and the cache are
 * not affected. */
LF_API int lf_decode_step_noalloc(const uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                                  uint16_t* kcache, uint16_t* vcache, int32_t* pos,
                                  int B, int Hq, int Hkv, int D, int budget, int sink, int window,
                                  float* out, int32_t* evicted_idx, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* LF_DECODE_H */
