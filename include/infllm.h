/*
 * infllm.h -- C ABI of a single-GPU (sm_100a) InfLLM block-memory sparse attention layer.
 *
 * One context holds one attention layer's context memory for one token stream.
 * Tokens arrive in chunks (prefill) or one at a time (decode).  Distant tokens are
 * grouped into fixed-size memory units, each represented by its top-n_reps
 * representative tokens; every chunk (or decode step) scores all units, keeps
 * the top_k per kv head, and attends with one exact softmax over the sink tokens,
 * the selected units and the local window.
 *
 * Method sources (InfLLM pages):
 *   - "InfLLM Guide: Training-Free Long-Context Memory Units", sections
 *     "Core Innovation 1: Structured Context Partitioning" (sinks / memory units /
 *     local window) and "Core Innovation 2: Semantic Representative Key Vectors &
 *     Dynamic Top-K Selection", items 2 "Query-Aware Top-K Scoring and Loading"
 *     (Score(M_j) = q . r_j / sqrt(d), top-k) and 3 "Exact Attention Evaluation"
 *     (working context = sinks U top-k units U local window).
 *   - "InfLLM: Training-Free Long-Context Extrapolation for LLMs with an Efficient
 *     Context Memory" (atlas.scime.ai summary), "Approach": units represented by
 *     their top-scoring representative tokens chosen by attention scores; lookup
 *     at every step.  Its ablation rows ("Measured effects") keep lookup during both
 *     encoding and decoding.
 *   - OpenReview rebuttal (paperhub.cn), Q2 "Comparison to Well-trained Long LLM":
 *     lookup during pre-filling is done per block (chunk).
 *
 * Conventions for every call:
 *   - q, k, v and out are CALLER-OWNED DEVICE pointers, contiguous [n][heads][head_dim]
 *     in the context's dtype (fp32 or bf16), 16-byte aligned.  q has n_q_heads heads,
 *     k and v have n_kv_heads heads.  k and v are raw (before RoPE): the library applies
 *     the position scheme.
 *   - All work is enqueued on the CUDA stream given to infllm_create and runs
 *     asynchronously; calls return after enqueueing.  Argument and state errors are
 *     detected on the host and returned before anything is enqueued.
 *   - The library owns every internal buffer (allocated by create, freed by destroy).
 *   - A device-side consistency check that fails latches an error word; the next call
 *     returns INFLLM_EDEVICE.  After any error, infllm_destroy stays valid.
 *   - Calls on one context are not thread-safe.  Contexts are independent.
 *
 * Position scheme (RoPE, rotate-half pairing (i, i + d/2), theta_i = rope_base^(-2i/d)):
 * a query at token t and a window key at token n interact at their true relative
 * distance t - n; every sink and memory key sits at one clamped distance equal to
 * `window` (query rotated by R(window), key unrotated).
 */
#ifndef INFLLM_H
#define INFLLM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    INFLLM_OK = 0,
    INFLLM_EINVAL = 1,    /* bad argument or configuration */
    INFLLM_ECAPACITY = 2, /* max_tokens or max_chunk would be exceeded */
    INFLLM_ESTATE = 3,    /* call out of order (e.g. attend without a matching append) */
    INFLLM_ECUDA = 4,     /* a CUDA runtime call failed (message in infllm_last_error) */
    INFLLM_EDEVICE = 5    /* a device-side check failed in an earlier launch */
} infllm_status;

typedef enum { INFLLM_F32 = 0, INFLLM_BF16 = 1 } infllm_dtype;

/* How a unit is scored against the chunk's queries.  REPS and REPSUM are the same number in exact
 * arithmetic (the dot product is linear in the key): REPS reads the n_reps representative keys of
 * every unit; REPSUM reads one fp32 sum of them per unit (half the bytes).  MEANKEY scores a unit by
 * the mean of all of its keys (one vector per unit in the context dtype, the sum taken in fp64 and
 * rounded once), the alternative representation that "InfLLM: Training-Free Long-Context
 * Extrapolation for LLMs with an Efficient Context Memory" (research-map summary, "Measured effects",
 * row "Use selected representative tokens instead of mean key-vector representations") compares
 * against; it selects different units than REPS. */
typedef enum { INFLLM_SCORE_REPS = 0, INFLLM_SCORE_REPSUM = 1, INFLLM_SCORE_MEANKEY = 2 } infllm_score_mode;

typedef struct {
    int32_t n_q_heads;   /* Hq; Hq % Hkv == 0; q head h uses kv head h / (Hq/Hkv) */
    int32_t n_kv_heads;  /* Hkv */
    int32_t head_dim;    /* d: 64 or 128 */
    int32_t n_sink;      /* S >= 0: initial tokens always attended */
    int32_t window;      /* W >= 1: local window length (and the clamped distance) */
    int32_t unit_size;   /* U in [1, 1024]: tokens per memory unit */
    int32_t n_reps;      /* r in [1, min(U, 32)]: representative tokens per unit */
    int32_t top_k;       /* k >= 0: units attended per chunk and kv head */
    int32_t max_chunk;   /* largest n accepted by append/attend */
    int64_t max_tokens;  /* capacity of the token stream; max_tokens / unit_size + 1 <= 16384 units */
    double rope_base;    /* RoPE base (> 1) */
    int32_t dtype;       /* infllm_dtype of q/k/v/out.  bf16 attention runs on the tcgen05 tensor
                          * cores, which take Hq / Hkv dividing 128 and top_k <= 4096: other bf16
                          * shapes are refused (EINVAL).  fp32 runs on the CUDA cores. */
    int32_t score_mode;  /* infllm_score_mode */
} infllm_config;

typedef struct {
    int64_t tokens;          /* tokens appended so far */
    int64_t units_with_reps; /* units whose representatives have been chosen */
    int32_t n_mem;           /* units eligible for the last attended chunk */
    int32_t n_selected;      /* min(top_k, n_mem) of the last attended chunk */
    int64_t window_base;     /* first window token of the last attended chunk */
    int64_t active_tokens;   /* keys attended by the last query of the last attended chunk */
    int64_t kernel_launches; /* kernels enqueued since create (or the last stats reset) */
    int32_t attend_path;     /* chunk attention kernel: 0 = CUDA cores (fp32), 1 = tcgen05 tensor cores (bf16) */
    int32_t score_mode;      /* infllm_score_mode in use */
    /* filled when profiling is on (infllm_set_profiling), device times from CUDA events: */
    double ms_append, ms_reps, ms_prep, ms_select, ms_attend, ms_decode;
    int64_t n_append, n_reps, n_prep, n_select, n_attend, n_decode;
} infllm_stats;

typedef struct infllm_ctx infllm_ctx; /* opaque */

/* Create a context: validates cfg, allocates every pool for max_tokens / max_chunk on the
 * current CUDA device (the K/V stores, the representative pool, the packed-query and lookup
 * buffers), and records `cuda_stream` (a cudaStream_t; NULL = legacy default stream) for all
 * later work.  The pools hold the three parts of the context that "InfLLM Guide: Training-Free
 * Long-Context Memory Units", "Core Innovation 1: Structured Context Partitioning", names:
 * initial (sink) tokens, memory units of unit_size tokens, and the local window.
 * Errors: EINVAL (cfg out of range, or a bf16 shape the tensor-core kernel does not take; message
 * on stderr), ECUDA (allocation failed).  On failure
 * *out is NULL and nothing stays allocated.  The caller owns the context until infllm_destroy. */
infllm_status infllm_create(const infllm_config* cfg, void* cuda_stream, infllm_ctx** out);

/* Free everything the context owns.  Waits for the context's pending work.  NULL is accepted. */
infllm_status infllm_destroy(infllm_ctx* ctx);

/* Start a new token stream in the same context (keeps allocations). */
infllm_status infllm_reset(infllm_ctx* ctx);

/* Append tokens [t, t+n) where t = tokens so far.  First, every unit that becomes eligible at t
 * (its last token at least `window` tokens before t) is turned into a memory unit: its n_reps
 * representative tokens are the ones with the largest attention logit summed over the `window`
 * queries that follow the unit and the q heads of the group ("InfLLM: Training-Free Long-Context
 * Extrapolation for LLMs with an Efficient Context Memory", research-map summary, "Approach":
 * units represented by representative tokens chosen by attention scores; ties to the lower
 * token).  Then the chunk's k and v are stored and its queries are kept (as block sums) for
 * later representative scores.
 *   q [n][Hq][d] device, k, v [n][Hkv][d] device, all in the context dtype; read during the call's
 *   kernels only (the caller may reuse them once the stream has passed this call).
 * n == 0 is a no-op.  A chunk that is appended and not attended before the next append, decode
 * step or prefill stays in the context without outputs of its own: that is how a memory is built
 * from a prompt whose outputs are not needed.
 * Errors: EINVAL (null pointer with n > 0, n > max_chunk, n < 0), ECAPACITY (tokens + n >
 * max_tokens), EDEVICE (an earlier kernel's check failed). */
infllm_status infllm_append_chunk(infllm_ctx* ctx, const void* q, const void* k, const void* v,
                                  int32_t n);

/* Attention output of the chunk just appended (same n), the chunk-wise lookup of the OpenReview
 * rebuttal (paperhub.cn), Q2 "Comparison to Well-trained Long LLM".  Unit lookup: every eligible
 * unit's score is the scaled logit q . r / sqrt(d) summed over the chunk's queries, the group's q
 * heads and the unit's representatives, with every memory token at relative distance `window`
 * ("InfLLM Guide...", "Core Innovation 2", item 2 "Query-Aware Top-K Scoring and Loading"); the top
 * min(top_k, n_mem) per kv head are kept, ties to the lower unit index.  Then one exact softmax
 * over sinks (n < S, causal) U selected units U window [B, t] (same page, item 3 "Exact Attention
 * Evaluation").
 *   q [n][Hq][d] device (the chunk's queries again); out [n][Hq][d] device, written by the call's
 *   kernels.
 * Errors: ESTATE (no matching append), EINVAL (null pointer), EDEVICE. */
infllm_status infllm_attend_chunk(infllm_ctx* ctx, const void* q, int32_t n, void* out);

/* Whole-prompt prefill: n tokens (q [n][Hq][d], k, v [n][Hkv][d], out [n][Hq][d], device) in chunks
 * of `chunk` tokens (the last one ragged), each chunk appended and then attended exactly as
 * infllm_append_chunk + infllm_attend_chunk would, in one call.  Chunk-wise pre-filling with
 * per-chunk unit lookup follows the OpenReview rebuttal (paperhub.cn), Q2 "Comparison to
 * Well-trained Long LLM", and "InfLLM Guide...", "Memory Efficiency"; this entry point adds no
 * arithmetic of its own.  Because every input is in place when the call starts, the kernels of
 * chunk c+1 that store its keys and pack its queries are chained to (and overlap) chunk c's
 * attention.  Results are identical, bit for bit, to the per-chunk calls.
 * Errors: EINVAL (null pointer with n > 0, chunk not in [1, max_chunk], n < 0), ECAPACITY (tokens
 * + n > max_tokens), EDEVICE. */
infllm_status infllm_prefill(infllm_ctx* ctx, const void* q, const void* k, const void* v,
                             int64_t n, int32_t chunk, void* out);

/* One decode step: append one token (q [1][Hq][d], k, v [1][Hkv][d], device) and attend it; out
 * [1][Hq][d] device.  Per generated token: lookup over every eligible unit and exact attention
 * over sinks U top-k units U window, as for a one-token chunk ("InfLLM Guide...", "Core Innovation
 * 2", items 2 and 3; lookup at every decoding step: "InfLLM: Training-Free Long-Context
 * Extrapolation...", research-map summary, "Approach").  The attention is split over key tiles
 * whose partial softmaxes are merged by log-sum-exp (exact).
 * Errors: EINVAL (null pointer), ECAPACITY (tokens + 1 > max_tokens), EDEVICE. */
infllm_status infllm_decode_step(infllm_ctx* ctx, const void* q, const void* k, const void* v,
                                 void* out);

/* --- introspection (synchronize the context's stream) --------------------------------- */

/* Selected units of the last attended chunk: host_sel [Hkv][top_k] int32, ascending unit
 * ids, padded with -1. */
infllm_status infllm_get_selection(infllm_ctx* ctx, int32_t* host_sel);

/* Unit scores of the last attended chunk: host_scores [Hkv][n_mem] float32 (includes the
 * 1/sqrt(d) factor).  *n_mem_out receives n_mem. */
infllm_status infllm_get_unit_scores(infllm_ctx* ctx, float* host_scores, int32_t capacity,
                                     int32_t* n_mem_out);

/* Representatives of units [unit_begin, unit_begin + n_units): host_ids [Hkv][n_units][n_reps]
 * int32, unit-local token offsets in ascending order.  The units must already have
 * representatives (ESTATE otherwise). */
infllm_status infllm_get_reps(infllm_ctx* ctx, int32_t unit_begin, int32_t n_units, int32_t* host_ids);

infllm_status infllm_get_stats(infllm_ctx* ctx, infllm_stats* out);

/* Switch the unit-scoring operand (infllm_score_mode) for later calls; every operand pool is always
 * maintained, so this is valid at any point of a stream. */
infllm_status infllm_set_score_mode(infllm_ctx* ctx, int32_t score_mode);

/* Record CUDA events around kernel launches and accumulate their device times into
 * infllm_stats.  enable: 0 = off, INFLLM_PROFILE_ALL = every kernel class, or an OR of the
 * INFLLM_PROFILE_* class bits below (events break the overlap between consecutive launches, so
 * profile only the classes being measured).  Any call clears the accumulated times and counts. */
enum {
    INFLLM_PROFILE_ALL = 1,
    INFLLM_PROFILE_APPEND = 2,  /* token store and query block sums */
    INFLLM_PROFILE_REPS = 4,    /* representative scoring of newly evicted units */
    INFLLM_PROFILE_PREP = 8,    /* rotated, packed queries of a chunk */
    INFLLM_PROFILE_SELECT = 16, /* unit scores and top-k */
    INFLLM_PROFILE_ATTEND = 32, /* chunk attention */
    INFLLM_PROFILE_DECODE = 64  /* decode attention (tiles and merge) */
};
infllm_status infllm_set_profiling(infllm_ctx* ctx, int32_t enable);

/* Unit lookup while pre-filling (default on).  enable = 0: chunks (infllm_attend_chunk,
 * infllm_prefill) attend to sinks and the local window only, while representatives are still
 * built for every evicted unit; infllm_decode_step always looks up.  This is the ablation
 * "memory lookup during both encoding and decoding instead of decoding only" of "InfLLM:
 * Training-Free Long-Context Extrapolation for LLMs with an Efficient Context Memory" (research-map
 * summary, "Measured effects"), run with lookup during decoding only. */
infllm_status infllm_set_prefill_lookup(infllm_ctx* ctx, int32_t enable);

/* Launch chaining (default on): inside one call, every kernel launch after the first is a
 * programmatic dependent launch, so a kernel that does not need its predecessor's results
 * starts while that predecessor runs; the first launch of a call always waits for the work
 * before it on the stream.  enable = 0 launches every kernel plainly (same results). */
infllm_status infllm_set_launch_chaining(infllm_ctx* ctx, int32_t enable);

/* Human-readable description of the last error on this context ("" if none). */
const char* infllm_last_error(infllm_ctx* ctx);

/* --- lookup without any device allocation --------------------------------------------- */

/* Unit scores and top-k selection for ONE query token, allocating nothing on the device.
 *
 * For callers that cannot call cudaMalloc: code running while a framework captures its stream
 * into a CUDA graph and forbids allocation there, engines whose memory planner owns every device
 * byte, and real-time loops where an allocation could synchronise the device.  No context is
 * needed.  The caller passes every input and output; the only other memory used is a fixed
 * scratch area inside the library (a static device array of about 1 MiB that every GPU which
 * loads the library holds until the process exits).  The InfLLM pages have no counterpart to this
 * call: it computes what the lookup step of infllm_decode_step computes, from caller buffers.
 *
 *   rep_keys  device [n_kv_heads][n_units][n_reps][head_dim], `dtype`: raw keys of every unit's
 *             representative tokens
 *             (16-byte aligned)
 *   q         device [n_q_heads][head_dim], `dtype`: the query token, before RoPE
 *   sel       device out [n_kv_heads][top_k] int32: ascending ids of the top min(top_k, n_units)
 *             units of each kv head (ties to the lower id), padded with -1
 *   scores    device out or NULL, [n_kv_heads][n_units] float32: the unit scores (query at
 *             relative distance `window`, factor 1/sqrt(head_dim) included)
 * Limits of the scratch area: n_kv_heads <= 64 and n_units <= 16384; larger sizes return
 * INFLLM_ECAPACITY before anything is enqueued.  Other bad arguments (top_k outside [1, 32],
 * head_dim not 64/128, ...) return INFLLM_EINVAL.  Work is enqueued on `cuda_stream`, which must
 * belong to the current device.
 * The first call on a device looks up the device address of the scratch array (once per device
 * and CUDA context, with that device current); make that first call before any stream capture.  A
 * device reset (cudaDeviceReset) gives the device a new context, and the next call looks the
 * address up again.  Every call shares
 * the scratch area and keeps the last call's contents (the call clears what must start at zero):
 * calls whose work overlaps on the GPU -- on different streams or from different host threads --
 * race and can return wrong results, so serialise them. */
infllm_status infllm_select_units_noalloc(const void* rep_keys, const void* q, int32_t n_q_heads,
                                          int32_t n_kv_heads, int32_t head_dim, int32_t n_units,
                                          int32_t n_reps, int32_t window, double rope_base, int32_t dtype,
                                          int32_t top_k, int32_t* sel, float* scores, void* cuda_stream);

/* Library version string. */
const char* infllm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* INFLLM_H */
