/*
 * sa.h -- indexed sparse attention for NVIDIA B200 (sm_100a): C ABI.
 *
 * The path has three steps, which the pages present as one pipeline
 * ("Optimizing Next-Gen LLM Inference: Sparse Attention and Mixed Parallelism
 * in Practice", §1 and §3; "Inference Acceleration for New Large Model
 * Architectures", §3):
 *
 *   1. a lightweight indexer scores every visible cached position s of a query
 *      t and weights the per-head scores by head weights:
 *          I[t,s] = sum_j w[t,j] * max(0, q_I[t,j,:] . k_I[s,:]);
 *   2. a per-query top-K keeps the K best positions;
 *   3. a sparse attention kernel reads only those rows of the MLA latent cache
 *      (512-d latent + 64-d rope, absorbed query) and returns the 512-d output.
 *
 * Both caches are paged and read in place through a page table
 * ("Optimizing Next-Gen LLM Inference" §3.1; "Inference Acceleration" §3.1).
 * Index keys and the latent cache may be FP8 ("Optimizing Next-Gen LLM
 * Inference" §4): index keys as e4m3 with one fp32 scale per token, the latent
 * as e4m3 with one fp32 scale per tile of tokens x latent dims (a whole page
 * by default; rope stays bf16).  Input preparation quantises the query and
 * appends new tokens in these formats.
 *
 * Conventions for every entry point
 *  - All pointers marked "device" are CUDA device pointers owned by the
 *    caller; the library allocates no memory.  Host structs are read during
 *    the call only.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and never synchronises, except sa_device_status().
 *  - Shapes and dtypes are checked on the host before anything is launched;
 *    a bad argument returns SA_ERR_INVALID_ARG (or SA_ERR_UNSUPPORTED for a
 *    valid but unimplemented combination) and launches nothing.
 *  - Data errors found on the device (a page id outside [0, num_pages), a
 *    query position past its sequence, a selected index outside the visible
 *    range) never fault: the offending work is skipped and a status word in
 *    the workspace records the first error; read it with sa_device_status().
 *  - Positions are logical (0 .. q_pos), never physical rows, so results do
 *    not depend on where pages sit in the pools.
 *  - Device pointers must be 16-byte aligned.
 *  - Nothing aborts, exits or traps.
 */
#ifndef SA_H
#define SA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SA_API __attribute__((visibility("default")))
#else
#define SA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sa_status {
    SA_OK = 0,
    SA_ERR_INVALID_ARG = 1,   /* shape, dtype, pointer or size rejected on the host */
    SA_ERR_UNSUPPORTED = 2,   /* valid combination the library does not implement */
    SA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than sa_workspace_size() */
    SA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    SA_ERR_DEVICE_FAULT = 5,  /* bad data detected on the device (see detail code) */
    SA_ERR_TIMEOUT = 6        /* a bounded device-side wait gave up */
} sa_status;

typedef enum sa_dtype {
    SA_F32 = 0,
    SA_BF16 = 1,
    SA_E4M3 = 2,              /* OCP e4m3fn code bytes, always paired with fp32 scales */
    SA_MXFP8 = 3              /* index query and keys only: e4m3fn code bytes with one E8M0
                               * scale byte per 32 consecutive values (the OCP MX format:
                               * scale = 2^(byte - 127); byte 255 is NaN) */
} sa_dtype;

/* Paged caches of one attention layer.
 *
 * Logical position s of sequence b lives in physical row
 *     page_table[b * max_pages + s / page_size] * page_size + s % page_size
 * of both pools below.  page_size must be 64.
 */
typedef struct sa_cache {
    const int32_t *page_table;   /* device int32 [batch, max_pages]; unused slots may hold -1 */
    const int32_t *seq_len;      /* device int32 [batch]: tokens cached per sequence */
    int32_t batch;
    int32_t max_pages;
    int32_t num_pages;           /* physical pages in each pool */
    int32_t page_size;           /* tokens per page (64) */

    /* indexer keys */
    /* SA_E4M3 (the quantised path) or SA_BF16 (the BF16 path, unscaled): the
     * indexer's two numerical paths ("Optimizing Next-Gen LLM Inference" §3.1;
     * "Inference Acceleration for New Large Model Architectures" §3.1); or
     * SA_MXFP8, the pages' group-wise quantisation with one scale per 32
     * values ("Inference Acceleration for New Large Model Architectures" §4.1;
     * "Long-Context LLM Inference Optimization", Layered Quantization); or
     * SA_F32 */
    sa_dtype index_dtype;
    const void *k_index;         /* device [num_pages, page_size, d_index] */
    const float *k_index_scale;  /* device SA_E4M3: fp32 [num_pages, page_size], one per token;
                                  * SA_MXFP8: E8M0 bytes [num_pages, page_size, d_index / 32]
                                  * (pass the byte array's address); NULL otherwise */
    int32_t d_index;

    /* MLA latent KV rows */
    sa_dtype kv_dtype;           /* SA_BF16, SA_E4M3 or SA_F32 */
    const void *kv;              /* SA_F32/SA_BF16: [num_pages, page_size, d_latent + d_rope]
                                  * SA_E4M3: latent codes [num_pages, page_size, d_latent] */
    const void *kv_rope;         /* SA_E4M3 only: bf16 [num_pages, page_size, d_rope] */
    const float *kv_scale;       /* SA_E4M3 only: fp32 [num_pages, page_size / kv_scale_tokens,
                                  * d_latent / kv_scale_dims], one scale per tile */
    int32_t d_latent;            /* 512 (production) */
    int32_t d_rope;              /* 64 (production) */
    /* SA_E4M3 scale tile: one fp32 scale per kv_scale_tokens tokens of a page
     * x kv_scale_dims latent dims.  The pages quantise the main cache per token
     * and per 128 elements ("Optimizing Next-Gen LLM Inference" §4, table;
     * "Inference Acceleration for New Large Model Architectures" §4.2;
     * "Long-Context LLM Inference Optimization", Layered Quantization): that is
     * (1, 128).  kv_scale_tokens divides page_size; kv_scale_dims divides
     * d_latent and is a multiple of 16.  0 and 0 mean one scale per page
     * (page_size x d_latent). */
    int32_t kv_scale_tokens;
    int32_t kv_scale_dims;
} sa_cache;

/* A batch of query tokens.  Query t belongs to sequence q_seq[t] and sits at
 * position q_pos[t]; it sees positions 0 .. q_pos[t] (V_t = q_pos[t] + 1,
 * causal and inclusive).  Decode is one query per sequence at seq_len - 1;
 * chunked prefill is many queries of one sequence. */
typedef struct sa_query {
    int32_t n_q;
    const int32_t *q_seq;        /* device int32 [n_q] */
    const int32_t *q_pos;        /* device int32 [n_q] */
    int32_t max_visible;         /* host: an upper bound of q_pos[t] + 1 over all t */

    /* indexer query, same dtype as the cache's index keys */
    const void *q_index;         /* device [n_q, h_index, d_index] */
    const float *q_index_scale;  /* device SA_E4M3: fp32 [n_q, h_index], one per (token, head);
                                  * SA_MXFP8: E8M0 bytes [n_q, h_index, d_index / 32] */
    const float *w;              /* device [n_q, h_index] head weights */
    int32_t h_index;

    /* absorbed MLA attention query */
    sa_dtype q_dtype;            /* SA_BF16 or SA_F32 */
    const void *q;               /* device [n_q, heads, d_latent + d_rope] */
    int32_t heads;
    float sm_scale;              /* softmax scale applied to q . kv */

    /* A promise for chunked prefill: queries 4i .. 4i+3 belong to one sequence
     * (the last group may be shorter).  Any value but 4 makes no promise;
     * negative values are rejected.  With 4 and e4m3 index keys, the indexer scores
     * each group against every key tile once (the tile shared by the four
     * queries); a group that breaks the promise is skipped and reported as
     * SA_DETAIL_BAD_POSITION. */
    int32_t q_group;
} sa_query;

/* Which entry point a workspace is sized for. */
enum {
    SA_WS_INDEXER = 1,
    SA_WS_TOPK = 2,
    SA_WS_ATTN = 4,
    SA_WS_DECODE = 8,
    SA_WS_APPEND = 16             /* sa_append_tokens alone: `query` may be NULL */
};

/* Bytes of device workspace the entry points in `uses` (an OR of SA_WS_*)
 * need for this cache/query/K.  Returns 0 if the arguments are invalid.  The
 * workspace must be 256-byte aligned; its contents need no initialisation and
 * are overwritten by every call.  Calls that share a workspace must be
 * ordered (same stream, or synchronised). */
SA_API size_t sa_workspace_size(const sa_cache *cache, const sa_query *query, int32_t top_k,
                         int32_t uses);

/* Step 1 -- indexer scores ("Optimizing Next-Gen LLM Inference" §3.1:
 * relevance scoring and head-weight weighting; "Inference Acceleration for New
 * Large Model Architectures" §3.1 steps 1-2).
 * Writes scores[t * ld_scores + s] (fp32) for every s < q_pos[t] + 1; other
 * entries are left untouched.  ld_scores >= query->max_visible. */
SA_API sa_status sa_indexer_score(const sa_cache *cache, const sa_query *query, float *scores,
                           int64_t ld_scores, void *workspace, size_t workspace_bytes,
                           void *stream);

/* Step 2 -- top-K ("Optimizing Next-Gen LLM Inference" §3.1 Top-K selection;
 * "Inference Acceleration" §3.1 step 3).
 * For each row t of scores (fp32 [n_q, ld_scores], first valid_len[t] entries
 * valid): writes idx[t * top_k .. +top_k) = the min(top_k, valid_len[t])
 * positions with the largest scores, ties broken towards the lower position,
 * in ascending position order, padded with -1.  Bit-exact.
 * valid_len: device int32 [n_q]; max_valid: host bound on valid_len. */
SA_API sa_status sa_topk(const float *scores, int64_t ld_scores, const int32_t *valid_len,
                  int32_t n_q, int32_t max_valid, int32_t top_k, int32_t *idx,
                  void *workspace, size_t workspace_bytes, void *stream);

/* Step 3 -- sparse MLA attention over the selected rows ("Optimizing Next-Gen
 * LLM Inference" §3.3; "Inference Acceleration" §3.2).
 * idx: device int32 [n_q, top_k] logical positions (ascending not required;
 * -1 entries are skipped).  For each query t and head h:
 *   z_s = sm_scale * q[t,h,:] . kv[s,:]   (latent + rope; an e4m3 latent is
 *                                          scaled by its page-tile scale)
 *   out[t,h,:] = sum_s softmax(z)_s * kv[s, 0:d_latent],  lse[t,h] = log sum_s exp(z_s)
 * out: device [n_q, heads, d_latent] in out_dtype (SA_BF16 or SA_F32);
 * lse: device fp32 [n_q, heads] (may be NULL).  A query with no valid index
 * gets out = 0 and lse = -inf. */
SA_API sa_status sa_sparse_mla_attn(const sa_cache *cache, const sa_query *query, const int32_t *idx,
                             int32_t top_k, void *out, sa_dtype out_dtype, float *lse,
                             void *workspace, size_t workspace_bytes, void *stream);

/* Steps 1-3 fused for decode and chunked prefill ("Optimizing Next-Gen LLM
 * Inference" §3.1: scoring, weighting and selection without writing
 * intermediates back; "Inference Acceleration" §3.1).
 * The only intermediate that reaches device memory is what the top-K needs.
 * idx_out (device int32 [n_q, top_k]) may be NULL; when given it receives the
 * selected positions exactly as sa_topk would return them. */
SA_API sa_status sa_decode(const sa_cache *cache, const sa_query *query, int32_t top_k,
                    int32_t *idx_out, void *out, sa_dtype out_dtype, float *lse,
                    void *workspace, size_t workspace_bytes, void *stream);

/* sa_decode with phase timing: when `phase_events` is non-NULL it points to
 * SA_DECODE_PHASES + 1 cudaEvent_t handles (created by the caller), which are
 * recorded on `stream` before the first phase and after each phase, so that
 * cudaEventElapsedTime between neighbours gives each phase's device time.
 * Phases: indexer, top-K, sparse attention. */
#define SA_DECODE_PHASES 3
SA_API sa_status sa_decode_traced(const sa_cache *cache, const sa_query *query, int32_t top_k,
                                  int32_t *idx_out, void *out, sa_dtype out_dtype, float *lse,
                                  void *workspace, size_t workspace_bytes, void *stream,
                                  void *const *phase_events);

/* sa_decode for callers that cannot allocate device memory -- e.g. a plugin
 * whose host application owns every device allocation, a pool with a hard cap
 * this library may not grow, or a latency-critical loop where cudaMalloc
 * (which can synchronise the device) is not allowed.  The paper has no
 * counterpart; this entry point only serves such deployments.
 * Same arguments and results as sa_decode, without a workspace: the scratch
 * lives in a static device array of SA_NOALLOC_SCRATCH_BYTES that every
 * device loading this library holds until the process exits.  The call
 * allocates nothing.
 *  - Requests needing more scratch than that (sa_workspace_size(...,
 *    SA_WS_DECODE) > SA_NOALLOC_SCRATCH_BYTES) return SA_ERR_WORKSPACE and
 *    launch nothing.
 *  - The first call on a device looks the array's address up with that
 *    device current; make it before any stream capture.  The address is
 *    kept per device and CUDA context, so a call after cudaDeviceReset looks
 *    it up again (that call, too, belongs before any capture).
 *  - All calls on a device share the array: calls whose GPU work overlaps
 *    race and must not be issued.  The device status word of these calls
 *    lives in the array: read it with sa_noalloc_status(). */
#define SA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
SA_API sa_status sa_decode_noalloc(const sa_cache *cache, const sa_query *query, int32_t top_k,
                                   int32_t *idx_out, void *out, sa_dtype out_dtype, float *lse,
                                   void *stream);

/* Device-side status of the most recent sa_decode_noalloc call on the current
 * device: what sa_device_status reports for a workspace, read from the status
 * word at the start of the static array.  Synchronises `stream`; allocates
 * nothing.  *detail (may be NULL) receives an SA_DETAIL_* code. */
SA_API sa_status sa_noalloc_status(void *stream, int32_t *detail);

/* ---- Context parallelism across GPUs -------------------------------------
 * One long sequence split along its context over G GPUs ("Inference
 * Acceleration for New Large Model Architectures" §5.1-5.2: each device
 * handles a contiguous portion of the sequence; "Long-Context LLM Inference
 * Optimization", Distributed Scaling).  Rank r holds positions
 * [lo_r, hi_r) of each sequence in its own paged caches, as local positions
 * 0 .. hi_r - lo_r - 1, with lo_0 = 0 and hi_r = lo_{r+1}.  A decode step:
 *   1. sa_local_candidates on every rank (its shard, its query positions
 *      clamped to the shard: the last local position for decode);
 *   2. all-gather of the candidates (the caller's collective) into
 *      [G, n_q, top_k], rank-major;
 *   3. sa_merge_candidates on every rank: the same global top-K everywhere,
 *      and the part this rank holds, as local positions;
 *   4. sa_sparse_mla_attn on every rank over its local part, fp32 output;
 *   5. all-gather of those outputs and lse into [G, n_q, heads, d] / [G, n_q,
 *      heads]; 6. sa_combine_partials.
 * Positions selected match the single-GPU sa_decode exactly (the scores of a
 * position do not depend on the shard); the output differs by the rounding
 * of the merge. */

/* Step 1: this rank's top_k by the fused indexer + top-K, as
 * cand_score (device fp32 [n_q, top_k]) and cand_pos (device int32 [n_q,
 * top_k]) = local position + position_offset[t] (device int32 [n_q]: the
 * shard's lo for query t's sequence), ascending, padded with (-inf, -1).
 * Workspace as for sa_decode (SA_WS_DECODE). */
SA_API sa_status sa_local_candidates(const sa_cache *cache, const sa_query *query, int32_t top_k,
                                     const int32_t *position_offset, float *cand_score,
                                     int32_t *cand_pos, void *workspace, size_t workspace_bytes,
                                     void *stream);

/* Step 3: cand_score / cand_pos are device [n_ranks, n_q, top_k] as step 1
 * wrote them on each rank, rank r's block r-th.  Per query the top_k
 * candidates by score (ties to the lower position; padding last) go to
 * idx_global (device int32 [n_q, top_k], ascending, -1 padded); idx_local
 * (same shape) holds position - pos_lo[t] where pos_lo[t] <= position <
 * pos_hi[t] (device int32 [n_q]: this rank's shard of query t's sequence),
 * else -1.  n_ranks * top_k <= 24576.  No workspace. */
SA_API sa_status sa_merge_candidates(const float *cand_score, const int32_t *cand_pos,
                                     int32_t n_ranks, int32_t n_q, int32_t top_k,
                                     const int32_t *pos_lo, const int32_t *pos_hi,
                                     int32_t *idx_global, int32_t *idx_local, void *stream);

/* Step 6: o_part device fp32 [n_parts, n_q, heads, d], lse_part device fp32
 * [n_parts, n_q, heads] (natural log; -inf for a part with no selected row)
 * -> out [n_q, heads, d] in out_dtype (SA_BF16 or SA_F32) and lse [n_q,
 * heads] (may be NULL): out = sum_r exp(lse_r - lse) o_r, lse = log sum_r
 * exp(lse_r).  n_parts <= 256.  No workspace. */
SA_API sa_status sa_combine_partials(const float *o_part, const float *lse_part, int32_t n_parts,
                                     int32_t n_q, int32_t heads, int32_t d, void *out,
                                     sa_dtype out_dtype, float *lse, void *stream);

/* ---- Input preparation -------------------------------------------------
 * Before the indexer runs, the query is quantised and the step's new tokens
 * are written into the paged caches ("Optimizing Next-Gen LLM Inference"
 * §3.2 input preparation and the §4 table; "Inference Acceleration for New
 * Large Model Architectures" §3.3 and §4.1-4.2).  Projections and key
 * normalisation stay with the caller (they need the model's weights); these
 * calls take their bf16 or fp32 outputs.
 *
 * FP8 rule, per group of values, in fp32: amax = max |x|, scale = amax / 448
 * (1 for an all-zero group), code = e4m3(x / scale) with an IEEE
 * round-to-nearest division, rounded to nearest even and saturated to +-448.
 * Inputs must be finite: a NaN or infinity gives unspecified codes. */

/* Indexer query -> e4m3 codes + one fp32 scale per (token, head): the form
 * sa_query.q_index / q_index_scale take for an SA_E4M3 index cache.
 *   q_in:    device [n_q, h_index, d_index] in in_dtype (SA_BF16 or SA_F32)
 *   q_out:   device uint8 [n_q, h_index, d_index]
 *   q_scale: device fp32 [n_q, h_index]
 * Needs no workspace and cannot fail on the device. */
SA_API sa_status sa_quantize_index_query(const void *q_in, sa_dtype in_dtype, int32_t n_q,
                                         int32_t h_index, int32_t d_index, void *q_out,
                                         float *q_scale, void *stream);

/* New tokens of one step: token i belongs to sequence seq[i] at logical
 * position pos[i]. */
typedef struct sa_new_tokens {
    int32_t n_new;
    const int32_t *seq;          /* device int32 [n_new] */
    const int32_t *pos;          /* device int32 [n_new] */
    sa_dtype in_dtype;           /* SA_BF16 or SA_F32, for both inputs below */
    const void *k_index;         /* device [n_new, d_index] index keys, or NULL (not written) */
    const void *kv;              /* device [n_new, d_latent + d_rope] latent + rope rows,
                                  * or NULL (not written) */
} sa_new_tokens;

/* Writes each new token into the pools of `cache` at its physical row
 * (page_table[seq * max_pages + pos / page_size] * page_size + pos % page_size):
 *  - index key: SA_E4M3 pool -> codes + the token's scale (one group of
 *    d_index values); SA_F32 pool -> the values;
 *  - latent row: SA_BF16 / SA_F32 pool -> the row (fp32 inputs rounded to
 *    nearest even for bf16); SA_E4M3 pool -> the latent quantised in groups of
 *    kv_scale_dims values with its scales, the rope as bf16.  An SA_E4M3 pool
 *    needs kv_scale_tokens == 1: a scale shared by several tokens would force
 *    the others to be requantised, so other tiles return SA_ERR_UNSUPPORTED.
 * The pools named by `cache` (k_index, k_index_scale, kv, kv_rope, kv_scale)
 * are written in place and must be writable device memory; seq_len is neither
 * read nor changed (the caller advances it), so a position is not checked
 * against it: appending at seq_len[seq] before advancing it is the normal use.
 * Tokens must not share a row: two tokens with the same (seq, pos), or whose
 * page-table entries point at the same page, are written by two CTAs at once,
 * and the row may end up with codes of one token and the scale of the other.
 * The call does not detect such a batch.
 * A token whose sequence is outside [0, batch), whose position is negative or
 * at or past max_pages * page_size, or whose page-table entry is outside
 * [0, num_pages) is skipped and recorded in the workspace status word
 * (SA_DETAIL_BAD_POSITION / SA_DETAIL_BAD_PAGE; read it with
 * sa_device_status).  workspace: at least
 * sa_workspace_size(cache, NULL, 0, SA_WS_APPEND) bytes, 256-byte aligned. */
SA_API sa_status sa_append_tokens(const sa_cache *cache, const sa_new_tokens *tokens,
                                  void *workspace, size_t workspace_bytes, void *stream);

/* Device-side status of the most recent call that used `workspace`.
 * Synchronises `stream`.  Returns SA_OK, SA_ERR_DEVICE_FAULT or
 * SA_ERR_TIMEOUT; *detail (may be NULL) receives an SA_DETAIL_* code. */
enum {
    SA_DETAIL_NONE = 0,
    SA_DETAIL_BAD_PAGE = 1,       /* page id outside [0, num_pages) */
    SA_DETAIL_BAD_POSITION = 2,   /* q_pos >= seq_len, or q_seq outside [0, batch) */
    SA_DETAIL_BAD_INDEX = 3,      /* selected index outside [0, q_pos] */
    SA_DETAIL_WAIT_TIMEOUT = 4    /* a bounded wait inside a kernel gave up */
};
SA_API sa_status sa_device_status(const void *workspace, size_t workspace_bytes, void *stream,
                           int32_t *detail);

/* Number of CUDA kernels this library has launched in this process so far
 * (all devices, all threads).  For tracing: the difference across a region
 * is the number of library kernels enqueued in it. */
SA_API uint64_t sa_kernel_launches(void);

/* Human-readable name of a status code (static storage). */
SA_API const char *sa_status_string(sa_status status);

/* Library version: major * 10000 + minor * 100 + patch. */
SA_API int32_t sa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SA_H */
