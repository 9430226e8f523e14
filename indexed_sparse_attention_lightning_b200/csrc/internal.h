// internal.h -- parameter blocks and launchers shared between the host API
// (sa_api.cu) and the kernel files.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <utility>

#include "sa.h"

namespace sa {

// Launches `kernel` with programmatic stream serialization, so that its
// launch overlaps the tail of the previous kernel in the stream (the kernel
// itself calls pdl_wait before touching anything that kernel wrote).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args &&...args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}


// Everything a kernel needs to know about the paged caches and the queries.
struct PathParams {
    // paging
    const int32_t *page_table;
    const int32_t *seq_len;
    int32_t batch, max_pages, num_pages;
    // indexer keys
    const void *k_index;
    const float *k_index_scale;
    int32_t d_index;
    int32_t index_dtype;  // sa_dtype: SA_E4M3, SA_BF16 (unscaled) or SA_F32
    // latent cache
    const void *kv;
    const void *kv_rope;
    const float *kv_scale;
    int32_t d_latent, d_rope;
    int32_t kv_dtype;  // sa_dtype
    int32_t kv_scale_tokens, kv_scale_dims;  // e4m3 scale tile (resolved, > 0)
    // queries
    int32_t n_q;
    const int32_t *q_seq, *q_pos;
    int32_t max_visible;
    const void *q_index;
    const float *q_index_scale;
    const float *w;
    int32_t h_index;
    const void *q;
    int32_t q_dtype;  // sa_dtype
    int32_t heads;
    float sm_scale;
    int32_t q_group;  // queries in runs of this many of one sequence (4: chunked prefill)
    // status word (first 2 ints of the workspace)
    int32_t *status;
};

// Visible length of query t after validating its sequence and position
// against the cache; returns 0 (and reports) for an invalid query.
__device__ __forceinline__ int32_t visible_len(const PathParams &p, int32_t t);

// Count one kernel launch (see sa_kernel_launches).
void count_launch();

// SM count of the current device (cached).
int num_sms();

// 2-D TMA tensor map over a row-major [outer, inner] array (elements of
// dtype_bytes = 1 (u8), 2 (bf16) or 4 (f32)), box [box_outer, box_inner].
bool encode_tmap_2d(CUtensorMap *map, int dtype_bytes, const void *base, uint64_t inner,
                    uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                    uint32_t box_outer, bool swizzle128);

// ---- launchers (each returns the launch error, if any) --------------------
// Visible length per query and the inclusive prefix of ceil(V / tile); also
// zeroes `zero_words` 32-bit words at `zero` (histograms and counters) and,
// with `clear_status`, the status word before anything can report into it.
cudaError_t launch_plan(const PathParams &p, int32_t *vis, int32_t *tile_end, int32_t tile,
                        uint32_t *zero, size_t zero_words, bool clear_status, cudaStream_t s,
                        int32_t group = 1);

cudaError_t launch_indexer_simt(const PathParams &p, float *scores, int64_t ld, cudaStream_t s);

// Tensor-core FP8 indexer (e4m3 keys, 64 heads x 128 dims); needs the plan.
// indexer_query_group(p): how many consecutive queries share each key tile
// (4 for flagged chunked prefill with e4m3 keys, else 1); the plan's tile
// prefix must run over groups of that size.
bool indexer_mma_supported(const PathParams &p);
int32_t indexer_query_group(const PathParams &p);
cudaError_t launch_indexer_mma(const PathParams &p, const int32_t *vis, const int32_t *tile_end,
                               float *scores, int64_t ld, uint32_t *hist, cudaStream_t s);

// Row-wise exact top-K.  Row t has valid_len[t] entries, or q_pos[t] + 1 when
// valid_len is null (rows then validated as queries of `p`).
cudaError_t launch_topk_rowwise(const float *scores, int64_t ld, const int32_t *valid_len,
                                int32_t max_valid, const PathParams *p, int32_t n_q,
                                int32_t top_k, int32_t *idx, int32_t *status, cudaStream_t s);

// Histogram-guided exact top-K for rows scored by the tensor-core indexer
// (which filled `hist`, [n_q, kHistBins]).  Scratch: sel [n_q, top_k],
// counts [n_q, kTopkCountsPerQuery] (zeroed), cand [n_q, cap], chunk_info.
constexpr int32_t kTopkCandCap = 8192;
constexpr int32_t kTopkCountsPerQuery = 2;
// Rows longer than this many positions per chunk split into chunks; chunk_info
// [n_q, topk_chunk_slots(ld)] (int4) holds each chunk's list slots.
constexpr int32_t kTopkChunk = 8192;
inline int64_t topk_chunk_slots(int64_t ld) { return (ld + kTopkChunk - 1) / kTopkChunk; }
// With `rows` non-null it also writes the physical cache rows of the
// selection for the tensor-core attention (compact_rows layout, tile 64,
// leading dimension ld_rows) and their count n_valid [n_q].
cudaError_t launch_topk_hist(const float *scores, int64_t ld, const int32_t *vis,
                             const uint32_t *hist, int32_t n_q, int32_t max_valid, int32_t top_k,
                             int32_t *sel, int32_t *counts, uint64_t *cand, int32_t cap,
                             int4 *chunk_info, int32_t *idx, const PathParams &p, int32_t *rows,
                             int32_t ld_rows, int32_t *n_valid, cudaStream_t s);

cudaError_t launch_attn_simt(const PathParams &p, const int32_t *idx, int32_t top_k, void *out,
                             int32_t out_dtype, float *lse, cudaStream_t s);

// Tensor-core sparse attention (bf16 cache and query, 128 heads, 512 + 64
// dims, K <= 2048): a compaction kernel turns the selected positions into
// physical rows (rows [n_q, sfa_rows_ld(K)], n_valid [n_q]; skipped when
// `rows_ready`, i.e. the top-K kernel already wrote them), then one CTA per
// 64 heads of a query and key split; with `splits` > 1 the partial outputs go
// to o_part [n_q, splits, 128, 512] / lse_part [n_q, splits, 128] and a third
// kernel merges them.
bool sfa_mma_supported(const PathParams &p, int32_t top_k);
int32_t sfa_splits(int32_t n_q, int32_t top_k);
int32_t sfa_rows_ld(int32_t top_k);
cudaError_t launch_sfa_mma(const PathParams &p, const int32_t *idx, int32_t top_k, int32_t splits,
                           int32_t *rows, int32_t *n_valid, bool rows_ready, void *out,
                           int32_t out_dtype, float *lse, float *o_part, float *lse_part,
                           cudaStream_t s);

// Context-parallel decode steps (cp.cu).
int32_t cp_merge_max_candidates();
int32_t cp_combine_max_parts();
cudaError_t launch_cand_emit(const float *scores, int64_t ld, const int32_t *idx, int32_t n_q,
                             int32_t top_k, const int32_t *offset, float *cand_score,
                             int32_t *cand_pos, cudaStream_t s);
cudaError_t launch_cp_merge(const float *cand_score, const int32_t *cand_pos, int32_t n_ranks,
                            int32_t n_q, int32_t top_k, const int32_t *pos_lo,
                            const int32_t *pos_hi, int32_t *idx_global, int32_t *idx_local,
                            cudaStream_t s);
cudaError_t launch_cp_combine(const float *o_part, const float *lse_part, int32_t n_parts,
                              int64_t rows, int32_t d, void *out, int32_t out_dtype, float *lse,
                              cudaStream_t s);

}  // namespace sa

// ---- inline device definitions -------------------------------------------
#ifdef __CUDACC__
#include "common.cuh"
namespace sa {
__device__ __forceinline__ int32_t visible_len(const PathParams &p, int32_t t) {
    int32_t b = __ldg(p.q_seq + t);
    int32_t pos = __ldg(p.q_pos + t);
    if (b < 0 || b >= p.batch || pos < 0 || pos >= __ldg(p.seq_len + b) ||
        pos >= p.max_visible) {
        report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_POSITION);
        return 0;
    }
    return pos + 1;
}

// Scale of latent dim d of physical row `row` of the e4m3 cache: one fp32 per
// tile of kv_scale_tokens tokens x kv_scale_dims dims of a 64-token page,
// laid out [num_pages, 64 / kv_scale_tokens, d_latent / kv_scale_dims].
__device__ __forceinline__ float kv_scale_at(const PathParams &p, int64_t row, int32_t d) {
    const int64_t page = row >> 6;
    const int32_t tok = static_cast<int32_t>(row & 63);
    const int32_t tiles_t = 64 / p.kv_scale_tokens, tiles_d = p.d_latent / p.kv_scale_dims;
    return __ldg(p.kv_scale + (page * tiles_t + tok / p.kv_scale_tokens) * tiles_d +
                 d / p.kv_scale_dims);
}

// Physical cache rows of query t's selected positions sel[0, K): list order,
// -1 entries dropped, out-of-range positions and bad page ids skipped and
// reported; then padded with the first row up to a multiple of `tile`.
// Writes rows[0, padded) and *n_valid.  Called by every thread of a CTA
// (blockDim.x a multiple of 32); `scratch` is shared memory of 33 ints.
__device__ __forceinline__ void compact_rows(const PathParams &p, int32_t t, const int32_t *sel,
                                             int32_t K, int32_t tile, int32_t *rows,
                                             int32_t *n_valid, int32_t *scratch) {
    const int nwarps = blockDim.x >> 5, w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t V = visible_len(p, t);
    const int32_t seq = __ldg(p.q_seq + t);
    int32_t base = 0;
    for (int32_t r0 = 0; r0 < K; r0 += blockDim.x) {
        const int32_t k = r0 + threadIdx.x;
        const int32_t s = k < K ? sel[k] : -1;
        int32_t v = -1;
        if (s >= V) {
            report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_INDEX);
        } else if (s >= 0) {
            const int64_t row = phys_row(p.page_table, p.max_pages, p.num_pages, seq, s);
            if (row < 0) report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_PAGE);
            else v = static_cast<int32_t>(row);
        }
        const unsigned bal = __ballot_sync(0xffffffffu, v >= 0);
        if (lane == 0) scratch[w] = __popc(bal);
        __syncthreads();
        int32_t off = base, tot = 0;
        for (int i = 0; i < nwarps; ++i) {
            if (i < w) off += scratch[i];
            tot += scratch[i];
        }
        const int32_t pos = off + __popc(bal & ((1u << lane) - 1u));
        if (v >= 0) {
            rows[pos] = v;
            if (pos == 0) scratch[32] = v;
        }
        __syncthreads();
        base += tot;
    }
    const int32_t padded = (base + tile - 1) / tile * tile;
    if (base > 0)
        for (int32_t c = base + threadIdx.x; c < padded; c += blockDim.x) rows[c] = scratch[32];
    if (threadIdx.x == 0) *n_valid = base;
}
}  // namespace sa
#endif
