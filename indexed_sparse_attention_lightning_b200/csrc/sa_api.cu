// sa_api.cu -- the C ABI: host-side validation, workspace layout, dispatch.
//
// Every entry point checks its arguments before touching the device, then
// enqueues its kernels on the caller's stream without synchronising.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "prep.h"
#include "sa.h"

namespace sa {
static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
}  // namespace sa

namespace {
using namespace sa;

constexpr int32_t kPageSize = 64;
constexpr int32_t kMaxQueries = 65535;
constexpr int32_t kMaxTopK = 1 << 20;
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

sa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

sa_status check_cache(const sa_cache *c) {
    if (c == nullptr) return SA_ERR_INVALID_ARG;
    if (c->page_size != kPageSize) return SA_ERR_UNSUPPORTED;
    if (c->batch <= 0 || c->max_pages <= 0 || c->num_pages <= 0) return SA_ERR_INVALID_ARG;
    if (!c->page_table || !c->seq_len || !c->k_index || !c->kv) return SA_ERR_INVALID_ARG;
    if (!aligned16(c->k_index) || !aligned16(c->kv)) return SA_ERR_INVALID_ARG;
    if (c->index_dtype != SA_F32 && c->index_dtype != SA_BF16 && c->index_dtype != SA_E4M3 &&
        c->index_dtype != SA_MXFP8)
        return SA_ERR_UNSUPPORTED;
    const bool scaled = c->index_dtype == SA_E4M3 || c->index_dtype == SA_MXFP8;
    if (scaled && (!c->k_index_scale || !aligned16(c->k_index_scale))) return SA_ERR_INVALID_ARG;
    if (c->d_index <= 0 || c->d_index % 16 != 0) return SA_ERR_INVALID_ARG;
    if (c->index_dtype == SA_MXFP8 && c->d_index % 32 != 0) return SA_ERR_INVALID_ARG;
    if (c->d_index > 256) return SA_ERR_UNSUPPORTED;
    if (c->kv_dtype != SA_F32 && c->kv_dtype != SA_BF16 && c->kv_dtype != SA_E4M3)
        return SA_ERR_UNSUPPORTED;  // SA_MXFP8 names index data only
    if (c->d_latent <= 0 || c->d_rope < 0) return SA_ERR_INVALID_ARG;
    if (c->d_latent > 512 || c->d_latent + c->d_rope > 1024) return SA_ERR_UNSUPPORTED;
    if (c->kv_dtype == SA_E4M3) {
        if (!c->kv_scale || (c->d_rope > 0 && !c->kv_rope)) return SA_ERR_INVALID_ARG;
        if (c->kv_rope && !aligned16(c->kv_rope)) return SA_ERR_INVALID_ARG;
        const bool page_tile = c->kv_scale_tokens == 0 && c->kv_scale_dims == 0;
        if (!page_tile) {
            if (c->kv_scale_tokens <= 0 || c->kv_scale_dims <= 0) return SA_ERR_INVALID_ARG;
            if (c->page_size % c->kv_scale_tokens != 0 || c->d_latent % c->kv_scale_dims != 0 ||
                c->kv_scale_dims % 16 != 0)
                return SA_ERR_UNSUPPORTED;
        }
    }
    return SA_OK;
}

sa_status check_query(const sa_query *q, const sa_cache *c, bool need_index, bool need_attn) {
    if (q == nullptr) return SA_ERR_INVALID_ARG;
    if (q->n_q < 0) return SA_ERR_INVALID_ARG;
    if (q->n_q > kMaxQueries) return SA_ERR_UNSUPPORTED;
    if (q->n_q == 0) return SA_OK;
    if (!q->q_seq || !q->q_pos || q->max_visible <= 0) return SA_ERR_INVALID_ARG;
    if ((int64_t)q->max_visible > (int64_t)c->max_pages * c->page_size) return SA_ERR_INVALID_ARG;
    if (need_index) {
        if (!q->q_index || !q->w || q->h_index <= 0) return SA_ERR_INVALID_ARG;
        if (q->h_index > 128) return SA_ERR_UNSUPPORTED;
        if (q->q_group < 0) return SA_ERR_INVALID_ARG;
        if ((c->index_dtype == SA_E4M3 || c->index_dtype == SA_MXFP8) && !q->q_index_scale)
            return SA_ERR_INVALID_ARG;
        if (c->index_dtype == SA_MXFP8 && !aligned16(q->q_index_scale)) return SA_ERR_INVALID_ARG;
    }
    if (need_attn) {
        if (!q->q || q->heads <= 0) return SA_ERR_INVALID_ARG;
        if (q->q_dtype != SA_F32 && q->q_dtype != SA_BF16) return SA_ERR_UNSUPPORTED;
        if (!std::isfinite(q->sm_scale)) return SA_ERR_INVALID_ARG;
    }
    return SA_OK;
}

PathParams make_params(const sa_cache *c, const sa_query *q, void *ws) {
    PathParams p{};
    p.page_table = c->page_table;
    p.seq_len = c->seq_len;
    p.batch = c->batch;
    p.max_pages = c->max_pages;
    p.num_pages = c->num_pages;
    p.k_index = c->k_index;
    p.k_index_scale = c->k_index_scale;
    p.d_index = c->d_index;
    p.index_dtype = c->index_dtype;
    p.kv = c->kv;
    p.kv_rope = c->kv_rope;
    p.kv_scale = c->kv_scale;
    p.d_latent = c->d_latent;
    p.d_rope = c->d_rope;
    p.kv_dtype = c->kv_dtype;
    const bool page_tile = c->kv_scale_tokens == 0 && c->kv_scale_dims == 0;
    p.kv_scale_tokens = page_tile ? c->page_size : c->kv_scale_tokens;
    p.kv_scale_dims = page_tile ? c->d_latent : c->kv_scale_dims;
    p.n_q = q->n_q;
    p.q_seq = q->q_seq;
    p.q_pos = q->q_pos;
    p.max_visible = q->max_visible;
    p.q_index = q->q_index;
    p.q_index_scale = q->q_index_scale;
    p.w = q->w;
    p.h_index = q->h_index;
    p.q = q->q;
    p.q_dtype = q->q_dtype;
    p.heads = q->heads;
    p.sm_scale = q->sm_scale;
    p.q_group = q->q_group;
    p.status = static_cast<int32_t *>(ws);
    return p;
}

// Workspace: status | vis [n_q] | tile_end [n_q] | scores [n_q, ld] | idx [n_q, K]
// | hist [n_q, 4096] | counts [n_q, 2] | sel [n_q, K] | cand [n_q, cap]
// | chunk_info [n_q, C] | rows [n_q, R] | n_valid [n_q] | o_part [n_q, S, 128, 512]
// | lse_part [n_q, S, 128]; the indexer needs the first three, the fused path
// all of them; the attention alone needs the status, the compacted rows and
// the split-KV partials (placed right after the status).
struct Layout {
    int64_t ld;
    int32_t splits;
    size_t vis, tile_end, scores, idx, hist, counts, sel, cand, chunk_info, rows, n_valid, o_part,
        lse_part;
    size_t indexer_total, decode_total;
    size_t attn_rows, attn_n_valid, attn_o_part, attn_lse_part, attn_total;
};

size_t part_bytes(size_t nq, int32_t splits, size_t per) {
    return splits > 1 ? per * nq * (size_t)splits : 0;
}

Layout make_layout(const sa_query *q, int32_t top_k) {
    Layout l{};
    const size_t nq = q->n_q > 0 ? (size_t)q->n_q : 0;
    l.ld = round_up(q->max_visible > 0 ? q->max_visible : 1, 128);
    l.splits = sfa_splits(q->n_q, top_k > 0 ? top_k : 1);
    const size_t o_bytes = part_bytes(nq, l.splits, sizeof(float) * 128 * 512);
    const size_t lse_bytes = part_bytes(nq, l.splits, sizeof(float) * 128);
    l.vis = align_up(kStatusBytes);
    l.tile_end = align_up(l.vis + sizeof(int32_t) * nq);
    l.indexer_total = align_up(l.tile_end + sizeof(int32_t) * nq);
    l.scores = l.indexer_total;
    const size_t kk = top_k > 0 ? (size_t)top_k : 0;
    l.idx = align_up(l.scores + sizeof(float) * nq * (size_t)l.ld);
    l.hist = align_up(l.idx + sizeof(int32_t) * nq * kk);
    l.counts = align_up(l.hist + sizeof(uint32_t) * nq * kHistBins);  // follows hist: one clear
    l.sel = align_up(l.counts + sizeof(int32_t) * kTopkCountsPerQuery * nq);
    l.cand = align_up(l.sel + sizeof(int32_t) * nq * kk);
    const size_t rows_bytes = sizeof(int32_t) * nq * (size_t)sfa_rows_ld(top_k);
    l.chunk_info = align_up(l.cand + sizeof(uint64_t) * nq * kTopkCandCap);
    l.rows = align_up(l.chunk_info + sizeof(int4) * nq * (size_t)topk_chunk_slots(l.ld));
    l.n_valid = align_up(l.rows + rows_bytes);
    l.o_part = align_up(l.n_valid + sizeof(int32_t) * nq);
    l.lse_part = align_up(l.o_part + o_bytes);
    l.decode_total = align_up(l.lse_part + lse_bytes);
    l.attn_rows = align_up(kStatusBytes);
    l.attn_n_valid = align_up(l.attn_rows + rows_bytes);
    l.attn_o_part = align_up(l.attn_n_valid + sizeof(int32_t) * nq);
    l.attn_lse_part = align_up(l.attn_o_part + o_bytes);
    l.attn_total = align_up(l.attn_lse_part + lse_bytes);
    return l;
}

// Sparse attention: the tensor-core kernel for its shape, CUDA cores otherwise.
sa_status run_attention(const PathParams &p, const Layout &l, bool fused, bool rows_ready,
                        void *ws, const int32_t *idx, int32_t top_k, void *out,
                        int32_t out_dtype, float *lse, cudaStream_t s) {
    if (sfa_mma_supported(p, top_k)) {
        char *base = static_cast<char *>(ws);
        return cuda_status(launch_sfa_mma(
            p, idx, top_k, l.splits,
            reinterpret_cast<int32_t *>(base + (fused ? l.rows : l.attn_rows)),
            reinterpret_cast<int32_t *>(base + (fused ? l.n_valid : l.attn_n_valid)), rows_ready,
            out, out_dtype, lse, reinterpret_cast<float *>(base + (fused ? l.o_part : l.attn_o_part)),
            reinterpret_cast<float *>(base + (fused ? l.lse_part : l.attn_lse_part)), s));
    }
    return cuda_status(launch_attn_simt(p, idx, top_k, out, out_dtype, lse, s));
}

// Indexer scores into `scores` (ld): the tensor-core kernel for its shape,
// the CUDA-core kernel otherwise.  With `want_hist` (fused path) the
// tensor-core kernel also fills the per-query score histograms, which the
// plan kernel clears first together with the counters behind them;
// *have_hist reports whether they were built.
sa_status clear_status(void *ws, cudaStream_t s);

// With `clear`, the status word is cleared first: by the plan kernel when
// there is one (saving a separate memset in front of it), else by a memset.
sa_status run_indexer(const PathParams &p, const Layout &l, void *ws, float *scores, int64_t ld,
                      bool want_hist, bool clear, bool *have_hist, cudaStream_t s) {
    *have_hist = false;
    if (indexer_mma_supported(p)) {
        char *base = static_cast<char *>(ws);
        int32_t *vis = reinterpret_cast<int32_t *>(base + l.vis);
        int32_t *tile_end = reinterpret_cast<int32_t *>(base + l.tile_end);
        uint32_t *hist = want_hist ? reinterpret_cast<uint32_t *>(base + l.hist) : nullptr;
        const size_t zero_words = want_hist ? (l.sel - l.hist) / 4 : 0;
        sa_status st = cuda_status(launch_plan(p, vis, tile_end, 128, hist, zero_words, clear, s,
                                               indexer_query_group(p)));
        if (st != SA_OK) return st;
        st = cuda_status(launch_indexer_mma(p, vis, tile_end, scores, ld, hist, s));
        *have_hist = want_hist && st == SA_OK;
        return st;
    }
    if (clear) {
        const sa_status st = clear_status(ws, s);
        if (st != SA_OK) return st;
    }
    return cuda_status(launch_indexer_simt(p, scores, ld, s));
}

sa_status check_workspace(void *ws, size_t bytes, size_t need) {
    if (ws == nullptr || bytes < need) return SA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return SA_ERR_WORKSPACE;
    return SA_OK;
}

sa_status clear_status(void *ws, cudaStream_t s) {
    return cuda_status(cudaMemsetAsync(ws, 0, kStatusBytes, s));
}

}  // namespace

extern "C" {

size_t sa_workspace_size(const sa_cache *cache, const sa_query *query, int32_t top_k,
                         int32_t uses) {
    if (check_cache(cache) != SA_OK) return 0;
    if (uses == SA_WS_APPEND) return align_up(kStatusBytes);
    const bool idx = (uses & (SA_WS_INDEXER | SA_WS_DECODE)) != 0;
    const bool att = (uses & (SA_WS_ATTN | SA_WS_DECODE)) != 0;
    if (check_query(query, cache, idx, att) != SA_OK) return 0;
    if ((uses & (SA_WS_TOPK | SA_WS_DECODE | SA_WS_ATTN)) && (top_k <= 0 || top_k > kMaxTopK))
        return 0;
    const Layout l = make_layout(query, top_k);
    size_t need = kStatusBytes;
    if (uses & SA_WS_INDEXER) need = std::max(need, l.indexer_total);
    if (uses & SA_WS_ATTN) need = std::max(need, l.attn_total);
    if (uses & SA_WS_DECODE) need = std::max(need, l.decode_total);
    return align_up(need);
}

sa_status sa_indexer_score(const sa_cache *cache, const sa_query *query, float *scores,
                           int64_t ld_scores, void *workspace, size_t workspace_bytes,
                           void *stream) {
    sa_status st = check_cache(cache);
    if (st != SA_OK) return st;
    if ((st = check_query(query, cache, true, false)) != SA_OK) return st;
    if (query->n_q > 0 && (!scores || ld_scores < query->max_visible)) return SA_ERR_INVALID_ARG;
    const Layout l = make_layout(query, 1);
    if ((st = check_workspace(workspace, workspace_bytes, l.indexer_total)) != SA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = clear_status(workspace, s)) != SA_OK) return st;
    if (query->n_q == 0) return SA_OK;
    PathParams p = make_params(cache, query, workspace);
    bool have_hist;
    return run_indexer(p, l, workspace, scores, ld_scores, false, false, &have_hist, s);
}

sa_status sa_topk(const float *scores, int64_t ld_scores, const int32_t *valid_len, int32_t n_q,
                  int32_t max_valid, int32_t top_k, int32_t *idx, void *workspace,
                  size_t workspace_bytes, void *stream) {
    if (n_q < 0 || top_k <= 0 || top_k > kMaxTopK) return SA_ERR_INVALID_ARG;
    if (n_q > kMaxQueries) return SA_ERR_UNSUPPORTED;
    if (n_q > 0 && (!scores || !valid_len || !idx || max_valid < 0 || ld_scores < max_valid))
        return SA_ERR_INVALID_ARG;
    sa_status st = check_workspace(workspace, workspace_bytes, kStatusBytes);
    if (st != SA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = clear_status(workspace, s)) != SA_OK) return st;
    return cuda_status(launch_topk_rowwise(scores, ld_scores, valid_len, max_valid, nullptr, n_q,
                                           top_k, idx, static_cast<int32_t *>(workspace), s));
}

sa_status sa_sparse_mla_attn(const sa_cache *cache, const sa_query *query, const int32_t *idx,
                             int32_t top_k, void *out, sa_dtype out_dtype, float *lse,
                             void *workspace, size_t workspace_bytes, void *stream) {
    sa_status st = check_cache(cache);
    if (st != SA_OK) return st;
    if ((st = check_query(query, cache, false, true)) != SA_OK) return st;
    if (top_k <= 0 || top_k > kMaxTopK) return SA_ERR_INVALID_ARG;
    if (out_dtype != SA_BF16 && out_dtype != SA_F32) return SA_ERR_UNSUPPORTED;
    if (query->n_q > 0 && (!idx || !out)) return SA_ERR_INVALID_ARG;
    const Layout l = make_layout(query, top_k);
    if ((st = check_workspace(workspace, workspace_bytes, l.attn_total)) != SA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = clear_status(workspace, s)) != SA_OK) return st;
    if (query->n_q == 0) return SA_OK;
    PathParams p = make_params(cache, query, workspace);
    return run_attention(p, l, false, false, workspace, idx, top_k, out, out_dtype, lse, s);
}

// Where sa_local_candidates wants the selection: (score, position + offset).
struct CandOut {
    const int32_t *offset;  // device [n_q]
    float *score;
    int32_t *pos;
};

static sa_status decode_impl(const sa_cache *cache, const sa_query *query, int32_t top_k,
                             int32_t *idx_out, void *out, sa_dtype out_dtype, float *lse,
                             void *workspace, size_t workspace_bytes, void *stream,
                             void *const *events, const CandOut *cand = nullptr) {
    sa_status st = check_cache(cache);
    if (st != SA_OK) return st;
    if ((st = check_query(query, cache, true, true)) != SA_OK) return st;
    if (top_k <= 0 || top_k > kMaxTopK) return SA_ERR_INVALID_ARG;
    if (out_dtype != SA_BF16 && out_dtype != SA_F32) return SA_ERR_UNSUPPORTED;
    if (query->n_q > 0 && !out && !cand) return SA_ERR_INVALID_ARG;
    const Layout l = make_layout(query, top_k);
    if ((st = check_workspace(workspace, workspace_bytes, l.decode_total)) != SA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto mark = [&](int i) -> sa_status {
        if (events == nullptr) return SA_OK;
        return cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s));
    };
    if (query->n_q == 0 && (st = clear_status(workspace, s)) != SA_OK) return st;
    if ((st = mark(0)) != SA_OK) return st;
    if (query->n_q > 0) {
        PathParams p = make_params(cache, query, workspace);
        char *base = static_cast<char *>(workspace);
        float *scores = reinterpret_cast<float *>(base + l.scores);
        int32_t *idx = idx_out ? idx_out : reinterpret_cast<int32_t *>(base + l.idx);
        bool have_hist = false;
        if ((st = run_indexer(p, l, workspace, scores, l.ld, true, true, &have_hist, s)) != SA_OK)
            return st;
        if ((st = mark(1)) != SA_OK) return st;
        // the top-K kernel also emits the physical rows for the tensor-core attention
        const bool rows_ready = have_hist && sfa_mma_supported(p, top_k);
        if (have_hist) {
            st = cuda_status(launch_topk_hist(
                scores, l.ld, reinterpret_cast<const int32_t *>(base + l.vis),
                reinterpret_cast<const uint32_t *>(base + l.hist), query->n_q, query->max_visible,
                top_k, reinterpret_cast<int32_t *>(base + l.sel),
                reinterpret_cast<int32_t *>(base + l.counts),
                reinterpret_cast<uint64_t *>(base + l.cand), kTopkCandCap,
                reinterpret_cast<int4 *>(base + l.chunk_info), idx, p,
                rows_ready ? reinterpret_cast<int32_t *>(base + l.rows) : nullptr,
                sfa_rows_ld(top_k),
                rows_ready ? reinterpret_cast<int32_t *>(base + l.n_valid) : nullptr, s));
        } else {
            st = cuda_status(launch_topk_rowwise(scores, l.ld, nullptr, query->max_visible, &p,
                                                 query->n_q, top_k, idx, p.status, s));
        }
        if (st != SA_OK) return st;
        if (cand != nullptr)  // this GPU's candidates for a context-parallel merge
            return cuda_status(launch_cand_emit(scores, l.ld, idx, query->n_q, top_k, cand->offset,
                                                cand->score, cand->pos, s));
        if ((st = mark(2)) != SA_OK) return st;
        if ((st = run_attention(p, l, true, rows_ready, workspace, idx, top_k, out, out_dtype,
                                lse, s)) != SA_OK)
            return st;
        return mark(3);
    }
    for (int i = 1; i <= SA_DECODE_PHASES; ++i)
        if ((st = mark(i)) != SA_OK) return st;
    return SA_OK;
}

sa_status sa_decode(const sa_cache *cache, const sa_query *query, int32_t top_k,
                    int32_t *idx_out, void *out, sa_dtype out_dtype, float *lse,
                    void *workspace, size_t workspace_bytes, void *stream) {
    return decode_impl(cache, query, top_k, idx_out, out, out_dtype, lse, workspace,
                       workspace_bytes, stream, nullptr);
}

sa_status sa_decode_traced(const sa_cache *cache, const sa_query *query, int32_t top_k,
                           int32_t *idx_out, void *out, sa_dtype out_dtype, float *lse,
                           void *workspace, size_t workspace_bytes, void *stream,
                           void *const *phase_events) {
    return decode_impl(cache, query, top_k, idx_out, out, out_dtype, lse, workspace,
                       workspace_bytes, stream, phase_events);
}

sa_status sa_local_candidates(const sa_cache *cache, const sa_query *query, int32_t top_k,
                              const int32_t *position_offset, float *cand_score,
                              int32_t *cand_pos, void *workspace, size_t workspace_bytes,
                              void *stream) {
    if (query != nullptr && query->n_q > 0 && (!cand_score || !cand_pos || !position_offset))
        return SA_ERR_INVALID_ARG;
    const CandOut cand{position_offset, cand_score, cand_pos};
    return decode_impl(cache, query, top_k, nullptr, nullptr, SA_BF16, nullptr, workspace,
                       workspace_bytes, stream, nullptr, &cand);
}

sa_status sa_merge_candidates(const float *cand_score, const int32_t *cand_pos, int32_t n_ranks,
                              int32_t n_q, int32_t top_k, const int32_t *pos_lo,
                              const int32_t *pos_hi, int32_t *idx_global, int32_t *idx_local,
                              void *stream) {
    if (n_ranks <= 0 || n_q < 0 || top_k <= 0) return SA_ERR_INVALID_ARG;
    if (n_q > kMaxQueries) return SA_ERR_UNSUPPORTED;
    if ((int64_t)n_ranks * top_k > cp_merge_max_candidates()) return SA_ERR_UNSUPPORTED;
    if (n_q == 0) return SA_OK;
    if (!cand_score || !cand_pos || !pos_lo || !pos_hi || !idx_global || !idx_local)
        return SA_ERR_INVALID_ARG;
    return cuda_status(launch_cp_merge(cand_score, cand_pos, n_ranks, n_q, top_k, pos_lo, pos_hi,
                                       idx_global, idx_local, static_cast<cudaStream_t>(stream)));
}

sa_status sa_combine_partials(const float *o_part, const float *lse_part, int32_t n_parts,
                              int32_t n_q, int32_t heads, int32_t d, void *out,
                              sa_dtype out_dtype, float *lse, void *stream) {
    if (n_parts <= 0 || n_q < 0 || heads <= 0 || d <= 0) return SA_ERR_INVALID_ARG;
    if (n_parts > cp_combine_max_parts()) return SA_ERR_UNSUPPORTED;
    if (out_dtype != SA_BF16 && out_dtype != SA_F32) return SA_ERR_UNSUPPORTED;
    if (n_q == 0) return SA_OK;
    if (!o_part || !lse_part || !out) return SA_ERR_INVALID_ARG;
    return cuda_status(launch_cp_combine(o_part, lse_part, n_parts, (int64_t)n_q * heads, d, out,
                                         out_dtype, lse, static_cast<cudaStream_t>(stream)));
}

sa_status sa_quantize_index_query(const void *q_in, sa_dtype in_dtype, int32_t n_q,
                                  int32_t h_index, int32_t d_index, void *q_out, float *q_scale,
                                  void *stream) {
    if (n_q < 0 || h_index <= 0 || d_index <= 0) return SA_ERR_INVALID_ARG;
    if (in_dtype != SA_BF16 && in_dtype != SA_F32) return SA_ERR_UNSUPPORTED;
    if (n_q == 0) return SA_OK;
    if (!q_in || !q_out || !q_scale) return SA_ERR_INVALID_ARG;
    if (!aligned16(q_in) || !aligned16(q_out) || !aligned16(q_scale)) return SA_ERR_INVALID_ARG;
    return cuda_status(launch_quantize_rows(q_in, in_dtype, (int64_t)n_q * h_index, d_index,
                                            static_cast<uint8_t *>(q_out), q_scale,
                                            static_cast<cudaStream_t>(stream)));
}

sa_status sa_append_tokens(const sa_cache *cache, const sa_new_tokens *tokens, void *workspace,
                           size_t workspace_bytes, void *stream) {
    sa_status st = check_cache(cache);
    if (st != SA_OK) return st;
    if (tokens == nullptr || tokens->n_new < 0) return SA_ERR_INVALID_ARG;
    if (tokens->in_dtype != SA_BF16 && tokens->in_dtype != SA_F32) return SA_ERR_UNSUPPORTED;
    const bool page_tile = cache->kv_scale_tokens == 0 && cache->kv_scale_dims == 0;
    if (tokens->kv && cache->kv_dtype == SA_E4M3 && (page_tile || cache->kv_scale_tokens != 1))
        return SA_ERR_UNSUPPORTED;  // a scale shared by several tokens cannot take one more
    if (tokens->k_index && cache->index_dtype == SA_MXFP8)
        return SA_ERR_UNSUPPORTED;  // no MXFP8 key encoder: such pools are filled by the caller
    if (tokens->n_new > 0) {
        if (!tokens->seq || !tokens->pos) return SA_ERR_INVALID_ARG;
        if ((tokens->k_index && !aligned16(tokens->k_index)) ||
            (tokens->kv && !aligned16(tokens->kv)))
            return SA_ERR_INVALID_ARG;
    }
    if ((st = check_workspace(workspace, workspace_bytes, kStatusBytes)) != SA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = clear_status(workspace, s)) != SA_OK) return st;
    if (tokens->n_new == 0 || (!tokens->k_index && !tokens->kv)) return SA_OK;
    AppendParams p{};
    p.page_table = cache->page_table;
    p.batch = cache->batch;
    p.max_pages = cache->max_pages;
    p.num_pages = cache->num_pages;
    p.n_new = tokens->n_new;
    p.seq = tokens->seq;
    p.pos = tokens->pos;
    p.in_bf16 = tokens->in_dtype == SA_BF16;
    p.k_new = tokens->k_index;
    p.kv_new = tokens->kv;
    // The pools are caller-owned writable device memory; sa_cache holds them
    // as const because the decode path only reads them.
    p.k_index = const_cast<void *>(cache->k_index);
    p.k_index_scale = const_cast<float *>(cache->k_index_scale);
    p.d_index = cache->d_index;
    p.index_dtype = cache->index_dtype;
    p.kv = const_cast<void *>(cache->kv);
    p.kv_rope = const_cast<void *>(cache->kv_rope);
    p.kv_scale = const_cast<float *>(cache->kv_scale);
    p.d_latent = cache->d_latent;
    p.d_rope = cache->d_rope;
    p.kv_dtype = cache->kv_dtype;
    p.kv_scale_dims = page_tile ? cache->d_latent : cache->kv_scale_dims;
    p.status = static_cast<int32_t *>(workspace);
    return cuda_status(launch_append(p, s));
}

sa_status sa_device_status(const void *workspace, size_t workspace_bytes, void *stream,
                           int32_t *detail) {
    if (workspace == nullptr || workspace_bytes < kStatusBytes) return SA_ERR_WORKSPACE;
    int32_t word[2] = {0, 0};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(word, workspace, sizeof word, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return SA_ERR_CUDA;
    if (detail) *detail = word[1];
    if (word[0] == 0) return SA_OK;
    if (word[0] == SA_ERR_TIMEOUT) return SA_ERR_TIMEOUT;
    return SA_ERR_DEVICE_FAULT;
}

const char *sa_status_string(sa_status status) {
    switch (status) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID_ARG: return "invalid argument";
    case SA_ERR_UNSUPPORTED: return "unsupported combination";
    case SA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SA_ERR_CUDA: return "CUDA error";
    case SA_ERR_DEVICE_FAULT: return "bad data detected on the device";
    case SA_ERR_TIMEOUT: return "bounded device wait timed out";
    }
    return "unknown status";
}

int32_t sa_version(void) { return 100; }

uint64_t sa_kernel_launches(void) { return sa::g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
