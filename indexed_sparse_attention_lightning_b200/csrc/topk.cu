// topk.cu -- exact per-row top-K by radix select ("Optimizing Next-Gen LLM
// Inference" §3.1, Top-K selection; "Inference Acceleration for New Large Model
// Architectures" §3.1 step 3).
//
// Scores map to order-preserving 32-bit keys.  Four 8-bit passes, each a
// shared-memory histogram over the keys that match the prefix found so far,
// fix the K-th largest key T and how many keys equal to T are still needed.
// A final in-order pass keeps every key > T and the first `need` keys == T
// (lowest positions win ties) and writes them in ascending position order --
// which also groups the selected rows of one cache page together for the
// gather ("Inference Acceleration" §3.2: aggregate indices into blocks).
// Warp ballots and prefix popcounts do the stream compaction.
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kThreads = 1024;

// Exclusive prefix of `flag` over the block in thread order; returns the
// block total through *total.  Uses warp ballots plus one scan of the warp
// totals.  All threads must call it.
__device__ __forceinline__ int block_exclusive_count(bool flag, int *warp_sums, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned ballot = __ballot_sync(0xffffffffu, flag);
    const int in_warp = __popc(ballot & ((1u << lane) - 1u));
    if (lane == 0) warp_sums[warp] = __popc(ballot);
    __syncthreads();
    if (warp == 0) {
        int v = warp_sums[lane];
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        warp_sums[lane] = incl - v;  // exclusive
        if (lane == 31) warp_sums[32] = incl;
    }
    __syncthreads();
    const int r = warp_sums[warp] + in_warp;
    *total = warp_sums[32];
    __syncthreads();
    return r;
}

// Exclusive prefix sum of `v` over the block in thread order (total through
// *total).  All threads must call it.
__device__ __forceinline__ int block_exclusive_prefix(int v, int *warp_sums, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int w = lane < nw ? warp_sums[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        warp_sums[lane] = wi - w;
        if (lane == 31) warp_sums[32] = wi;
    }
    __syncthreads();
    const int r = warp_sums[warp] + incl - v;
    *total = warp_sums[32];
    __syncthreads();
    return r;
}

// Exact top-K of one row by four 8-bit radix passes, written in ascending
// position order.  All kThreads threads of the block call it.
__device__ void select_row(const float *__restrict__ row, int32_t V, int32_t top_k,
                           int32_t *__restrict__ out) {
    __shared__ unsigned hist[256];
    __shared__ int warp_sums[33];
    __shared__ unsigned sel_digit, sel_above;

    if (V <= top_k) {
        for (int i = threadIdx.x; i < top_k; i += kThreads) out[i] = i < V ? i : -1;
        return;
    }
    uint32_t prefix = 0, mask = 0;
    unsigned remaining = top_k;  // how many still to take at or below the prefix
    const int lane = threadIdx.x & 31;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += kThreads) hist[i] = 0;
        __syncthreads();
        for (int64_t base = 0; base < V; base += kThreads) {
            const int64_t i = base + threadIdx.x;
            uint32_t key = i < V ? order_key(row[i]) : 0u;
            bool match = i < V && (key & mask) == prefix;
            unsigned digit = match ? (key >> shift) & 255u : 256u;
            unsigned same = __match_any_sync(0xffffffffu, digit);
            if (match && lane == __ffs(same) - 1) atomicAdd(&hist[digit], __popc(same));
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // lane l owns bins 8l..8l+7; find the bin where the count from the
            // top reaches `remaining`
            unsigned c[8], lane_sum = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                c[b] = hist[8 * lane + b];
                lane_sum += c[b];
            }
            unsigned suffix = lane_sum;  // inclusive sum of lanes >= lane
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                unsigned n = __shfl_down_sync(0xffffffffu, suffix, o);
                if (lane + o < 32) suffix += n;
            }
            const unsigned above_lane = suffix - lane_sum;  // lanes > lane
            if (above_lane < remaining && remaining <= suffix) {
                unsigned acc = above_lane;
                for (int b = 7; b >= 0; --b) {
                    if (acc + c[b] >= remaining) {
                        sel_digit = 8 * lane + b;
                        sel_above = acc;
                        break;
                    }
                    acc += c[b];
                }
            }
        }
        __syncthreads();
        prefix |= sel_digit << shift;
        mask |= 255u << shift;
        remaining -= sel_above;
        __syncthreads();
    }
    // prefix == T, the K-th largest key; `remaining` ties must be taken.
    const uint32_t T = prefix;
    int written = 0, ties_seen = 0;
    for (int64_t base = 0; base < V && written < top_k; base += kThreads) {
        const int64_t i = base + threadIdx.x;
        const uint32_t key = i < V ? order_key(row[i]) : 0u;
        const bool eq = i < V && key == T;
        int eq_total;
        const int eq_rank = block_exclusive_count(eq, warp_sums, &eq_total);
        const bool take = (i < V && key > T) || (eq && ties_seen + eq_rank < (int)remaining);
        int take_total;
        const int pos = block_exclusive_count(take, warp_sums, &take_total);
        if (take && written + pos < top_k) out[written + pos] = static_cast<int32_t>(i);
        written += take_total;
        ties_seen += eq_total;
    }
}

__global__ void __launch_bounds__(kThreads)
topk_rowwise_kernel(const float *__restrict__ scores, int64_t ld,
                    const int32_t *__restrict__ valid_len, int32_t max_valid, const PathParams p,
                    int32_t top_k, int32_t *__restrict__ idx, int32_t *status) {
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.x;
    int32_t V;
    if (valid_len != nullptr) {
        V = valid_len[t];
        if (V < 0 || V > max_valid) {
            if (threadIdx.x == 0) report(status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_POSITION);
            V = 0;
        }
    } else {
        V = visible_len(p, t);
    }
    select_row(scores + (int64_t)t * ld, V, top_k, idx + (int64_t)t * top_k);
}

// ---------------------------------------------------------------------------
// Histogram-guided top-K for the fused path.  The indexer has counted every
// query's score keys in kHistBins radix buckets (the top kHistBits bits of
// the order-preserving key).  The bucket b* where the count from the top
// reaches K splits the row: keys above it are selected outright, keys inside
// it are candidates whose exact order is settled later, keys below are out.
// ---------------------------------------------------------------------------
constexpr int kCollectThreads = 256;

// Bucket b* and the number of keys in buckets above it, for a histogram of
// kHistBins bins with at least K keys.  All threads of the block call it.
__device__ void threshold_bucket(const uint32_t *__restrict__ h, int32_t K, int *b_out,
                                 uint32_t *above_out) {
    constexpr int kPer = kHistBins / kCollectThreads;  // 16 bins per thread
    __shared__ uint32_t part[kCollectThreads];
    __shared__ int sb;
    __shared__ uint32_t sa;
    const int tid = threadIdx.x;
    uint32_t c[kPer], mine = 0;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        c[j] = h[tid * kPer + j];
        mine += c[j];
    }
    part[tid] = mine;
    if (tid == 0) {
        sb = 0;   // only used when the histogram holds fewer than K keys; the
        sa = 0;   // finalize step then falls back to the row-wise select
    }
    __syncthreads();
    if (tid < 32) {
        // suffix sums over the 256 thread partials, 8 per lane
        uint32_t v[8], s8 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            v[j] = part[tid * 8 + j];
            s8 += v[j];
        }
        uint32_t suffix = s8;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t n = __shfl_down_sync(0xffffffffu, suffix, o);
            if (tid + o < 32) suffix += n;
        }
        uint32_t acc = suffix - s8;  // partials of threads > 8 * tid + 7
#pragma unroll
        for (int j = 7; j >= 0; --j) {
            const uint32_t hi = acc;  // partials strictly above thread 8*tid+j
            acc += v[j];
            part[tid * 8 + j] = hi;   // counts in buckets above this thread's range
        }
    }
    __syncthreads();
    uint32_t acc = part[tid];
    if (acc < (uint32_t)K && acc + mine >= (uint32_t)K) {
#pragma unroll
        for (int j = kPer - 1; j >= 0; --j) {
            if (acc + c[j] >= (uint32_t)K) {
                sb = tid * kPer + j;
                sa = acc;
                break;
            }
            acc += c[j];
        }
    }
    __syncthreads();
    *b_out = sb;
    *above_out = sa;
}

// Exclusive prefix of v over the kCollectThreads threads of the block (total
// through *total).  All threads call it.
__device__ __forceinline__ int collect_prefix(int v, int *warp_sums, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kCollectThreads / 32;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    int before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const int x = warp_sums[w];
        before += w < warp ? x : 0;
        all += x;
    }
    __syncthreads();
    *total = all;
    return before + incl - v;
}

// Long rows (more than kSingleMaxV positions) take two kernels:
//   count     many CTAs per query, one per 8192-position chunk: the chunk's keys
//             above the threshold bucket go, in ascending position order, to
//             a per-query list (one reservation per chunk), its keys inside the
//             bucket to the candidate list as composite keys (likewise), and
//             the chunk's four numbers (first slot and count in each list) to
//             chunk_info;
//   finalize  one CTA per query: the exact need-th largest candidate (an exact
//             composite threshold), then every selected position's output slot
//             from its chunk's first slot, its place in its own list and a
//             binary search in the chunk's other list -- positions ascending,
//             no pass over the row -- with its physical cache row.
// Per-query counters (counts, [n_q, kTopkCountsPerQuery] int32, zeroed with
// the histograms): [0] keys above the bucket, [1] candidates.
constexpr int kChunk = kTopkChunk;                       // positions per count CTA
constexpr int kChunkPer = kChunk / kCollectThreads;      // 32 consecutive positions a thread
static_assert(kChunkPer == 32, "a thread's run is one 32-bit selection mask");

// The 32 scores of positions [p0, p0 + 32) of `row` (entries at or past V
// are never selected; they read as 0).
__device__ __forceinline__ void load_run(const float *row, int64_t p0, int64_t V, float (&x)[32]) {
    if (p0 + 32 <= V) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float4 v = *reinterpret_cast<const float4 *>(row + p0 + 4 * u);
            x[4 * u] = v.x;
            x[4 * u + 1] = v.y;
            x[4 * u + 2] = v.z;
            x[4 * u + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = p0 + i < V ? row[p0 + i] : 0.f;
    }
}

__global__ void __launch_bounds__(kCollectThreads)
topk_count_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ vis,
                  const uint32_t *__restrict__ hist, int32_t top_k, int32_t *__restrict__ above_pos,
                  int4 *__restrict__ chunk_info, int32_t ld_chunks, int32_t *__restrict__ counts,
                  uint64_t *__restrict__ cand, int32_t cap) {
    pdl_wait();
    pdl_trigger();
    __shared__ int warp_sums[kCollectThreads / 32];
    __shared__ int32_t base_s[2];
    const int t = blockIdx.y, tid = threadIdx.x;
    const int32_t V = vis[t];
    const int64_t c0 = (int64_t)blockIdx.x * kChunk;
    if (V <= top_k || c0 >= V) return;
    const int64_t p0 = c0 + (int64_t)kChunkPer * tid;
    float x[32];
    load_run(scores + (int64_t)t * ld, p0, V, x);
    int bstar;
    uint32_t above;
    threshold_bucket(hist + (int64_t)t * kHistBins, top_k, &bstar, &above);
    uint32_t hi = 0, eq = 0;  // this thread's keys above / inside the bucket
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int b = static_cast<int>(order_key(x[i]) >> (32 - kHistBits));
        if (p0 + i < V && b > bstar) hi |= 1u << i;
        if (p0 + i < V && b == bstar) eq |= 1u << i;
    }
    int tot_h, tot_e;
    int oh = collect_prefix(__popc(hi), warp_sums, &tot_h);
    int oe = collect_prefix(__popc(eq), warp_sums, &tot_e);
    int32_t *ct = counts + (int64_t)t * kTopkCountsPerQuery;
    if (tid == 0) {
        base_s[0] = tot_h > 0 ? atomicAdd(&ct[0], tot_h) : 0;
        base_s[1] = tot_e > 0 ? atomicAdd(&ct[1], tot_e) : 0;
        // a row of more chunks than slots is left to the finalize kernel's fallback
        if ((int)blockIdx.x < ld_chunks)
            chunk_info[(int64_t)t * ld_chunks + blockIdx.x] =
                make_int4(base_s[0], tot_h, base_s[1], tot_e);
    }
    __syncthreads();
    oh += base_s[0];
    oe += base_s[1];
    int32_t *sel_t = above_pos + (int64_t)t * top_k;
    while (hi != 0) {
        const int i = __ffs(hi) - 1;
        hi &= hi - 1;
        if (oh < top_k) sel_t[oh] = static_cast<int32_t>(p0 + i);
        ++oh;
    }
    if (eq == 0) return;
    uint64_t *cand_t = cand + (int64_t)t * cap;
#pragma unroll
    for (int i = 0; i < 32; ++i) {  // static indices: x stays in registers
        if ((eq >> i) & 1u) {
            if (oe < cap)
                cand_t[oe] = (static_cast<uint64_t>(order_key(x[i])) << 32) |
                             (0xFFFFFFFFu - static_cast<uint32_t>(p0 + i));
            ++oe;
        }
    }
}

// The `need` largest of the n_cand composite candidate keys cs[] --
// order-preserving score key in the high word, inverted position in the low
// word, so all distinct and ties go to the lower position -- which all share
// their top kHistBits bits (the threshold bucket `bstar`): on return exactly
// `need` of them satisfy (k & *mask) >= *prefix.  Radix passes of 10-bit
// digits below the bucket bits find the need-th largest key, stopping as soon
// as a whole digit bin is taken (normally after two passes); the bucket bits
// themselves are never counted, so no pass piles every candidate onto one
// histogram bin.  Any composite key of the row above the bucket also passes
// the test, any below fails it.  1 <= need <= n_cand.  All threads of the
// block call it; dh holds 1024 counters.
__device__ void candidate_threshold(const uint64_t *cs, int n_cand, int need, int bstar,
                                    unsigned *dh, int *warp_sums, uint64_t *mask_out,
                                    uint64_t *prefix_out) {
    __shared__ int sel_digit_s, sel_above_s, sel_count_s;
    const int tid = threadIdx.x;
    uint64_t prefix = static_cast<uint64_t>(bstar) << (64 - kHistBits);
    uint64_t mask = ~0ull << (64 - kHistBits);
    int remaining = need, tot;
    int shift = 64 - kHistBits - 10, width = 10;
    for (;;) {
        const uint64_t dmask = (1ull << width) - 1;
        dh[tid] = 0;
        __syncthreads();
        for (int i = tid; i < n_cand; i += kThreads) {
            const uint64_t k = cs[i];
            if ((k & mask) == prefix) atomicAdd(&dh[(k >> shift) & dmask], 1u);
        }
        __syncthreads();
        const int d = 1023 - tid;  // digits in descending order
        const int cd = static_cast<int>(dh[d]);
        const int ex = block_exclusive_prefix(cd, warp_sums, &tot);
        if (ex < remaining && ex + cd >= remaining) {
            sel_digit_s = d;
            sel_above_s = ex;
            sel_count_s = cd;
        }
        __syncthreads();
        prefix |= static_cast<uint64_t>(sel_digit_s) << shift;
        mask |= dmask << shift;
        remaining -= sel_above_s;
        const bool whole = remaining == sel_count_s;
        __syncthreads();
        if (whole || shift == 0) break;
        if (shift >= 10) {
            shift -= 10;
        } else {
            width = shift;
            shift = 0;
        }
    }
    *mask_out = mask;
    *prefix_out = prefix;
}

// Marks in `bits` (by position) the `need` largest candidates (see
// candidate_threshold).  All threads of the block call it.
__device__ void mark_top_candidates(const uint64_t *cs, int n_cand, int need, int bstar,
                                    uint32_t *bits, unsigned *dh, int *warp_sums) {
    const int tid = threadIdx.x;
    uint64_t mask, prefix;
    candidate_threshold(cs, n_cand, need, bstar, dh, warp_sums, &mask, &prefix);
    for (int i = tid; i < n_cand; i += kThreads) {
        const uint64_t k = cs[i];
        if ((k & mask) >= prefix) {
            const uint32_t pos = 0xFFFFFFFFu - static_cast<uint32_t>(k);
            atomicOr(&bits[pos >> 5], 1u << (pos & 31));
        }
    }
}

// Writes the selected positions (bits set in `bits`, `words` words) to out in
// ascending order, -1 after them, and -- when rows != null -- their physical
// cache rows (compact_rows layout, tile 64) and count.  Positions first (each
// thread owns a run of words; selected keys may crowd into a few runs), then
// the rows in a second pass spread evenly over the threads, so no thread
// serialises many page-table loads.  All threads call it.
__device__ void emit_selection(const uint32_t *bits, int words, int32_t top_k, int32_t *out,
                               const PathParams &p, int32_t t, int32_t *rows, int32_t *n_valid,
                               int *warp_sums, const int32_t *pt_smem = nullptr) {
    // each warp owns a run of words and walks it 32 words at a time, one
    // word per lane, so a run dense with selected keys is shared by 32 lanes
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int kWarps = kThreads / 32;
    const int per = (words + kWarps - 1) / kWarps;
    const int w0 = min(words, warp * per), w1 = min(words, w0 + per);
    int cnt = 0;
    for (int w = w0 + lane; w < w1; w += 32) cnt += __popc(bits[w]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    int total;
    int pos = block_exclusive_prefix(lane == 0 ? cnt : 0, warp_sums, &total);
    pos = __shfl_sync(0xffffffffu, pos, 0);  // the warp's first slot
    for (int c0 = w0; c0 < w1; c0 += 32) {
        const int w = c0 + lane;
        uint32_t b = w < w1 ? bits[w] : 0u;
        if (!__any_sync(0xffffffffu, b != 0u)) continue;  // sparse long rows: most chunks empty
        const int c = __popc(b);
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int q = pos + incl - c;
        while (b) {
            const int j = __ffs(b) - 1;
            b &= b - 1;
            if (q < top_k) out[q] = w * 32 + j;
            ++q;
        }
        pos += __shfl_sync(0xffffffffu, incl, 31);
    }
    const int32_t nv = min(total, top_k);
    for (int i = nv + threadIdx.x; i < top_k; i += kThreads) out[i] = -1;
    if (rows == nullptr) return;
    __syncthreads();  // the positions are visible to the whole block
    const int32_t seq = __ldg(p.q_seq + t);
    int bad_page = 0;
    for (int i = threadIdx.x; i < nv; i += kThreads) {
        const int32_t s = out[i];
        int64_t row;
        if (pt_smem != nullptr) {  // the sequence's page-table row, staged by the caller
            const int32_t page = pt_smem[s >> 6];
            row = (page < 0 || page >= p.num_pages) ? -1 : (int64_t)page * 64 + (s & 63);
        } else {
            row = phys_row(p.page_table, p.max_pages, p.num_pages, seq, s);
        }
        if (row < 0) bad_page = 1;
        else rows[i] = static_cast<int32_t>(row);
    }
    if (__syncthreads_or(bad_page)) {  // rare: drop (and report) the unmapped rows
        compact_rows(p, t, out, top_k, 64, rows, n_valid, warp_sums);
        return;
    }
    const int32_t padded = (nv + 63) / 64 * 64;
    if (nv > 0)
        for (int c = nv + threadIdx.x; c < padded; c += kThreads) rows[c] = rows[0];
    if (threadIdx.x == 0) *n_valid = nv;
}

// First index of the ascending list v[0, n) holding a value >= x.
__device__ __forceinline__ int lower_bound(const int32_t *v, int n, int32_t x) {
    int lo = 0;
    while (n > 0) {
        const int half = n >> 1;
        if (v[lo + half] < x) {
            lo += half + 1;
            n -= half + 1;
        } else {
            n = half;
        }
    }
    return lo;
}

// One CTA per query (see topk_count_kernel).  Rows the candidate buffer or the
// above list cannot hold (massive exact ties, very large K), short rows and
// rows of more chunks than one CTA handles take the row-wise radix select,
// whole.
constexpr int kMaxChunks = kThreads;
constexpr int kMaxAbove = 8192;
__host__ __device__ constexpr size_t finalize_smem_bytes(int cap) {
    return (size_t)cap * 8 + (size_t)kMaxAbove * 4 + (size_t)(cap + 1) * 4 + (size_t)cap * 4 +
           (size_t)kMaxChunks * 16 + 16;
}
__global__ void __launch_bounds__(kThreads)
topk_finalize_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ vis,
                     int32_t top_k, const int32_t *__restrict__ above_pos,
                     const int4 *__restrict__ chunk_info, int32_t ld_chunks,
                     const int32_t *__restrict__ counts, const uint64_t *__restrict__ cand,
                     int32_t cap, int32_t *__restrict__ idx, const PathParams p,
                     int32_t *__restrict__ rows_all, int32_t ld_rows,
                     int32_t *__restrict__ n_valid_all) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint64_t fin_smem[];
    __shared__ unsigned dh[1024];
    __shared__ int warp_sums[33];
    __shared__ int slot_s[kMaxChunks], bbase_s[kMaxChunks], bcount_s[kMaxChunks];
    const int t = blockIdx.x, tid = threadIdx.x;
    const int32_t V = vis[t];
    int32_t *out = idx + (int64_t)t * top_k;
    int32_t *rows = rows_all != nullptr ? rows_all + (int64_t)t * ld_rows : nullptr;
    const int32_t *ct = counts + (int64_t)t * kTopkCountsPerQuery;
    const int32_t n_above = ct[0], n_cand = ct[1];
    const int32_t need = top_k - n_above;
    const int chunks = static_cast<int>((V + kChunk - 1) / kChunk);
    const bool fits = V > top_k && n_cand <= cap && n_above <= kMaxAbove && need > 0 &&
                      need <= n_cand && chunks <= min(kMaxChunks, ld_chunks);
    if (!fits) {
        select_row(scores + (int64_t)t * ld, V, top_k, out);
        if (rows != nullptr) {
            __syncthreads();
            compact_rows(p, t, out, top_k, 64, rows, n_valid_all + t, warp_sums);
        }
        return;
    }
    uint64_t *cs = fin_smem;                                    // [cap] candidates
    int32_t *A = reinterpret_cast<int32_t *>(cs + cap);         // [kMaxAbove] above positions
    int32_t *pre = A + kMaxAbove;                               // [cap + 1] selected before i
    int32_t *B = pre + cap + 1;                                 // [cap] selected positions
    int4 *ci = reinterpret_cast<int4 *>(
        (reinterpret_cast<uintptr_t>(B + cap) + 15) & ~uintptr_t(15));  // [kMaxChunks]
    const uint64_t *cg = cand + (int64_t)t * cap;
    const int32_t *ag = above_pos + (int64_t)t * top_k;
    for (int i = tid; i < n_cand; i += kThreads) cs[i] = cg[i];
    for (int i = tid; i < n_above; i += kThreads) A[i] = ag[i];
    if (tid < chunks) ci[tid] = chunk_info[(int64_t)t * ld_chunks + tid];
    __syncthreads();
    uint64_t mask, prefix;
    candidate_threshold(cs, n_cand, need, static_cast<int>(cs[0] >> (64 - kHistBits)), dh,
                        warp_sums, &mask, &prefix);
    // the selected candidates, compacted in list order (each chunk's stay
    // contiguous and ascending)
    const int per = (n_cand + kThreads - 1) / kThreads;
    const int i0 = tid * per;
    int mine = 0;
    for (int k = 0; k < per; ++k) {
        const int i = i0 + k;
        if (i < n_cand && (cs[i] & mask) >= prefix) ++mine;
    }
    int total;
    int q = block_exclusive_prefix(mine, warp_sums, &total);
    for (int k = 0; k < per; ++k) {
        const int i = i0 + k;
        if (i >= n_cand) break;
        pre[i] = q;
        if ((cs[i] & mask) >= prefix) B[q++] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(cs[i]));
    }
    if (tid == 0) pre[n_cand] = total;
    __syncthreads();
    // each chunk's first output slot
    int cnt = 0;
    if (tid < chunks) {
        const int4 f = ci[tid];
        bbase_s[tid] = pre[f.z];
        bcount_s[tid] = pre[f.z + f.w] - pre[f.z];
        cnt = f.y + bcount_s[tid];
    }
    const int first = block_exclusive_prefix(cnt, warp_sums, &total);
    if (tid < chunks) slot_s[tid] = first;
    __syncthreads();
    // every selected position to its slot, with its physical row
    const int32_t seq = __ldg(p.q_seq + t);
    int bad = 0;
    for (int e = tid; e < n_above + need; e += kThreads) {
        int32_t pos;
        int slot;
        if (e < n_above) {
            pos = A[e];
            const int c = pos / kChunk;
            slot = slot_s[c] + (e - ci[c].x) + lower_bound(B + bbase_s[c], bcount_s[c], pos);
        } else {
            const int j = e - n_above;
            pos = B[j];
            const int c = pos / kChunk;
            const int4 f = ci[c];
            slot = slot_s[c] + (j - bbase_s[c]) + lower_bound(A + f.x, f.y, pos);
        }
        if (slot < 0 || slot >= top_k) continue;  // only if the lists disagree with the counts
        out[slot] = pos;
        if (rows != nullptr) {
            const int64_t r = phys_row(p.page_table, p.max_pages, p.num_pages, seq, pos);
            if (r < 0) bad = 1;
            else rows[slot] = static_cast<int32_t>(r);
        }
    }
    if (rows == nullptr) return;
    if (__syncthreads_or(bad)) {  // rare: drop (and report) the unmapped rows
        compact_rows(p, t, out, top_k, 64, rows, n_valid_all + t, warp_sums);
        return;
    }
    const int32_t padded = (top_k + 63) / 64 * 64;
    for (int c = top_k + tid; c < padded; c += kThreads) rows[c] = rows[0];
    if (tid == 0) n_valid_all[t] = top_k;
}

// ---------------------------------------------------------------------------
// Rows of at most kSingleMaxV positions (decode at up to 64K context): the
// whole selection in one CTA per query.  One pass over the row (from L2: the
// indexer has just written it; the first 32K positions' loads are issued
// before the threshold bucket is even known) marks the keys above the
// threshold bucket in a shared-memory bitmap and collects the bucket's keys,
// each thread's at a slot from one block-wide prefix (no shared counter); the
// need-th largest candidate follows from 10-bit radix passes over composite
// keys (score key, inverted position: distinct, ties to the lower position),
// normally two; the bitmap is then read back in ascending order, the physical
// rows looked up in a copy of the sequence's page-table row in shared memory.
// ---------------------------------------------------------------------------
constexpr int32_t kSingleMaxV = 65536;
constexpr int32_t kSingleCap = 8192;  // candidates held in shared memory
constexpr size_t kSingleSmem =
    (size_t)kSingleCap * 8 + (size_t)kSingleMaxV / 8 + (size_t)kSingleMaxV / 64 * 4;

// Scores b0 + 4 (threadIdx.x + u kThreads) .. + 3 of `row` for u < kSingleBatch
// (entries at or past V read as 0 and are never selected), all loads issued
// before any is used.
constexpr int kSingleBatch = 8;
__device__ __forceinline__ void load_single_batch(const float *row, int32_t b0, int32_t V,
                                                  float4 (&xs)[kSingleBatch]) {
#pragma unroll
    for (int u = 0; u < kSingleBatch; ++u) {
        const int32_t i0 = b0 + 4 * (threadIdx.x + u * kThreads);
        if (i0 + 4 <= V) {
            xs[u] = *reinterpret_cast<const float4 *>(row + i0);
        } else {
            xs[u].x = i0 < V ? row[i0] : 0.f;
            xs[u].y = i0 + 1 < V ? row[i0 + 1] : 0.f;
            xs[u].z = i0 + 2 < V ? row[i0 + 2] : 0.f;
            xs[u].w = i0 + 3 < V ? row[i0 + 3] : 0.f;
        }
    }
}

__global__ void __launch_bounds__(kThreads)
topk_single_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ vis,
                   const uint32_t *__restrict__ hist, int32_t top_k, int32_t *__restrict__ idx,
                   const PathParams p, int32_t *__restrict__ rows_all, int32_t ld_rows,
                   int32_t *__restrict__ n_valid_all) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint64_t single_smem[];
    uint64_t *cs = single_smem;                                               // [kSingleCap]
    uint32_t *bits = reinterpret_cast<uint32_t *>(single_smem + kSingleCap);  // [V / 32]
    int32_t *pt = reinterpret_cast<int32_t *>(bits + kSingleMaxV / 32);       // [V / 64]
    __shared__ unsigned dh[1024];
    __shared__ int warp_sums[33];
    __shared__ int bstar_s, above_s;
    const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const int32_t V = vis[t];
    int32_t *out = idx + (int64_t)t * top_k;
    int32_t *rows = rows_all != nullptr ? rows_all + (int64_t)t * ld_rows : nullptr;
    int32_t *nv_out = n_valid_all != nullptr ? n_valid_all + t : nullptr;
    const int words = (V + 31) / 32;
    // the sequence's page-table row, for the physical rows at the end (rows
    // past max_pages are looked up, and reported, the usual way)
    const int slots = min((V + 63) / 64, p.max_pages);
    if (rows != nullptr) {
        const int32_t *ptg = p.page_table + (int64_t)__ldg(p.q_seq + t) * p.max_pages;
        for (int i = tid; i < slots; i += kThreads) pt[i] = __ldg(ptg + i);
    }
    const int32_t *pts = (rows != nullptr && (V + 63) / 64 <= p.max_pages) ? pt : nullptr;
    if (V <= top_k) {  // everything visible is selected
        for (int w = tid; w < words; w += kThreads)
            bits[w] = (32 * w + 32 <= V) ? 0xFFFFFFFFu : ((1u << (V & 31)) - 1u);
        __syncthreads();
        emit_selection(bits, words, top_k, out, p, t, rows, nv_out, warp_sums, pts);
        return;
    }
    // the first batch of the row (a row of up to 32K positions is one batch;
    // the trip count is the same in every lane) -- issued before the bucket
    // search
    const float *row = scores + (int64_t)t * ld;
    float4 xs[kSingleBatch];
    load_single_batch(row, 0, V, xs);
    // threshold bucket b*: thread i holds the buckets of rank 4i .. 4i+3 from the top
    const uint32_t *h = hist + (int64_t)t * kHistBins;
    uint32_t c[4], mine = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        c[j] = h[kHistBins - 1 - 4 * tid - j];
        mine += c[j];
    }
    if (tid == 0) {
        bstar_s = -1;
        above_s = 0;
    }
    int tot;
    int excl = block_exclusive_prefix((int)mine, warp_sums, &tot);
    if (excl < top_k && excl + (int)mine >= top_k) {
        int acc = excl;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (acc + (int)c[j] >= top_k) {
                bstar_s = kHistBins - 1 - 4 * tid - j;
                above_s = acc;
                break;
            }
            acc += c[j];
        }
    }
    for (int w = tid; w < words; w += kThreads) bits[w] = 0;
    __syncthreads();
    const int bstar = bstar_s;
    const int32_t need = top_k - above_s;
    bool fallback = bstar < 0;
    int n_cand = 0;
    if (!fallback) {
        // one pass over the row: keys above b* into the bitmap, b*'s keys collected
        for (int32_t b0 = 0; b0 < V; b0 += 4 * kThreads * kSingleBatch) {
            if (b0 > 0) load_single_batch(row, b0, V, xs);
            uint32_t cmask = 0;  // this thread's keys in the bucket: bit 4u + e
#pragma unroll
            for (int u = 0; u < kSingleBatch; ++u) {
                const int32_t i0 = b0 + 4 * (tid + u * kThreads);
                const float x[4] = {xs[u].x, xs[u].y, xs[u].z, xs[u].w};
                uint32_t above_mask = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int b = static_cast<int>(order_key(x[e]) >> (32 - kHistBits));
                    const bool valid = i0 + e < V;
                    if (valid && b > bstar) above_mask |= 1u << e;
                    if (valid && b == bstar) cmask |= 1u << (4 * u + e);
                }
                // the 8 lanes of a 32-position word combine their 4-bit masks
                // (lane l holds positions 4l .. 4l + 3 of the warp's 128), and
                // the group's first lane stores the word: no atomics
                uint32_t word = above_mask << (4 * (lane & 7));
                word |= __shfl_xor_sync(0xffffffffu, word, 1);
                word |= __shfl_xor_sync(0xffffffffu, word, 2);
                word |= __shfl_xor_sync(0xffffffffu, word, 4);
                if ((lane & 7) == 0 && i0 < V) bits[i0 >> 5] = word;
            }
            // the bucket's keys (a few per thread, their scores read again from
            // L2): every thread's at its slot of one block prefix
            int total;
            int base = n_cand + block_exclusive_prefix(__popc(cmask), warp_sums, &total);
            n_cand += total;
            while (cmask != 0) {
                const int j = __ffs(cmask) - 1;
                cmask &= cmask - 1;
                const int32_t pos = b0 + 4 * (tid + (j >> 2) * kThreads) + (j & 3);
                if (base < kSingleCap)
                    cs[base] = (static_cast<uint64_t>(order_key(row[pos])) << 32) |
                               (0xFFFFFFFFu - static_cast<uint32_t>(pos));
                ++base;
            }
        }
        __syncthreads();
        fallback = n_cand > kSingleCap || need < 1 || need > n_cand;
    }
    if (fallback) {  // histogram and scores disagree, or too many candidates
        select_row(scores + (int64_t)t * ld, V, top_k, out);
        if (rows != nullptr) {
            __syncthreads();
            compact_rows(p, t, out, top_k, 64, rows, nv_out, warp_sums);
        }
        return;
    }
    mark_top_candidates(cs, n_cand, need, bstar, bits, dh, warp_sums);
    __syncthreads();
    emit_selection(bits, words, top_k, out, p, t, rows, nv_out, warp_sums, pts);
}

}  // namespace

cudaError_t launch_topk_hist(const float *scores, int64_t ld, const int32_t *vis,
                             const uint32_t *hist, int32_t n_q, int32_t max_valid, int32_t top_k,
                             int32_t *sel, int32_t *counts, uint64_t *cand, int32_t cap,
                             int4 *chunk_info, int32_t *idx, const PathParams &p, int32_t *rows,
                             int32_t ld_rows, int32_t *n_valid, cudaStream_t s) {
    if (n_q == 0) return cudaSuccess;
    if (max_valid <= kSingleMaxV) {
        cudaError_t e = cudaFuncSetAttribute(
            topk_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSingleSmem);
        if (e != cudaSuccess) return e;
        count_launch();
        return launch_pdl(topk_single_kernel, dim3(n_q), dim3(kThreads), kSingleSmem, s, scores,
                          ld, vis, hist, top_k, idx, p, rows, ld_rows, n_valid);
    }
    const int32_t chunks = static_cast<int32_t>(ceil_div(std::max(max_valid, 1), kChunk));
    const dim3 grid_c(static_cast<unsigned>(chunks), n_q);
    const int32_t ld_chunks = static_cast<int32_t>(topk_chunk_slots(ld));
    count_launch();
    cudaError_t e = launch_pdl(topk_count_kernel, grid_c, dim3(kCollectThreads), 0, s, scores, ld,
                               vis, hist, top_k, sel, chunk_info, ld_chunks, counts, cand, cap);
    if (e != cudaSuccess) return e;
    const size_t smem = finalize_smem_bytes(cap);
    e = cudaFuncSetAttribute(topk_finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    return launch_pdl(topk_finalize_kernel, dim3(n_q), dim3(kThreads), smem, s, scores, ld, vis,
                      top_k, (const int32_t *)sel, (const int4 *)chunk_info, ld_chunks,
                      (const int32_t *)counts, (const uint64_t *)cand, cap, idx, p, rows,
                      ld_rows, n_valid);
}

cudaError_t launch_topk_rowwise(const float *scores, int64_t ld, const int32_t *valid_len,
                                int32_t max_valid, const PathParams *p, int32_t n_q,
                                int32_t top_k, int32_t *idx, int32_t *status, cudaStream_t s) {
    if (n_q == 0) return cudaSuccess;
    PathParams pp{};
    if (p != nullptr) pp = *p;
    count_launch();
    return launch_pdl(topk_rowwise_kernel, dim3(n_q), dim3(kThreads), 0, s, scores, ld, valid_len,
                      max_valid, pp, top_k, idx, status);
}

}  // namespace sa
