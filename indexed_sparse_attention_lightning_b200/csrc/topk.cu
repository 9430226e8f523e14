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

__global__ void __launch_bounds__(kThreads)
topk_rowwise_kernel(const float *__restrict__ scores, int64_t ld,
                    const int32_t *__restrict__ valid_len, int32_t max_valid, const PathParams p,
                    int32_t top_k, int32_t *__restrict__ idx, int32_t *status) {
    __shared__ unsigned hist[256];
    __shared__ int warp_sums[33];
    __shared__ unsigned sel_digit, sel_above;

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
    const float *row = scores + (int64_t)t * ld;
    int32_t *out = idx + (int64_t)t * top_k;

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
            unsigned digit = match ? (key >> shift) & 255u : 256u + 0u;
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

}  // namespace

cudaError_t launch_topk_rowwise(const float *scores, int64_t ld, const int32_t *valid_len,
                                int32_t max_valid, const PathParams *p, int32_t n_q,
                                int32_t top_k, int32_t *idx, int32_t *status, cudaStream_t s) {
    if (n_q == 0) return cudaSuccess;
    PathParams pp{};
    if (p != nullptr) pp = *p;
    count_launch();
    topk_rowwise_kernel<<<n_q, kThreads, 0, s>>>(scores, ld, valid_len, max_valid, pp, top_k,
                                                 idx, status);
    return cudaGetLastError();
}

}  // namespace sa
