// cp.cu -- the exchange steps of context-parallel decode over several GPUs.
//
// One long sequence's context is split into contiguous shards, one per GPU;
// each GPU scores the positions it holds and keeps its own top-K, the
// candidates of all GPUs are gathered, every GPU merges them into the same
// global top-K, attends over the selected rows it holds, and the partial
// outputs are merged by their log-sum-exp ("Inference Acceleration for New
// Large Model Architectures" §5.1-5.2: context parallelism splits the
// sequence, each device handles a portion; "Long-Context LLM Inference
// Optimization", Distributed Scaling).  The collectives themselves (two
// all-gathers) belong to the caller; these kernels are the steps around them:
//   cand_emit_kernel   this GPU's top-K as (score, global position) pairs;
//   merge_kernel       the global top-K of all GPUs' candidates, and the part
//                      of it this GPU holds, as local positions;
//   combine_kernel     out = sum_r exp(lse_r - lse) o_r, lse = log sum_r exp(lse_r).
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kEmitThreads = 256;
constexpr int kMergeThreads = 1024;
constexpr int kCombineThreads = 128;

__global__ void __launch_bounds__(kEmitThreads)
cand_emit_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ idx,
                 int32_t top_k, const int32_t *__restrict__ offsets,
                 float *__restrict__ cand_score, int32_t *__restrict__ cand_pos) {
    pdl_wait();
    pdl_trigger();
    const int64_t t = blockIdx.x;
    const int32_t offset = offsets[t];
    for (int k = threadIdx.x; k < top_k; k += kEmitThreads) {
        const int32_t i = idx[t * top_k + k];
        cand_score[t * top_k + k] = i >= 0 ? scores[t * ld + i] : -INFINITY;
        cand_pos[t * top_k + k] = i >= 0 ? i + offset : -1;
    }
}

// Exclusive prefix of v over the block (1024 threads) in thread order.
__device__ __forceinline__ int block_prefix(int v, int *warp_sums, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = warp_sums[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, wi, o);
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

// One CTA per query.  Candidate i of the query (rank-major: rank i / K, slot
// i % K) gets the composite key (order-preserving score key, inverted
// position): distinct for distinct positions, larger for a higher score and,
// at equal scores, for the lower position; padding (position -1) gets 0 and
// ranks last.  The K largest keys are selected by radix passes of 8-bit
// digits from the top (stopping once a whole digit bin is taken), then
// written in candidate order -- ascending positions, because every rank's
// list is ascending and the ranks' shards follow one another.
__global__ void __launch_bounds__(kMergeThreads)
merge_kernel(const float *__restrict__ cand_score, const int32_t *__restrict__ cand_pos,
             int32_t n_ranks, int32_t n_q, int32_t top_k, const int32_t *__restrict__ pos_lo,
             const int32_t *__restrict__ pos_hi, int32_t *__restrict__ idx_global,
             int32_t *__restrict__ idx_local) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint64_t keys[];  // [n_ranks * top_k]
    __shared__ unsigned hist[256];
    __shared__ int warp_sums[33];
    __shared__ int sel_digit, sel_above, sel_count;
    const int t = blockIdx.x, tid = threadIdx.x;
    const int n = n_ranks * top_k;
    int n_valid = 0;
    for (int i = tid; i < n; i += kMergeThreads) {
        const int64_t g = ((int64_t)(i / top_k) * n_q + t) * top_k + i % top_k;
        const int32_t pos = cand_pos[g];
        uint64_t key = 0;
        if (pos >= 0) {
            key = (static_cast<uint64_t>(order_key(cand_score[g])) << 32) |
                  (0xFFFFFFFFu - static_cast<uint32_t>(pos));
            ++n_valid;
        }
        keys[i] = key;
    }
    int total;
    block_prefix(n_valid, warp_sums, &total);  // also orders the key stores
    n_valid = total;
    // threshold: the K-th largest key (every valid key when there are fewer)
    uint64_t prefix = 0, mask = 0;
    if (n_valid > top_k) {
        int remaining = top_k;
        for (int shift = 56; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += kMergeThreads) hist[i] = 0;
            __syncthreads();
            for (int i = tid; i < n; i += kMergeThreads) {
                const uint64_t k = keys[i];
                if (k != 0 && (k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
            }
            __syncthreads();
            const int d = 255 - tid;  // digits in descending order (threads 0..255)
            const int cd = tid < 256 ? static_cast<int>(hist[d]) : 0;
            const int ex = block_prefix(cd, warp_sums, &total);
            if (tid < 256 && ex < remaining && ex + cd >= remaining) {
                sel_digit = d;
                sel_above = ex;
                sel_count = cd;
            }
            __syncthreads();
            prefix |= static_cast<uint64_t>(sel_digit) << shift;
            mask |= static_cast<uint64_t>(255u) << shift;
            remaining -= sel_above;
            const bool whole = remaining == sel_count;
            __syncthreads();
            if (whole) break;
        }
    }
    // selected: valid and (k & mask) >= prefix; exactly min(K, n_valid) of them
    const int32_t lo = pos_lo[t], hi = pos_hi[t];
    int base = 0;
    for (int i0 = 0; i0 < n; i0 += kMergeThreads) {
        const int i = i0 + tid;
        const uint64_t k = i < n ? keys[i] : 0;
        const bool take = k != 0 && (k & mask) >= prefix;
        const int slot = base + block_prefix(take ? 1 : 0, warp_sums, &total);
        if (take && slot < top_k) {
            const int32_t pos = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(k));
            idx_global[(int64_t)t * top_k + slot] = pos;
            idx_local[(int64_t)t * top_k + slot] = (pos >= lo && pos < hi) ? pos - lo : -1;
        }
        base += total;
    }
    for (int s = base + tid; s < top_k; s += kMergeThreads) {
        idx_global[(int64_t)t * top_k + s] = -1;
        idx_local[(int64_t)t * top_k + s] = -1;
    }
}

// One CTA per (query, head): the part weights once in shared memory, then the
// threads sweep the head's d output values.
constexpr int kMaxParts = 256;
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const float *__restrict__ o_part, const float *__restrict__ lse_part,
               int32_t n_parts, int64_t rows, int32_t d, void *out, int32_t out_dtype,
               float *lse) {
    pdl_wait();
    pdl_trigger();
    __shared__ float w_s[kMaxParts];
    const int64_t row = blockIdx.x;  // t * heads + h
    for (int r = threadIdx.x; r < n_parts; r += kCombineThreads)
        w_s[r] = lse_part[(int64_t)r * rows + row];
    __syncthreads();
    if (threadIdx.x < 32) {
        float m = -INFINITY;
        for (int r = threadIdx.x; r < n_parts; r += 32) m = fmaxf(m, w_s[r]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float sum = 0.f;
        for (int r = threadIdx.x; r < n_parts; r += 32) {
            const float ls = w_s[r];
            const float w = (m == -INFINITY || ls == -INFINITY) ? 0.f : expf(ls - m);
            w_s[r] = w;
            sum += w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float inv = sum > 0.f ? 1.f / sum : 0.f;
        for (int r = threadIdx.x; r < n_parts; r += 32) w_s[r] *= inv;
        if (lse != nullptr && threadIdx.x == 0) lse[row] = sum > 0.f ? m + logf(sum) : -INFINITY;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < d; c += kCombineThreads) {
        float acc = 0.f;
        for (int r = 0; r < n_parts; ++r) {
            const float w = w_s[r];
            if (w != 0.f) acc += w * o_part[((int64_t)r * rows + row) * d + c];
        }
        if (out_dtype == SA_BF16)
            static_cast<__nv_bfloat16 *>(out)[row * d + c] = __float2bfloat16_rn(acc);
        else
            static_cast<float *>(out)[row * d + c] = acc;
    }
}

}  // namespace

int32_t cp_merge_max_candidates() { return 24576; }
int32_t cp_combine_max_parts() { return kMaxParts; }

cudaError_t launch_cand_emit(const float *scores, int64_t ld, const int32_t *idx, int32_t n_q,
                             int32_t top_k, const int32_t *offset, float *cand_score,
                             int32_t *cand_pos, cudaStream_t s) {
    if (n_q == 0) return cudaSuccess;
    count_launch();
    return launch_pdl(cand_emit_kernel, dim3(n_q), dim3(kEmitThreads), 0, s, scores, ld, idx,
                      top_k, offset, cand_score, cand_pos);
}

cudaError_t launch_cp_merge(const float *cand_score, const int32_t *cand_pos, int32_t n_ranks,
                            int32_t n_q, int32_t top_k, const int32_t *pos_lo,
                            const int32_t *pos_hi, int32_t *idx_global, int32_t *idx_local,
                            cudaStream_t s) {
    if (n_q == 0) return cudaSuccess;
    const size_t smem = sizeof(uint64_t) * (size_t)n_ranks * top_k;
    cudaError_t e =
        cudaFuncSetAttribute(merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    return launch_pdl(merge_kernel, dim3(n_q), dim3(kMergeThreads), smem, s, cand_score, cand_pos,
                      n_ranks, n_q, top_k, pos_lo, pos_hi, idx_global, idx_local);
}

cudaError_t launch_cp_combine(const float *o_part, const float *lse_part, int32_t n_parts,
                              int64_t rows, int32_t d, void *out, int32_t out_dtype, float *lse,
                              cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    count_launch();
    return launch_pdl(combine_kernel, dim3(static_cast<unsigned>(rows)), dim3(kCombineThreads), 0,
                      s, o_part, lse_part, n_parts, rows, d, out, out_dtype, lse);
}

}  // namespace sa
