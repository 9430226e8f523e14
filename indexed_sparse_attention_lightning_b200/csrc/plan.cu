// plan.cu -- per-call schedule: validated visible length of every query and
// the inclusive prefix of its 128-key tile count, which the persistent
// kernels use to split the concatenated tiles of all queries evenly.  The
// same launch clears the per-call histograms and counters.  With groups of
// `group` queries (chunked prefill: consecutive queries of one sequence that
// share every key tile), the prefix runs over groups instead: a group's tile
// count is that of its longest query, and tile_end[g] is written for group g.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kThreads = 1024;

__global__ void __launch_bounds__(kThreads)
plan_kernel(const PathParams p, int32_t *vis, int32_t *tile_end, int32_t tile, uint32_t *zero,
            size_t zero_words, int32_t clear_status, int32_t group) {
    pdl_wait();
    pdl_trigger();
    // CTA 0 is the only one that reports, so it clears the status word first
    if (clear_status && blockIdx.x == 0 && threadIdx.x < kStatusBytes / 4) p.status[threadIdx.x] = 0;
    for (size_t i = (size_t)blockIdx.x * kThreads + threadIdx.x; i < zero_words;
         i += (size_t)gridDim.x * kThreads)
        zero[i] = 0u;
    if (blockIdx.x != 0) return;
    __syncthreads();
    __shared__ int32_t warp_sums[32];
    __shared__ int32_t carry;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    for (int base = 0; base < p.n_q; base += kThreads) {
        const int t = base + threadIdx.x;
        int32_t V = t < p.n_q ? visible_len(p, t) : 0;
        int32_t tiles = (V + tile - 1) / tile;
        if (group == 4) {  // groups of 4 lanes: the longest query, one sequence
            const int32_t seq = t < p.n_q ? __ldg(p.q_seq + t) : -1;
            const int32_t seq0 = __shfl_sync(0xffffffffu, seq, lane & ~3);
            int bad = (t < p.n_q && seq != seq0) ? 1 : 0;
            bad |= __shfl_xor_sync(0xffffffffu, bad, 1);
            bad |= __shfl_xor_sync(0xffffffffu, bad, 2);
            int32_t m = tiles;
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
            m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
            if (bad) {  // a group must hold one sequence: report it, and its queries see nothing
                if ((lane & 3) == 0) report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_POSITION);
                m = 0;
                V = 0;
            }
            tiles = (lane & 3) == 0 ? m : 0;
        }
        int32_t x = tiles;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_sums[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int32_t w = warp_sums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int32_t y = __shfl_up_sync(0xffffffffu, w, o);
                if (lane >= o) w += y;
            }
            warp_sums[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        const int32_t incl = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + x;
        if (t < p.n_q) {
            vis[t] = V;
            if (group == 4) {
                if ((t & 3) == 0) tile_end[t >> 2] = incl;
            } else {
                tile_end[t] = incl;
            }
        }
        __syncthreads();
        if (threadIdx.x == kThreads - 1) carry = incl;
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_plan(const PathParams &p, int32_t *vis, int32_t *tile_end, int32_t tile,
                        uint32_t *zero, size_t zero_words, bool clear_status, cudaStream_t s,
                        int32_t group) {
    if (p.n_q == 0) return cudaSuccess;
    const int64_t blocks =
        std::max<int64_t>(1, std::min<int64_t>(num_sms(), ceil_div(zero_words, 4 * kThreads)));
    count_launch();
    return launch_pdl(plan_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0, s, p,
                      vis, tile_end, tile, zero, zero_words, clear_status ? 1 : 0, group);
}

int num_sms() {
    // one slot per device, safe to read and fill from any host thread (the
    // value is the same whoever stores it)
    constexpr int kMaxDevices = 64;
    static std::atomic<int> cached[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < kMaxDevices) {
        const int n = cached[dev].load(std::memory_order_relaxed);
        if (n > 0) return n;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev >= 0 && dev < kMaxDevices) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace sa
