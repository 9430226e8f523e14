// sfa_mma.cu -- sparse MLA attention on the 5th-generation tensor cores.
//
// For query t and its selected latent rows s ("Optimizing Next-Gen LLM
// Inference" §3.3: attention only on the selected positions, reading the cache
// by index; "Inference Acceleration for New Large Model Architectures" §3.2:
// aggregated, vectorised sparse reads; "Engineering Practices for Optimizing
// Ultra-Large Sparse Attention Model Inference" §3.1: index construction, block
// loading with asynchronous prefetch, local attention on matrix units):
//     z_s = sm_scale * q[t,h,:] . kv[s,:]   (576-d: 512 latent + 64 rope)
//     out[t,h,:] = sum_s softmax(z)_s kv[s, 0:512],   lse = log sum_s exp(z_s)
//
// B200 mapping.  All 128 absorbed-query heads share the selected rows, so both
// contractions are dense per key tile.  One CTA owns 64 heads of one query
// (two CTAs per query) and walks 64-key tiles of its selected rows:
//     S  = Q K^T   M = 64 heads, N = 64 keys, K = 576   (A = Q from TMEM)
//     O += P V     M = 64 heads, N = 2 x 256 dims, K = 64 keys
// An M = 64 accumulator fills lanes 0-15 of each 32-lane TMEM subpartition; a
// second one may sit on lanes 16-31.  So Q (288 columns of bf16 pairs) and two
// S buffers live on the lower half-lanes and O (64 x 512 fp32, all 512
// columns) on the upper half-lanes: head m's S row is lane 32(m/16) + m%16,
// its O row that lane + 16, i.e. the same warp.  Each tile's 64 full 1152-byte
// rows are copied once into a 128-byte-swizzled stage that is the K-major B
// operand of S and, read MN-major, the B operand of P V.
//
// Roles (256 threads, one CTA per SM):
//   warp 0     lane 0 issues the MMAs from a non-blocking loop -- S of a tile
//              as soon as its rows are in and an S buffer is free, P V as soon
//              as P is written -- and commits them to mbarriers;
//   warps 1-3  copy the selected rows (16-byte cp.async, the swizzle applied
//              in the addresses) into a 3-stage ring freed by each tile's P V;
//   warps 4-7  put Q into TMEM, then run the online softmax: lane l < 16 of
//              warp 4 + j owns head 16j + l (a whole 64-key S row, no
//              exchange); P goes to shared memory as bf16; O is rescaled in
//              TMEM (16-lane accesses that leave Q and S alone) only when a
//              head's running maximum grows by more than 2^8; finally lanes
//              16-31 write O / l.
// Selected positions are turned into physical cache rows by a small kernel
// first (sfa_rows_kernel).  All waits are bounded; a timeout is reported in
// the workspace status word.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace sa {
namespace {
using namespace sm100;

constexpr int kHeadsCta = 64;
constexpr int kDl = 512, kDr = 64, kD = kDl + kDr;
constexpr int kBlocks = kD / 64;  // 64-dim (128-byte) column blocks of a row
constexpr int kTile = 64;         // selected keys per tile
constexpr int kStages = 3;
constexpr int kProducerWarps = 3;
constexpr int kThreads = 256;
constexpr int kMaxK = 2048;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;    // lower half-lanes: Q, 288 columns
constexpr uint32_t kColS = 288;  // lower half-lanes: two S buffers of 64 columns
constexpr uint32_t kLaneO = 16;  // O: upper half-lanes, columns [0, 512)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kChunksPerRow = kD * 2 / 16;  // 72 sixteen-byte pieces of a row

struct SfaSmem {
    uint8_t kv[kStages][kBlocks][kTile * 128];  // 64 full rows, 128-byte swizzle per block
    uint8_t p[kHeadsCta * 128];                 // P (bf16), K-major, 128-byte swizzle
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t s_full[2], p_full, o_done, q_ready;
    uint32_t tmem_base;
    int abort;
};

static_assert(sizeof(SfaSmem) + 1024 <= 232448, "shared memory budget of one CTA");
static_assert(kColS + 2 * kTile <= kTmemCols && kBlocks * 32 == (int)kColS, "TMEM columns");

struct SfaArgs {
    PathParams p;
    const int32_t *rows;     // [n_q, ld_rows] physical rows, padded to whole tiles
    const int32_t *n_valid;  // [n_q]
    int32_t ld_rows;
    int32_t splits;
    void *out;               // [n_q, 128, 512] (splits == 1)
    int32_t out_dtype;
    float *lse;              // [n_q, 128] or null (splits == 1)
    float *o_part;           // [n_q, splits, 128, 512] (splits > 1)
    float *lse_part;         // [n_q, splits, 128]      (splits > 1)
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *status) {
    bool ok = true;
    if (lane_id() == 0) ok = mbar_wait(bar, parity, abort_flag, status);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

// Tiles [j0, j1) of the compacted key list handled by this split.
__device__ __forceinline__ void split_range(int32_t n_valid, int32_t split, int32_t splits,
                                            int32_t &j0, int32_t &j1) {
    const int32_t tiles = (n_valid + kTile - 1) / kTile;
    j0 = (int32_t)((int64_t)tiles * split / splits);
    j1 = (int32_t)((int64_t)tiles * (split + 1) / splits);
}

// Query t's selected positions -> physical cache rows, in list order with the
// -1 padding dropped, then padded with the first row to whole tiles (the
// softmax masks the padding).  Out-of-range positions and bad page ids are
// skipped and reported.  One CTA of 128 threads per query.
__global__ void __launch_bounds__(128)
sfa_rows_kernel(const PathParams p, const int32_t *__restrict__ idx, int32_t K, int32_t ld_rows,
                int32_t *__restrict__ rows, int32_t *__restrict__ n_valid_out) {
    __shared__ int32_t warp_cnt[4];
    __shared__ int32_t first_row;
    const int t = blockIdx.x, et = threadIdx.x, ew = et >> 5, lane = et & 31;
    const int32_t V = visible_len(p, t);
    const int32_t seq = p.q_seq[t];
    const int32_t *sel = idx + (int64_t)t * K;
    int32_t *out = rows + (int64_t)t * ld_rows;
    // all index and page-table loads in flight at once (16 per thread), then
    // an ordered compaction over the 16 rounds of 128 entries
    constexpr int kRounds = kMaxK / 128;
    int32_t phys[kRounds];
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
        const int k = r * 128 + et;
        phys[r] = k < K ? __ldg(sel + k) : -1;
    }
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
        const int32_t s = phys[r];
        int32_t v = -1;
        if (s >= V) {
            report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_INDEX);
        } else if (s >= 0) {
            const int64_t row = phys_row(p.page_table, p.max_pages, p.num_pages, seq, s);
            if (row < 0) report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_PAGE);
            else v = static_cast<int32_t>(row);
        }
        phys[r] = v;
    }
    int32_t base = 0;
#pragma unroll
    for (int r = 0; r < kRounds; ++r) {
        const unsigned bal = __ballot_sync(0xffffffffu, phys[r] >= 0);
        if (lane == 0) warp_cnt[ew] = __popc(bal);
        __syncthreads();
        int32_t off = base, tot = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            if (w < ew) off += warp_cnt[w];
            tot += warp_cnt[w];
        }
        const int32_t pos = off + __popc(bal & ((1u << lane) - 1u));
        if (phys[r] >= 0) {
            out[pos] = phys[r];
            if (pos == 0) first_row = phys[r];
        }
        __syncthreads();
        base += tot;
    }
    const int32_t n_valid = base;
    const int32_t padded = ((n_valid + kTile - 1) / kTile) * kTile;
    if (n_valid > 0) {
        const int32_t r0 = first_row;  // written before the last barrier above
        for (int c = n_valid + et; c < padded; c += 128) out[c] = r0;
    }
    if (et == 0) n_valid_out[t] = n_valid;
}

__global__ void __launch_bounds__(kThreads, 1) sfa_mma_kernel(const SfaArgs a) {
    extern __shared__ uint8_t smem_raw[];
    SfaSmem &sm = *reinterpret_cast<SfaSmem *>(align1024(smem_raw));
    const PathParams &p = a.p;
    const int hh = blockIdx.x & 1;  // which 64 heads
    const int unit = blockIdx.x >> 1;
    const int t = unit / a.splits, split = unit % a.splits;
    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.kv_full[s], 32 * kProducerWarps);  // one cp.async arrival per lane
            mbar_init(&sm.kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) mbar_init(&sm.s_full[b], 1);
        mbar_init(&sm.p_full, 4);  // the four softmax warps
        mbar_init(&sm.o_done, 1);
        mbar_init(&sm.q_ready, 4);
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort;
    int32_t *status = p.status;
    const int32_t n_valid = a.n_valid[t];
    int32_t j0, j1;
    split_range(n_valid, split, a.splits, j0, j1);
    const int T = j1 - j0;

    if (warp >= 4) {
        const int j = warp & 3;  // TMEM subpartition of this warp
        const bool owner = lane < 16;
        const int h = 16 * j + (lane & 15);  // head within this CTA (owner: S row, else O row)
        const uint32_t lane_lo = static_cast<uint32_t>(32 * j) << 16;
        const uint32_t lane_hi = static_cast<uint32_t>(32 * j + kLaneO) << 16;
        // ----------------------------------------------- Q into TMEM ---
        // 32-lane stores: lanes 16-31 receive a copy on O's columns, which
        // the first P V overwrites.
        if (T > 0) {
            const uint4 *qrow = reinterpret_cast<const uint4 *>(
                static_cast<const __nv_bfloat16 *>(p.q) +
                ((int64_t)t * 128 + kHeadsCta * hh + h) * kD);
#pragma unroll 1
            for (int c = 0; c < kBlocks; ++c) {
                uint32_t v[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint4 x = __ldg(qrow + 8 * c + i);
                    v[4 * i] = x.x;
                    v[4 * i + 1] = x.y;
                    v[4 * i + 2] = x.z;
                    v[4 * i + 3] = x.w;
                }
                tmem_st32_u(tmem + lane_lo + kColQ + 32 * c, v);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.q_ready);
        }

        // ----------------------------------------------- online softmax ---
        // The loop never leaves early: after a failed wait (a timeout raised
        // the abort flag) it keeps going without waiting or touching TMEM.
        const float sl2 = p.sm_scale * kLog2e;
        float m_run = -INFINITY, l_sum = 0.f;
        bool ok = true;
        for (int n = 0; n < T; ++n) {
            const int sb = n & 1;
            if (ok) ok = warp_wait(&sm.s_full[sb], (n >> 1) & 1, abort_flag, status);
            float s0[32], s1[32];
            if (ok) {
                tc_fence_after();
                tmem_ld32(tmem + lane_lo + kColS + kTile * sb, s0);
                tmem_ld32(tmem + lane_lo + kColS + kTile * sb + 32, s1);
                tmem_wait_ld();
            }
            const int kvalid = owner ? n_valid - (j0 + n) * kTile : 0;
            float tmax = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                s0[i] = (ok && i < kvalid) ? s0[i] * sl2 : -INFINITY;
                s1[i] = (ok && i + 32 < kvalid) ? s1[i] * sl2 : -INFINITY;
                tmax = fmaxf(tmax, fmaxf(s0[i], s1[i]));
            }
            // lazy rescaling: the running maximum moves only on a large jump
            const bool grow = tmax > m_run + kRescaleLog2;
            const float m_new = grow ? tmax : m_run;
            const float f = (grow && n > 0) ? exp2f(m_run - m_new) : 1.f;
            uint32_t packed[32];
            float l_tile = 0.f;
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const float a0 = exp2f(s0[i] - m_new), a1 = exp2f(s0[i + 1] - m_new);
                const float b0 = exp2f(s1[i] - m_new), b1 = exp2f(s1[i + 1] - m_new);
                l_tile += (a0 + a1) + (b0 + b1);
                __nv_bfloat162 x = __floats2bfloat162_rn(a0, a1);
                __nv_bfloat162 y = __floats2bfloat162_rn(b0, b1);
                packed[i / 2] = *reinterpret_cast<uint32_t *>(&x);
                packed[16 + i / 2] = *reinterpret_cast<uint32_t *>(&y);
            }
            // O and the P buffer belong to P V of the previous tile until it is done
            if (n > 0 && ok) ok = warp_wait(&sm.o_done, (n - 1) & 1, abort_flag, status);
            if (ok && __any_sync(0xffffffffu, grow && n > 0)) {
                tc_fence_after();
                // 16-lane accesses to lanes 16-31: thread i holds rows i/4
                // and i/4 + 8 of them (registers 4r, 4r+1 and 4r+2, 4r+3)
                const float fa = __shfl_sync(0xffffffffu, f, lane >> 2);
                const float fb = __shfl_sync(0xffffffffu, f, (lane >> 2) + 8);
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t v[64];
                    tmem_ld_16x256b_x16(tmem + lane_hi + 128 * c, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        v[4 * r] = __float_as_uint(__uint_as_float(v[4 * r]) * fa);
                        v[4 * r + 1] = __float_as_uint(__uint_as_float(v[4 * r + 1]) * fa);
                        v[4 * r + 2] = __float_as_uint(__uint_as_float(v[4 * r + 2]) * fb);
                        v[4 * r + 3] = __float_as_uint(__uint_as_float(v[4 * r + 3]) * fb);
                    }
                    tmem_st_16x256b_x16(tmem + lane_hi + 128 * c, v);
                }
                tmem_wait_st();
            }
            l_sum = l_sum * f + l_tile;
            m_run = m_new;
            if (owner) {
                uint8_t *prow = sm.p + h * 128;
                const int sw = h & 7;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(prow + ((c ^ sw) << 4)) =
                        make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2],
                                   packed[4 * c + 3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.p_full);
        }
        if (ok && T > 0) ok = warp_wait(&sm.o_done, (T - 1) & 1, abort_flag, status);
        tc_fence_after();
        const float inv = (ok && l_sum > 0.f) ? 1.f / l_sum : 0.f;
        const float lse_v = (ok && l_sum > 0.f) ? (m_run + log2f(l_sum)) * kLn2 : -INFINITY;
        const float inv_o = __shfl_sync(0xffffffffu, inv, lane & 15);
        const int head = kHeadsCta * hh + h;
        const int64_t row = (int64_t)t * 128 + head;
        // 32-lane loads: lanes 16-31 receive the O rows
#pragma unroll 1
        for (int c = 0; c < kDl / 32; ++c) {
            float v[32];
            if (ok && T > 0) {
                tmem_ld32(tmem + lane_lo + 32 * c, v);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.f;
            }
            if (owner) continue;
            const int dv = 32 * c;
            if (a.splits == 1) {
                if (a.out_dtype == SA_BF16) {
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        __nv_bfloat162 b2 =
                            __floats2bfloat162_rn(v[i] * inv_o, v[i + 1] * inv_o);
                        w[i / 2] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.out) +
                                                           row * kDl + dv);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
                } else {
                    float4 *dst =
                        reinterpret_cast<float4 *>(static_cast<float *>(a.out) + row * kDl + dv);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(v[4 * i] * inv_o, v[4 * i + 1] * inv_o,
                                             v[4 * i + 2] * inv_o, v[4 * i + 3] * inv_o);
                }
            } else {
                const int64_t prow_i = ((int64_t)t * a.splits + split) * 128 + head;
                float4 *dst = reinterpret_cast<float4 *>(a.o_part + prow_i * kDl + dv);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(v[4 * i] * inv_o, v[4 * i + 1] * inv_o,
                                         v[4 * i + 2] * inv_o, v[4 * i + 3] * inv_o);
            }
        }
        if (owner) {
            if (a.splits == 1) {
                if (a.lse != nullptr) a.lse[row] = lse_v;
            } else {
                a.lse_part[((int64_t)t * a.splits + split) * 128 + head] = lse_v;
            }
        }
    } else if (warp >= 1) {
        // ---------------------------------------------- row producers ---
        // warp 1 + w copies keys w, w + 3, ... of each tile; a key's 72
        // sixteen-byte pieces go to lanes (piece % 32) in three steps.
        const int pw = warp - 1;
        const uint8_t *kv = static_cast<const uint8_t *>(p.kv);
        const int32_t *rows = a.rows + (int64_t)t * a.ld_rows;
        for (int n = 0; n < T; ++n) {
            const int st = n % kStages;
            if (!warp_wait(&sm.kv_empty[st], ((n / kStages) & 1) ^ 1, abort_flag, status)) break;
            const int32_t *rr = rows + (j0 + n) * kTile;
            const int32_t r_lo = __ldg(rr + lane), r_hi = __ldg(rr + 32 + lane);
            const uint32_t dst0 = smem_u32(sm.kv[st][0]);
#pragma unroll 2
            for (int k = pw; k < kTile; k += kProducerWarps) {
                const int32_t r = __shfl_sync(0xffffffffu, k < 32 ? r_lo : r_hi, k & 31);
                const uint8_t *src = kv + (int64_t)r * (kD * 2);
                const uint32_t dk = dst0 + k * 128;
                const int sw = k & 7;
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                    const int c = lane + 32 * i;
                    if (c < kChunksPerRow)
                        cp_async16(dk + (c >> 3) * (kTile * 128) + (((c & 7) ^ sw) << 4),
                                   src + c * 16);
                }
            }
            cp_async_arrive(&sm.kv_full[st]);
        }
        cp_async_wait_all();
    } else if (lane == 0 && T > 0) {
        // ---------------------------------------------------- MMA issuer ---
        constexpr uint32_t id_s = instr_desc(64, kTile, 1 /*bf16*/, 0, 0);
        constexpr uint32_t id_pv = instr_desc(64, 256, 1 /*bf16*/, 0, 1);
        bool ok = mbar_wait(&sm.q_ready, 0, abort_flag, status);
        int ns = 0, np = 0;  // next S and next P V to issue
        long long t0 = clock64();
        uint32_t idle = 0;
        while (ok && np < T) {
            bool progressed = false;
            // S(ns) needs its rows and a free S buffer: the softmax of tile
            // ns - 2 is over once P V of it was issued
            if (ns < T && ns < np + 2) {
                const int st = ns % kStages;
                if (mbar_test(&sm.kv_full[st], (ns / kStages) & 1)) {
                    fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t d = tmem + kColS + kTile * (ns & 1);
#pragma unroll 1
                    for (int b = 0; b < kBlocks; ++b) {
                        const uint64_t bd = desc_kmajor_sw128(smem_u32(sm.kv[st][b]));
#pragma unroll
                        for (int k = 0; k < 4; ++k)  // 16 dims (32 bytes) per instruction
                            mma_bf16_ts(d, tmem + kColQ + 32 * b + 8 * k, bd + 2 * k, id_s,
                                        (b | k) != 0);
                    }
                    mma_commit(&sm.s_full[ns & 1]);
                    ++ns;
                    progressed = true;
                }
            }
            // P V(np) needs P of tile np
            if (np < ns && mbar_test(&sm.p_full, np & 1)) {
                fence_proxy_async_smem();
                tc_fence_after();
                const int st = np % kStages;
                const uint64_t ad = desc_kmajor_sw128(smem_u32(sm.p));
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const uint32_t vb = smem_u32(sm.kv[st][4 * half]);
#pragma unroll
                    for (int k = 0; k < 4; ++k)  // 16 keys per instruction
                        mma_bf16(tmem + (kLaneO << 16) + 256 * half, ad + 2 * k,
                                 desc_mnmajor_sw128(vb + 2048 * k, kTile * 128, 1024), id_pv,
                                 (np > 0 || k > 0) ? 1u : 0u);
                }
                mma_commit(&sm.o_done);
                if (np + kStages < T) mma_commit(&sm.kv_empty[st]);
                ++np;
                progressed = true;
            }
            if (progressed) {
                t0 = clock64();
                idle = 0;
            } else if ((++idle & 63) == 0 && wait_expired(t0, abort_flag, status)) {
                break;
            }
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// out = sum_s w_s o_s with w_s = exp(lse_s - lse), lse = log sum_s exp(lse_s).
__global__ void __launch_bounds__(128)
sfa_combine_kernel(const float *__restrict__ o_part, const float *__restrict__ lse_part,
                   int32_t splits, void *out, int32_t out_dtype, float *lse) {
    const int64_t row = blockIdx.x;  // t * 128 + head
    const int64_t t = row >> 7, head = row & 127;
    float m = -INFINITY;
    for (int s = 0; s < splits; ++s) m = fmaxf(m, lse_part[(t * splits + s) * 128 + head]);
    float acc[4] = {0.f, 0.f, 0.f, 0.f}, wsum = 0.f;
    if (m != -INFINITY) {
        for (int s = 0; s < splits; ++s) {
            const float ls = lse_part[(t * splits + s) * 128 + head];
            const float w = ls == -INFINITY ? 0.f : __expf(ls - m);
            wsum += w;
            const float4 v = reinterpret_cast<const float4 *>(
                o_part + ((t * splits + s) * 128 + head) * kDl)[threadIdx.x];
            acc[0] += w * v.x;
            acc[1] += w * v.y;
            acc[2] += w * v.z;
            acc[3] += w * v.w;
        }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    if (out_dtype == SA_BF16) {
        __nv_bfloat162 a = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
        __nv_bfloat162 b = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
        uint2 w = make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
        reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(out) + row * kDl)[threadIdx.x] = w;
    } else {
        reinterpret_cast<float4 *>(static_cast<float *>(out) + row * kDl)[threadIdx.x] =
            make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    }
    if (lse != nullptr && threadIdx.x == 0) lse[row] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

}  // namespace

bool sfa_mma_supported(const PathParams &p, int32_t top_k) {
    return p.kv_dtype == SA_BF16 && p.q_dtype == SA_BF16 && p.heads == 128 &&
           p.d_latent == kDl && p.d_rope == kDr && top_k <= kMaxK &&
           (int64_t)p.num_pages * 64 < (int64_t(1) << 31);
}

int32_t sfa_splits(int32_t n_q, int32_t top_k) {
    const int32_t ctas = std::max(1, num_sms());
    const int32_t max_tiles = (top_k + kTile - 1) / kTile;
    if (n_q <= 0) return 1;
    return std::max(1, std::min(max_tiles, ctas / (2 * n_q)));
}

int32_t sfa_rows_ld(int32_t top_k) { return (int32_t)round_up(top_k > 0 ? top_k : 1, kTile); }

cudaError_t launch_sfa_mma(const PathParams &p, const int32_t *idx, int32_t top_k, int32_t splits,
                           int32_t *rows, int32_t *n_valid, void *out, int32_t out_dtype,
                           float *lse, float *o_part, float *lse_part, cudaStream_t s) {
    if (p.n_q == 0) return cudaSuccess;
    const int32_t ld_rows = sfa_rows_ld(top_k);
    count_launch();
    sfa_rows_kernel<<<static_cast<unsigned>(p.n_q), 128, 0, s>>>(p, idx, top_k, ld_rows, rows,
                                                                 n_valid);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    SfaArgs a{p, rows, n_valid, ld_rows, splits, out, out_dtype, lse, o_part, lse_part};
    const size_t smem = sizeof(SfaSmem) + 1024;
    e = cudaFuncSetAttribute(sfa_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = 2 * (int64_t)p.n_q * splits;
    count_launch();
    sfa_mma_kernel<<<static_cast<unsigned>(grid), kThreads, smem, s>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess || splits == 1) return e;
    count_launch();
    sfa_combine_kernel<<<static_cast<unsigned>(p.n_q * 128), 128, 0, s>>>(o_part, lse_part, splits,
                                                                         out, out_dtype, lse);
    return cudaGetLastError();
}

}  // namespace sa
