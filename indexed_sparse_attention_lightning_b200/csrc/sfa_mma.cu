// sfa_mma.cu -- sparse MLA attention on the 5th-generation tensor cores,
// one CTA pair (cluster of two) per (query, key split).
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
// contractions are dense per key tile: S = Q K^T (M = 128 heads, N = 32 keys,
// K = 576) and O += P V (M = 128 heads, N = 512, K = 32 keys).  O is 128 x 512
// fp32 = all of one SM's TMEM, so the heads are split over a CTA pair with
// tcgen05.mma.cta_group::2 (M = 128 = 64 heads per CTA, full rate): each CTA
// keeps its 64 heads x 512 dims of O in its own TMEM (256 columns), the even
// CTA issues every MMA for both.  The B operand of each MMA is split by
// columns across the pair: for S each CTA holds 16 of the 32 keys (full
// 576-d rows), for P V each CTA holds 128 of every 256 output dims of all 32
// keys.  Rows are copied straight from the paged cache into the swizzled
// operand layouts, so no gathered copy of the cache is written to global
// memory.
//
// Roles per CTA (224 threads):
//   warp 0     producer of the S operand: the query block once (TMA), then per
//              tile this CTA's 16 keys x 9 column blocks as 16-byte cp.async
//              copies (the 128-byte swizzle applied in the addresses) into a
//              4-stage ring that is freed as soon as that tile's S is done;
//   warp 6     producer of the P V operand: per tile this CTA's 4 output-dim
//              blocks of all 32 keys, likewise, into a 3-stage ring;
//   warp 1     even CTA: issues the MMAs for both CTAs from a non-blocking
//              loop -- S of a tile as soon as its keys are in, P V as soon as
//              P is written -- and commits them to both CTAs' barriers;
//              odd CTA: forwards "stage loaded" to the even CTA;
//   warps 2-5  compact the index list into physical rows, then run the online
//              softmax: thread L owns TMEM lane L = (head L % 64, key half /
//              output half L / 64); the two halves of a head exchange their
//              tile maxima through shared memory; O is rescaled in TMEM only
//              when the running maximum grows by more than 2^8; P goes to
//              shared memory as bf16 for the P V MMA; finally O / l is written.
// Selected rows are gathered with the LSU (cp.async) rather than TMA
// tile::gather4: each row contributes only 128-byte pieces, and at that size
// the TMA issue rate, not bandwidth, limits a gather.
// All waits are bounded; a timeout is reported in the workspace status word.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace sa {
namespace {
using namespace sm100;

constexpr int kHeadsCta = 64;
constexpr int kDl = 512, kDr = 64, kD = kDl + kDr;
constexpr int kBlocks = kD / 64;  // 64-dim (128-byte) column blocks of a row
constexpr int kTile = 32;         // selected keys per tile
constexpr int kHalf = kTile / 2;  // keys per CTA in the S operand
constexpr int kKsStages = 4;      // S-operand ring (freed after S)
constexpr int kPvStages = 3;      // P V-operand ring (freed after P V)
constexpr int kThreads = 224;
constexpr int kMaxK = 2048;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;     // 256 columns: two 128-column halves of 256 output dims
constexpr uint32_t kColS = 256;   // three S buffers of 16 columns
constexpr int kBufs = 3;          // S (TMEM) and P (shared memory) buffers in flight
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kKsBytes = kHalf * kD * 2;       // 16 keys x 1152 bytes
constexpr uint32_t kPvBytes = kTile * 256 * 2;      // 32 keys x 256 dims x 2 bytes
constexpr int kKsChunks = kKsBytes / 16 / 32;      // 16-byte copies per lane per tile
constexpr int kChunksPerRow = kD * 2 / 16;          // 72
constexpr uint32_t kQBytes = kBlocks * kHeadsCta * 128;

struct SfaSmem {
    uint8_t q[kBlocks][kHeadsCta * 128];
    uint8_t ks[kKsStages][kBlocks][kHalf * 128];  // this CTA's 16 keys, full rows, K-major
    uint8_t pv[kPvStages][4][kTile * 128];        // this CTA's 256 output dims of all 32 keys
    uint8_t p[kBufs][kHeadsCta * 128];  // P (bf16), 32 keys used of each 128-byte row
    int32_t rows[kMaxK];                // compacted physical rows of the selected keys
    float xmax[2][128];
    float lsum[128];
    int32_t warp_cnt[4];
    int32_t n_valid;
    uint64_t q_full, rows_ready;
    uint64_t ks_loaded[kKsStages], ks_peer[kKsStages], ks_empty[kKsStages];
    uint64_t pv_loaded[kPvStages], pv_peer[kPvStages], pv_empty[kPvStages];
    uint64_t s_full[kBufs], p_full[kBufs], o_done[kBufs];
    uint32_t tmem_base;
    int abort;
};

static_assert(sizeof(SfaSmem) + 1024 <= 232448, "shared memory budget of one CTA");
static_assert(kKsBytes == sizeof(SfaSmem::ks[0]) && kPvBytes == sizeof(SfaSmem::pv[0]),
              "copies fill the stages exactly");

struct SfaArgs {
    PathParams p;
    const int32_t *idx;  // [n_q, K]
    int32_t K;
    int32_t splits;
    void *out;           // [n_q, 128, 512] (splits == 1)
    int32_t out_dtype;
    float *lse;          // [n_q, 128] or null (splits == 1)
    float *o_part;       // [n_q, splits, 128, 512] (splits > 1)
    float *lse_part;     // [n_q, splits, 128]      (splits > 1)
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *status, bool cluster_scope = false) {
    bool ok = true;
    if (lane_id() == 0)
        ok = cluster_scope ? mbar_wait_cluster(bar, parity, abort_flag, status)
                           : mbar_wait(bar, parity, abort_flag, status);
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
sfa_mma_kernel(const __grid_constant__ CUtensorMap tm_q, const SfaArgs a) {
    extern __shared__ uint8_t smem_raw[];
    SfaSmem &sm = *reinterpret_cast<SfaSmem *>(align1024(smem_raw));
    const PathParams &p = a.p;
    const uint32_t rank = cluster_ctarank();
    const int unit = blockIdx.x >> 1;
    const int t = unit / a.splits, split = unit % a.splits;
    const int warp = warp_id(), lane = lane_id();

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.rows_ready, 1);
        for (int s = 0; s < kKsStages; ++s) {
            mbar_init(&sm.ks_loaded[s], 32);  // one cp.async arrival per producer lane
            mbar_init(&sm.ks_peer[s], 1);
            mbar_init(&sm.ks_empty[s], 1);
        }
        for (int s = 0; s < kPvStages; ++s) {
            mbar_init(&sm.pv_loaded[s], 32);
            mbar_init(&sm.pv_peer[s], 1);
            mbar_init(&sm.pv_empty[s], 1);
        }
        for (int b = 0; b < kBufs; ++b) {
            mbar_init(&sm.s_full[b], 1);
            mbar_init(&sm.p_full[b], 8);  // 4 softmax warps in each CTA of the pair
            mbar_init(&sm.o_done[b], 1);
        }
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc_pair(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before anyone signals remotely
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort;
    int32_t *status = p.status;

    if (warp >= 2 && warp <= 5) {
        // --------------------------------------------- row compaction ---
        const int et = threadIdx.x - 64, ew = et >> 5;
        const int32_t V = visible_len(p, t);
        const int32_t seq = p.q_seq[t];
        const int32_t *sel = a.idx + (int64_t)t * a.K;
        // all index and page-table loads in flight at once (16 per thread),
        // then an ordered compaction over the 16 rounds of 128 entries
        constexpr int kRounds = kMaxK / 128;
        int32_t phys[kRounds];
#pragma unroll
        for (int r = 0; r < kRounds; ++r) {
            const int k = r * 128 + et;
            phys[r] = k < a.K ? __ldg(sel + k) : -1;
        }
#pragma unroll
        for (int r = 0; r < kRounds; ++r) {
            const int32_t s = phys[r];
            int32_t v = -1;
            if (s >= V) {
                report(status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_INDEX);
            } else if (s >= 0) {
                const int64_t row = phys_row(p.page_table, p.max_pages, p.num_pages, seq, s);
                if (row < 0) report(status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_PAGE);
                else v = static_cast<int32_t>(row);
            }
            phys[r] = v;
        }
        int32_t base = 0;
#pragma unroll
        for (int r = 0; r < kRounds; ++r) {
            const unsigned bal = __ballot_sync(0xffffffffu, phys[r] >= 0);
            if (lane == 0) sm.warp_cnt[ew] = __popc(bal);
            named_barrier(1, 128);
            int32_t off = base, tot = 0;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                if (w < ew) off += sm.warp_cnt[w];
                tot += sm.warp_cnt[w];
            }
            if (phys[r] >= 0) sm.rows[off + __popc(bal & ((1u << lane) - 1u))] = phys[r];
            named_barrier(1, 128);
            base += tot;
        }
        const int32_t n_valid = min(base, (int32_t)kMaxK);
        const int32_t padded = ((n_valid + kTile - 1) / kTile) * kTile;
        for (int c = n_valid + et; c < padded; c += 128) sm.rows[c] = sm.rows[0];
        named_barrier(1, 128);
        if (et == 0) {
            sm.n_valid = n_valid;
            mbar_arrive(&sm.rows_ready);  // release: rows and n_valid are visible
        }

        // ----------------------------------------------- online softmax ---
        // The loop never leaves early: after a failed wait (a timeout raised
        // the abort flag) it keeps going without waiting, so the four warps
        // always meet at the same named barriers.
        int32_t j0, j1;
        split_range(n_valid, split, a.splits, j0, j1);
        const int T = j1 - j0;
        const int L = 32 * (warp & 3) + lane;  // TMEM lane owned by this thread
        const int h = L & 63, hf = L >> 6;
        const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        const float sl2 = p.sm_scale * kLog2e;
        const uint32_t p_full_addr0 = map_to_rank(smem_u32(&sm.p_full[0]), 0);
        float m_run = -INFINITY, l_half = 0.f;
        bool ok = true;
        for (int n = 0; n < T; ++n) {
            const int sb = n % kBufs;
            if (ok) ok = warp_wait(&sm.s_full[sb], (n / kBufs) & 1, abort_flag, status, true);
            float s[16];
            if (ok) {
                tc_fence_after();
                tmem_ld16(tmem + lane_base + kColS + 16 * sb, s);
                tmem_wait_ld();
            }
            const int kvalid = n_valid - ((j0 + n) * kTile + kHalf * hf);
            float tmax = -INFINITY;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                s[i] = (ok && i < kvalid) ? s[i] * sl2 : -INFINITY;
                tmax = fmaxf(tmax, s[i]);
            }
            sm.xmax[n & 1][L] = tmax;
            named_barrier(1, 128);
            const float mt = fmaxf(tmax, sm.xmax[n & 1][L ^ 64]);
            if (mt > m_run + kRescaleLog2) {
                if (n > 0) {
                    // O holds P V of earlier tiles: wait for the last one, then rescale
                    if (ok)
                        ok = warp_wait(&sm.o_done[(n - 1) % kBufs], ((n - 1) / kBufs) & 1,
                                       abort_flag, status, true);
                    if (ok) {
                        tc_fence_after();
                        const float f = exp2f(m_run - mt);
#pragma unroll 1
                        for (int c = 0; c < 8; ++c) {
                            float v[32];
                            tmem_ld32(tmem + lane_base + kColO + 32 * c, v);
                            tmem_wait_ld();
#pragma unroll
                            for (int i = 0; i < 32; ++i) v[i] *= f;
                            tmem_st32(tmem + lane_base + kColO + 32 * c, v);
                        }
                        tmem_wait_st();
                        l_half *= f;
                    }
                }
                m_run = mt;
            }
            uint32_t packed[8];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                const float p0 = exp2f(s[i] - m_run), p1 = exp2f(s[i + 1] - m_run);
                l_half += p0 + p1;
                __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
                packed[i / 2] = *reinterpret_cast<uint32_t *>(&b2);
            }
            // P buffer sb was last read by the P V MMA of tile n - kBufs
            if (n >= kBufs && ok)
                ok = warp_wait(&sm.o_done[sb], ((n - kBufs) / kBufs) & 1, abort_flag, status, true);
            uint8_t *prow = sm.p[sb] + h * 128;
            const int sw = h & 7;
            *reinterpret_cast<uint4 *>(prow + (((2 * hf) ^ sw) << 4)) =
                make_uint4(packed[0], packed[1], packed[2], packed[3]);
            *reinterpret_cast<uint4 *>(prow + (((2 * hf + 1) ^ sw) << 4)) =
                make_uint4(packed[4], packed[5], packed[6], packed[7]);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(&sm.p_full[sb]);
                else mbar_arrive_remote(p_full_addr0 + sb * sizeof(uint64_t));
            }
        }
        if (ok && T > 0)
            ok = warp_wait(&sm.o_done[(T - 1) % kBufs], ((T - 1) / kBufs) & 1, abort_flag, status,
                           true);
        tc_fence_after();
        // both halves of a head hold part of its softmax denominator
        sm.lsum[L] = l_half;
        named_barrier(1, 128);
        const float l = l_half + sm.lsum[L ^ 64];
        const float inv = (ok && l > 0.f) ? 1.f / l : 0.f;
        const float lse_v = (ok && l > 0.f) ? (m_run + log2f(l)) * kLn2 : -INFINITY;
        const int head = kHeadsCta * rank + h;
        const int64_t row = (int64_t)t * 128 + head;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
            float v[32];
            if (ok && T > 0) {
                tmem_ld32(tmem + lane_base + kColO + 32 * c, v);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.f;
            }
            const int dv = 256 * (c >> 2) + 128 * hf + 32 * (c & 3);
            if (a.splits == 1) {
                if (a.out_dtype == SA_BF16) {
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(v[i] * inv, v[i + 1] * inv);
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
                        dst[i] = make_float4(v[4 * i] * inv, v[4 * i + 1] * inv, v[4 * i + 2] * inv,
                                             v[4 * i + 3] * inv);
                }
            } else {
                const int64_t prow_i = ((int64_t)t * a.splits + split) * 128 + head;
                float4 *dst = reinterpret_cast<float4 *>(a.o_part + prow_i * kDl + dv);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(v[4 * i] * inv, v[4 * i + 1] * inv, v[4 * i + 2] * inv,
                                         v[4 * i + 3] * inv);
            }
        }
        if (hf == 0) {
            if (a.splits == 1) {
                if (a.lse != nullptr) a.lse[row] = lse_v;
            } else {
                a.lse_part[((int64_t)t * a.splits + split) * 128 + head] = lse_v;
            }
        }
    } else {
        // the producers and the MMA warp need this split's tile range
        const bool ready = warp_wait(&sm.rows_ready, 0, abort_flag, status);
        int32_t j0 = 0, j1 = 0;
        if (ready) split_range(sm.n_valid, split, a.splits, j0, j1);
        const int T = j1 - j0;
        const uint8_t *kv = static_cast<const uint8_t *>(p.kv);
        if (warp == 0 && T > 0) {
            // ------------------------------------ S-operand producer ---
            if (lane == 0) {
                // both CTAs' query halves complete on the even CTA's barrier
                const uint32_t q_full0 = map_to_rank(smem_u32(&sm.q_full), 0);
                if (rank == 0) mbar_arrive_expect_tx(&sm.q_full, 2 * kQBytes);
                for (int b = 0; b < kBlocks; ++b)
                    tma_load_2d_pair(sm.q[b], &tm_q, 64 * b, t * 128 + kHeadsCta * rank, q_full0);
            }
            for (int n = 0; n < T; ++n) {
                const int st = n % kKsStages;
                if (!warp_wait(&sm.ks_empty[st], ((n / kKsStages) & 1) ^ 1, abort_flag, status,
                               true))
                    break;
                const int32_t *rr = &sm.rows[(j0 + n) * kTile + kHalf * rank];
                const uint32_t dst0 = smem_u32(sm.ks[st][0]);
#pragma unroll 4
                for (int it = 0; it < kKsChunks; ++it) {
                    const int g = it * 32 + lane;
                    const int k = g / kChunksPerRow, rem = g - k * kChunksPerRow;
                    const int b = rem >> 3, c = rem & 7;
                    cp_async16(dst0 + b * (kHalf * 128) + k * 128 + ((c ^ (k & 7)) << 4),
                               kv + (int64_t)rr[k] * (kD * 2) + rem * 16);
                }
                cp_async_arrive(&sm.ks_loaded[st]);
            }
        } else if (warp == 6 && T > 0) {
            // ---------------------------------- P V-operand producer ---
            const int c4 = lane >> 3, c = lane & 7;                 // block of 4, 16-byte chunk
            const int dvb = (c4 < 2 ? 0 : 4) + 2 * rank + (c4 & 1);  // 64-dim block of the row
            for (int n = 0; n < T; ++n) {
                const int st = n % kPvStages;
                if (!warp_wait(&sm.pv_empty[st], ((n / kPvStages) & 1) ^ 1, abort_flag, status,
                               true))
                    break;
                const int32_t *rr = &sm.rows[(j0 + n) * kTile];
                const uint32_t dst0 = smem_u32(sm.pv[st][c4]);
#pragma unroll 4
                for (int k = 0; k < kTile; ++k)  // one key per step, 512 bytes per warp
                    cp_async16(dst0 + k * 128 + ((c ^ (k & 7)) << 4),
                               kv + (int64_t)rr[k] * (kD * 2) + dvb * 128 + c * 16);
                cp_async_arrive(&sm.pv_loaded[st]);
            }
        } else if (warp == 1 && T > 0 && lane == 0 && rank == 1) {
            // ------------------------------------------------- relay ---
            const uint32_t ks_peer0 = map_to_rank(smem_u32(&sm.ks_peer[0]), 0);
            const uint32_t pv_peer0 = map_to_rank(smem_u32(&sm.pv_peer[0]), 0);
            int nk = 0, nv = 0;
            long long t0 = clock64();
            uint32_t idle = 0;
            while (nk < T || nv < T) {
                bool progressed = false;
                if (nk < T && mbar_test(&sm.ks_loaded[nk % kKsStages], (nk / kKsStages) & 1)) {
                    fence_proxy_async_smem();
                    mbar_arrive_remote(ks_peer0 + (nk % kKsStages) * sizeof(uint64_t));
                    ++nk;
                    progressed = true;
                }
                if (nv < T && mbar_test(&sm.pv_loaded[nv % kPvStages], (nv / kPvStages) & 1)) {
                    fence_proxy_async_smem();
                    mbar_arrive_remote(pv_peer0 + (nv % kPvStages) * sizeof(uint64_t));
                    ++nv;
                    progressed = true;
                }
                if (progressed) {
                    t0 = clock64();
                } else if ((++idle & 63) == 0 && wait_expired(t0, abort_flag, status)) {
                    break;
                }
            }
        } else if (warp == 1 && T > 0 && lane == 0 && rank == 0) {
            // ---------------------------------------------- MMA issuer ---
            constexpr uint32_t id_s = instr_desc(128, kTile, 1 /*bf16*/, 0, 0);
            constexpr uint32_t id_pv = instr_desc(128, 256, 1 /*bf16*/, 0, 1);
            bool ok = mbar_wait_cluster(&sm.q_full, 0, abort_flag, status);
            int ns = 0, np = 0;  // next S and next P V to issue
            long long t0 = clock64();
            uint32_t idle = 0;
            while (ok && np < T) {
                bool progressed = false;
                // S(ns) needs its keys in both CTAs and a free S buffer: the
                // softmax of tile ns - kBufs is done once P V of it was issued
                if (ns < T && ns < np + kBufs) {
                    const int st = ns % kKsStages;
                    const uint32_t ph = (ns / kKsStages) & 1;
                    if (mbar_test(&sm.ks_loaded[st], ph) && mbar_test_cluster(&sm.ks_peer[st], ph)) {
                        fence_proxy_async_smem();
                        tc_fence_after();
                        const uint32_t d = tmem + kColS + 16 * (ns % kBufs);
#pragma unroll 1
                        for (int b = 0; b < kBlocks; ++b) {
                            const uint64_t ad = desc_kmajor_sw128(smem_u32(sm.q[b]));
                            const uint64_t bd = desc_kmajor_sw128(smem_u32(sm.ks[st][b]));
#pragma unroll
                            for (int k = 0; k < 4; ++k)  // 16 bf16 (32 bytes) of K each
                                mma_bf16_pair(d, ad + 2 * k, bd + 2 * k, id_s, (b | k) != 0);
                        }
                        mma_commit_pair_multicast(&sm.s_full[ns % kBufs], 0x3);
                        if (ns + kKsStages < T) mma_commit_pair_multicast(&sm.ks_empty[st], 0x3);
                        ++ns;
                        progressed = true;
                    }
                }
                // P V(np) needs P from both CTAs and its value rows in both CTAs
                if (np < ns) {
                    const int st = np % kPvStages;
                    const uint32_t ph = (np / kPvStages) & 1;
                    if (mbar_test_cluster(&sm.p_full[np % kBufs], (np / kBufs) & 1) &&
                        mbar_test(&sm.pv_loaded[st], ph) && mbar_test_cluster(&sm.pv_peer[st], ph)) {
                        fence_proxy_async_smem();
                        tc_fence_after();
                        const uint64_t ad = desc_kmajor_sw128(smem_u32(sm.p[np % kBufs]));
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const uint32_t va = smem_u32(sm.pv[st][2 * half]);
#pragma unroll
                            for (int k = 0; k < 2; ++k)  // 16 keys per instruction
                                mma_bf16_pair(tmem + kColO + 128 * half, ad + 2 * k,
                                              desc_mnmajor_sw128(va + 2048 * k, kTile * 128, 1024),
                                              id_pv, (np > 0 || k > 0) ? 1u : 0u);
                        }
                        mma_commit_pair_multicast(&sm.o_done[np % kBufs], 0x3);
                        if (np + kPvStages < T) mma_commit_pair_multicast(&sm.pv_empty[st], 0x3);
                        ++np;
                        progressed = true;
                    }
                }
                if (progressed) {
                    t0 = clock64();
                } else if ((++idle & 63) == 0 && wait_expired(t0, abort_flag, status)) {
                    break;
                }
            }
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the pair no longer touches each other's shared memory or TMEM
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
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
    const int32_t pairs = std::max(1, num_sms() / 2);
    const int32_t max_tiles = (top_k + kTile - 1) / kTile;
    if (n_q <= 0) return 1;
    return std::max(1, std::min(max_tiles, pairs / n_q));
}

cudaError_t launch_sfa_mma(const PathParams &p, const int32_t *idx, int32_t top_k, int32_t splits,
                           void *out, int32_t out_dtype, float *lse, float *o_part,
                           float *lse_part, cudaStream_t s) {
    if (p.n_q == 0) return cudaSuccess;
    CUtensorMap tq;
    if (!encode_tmap_2d(&tq, 2, p.q, kD, (uint64_t)p.n_q * 128, kD * 2, 64, kHeadsCta, true))
        return cudaErrorInvalidValue;
    SfaArgs a{p, idx, top_k, splits, out, out_dtype, lse, o_part, lse_part};
    const size_t smem = sizeof(SfaSmem) + 1024;
    cudaError_t e =
        cudaFuncSetAttribute(sfa_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = 2 * (int64_t)p.n_q * splits;
    count_launch();
    sfa_mma_kernel<<<static_cast<unsigned>(grid), kThreads, smem, s>>>(tq, a);
    if ((e = cudaGetLastError()) != cudaSuccess || splits == 1) return e;
    count_launch();
    sfa_combine_kernel<<<static_cast<unsigned>(p.n_q * 128), 128, 0, s>>>(o_part, lse_part, splits,
                                                                         out, out_dtype, lse);
    return cudaGetLastError();
}

}  // namespace sa
