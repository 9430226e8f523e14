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
// operand of S and, read MN-major, the B operand of P V.  The stage's rope
// block (the last 64 dims of every row, 8 KB) is read by S only, so once S is
// done the softmax writes that tile's P (64 heads x 64 keys bf16, also 8 KB)
// over it: every stage carries its own P, and the softmax of the next tile
// never waits for P V of this one to release a shared P buffer.
//
// Roles (384 threads, one CTA per SM):
//   warp 0     lane 0 loads Q by TMA (into the third ring stage; this copy
//              starts before the wait on the top-K kernel), then issues
//              the MMAs from a non-blocking loop -- S of a tile as soon as its
//              rows are in and an S buffer is free, P V as soon as P is
//              written -- and commits them to mbarriers;
//   warps 1-7  copy the selected rows (16-byte cp.async, the swizzle applied
//              in the addresses) into a 3-stage ring freed by each tile's P V;
//              random 1152-byte rows reach shared memory fastest this way;
//   warps 8-11 move Q into TMEM, then run the online softmax.  Warp 8 + j
//              owns heads 16j .. 16j + 15 and reads their S rows with 16-lane
//              loads: thread i holds heads 16j + i/4 and 16j + i/4 + 8, keys
//              8r + 2(i%4) and 8r + 2(i%4) + 1 of each 8-key group r, so a row
//              maximum takes two shuffles and P goes to shared memory in
//              bf16 pairs.  O is rescaled in TMEM (16-lane accesses with the
//              same thread-to-head mapping, leaving Q and S alone) only when a
//              head's running maximum grows by more than 2^8; finally lanes
//              16-31 read O with 32-lane loads and write O / l.
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
// tiles of rows prefetched into L2 ahead of the copies (1 measured faster
// than 2, 3, 4 or 6 on the 32K decode: 0.0945 against 0.0977 ms at 4)
constexpr int kPrefetch = 1;
constexpr int kProducerWarps = 7;
constexpr int kSoftmaxWarp0 = 8;  // warps 8-11, one per TMEM subpartition
constexpr int kThreads = 384;
constexpr int kMaxK = 2048;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;    // lower half-lanes: Q, 288 columns
constexpr uint32_t kColS = 288;  // lower half-lanes: two S buffers of 64 columns
constexpr uint32_t kLaneO = 16;  // O: upper half-lanes, columns [0, 512)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;
constexpr int kChunksPerRow = kD * 2 / 16;  // 72 sixteen-byte pieces of a row
// Stage layout: key k of a tile, 64-dim block b -> byte (k/8)*kGroupBytes +
// b*1024 + (k%8)*128 (+ the 16-byte swizzle): the S view (K-major, 8-key
// groups kGroupBytes apart) and the P V view (MN-major, 64-dim atoms 1024
// bytes apart, 8-key groups kGroupBytes apart) read the same bytes.  After S,
// block 8 (the rope) holds P: head h's 64 keys at (h/8)*kGroupBytes + 8*1024 +
// (h%8)*128 (+ swizzle), the K-major A operand of P V with 8-head groups
// kGroupBytes apart.
constexpr uint32_t kGroupBytes = kBlocks * 1024;             // 9216
constexpr uint32_t kStageBytes = (kTile / 8) * kGroupBytes;  // 73728
constexpr uint32_t kPOffset = (kBlocks - 1) * 1024;          // the rope block

struct SfaSmem {
    // ring stage: 8 groups of 8 rows; a group holds the 9 column blocks of its
    // rows, each 8 x 128 bytes with the 128-byte swizzle (see kGroupBytes)
    uint8_t kv[kStages][kStageBytes];
    uint64_t kv_full[kStages], kv_empty[kStages];
    // o_done: one phase per P V (a rescale waits for the previous tile's);
    // o_final: once, after the last P V, for the final read of O (P V of the
    // last two tiles may both be in flight then, which o_done's parity cannot
    // tell apart)
    uint64_t s_full[2], p_full[kStages], o_done, o_final, q_full, q_ready;
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
    int32_t fp8;             // e4m3 latent + fp32 page scale + bf16 rope (else bf16 rows)
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

// 2^x on the special-function unit (ex2.approx: relative error ~2^-22, -inf -> 0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Tiles [j0, j1) of the compacted key list handled by this split.
__device__ __forceinline__ void split_range(int32_t n_valid, int32_t split, int32_t splits,
                                            int32_t &j0, int32_t &j1) {
    const int32_t tiles = (n_valid + kTile - 1) / kTile;
    j0 = (int32_t)((int64_t)tiles * split / splits);
    j1 = (int32_t)((int64_t)tiles * (split + 1) / splits);
}

// Query t's selected positions -> physical cache rows (compact_rows): one
// CTA per query.  The fused decode path gets the rows from the top-K kernel.
constexpr int kRowsThreads = 512;
__global__ void __launch_bounds__(kRowsThreads)
sfa_rows_kernel(const PathParams p, const int32_t *__restrict__ idx, int32_t K, int32_t ld_rows,
                int32_t *__restrict__ rows, int32_t *__restrict__ n_valid_out) {
    pdl_wait();
    pdl_trigger();
    __shared__ int32_t scratch[33];
    const int t = blockIdx.x;
    compact_rows(p, t, idx + (int64_t)t * K, K, kTile, rows + (int64_t)t * ld_rows,
                 n_valid_out + t, scratch);
}

__global__ void __launch_bounds__(kThreads, 1)
sfa_mma_kernel(const __grid_constant__ CUtensorMap tm_q, const SfaArgs a) {
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
        for (int s = 0; s < kStages; ++s) mbar_init(&sm.p_full[s], 4);  // the four softmax warps
        mbar_init(&sm.o_done, 1);
        mbar_init(&sm.o_final, 1);
        mbar_init(&sm.q_full, 1);
        mbar_init(&sm.q_ready, 4);
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) tmem_alloc(&sm.tmem_base, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_trigger();  // after the TMEM allocation: a waiting successor holds none
    // Q is an input, not the previous kernel's output: its copy (into ring
    // stage 2) starts before the wait on that kernel
    if (warp == 0 && lane == 0) {
        mbar_arrive_expect_tx(&sm.q_full, kBlocks * kHeadsCta * 128);
        for (int b = 0; b < kBlocks; ++b)
            tma_load_2d(sm.kv[2] + b * (kHeadsCta * 128), &tm_q, 64 * b, t * 128 + kHeadsCta * hh,
                        &sm.q_full);
    }
    pdl_wait();  // the selected rows come from the top-K kernel
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort;
    int32_t *status = p.status;
    const int32_t n_valid = a.n_valid[t];
    int32_t j0, j1;
    split_range(n_valid, split, a.splits, j0, j1);
    const int T = j1 - j0;

    if (warp >= kSoftmaxWarp0) {
        const int j = warp & 3;  // TMEM subpartition of this warp
        const int q4 = lane & 3;
        const int ha = 16 * j + (lane >> 2), hb = ha + 8;  // the two heads of this thread
        const uint32_t lane_lo = static_cast<uint32_t>(32 * j) << 16;
        const uint32_t lane_hi = static_cast<uint32_t>(32 * j + kLaneO) << 16;
        bool ok = true;
        // ----------------------------------------------- Q into TMEM ---
        // Q (128-byte-swizzled, in ring stage 2) -> lanes 32j .. 32j + 15;
        // the 32-lane stores also put a copy on O's columns of lanes 16-31,
        // which the first P V overwrites.
        if (T > 0) {
            ok = warp_wait(&sm.q_full, 0, abort_flag, status);
            if (ok) {
                const int h = 16 * j + (lane & 15);
#pragma unroll 1
                for (int b = 0; b < kBlocks; ++b) {
                    const uint8_t *qr = sm.kv[2] + b * (kHeadsCta * 128) + h * 128;
                    uint32_t v[32];
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 x = *reinterpret_cast<const uint4 *>(qr + ((c ^ (h & 7)) << 4));
                        v[4 * c] = x.x;
                        v[4 * c + 1] = x.y;
                        v[4 * c + 2] = x.z;
                        v[4 * c + 3] = x.w;
                    }
                    tmem_st32_u(tmem + lane_lo + kColQ + 32 * b, v);
                }
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.q_ready);  // also frees ring stage 2
        }

        // ----------------------------------------------- online softmax ---
        // The loop never leaves early: after a failed wait (a timeout raised
        // the abort flag) it keeps going without waiting or touching TMEM.
        const float sl2 = p.sm_scale * kLog2e;
        float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
        for (int n = 0; n < T; ++n) {
            const int sb = n & 1;
            if (ok) ok = warp_wait(&sm.s_full[sb], (n >> 1) & 1, abort_flag, status);
            uint32_t v[32];
            if (ok) {
                tc_fence_after();
                tmem_ld_16x256b_x8(tmem + lane_lo + kColS + kTile * sb, v);
                tmem_wait_ld();
            }
            const int kvalid = ok ? n_valid - (j0 + n) * kTile : 0;
            float xa[16], xb[16];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    xa[2 * r + e] = __uint_as_float(v[4 * r + e]) * sl2;
                    xb[2 * r + e] = __uint_as_float(v[4 * r + 2 + e]) * sl2;
                }
            }
            if (kvalid < kTile) {  // the last tile: mask the padding
#pragma unroll
                for (int r = 0; r < 8; ++r) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const bool valid = 8 * r + 2 * q4 + e < kvalid;
                        xa[2 * r + e] = valid ? xa[2 * r + e] : -INFINITY;
                        xb[2 * r + e] = valid ? xb[2 * r + e] : -INFINITY;
                    }
                }
            }
            float ta = xa[0], tb = xb[0];
#pragma unroll
            for (int i = 1; i < 16; ++i) {
                ta = fmaxf(ta, xa[i]);
                tb = fmaxf(tb, xb[i]);
            }
            ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, 1));
            ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, 2));
            tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, 1));
            tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, 2));
            // lazy rescaling: a running maximum moves only on a large jump
            const bool grow_a = ta > m_a + kRescaleLog2, grow_b = tb > m_b + kRescaleLog2;
            const float mn_a = grow_a ? ta : m_a, mn_b = grow_b ? tb : m_b;
            const float f_a = (grow_a && n > 0) ? exp2f(m_a - mn_a) : 1.f;
            const float f_b = (grow_b && n > 0) ? exp2f(m_b - mn_b) : 1.f;
            uint32_t pa[8], pb[8];
            float la = 0.f, lb = 0.f;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float a0 = ex2(xa[2 * r] - mn_a), a1 = ex2(xa[2 * r + 1] - mn_a);
                const float b0 = ex2(xb[2 * r] - mn_b), b1 = ex2(xb[2 * r + 1] - mn_b);
                la += a0 + a1;
                lb += b0 + b1;
                __nv_bfloat162 x = __floats2bfloat162_rn(a0, a1);
                __nv_bfloat162 y = __floats2bfloat162_rn(b0, b1);
                pa[r] = *reinterpret_cast<uint32_t *>(&x);
                pb[r] = *reinterpret_cast<uint32_t *>(&y);
            }
            // O belongs to P V of the previous tile until it is done: only a
            // rescale has to wait for it (P goes to this tile's own stage)
            const bool rescale = __any_sync(0xffffffffu, (grow_a || grow_b) && n > 0);
            if (rescale && ok) ok = warp_wait(&sm.o_done, (n - 1) & 1, abort_flag, status);
            if (ok && rescale) {
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t w[64];
                    tmem_ld_16x256b_x16(tmem + lane_hi + 128 * c, w);
                    tmem_wait_ld();
#pragma unroll
                    for (int r = 0; r < 16; ++r) {
                        w[4 * r] = __float_as_uint(__uint_as_float(w[4 * r]) * f_a);
                        w[4 * r + 1] = __float_as_uint(__uint_as_float(w[4 * r + 1]) * f_a);
                        w[4 * r + 2] = __float_as_uint(__uint_as_float(w[4 * r + 2]) * f_b);
                        w[4 * r + 3] = __float_as_uint(__uint_as_float(w[4 * r + 3]) * f_b);
                    }
                    tmem_st_16x256b_x16(tmem + lane_hi + 128 * c, w);
                }
                tmem_wait_st();
            }
            l_a = l_a * f_a + la;
            l_b = l_b * f_b + lb;
            m_a = mn_a;
            m_b = mn_b;
            // P rows ha, hb: keys 8r + 2 q4 (+1) -> bytes 16r + 4 q4 of the row,
            // in the rope block of this tile's stage (S has read it: s_full)
            uint8_t *pbase = sm.kv[n % kStages] + kPOffset;
            uint8_t *row_a = pbase + (ha >> 3) * kGroupBytes + (ha & 7) * 128 + 4 * q4;
            uint8_t *row_b = pbase + (hb >> 3) * kGroupBytes + (hb & 7) * 128 + 4 * q4;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                *reinterpret_cast<uint32_t *>(row_a + ((r ^ (ha & 7)) << 4)) = pa[r];
                *reinterpret_cast<uint32_t *>(row_b + ((r ^ (hb & 7)) << 4)) = pb[r];
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.p_full[n % kStages]);
        }
        if (ok && T > 0) ok = warp_wait(&sm.o_final, 0, abort_flag, status);
        tc_fence_after();
        // full row sums: the four threads of a head each hold a quarter
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
        const float inv_a = (ok && l_a > 0.f) ? 1.f / l_a : 0.f;
        const float inv_b = (ok && l_b > 0.f) ? 1.f / l_b : 0.f;
        // 32-lane loads: lane 16 + r receives the O row of head 16j + r, whose
        // sums sit in thread 4(r % 8) (as its first head for r < 8)
        const int r_o = lane & 15;
        const float inv_ra = __shfl_sync(0xffffffffu, inv_a, 4 * (r_o & 7));
        const float inv_rb = __shfl_sync(0xffffffffu, inv_b, 4 * (r_o & 7));
        const float inv_o = r_o < 8 ? inv_ra : inv_rb;
        const bool o_lane = lane >= 16;
        const int head = kHeadsCta * hh + 16 * j + r_o;
        const int64_t row = (int64_t)t * 128 + head;
#pragma unroll 2  // two TMEM loads in flight: measured faster than one
        for (int c = 0; c < kDl / 32; ++c) {
            float v[32];
            if (ok && T > 0) {
                tmem_ld32(tmem + lane_lo + 32 * c, v);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.f;
            }
            if (!o_lane) continue;
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
        if (q4 == 0) {
            const float lse_a = (ok && l_a > 0.f) ? (m_a + log2f(l_a)) * kLn2 : -INFINITY;
            const float lse_b = (ok && l_b > 0.f) ? (m_b + log2f(l_b)) * kLn2 : -INFINITY;
            const int64_t row_a = (int64_t)t * 128 + kHeadsCta * hh + ha;
            const int64_t row_b = row_a + 8;
            if (a.splits == 1) {
                if (a.lse != nullptr) {
                    a.lse[row_a] = lse_a;
                    a.lse[row_b] = lse_b;
                }
            } else {
                const int64_t base = ((int64_t)t * a.splits + split) * 128 + kHeadsCta * hh;
                a.lse_part[base + ha] = lse_a;
                a.lse_part[base + hb] = lse_b;
            }
        }
    } else if (warp >= 1) {
        // ---------------------------------------------- row producers ---
        // warp 1 + w copies keys w, w + 7, ... of each tile; a key's 72
        // sixteen-byte pieces go to lanes (piece % 32) in three steps.  Ring
        // stage 2 holds Q until the softmax warps have moved it to TMEM.
        const int pw = warp - 1;
        const uint8_t *kv = static_cast<const uint8_t *>(p.kv);
        const int32_t *rows = a.rows + (int64_t)t * a.ld_rows;
        // The ring holds about one tile in flight per SM, too little to cover
        // the latency of random row reads from HBM; so the rows of tile
        // n + kPrefetch are pulled into L2 (one bulk prefetch per row, by
        // warps 1-2) while tile n is copied, and the next copies start from L2.
        // Row indices are loaded one iteration before they are used, so no
        // global load latency sits between a freed stage and its copies.
        const int pk = pw * 32 + lane;  // key prefetched by this thread
        const bool prefetcher = pk < kTile;
        const int32_t *tile_rows = rows + (int64_t)j0 * kTile;
        const uint8_t *rope = static_cast<const uint8_t *>(p.kv_rope);
        auto prefetch_row = [&](int32_t r) {
            if (a.fp8) {
                prefetch_l2(kv + (int64_t)r * kDl, kDl);
                prefetch_l2(rope + (int64_t)r * (kDr * 2), kDr * 2);
            } else {
                prefetch_l2(kv + (int64_t)r * (kD * 2), kD * 2);
            }
        };
        if (prefetcher) {
            int32_t r0[kPrefetch];
#pragma unroll
            for (int n = 0; n < kPrefetch; ++n) r0[n] = n < T ? __ldg(tile_rows + n * kTile + pk) : 0;
#pragma unroll
            for (int n = 0; n < kPrefetch; ++n)
                if (n < T) prefetch_row(r0[n]);
        }
        int32_t pf_row =
            (prefetcher && kPrefetch < T) ? __ldg(tile_rows + kPrefetch * kTile + pk) : 0;
        int32_t r_lo = T > 0 ? __ldg(tile_rows + lane) : 0;
        int32_t r_hi = T > 0 ? __ldg(tile_rows + 32 + lane) : 0;
        for (int n = 0; n < T; ++n) {
            const int st = n % kStages;
            if (prefetcher && n + kPrefetch < T) prefetch_row(pf_row);
            const bool more = n + 1 < T;
            const int32_t pf_next = (prefetcher && n + 1 + kPrefetch < T)
                                        ? __ldg(tile_rows + (n + 1 + kPrefetch) * kTile + pk)
                                        : 0;
            const int32_t lo_next = more ? __ldg(tile_rows + (n + 1) * kTile + lane) : 0;
            const int32_t hi_next = more ? __ldg(tile_rows + (n + 1) * kTile + 32 + lane) : 0;
            if (!warp_wait(&sm.kv_empty[st], ((n / kStages) & 1) ^ 1, abort_flag, status)) break;
            if (n == 2 && !warp_wait(&sm.q_ready, 0, abort_flag, status)) break;
            if (!a.fp8) {
                const uint32_t dst0 = smem_u32(sm.kv[st]);
#pragma unroll 1  // measured faster than unrolling by 2 or 4 (32K decode: 0.087 against 0.095 ms)
                for (int k = pw; k < kTile; k += kProducerWarps) {
                    const int32_t r = __shfl_sync(0xffffffffu, k < 32 ? r_lo : r_hi, k & 31);
                    const uint8_t *src = kv + (int64_t)r * (kD * 2);
                    const uint32_t dk = dst0 + (k >> 3) * kGroupBytes + (k & 7) * 128;
                    const int sw = k & 7;
#pragma unroll
                    for (int i = 0; i < 3; ++i) {
                        const int c = lane + 32 * i;
                        if (c < kChunksPerRow)
                            cp_async16(dk + (c >> 3) * 1024 + (((c & 7) ^ sw) << 4), src + c * 16);
                    }
                }
                cp_async_arrive(&sm.kv_full[st]);
            } else {
                // e4m3 latent: lane c dequantises dims 16c .. 16c + 15 of a row
                // (x its page's scale, rounded to bf16) into the same swizzled
                // layout; lanes 0-7 copy the bf16 rope.  Plain stores, so a
                // proxy fence and an ordinary arrive publish them.
                uint8_t *stage = sm.kv[st];
#pragma unroll 2  // measured faster than no unrolling here (1M decode: 0.0327 against 0.0337 ms)
                for (int k = pw; k < kTile; k += kProducerWarps) {
                    const int32_t r = __shfl_sync(0xffffffffu, k < 32 ? r_lo : r_hi, k & 31);
                    const float sc = kv_scale_at(p, r, 16 * lane);  // this lane's 16 dims
                    const uint4 x = __ldg(reinterpret_cast<const uint4 *>(kv + (int64_t)r * kDl) + lane);
                    uint4 rp = make_uint4(0, 0, 0, 0);
                    if (lane < 8)
                        rp = __ldg(reinterpret_cast<const uint4 *>(rope + (int64_t)r * (kDr * 2)) + lane);
                    const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
                    uint32_t o[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const uint16_t two = static_cast<uint16_t>(xw[i >> 1] >> (16 * (i & 1)));
                        const float2 f = e4m3x2_to_float2(two);
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(f.x * sc, f.y * sc);
                        o[i] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    uint8_t *dk = stage + (k >> 3) * kGroupBytes + (k & 7) * 128;
                    const int sw = k & 7, b = lane >> 2, c0 = 2 * (lane & 3);
                    *reinterpret_cast<uint4 *>(dk + b * 1024 + ((c0 ^ sw) << 4)) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4 *>(dk + b * 1024 + (((c0 + 1) ^ sw) << 4)) =
                        make_uint4(o[4], o[5], o[6], o[7]);
                    if (lane < 8)
                        *reinterpret_cast<uint4 *>(dk + 8 * 1024 + ((lane ^ sw) << 4)) = rp;
                }
                fence_proxy_async_smem();
                mbar_arrive(&sm.kv_full[st]);
            }
            pf_row = pf_next;
            r_lo = lo_next;
            r_hi = hi_next;
        }
        cp_async_wait_all();
    } else if (lane == 0 && T > 0) {
        // ------------------------------------------------- MMA issuer ---
        constexpr uint32_t id_s = instr_desc(64, kTile, 1 /*bf16*/, 0, 0);
        constexpr uint32_t id_pv = instr_desc(64, 256, 1 /*bf16*/, 0, 1);
        bool ok = mbar_wait(&sm.q_ready, 0, abort_flag, status);
        int ns = 0, np = 0;  // next S and next P V to issue
        // P V(np) needs P of tile np
        auto try_pv = [&]() -> bool {
            const int st = np % kStages;
            if (!(np < ns && mbar_test(&sm.p_full[st], (np / kStages) & 1))) return false;
            fence_proxy_async_smem();
            tc_fence_after();
            const uint64_t ad = desc_kmajor_sw128_sbo(smem_u32(sm.kv[st]) + kPOffset, kGroupBytes);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const uint32_t vb = smem_u32(sm.kv[st]) + 4 * half * 1024;
#pragma unroll
                for (int k = 0; k < 4; ++k)  // 16 keys (two groups) per instruction
                    mma_bf16(tmem + (kLaneO << 16) + 256 * half, ad + 2 * k,
                             desc_mnmajor_sw128(vb + 2 * k * kGroupBytes, 1024, kGroupBytes),
                             id_pv, (np > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit(&sm.o_done);
            if (np + kStages < T) mma_commit(&sm.kv_empty[st]);
            ++np;
            return true;
        };
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
                    const uint32_t stage = smem_u32(sm.kv[st]);
#pragma unroll  // 36 MMAs straight-line: measured faster than a loop over the blocks
                    for (int b = 0; b < kBlocks; ++b) {
                        const uint64_t bd = desc_kmajor_sw128_sbo(stage + b * 1024, kGroupBytes);
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
            if (try_pv()) progressed = true;
            if (progressed) {
                t0 = clock64();
                idle = 0;
            } else if ((++idle & 63) == 0 && wait_expired(t0, abort_flag, status)) {
                break;
            }
        }
        // o_final: every MMA issued above (all P V of the tiles) has completed;
        // after a timeout too, so that TMEM is never released under an MMA
        mma_commit(&sm.o_final);
        int never = 0;
        mbar_wait(&sm.o_final, 0, &never, status);
    }
    // with no tiles nobody waited for Q: its copy must land before the CTA ends
    if (warp == 0 && lane == 0 && T == 0) mbar_wait(&sm.q_full, 0, abort_flag, status);
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// out = sum_s w_s o_s with w_s = exp(lse_s - lse), lse = log sum_s exp(lse_s).
// One CTA per (query, head): the split weights are computed once in shared
// memory, then each thread merges four output dims over all splits with the
// partial loads unrolled.
constexpr int kMaxSplits = 128;
__global__ void __launch_bounds__(128)
sfa_combine_kernel(const float *__restrict__ o_part, const float *__restrict__ lse_part,
                   int32_t splits, void *out, int32_t out_dtype, float *lse) {
    pdl_wait();
    pdl_trigger();
    __shared__ float w_s[kMaxSplits];
    const int64_t row = blockIdx.x;  // t * 128 + head
    const int64_t t = row >> 7, head = row & 127;
    if (threadIdx.x < splits) w_s[threadIdx.x] = lse_part[(t * splits + threadIdx.x) * 128 + head];
    __syncthreads();
    if (threadIdx.x < 32) {
        float m = -INFINITY;
        for (int s = threadIdx.x; s < splits; s += 32) m = fmaxf(m, w_s[s]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float sum = 0.f;
        for (int s = threadIdx.x; s < splits; s += 32) {
            const float ls = w_s[s];
            const float w = (m == -INFINITY || ls == -INFINITY) ? 0.f : __expf(ls - m);
            w_s[s] = w;
            sum += w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const float inv = sum > 0.f ? 1.f / sum : 0.f;
        for (int s = threadIdx.x; s < splits; s += 32) w_s[s] *= inv;
        if (lse != nullptr && threadIdx.x == 0) lse[row] = sum > 0.f ? m + logf(sum) : -INFINITY;
    }
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const float4 *src = reinterpret_cast<const float4 *>(o_part + (t * splits * 128 + head) * kDl) +
                        threadIdx.x;
    const int64_t stride = 128 * kDl / 4;  // one split, in float4
#pragma unroll 8
    for (int s = 0; s < splits; ++s) {
        const float w = w_s[s];
        const float4 v = src[s * stride];
        acc[0] += w * v.x;
        acc[1] += w * v.y;
        acc[2] += w * v.z;
        acc[3] += w * v.w;
    }
    if (out_dtype == SA_BF16) {
        __nv_bfloat162 a = __floats2bfloat162_rn(acc[0], acc[1]);
        __nv_bfloat162 b = __floats2bfloat162_rn(acc[2], acc[3]);
        uint2 w = make_uint2(*reinterpret_cast<uint32_t *>(&a), *reinterpret_cast<uint32_t *>(&b));
        reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(out) + row * kDl)[threadIdx.x] = w;
    } else {
        reinterpret_cast<float4 *>(static_cast<float *>(out) + row * kDl)[threadIdx.x] =
            make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
}

}  // namespace

bool sfa_mma_supported(const PathParams &p, int32_t top_k) {
    const bool kv_ok = p.kv_dtype == SA_BF16 ||
                       (p.kv_dtype == SA_E4M3 && p.kv_rope != nullptr && p.kv_scale != nullptr);
    return kv_ok && p.q_dtype == SA_BF16 && p.heads == 128 &&
           p.d_latent == kDl && p.d_rope == kDr && top_k <= kMaxK &&
           (int64_t)p.num_pages * 64 < (int64_t(1) << 31);
}

int32_t sfa_splits(int32_t n_q, int32_t top_k) {
    const int32_t ctas = std::max(1, num_sms());
    const int32_t max_tiles = (top_k + kTile - 1) / kTile;
    if (n_q <= 0) return 1;
    return std::max(1, std::min({max_tiles, ctas / (2 * n_q), kMaxSplits}));
}

int32_t sfa_rows_ld(int32_t top_k) { return (int32_t)round_up(top_k > 0 ? top_k : 1, kTile); }

cudaError_t launch_sfa_mma(const PathParams &p, const int32_t *idx, int32_t top_k, int32_t splits,
                           int32_t *rows, int32_t *n_valid, bool rows_ready, void *out,
                           int32_t out_dtype, float *lse, float *o_part, float *lse_part,
                           cudaStream_t s) {
    if (p.n_q == 0) return cudaSuccess;
    const int32_t ld_rows = sfa_rows_ld(top_k);
    cudaError_t e;
    if (!rows_ready) {
        count_launch();
        e = launch_pdl(sfa_rows_kernel, dim3(static_cast<unsigned>(p.n_q)), dim3(kRowsThreads), 0,
                       s, p, idx, top_k, ld_rows, rows, n_valid);
        if (e != cudaSuccess) return e;
    }
    CUtensorMap tq;
    if (!encode_tmap_2d(&tq, 2, p.q, kD, (uint64_t)p.n_q * 128, kD * 2, 64, kHeadsCta, true))
        return cudaErrorInvalidValue;
    SfaArgs a{p,         rows,   n_valid,  ld_rows,  splits, p.kv_dtype == SA_E4M3,
              out,       out_dtype, lse,    o_part,   lse_part};
    const size_t smem = sizeof(SfaSmem) + 1024;
    e = cudaFuncSetAttribute(sfa_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = 2 * (int64_t)p.n_q * splits;
    count_launch();
    e = launch_pdl(sfa_mma_kernel, dim3(static_cast<unsigned>(grid)), dim3(kThreads), smem, s, tq,
                   a);
    if (e != cudaSuccess || splits == 1) return e;
    count_launch();
    return launch_pdl(sfa_combine_kernel, dim3(static_cast<unsigned>(p.n_q * 128)), dim3(128), 0,
                      s, (const float *)o_part, (const float *)lse_part, splits, out, out_dtype,
                      lse);
}

}  // namespace sa
