// indexer_mma.cu -- lightning indexer on the 5th-generation tensor cores.
//
// Scores every visible cached position of every query ("Optimizing Next-Gen
// LLM Inference" §3.1: relevance scoring, head-weight weighting, and its two
// numerical paths; §4: index keys quantised to 8-bit floats):
//     I[t,s] = ks[s] * sum_j (w[t,j] * qs[t,j]) * max(0, q8[t,j,:] . k8[s,:])
// which equals sum_j w * max(0, q_I . k_I) because the scales are positive;
// on the BF16 path ("Inference Acceleration for New Large Model Architectures"
// §3.1) the query and keys are unscaled bf16 and ks = qs = 1.
//
// The contraction of 64 heads x 128 dims against every key is a dense GEMM
// (M = 128 keys of a two-page tile, N = 64 heads, K = 128), so it runs as
// tcgen05.mma kind::f8f6f4 (e4m3 x e4m3 -> fp32 in TMEM), or kind::f16 with
// bf16 operands.  A bf16 key row is 256 bytes, two 128-byte swizzle atoms
// wide, so its tiles are stored as two 64-column halves.  The kernel is
// persistent: the tiles of all queries are laid end to end and every CTA takes
// an equal contiguous share, so short and long contexts balance across SMs.
// Roles per CTA (320 threads; two CTAs per SM for e4m3, one for bf16):
//   warp 0     TMA producer: key pages (8 KB e4m3, or two 8 KB halves bf16,
//              128-byte swizzle) straight from the paged cache into a 4-stage
//              ring, with their per-token scales (bulk copy, e4m3 only) in a
//              ring of their own, and the query's 64x128 block when the query
//              changes; page-table entries are read one tile ahead;
//   warp 1     one thread issues the MMAs into four TMEM accumulators and
//              commits them to mbarriers;
//   warps 2-9  epilogue, two groups of four warps taking alternate tiles: each
//              thread owns one key row of the tile, reads its 64 head scores
//              from TMEM (tcgen05.ld), applies ReLU, the head weights and the
//              staged key scale, and writes one fp32 score; for the fused top-K
//              it also counts the score's 12-bit radix bucket in a shared-memory
//              histogram per query, which is added to the query's global
//              histogram when the CTA leaves the query.
// Every wait is bounded; a timeout is reported in the workspace status word.
#include <cstddef>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace sa {
namespace {
using namespace sm100;

constexpr int kKeys = 128;    // MMA M: keys per tile (two pages)
constexpr int kHeads = 64;    // MMA N: indexer heads
constexpr int kDim = 128;     // MMA K: index dimension
constexpr int kAcc = 4;       // TMEM accumulators (64 columns each)
constexpr int kScaleSlots = 8;  // key-scale ring: the epilogue frees these, not the key stages
constexpr int kEpiGroups = 2;  // epilogue warp groups, alternating tiles
constexpr int kThreads = 64 + kEpiGroups * 128;
constexpr uint32_t kTmemCols = kAcc * kHeads;
constexpr uint32_t kAtom = 128;  // bytes of a row in one 128-byte swizzle atom

// Storage of one index element type.  A row of kDim elements is kChunks
// 128-byte column chunks; a tile stores chunk c of all 128 keys contiguously
// (16 KB, page h at + 8 KB * h), the query chunk c of its 64 heads likewise.
template <bool kBf16>
struct IxCfg {
    static constexpr int kElem = kBf16 ? 2 : 1;
    static constexpr int kChunks = kDim * kElem / kAtom;
    static constexpr int kChunkElems = kAtom / kElem;              // TMA box width
    static constexpr uint32_t kPageBytes = 64 * kDim * kElem;
    static constexpr uint32_t kTileBytes = 2 * kPageBytes;
    static constexpr uint32_t kQBytes = kHeads * kDim * kElem;
    static constexpr int kKPerMma = 32 / kElem;                      // K of one instruction
    static constexpr int kMmas = kDim / kKPerMma;
    static constexpr int kCtasPerSm = kBf16 ? 1 : 2;
    // key stages in flight per CTA: 2 x 4 x 16 KB (e4m3) or 4 x 32 KB (bf16) per SM
    // (a fifth bf16 stage measured no faster)
    static constexpr int kStages = 4;
};

template <bool kBf16>
struct IndexerSmem {
    uint8_t keys[IxCfg<kBf16>::kStages][IxCfg<kBf16>::kTileBytes];  // 1024-byte aligned (swizzle atoms)
    uint32_t hist[kHistBins];              // score-key histogram of the current query
    uint8_t q[2][IxCfg<kBf16>::kQBytes];   // 1024-byte aligned like the key stages
    float wq[kEpiGroups][kHeads];          // head weights x query scales of that query
    float kscale[kScaleSlots][kKeys];   // per-token key scales of the staged pages
    int32_t page_ok[kScaleSlots][2];    // 1 when the staged page id was valid
    uint64_t full[IxCfg<kBf16>::kStages], empty[IxCfg<kBf16>::kStages];
    uint64_t sc_full[kScaleSlots], sc_empty[kScaleSlots];
    uint64_t acc_full[kAcc], acc_empty[kAcc];
    uint64_t q_full[2], q_empty[2];
    uint64_t done;
    uint32_t tmem_base;
    int32_t start_t, start_i;           // this CTA's first tile (query, tile in query)
    int abort;
};

static_assert(offsetof(IndexerSmem<false>, q) % 1024 == 0 &&
                  offsetof(IndexerSmem<true>, q) % 1024 == 0,
              "128-byte-swizzled Q tiles need 1024-byte alignment");
static_assert(offsetof(IndexerSmem<false>, wq) % 16 == 0 &&
                  offsetof(IndexerSmem<true>, wq) % 16 == 0,
              "head weights are read as float4");
static_assert(2 * (sizeof(IndexerSmem<false>) + 2048) <= 233472, "e4m3: two CTAs per SM");
static_assert(sizeof(IndexerSmem<true>) + 1024 <= 232448, "bf16: one CTA per SM");

struct IndexerArgs {
    PathParams p;
    const int32_t *vis;       // [n_q] visible length (0 = invalid query)
    const int32_t *tile_end;  // [n_q] inclusive prefix of ceil(vis / 128)
    float *scores;
    int64_t ld;
    uint32_t *hist;           // [n_q, kHistBins] (zeroed by the caller) or null
};

// Walks this CTA's contiguous share [k, k_end) of the global tile list.
struct TileCursor {
    int64_t k, k_end;
    int32_t t, i, seg;
    int32_t t_end;  // tile_end[t], loaded once per query

    __device__ void init_at(const int32_t *tile_end, int32_t t0, int32_t i0, int64_t k0,
                            int64_t k1) {
        k = k0;
        k_end = k1;
        seg = 0;
        t = t0;
        i = i0;
        t_end = tile_end[t0];
    }
    __device__ bool valid() const { return k < k_end; }
    // Advance one tile; returns true when the next tile starts a new query.
    __device__ bool next(const int32_t *tile_end) {
        ++k;
        ++i;
        if (k >= k_end) return false;
        if (k < t_end) return false;
        do {  // skip queries without tiles
            ++t;
            t_end = tile_end[t];
        } while (k >= t_end);
        i = 0;
        ++seg;
        return true;
    }
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// One lane polls, the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *status) {
    bool ok = true;
    if (lane_id() == 0) ok = mbar_wait(bar, parity, abort_flag, status);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

template <bool kBf16>
__global__ void __launch_bounds__(kThreads, IxCfg<kBf16>::kCtasPerSm)
indexer_mma_kernel(const __grid_constant__ CUtensorMap tm_keys,
                   const __grid_constant__ CUtensorMap tm_q, const IndexerArgs a) {
    using C = IxCfg<kBf16>;
    pdl_wait();
    extern __shared__ uint8_t smem_raw[];
    IndexerSmem<kBf16> &sm = *reinterpret_cast<IndexerSmem<kBf16> *>(align1024(smem_raw));
    const PathParams &p = a.p;
    const int warp = warp_id(), lane = lane_id();
    const int64_t total = p.n_q > 0 ? a.tile_end[p.n_q - 1] : 0;
    const int64_t k0 = total * blockIdx.x / gridDim.x;
    const int64_t k1 = total * (blockIdx.x + 1) / gridDim.x;
    if (k0 >= k1) return;  // uniform over the CTA, before any allocation

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int s = 0; s < kScaleSlots; ++s) {
            mbar_init(&sm.sc_full[s], 1);
            mbar_init(&sm.sc_empty[s], 4);
        }
        for (int c = 0; c < kAcc; ++c) {
            mbar_init(&sm.acc_full[c], 1);
            mbar_init(&sm.acc_empty[c], 4);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.q_full[b], 1);
            mbar_init(&sm.q_empty[b], 1);
        }
        mbar_init(&sm.done, 1);
        sm.abort = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        // this CTA's first tile: the first query t with tile_end[t] > k0, by a
        // 32-way search (a few dependent loads instead of a binary search's
        // dozen), shared with the other roles through shared memory
        int lo = 0, hi = p.n_q - 1;
        while (lo < hi) {
            const int step = (hi - lo + 32) / 32;
            const int q = min(hi, lo + (lane + 1) * step - 1);
            const unsigned bal = __ballot_sync(0xffffffffu, a.tile_end[q] > k0);
            const int j = __ffs(bal) - 1;  // lane 31 probes hi, which qualifies
            hi = min(hi, lo + (j + 1) * step - 1);
            lo += j * step;
        }
        if (lane == 0) {
            sm.start_t = lo;
            sm.start_i = static_cast<int32_t>(k0 - (lo > 0 ? a.tile_end[lo - 1] : 0));
        }
        tmem_alloc(&sm.tmem_base, kTmemCols);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_trigger();  // after the TMEM allocation: a waiting successor holds none
    const uint32_t tmem = sm.tmem_base;
    volatile int *abort_flag = &sm.abort;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer ---
        if (lane == 0) {
            // Page-table entries are looked up one tile ahead, so their load
            // latency overlaps the wait for a free stage instead of sitting
            // between that wait and the TMA copies.
            TileCursor c;
            c.init_at(a.tile_end, sm.start_t, sm.start_i, k0, k1);
            bool seg_start = true;
            int32_t seq = p.q_seq[c.t], V = a.vis[c.t];
            int32_t pg[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t s = (int64_t)c.i * kKeys + 64 * h;
                pg[h] = s < V ? p.page_table[(int64_t)seq * p.max_pages + (s >> 6)] : -1;
            }
            for (int n = 0; c.valid(); ++n) {
                // look-ahead: the next tile of this CTA
                TileCursor nx = c;
                const bool nx_seg = nx.next(a.tile_end);
                int32_t nseq = seq, nV = V, npg[2] = {-1, -1};
                if (nx.valid()) {
                    if (nx_seg) {
                        nseq = p.q_seq[nx.t];
                        nV = a.vis[nx.t];
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int64_t s = (int64_t)nx.i * kKeys + 64 * h;
                        if (s < nV) npg[h] = p.page_table[(int64_t)nseq * p.max_pages + (s >> 6)];
                    }
                }
                if (seg_start) {
                    const int b = c.seg & 1;
                    if (!mbar_wait(&sm.q_empty[b], ((c.seg >> 1) & 1) ^ 1, abort_flag, p.status))
                        break;
                    mbar_arrive_expect_tx(&sm.q_full[b], C::kQBytes);
#pragma unroll
                    for (int ch = 0; ch < C::kChunks; ++ch)
                        tma_load_2d(sm.q[b] + ch * (kHeads * kAtom), &tm_q, ch * C::kChunkElems,
                                    c.t * kHeads, &sm.q_full[b]);
                }
                const int stage = n % C::kStages;
                // the stage is free once its MMAs and its epilogue are done
                if (!mbar_wait(&sm.empty[stage], ((n / C::kStages) & 1) ^ 1, abort_flag, p.status))
                    break;
                const int slot = n % kScaleSlots;
                if (!mbar_wait(&sm.sc_empty[slot], ((n / kScaleSlots) & 1) ^ 1, abort_flag,
                               p.status))
                    break;
                int32_t rows[2] = {-1, -1};
                uint32_t bytes = 0;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int64_t s = (int64_t)c.i * kKeys + 64 * h;
                    if (s < V && pg[h] >= 0 && pg[h] < p.num_pages) {
                        rows[h] = pg[h] * 64;
                        bytes += C::kPageBytes;
                    }
                    sm.page_ok[slot][h] = rows[h] >= 0;  // published by the arrive below
                }
                // the bf16 path has no key scales: the slot then only
                // publishes the page validity
                mbar_arrive_expect_tx(&sm.sc_full[slot],
                                      kBf16 ? 0u : (bytes / C::kPageBytes) * 64 * sizeof(float));
                mbar_arrive_expect_tx(&sm.full[stage], bytes);
#pragma unroll
                for (int h = 0; h < 2; ++h)
                    if (rows[h] >= 0) {
#pragma unroll
                        for (int ch = 0; ch < C::kChunks; ++ch)
                            tma_load_2d(sm.keys[stage] + ch * (kKeys * kAtom) + h * (64 * kAtom),
                                        &tm_keys, ch * C::kChunkElems, rows[h], &sm.full[stage]);
                        if (!kBf16)
                            bulk_load(&sm.kscale[slot][64 * h], p.k_index_scale + rows[h],
                                      64 * sizeof(float), &sm.sc_full[slot]);
                    }
                c = nx;
                seg_start = nx_seg;
                seq = nseq;
                V = nV;
                pg[0] = npg[0];
                pg[1] = npg[1];
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            // kind::f8f6f4 format 0 = e4m3; kind::f16 format 1 = bf16
            constexpr uint32_t idesc = instr_desc(kKeys, kHeads, kBf16 ? 1 : 0, 0, 0);
            TileCursor c;
            c.init_at(a.tile_end, sm.start_t, sm.start_i, k0, k1);
            bool seg_start = true;
            for (int n = 0; c.valid(); ++n) {
                if (seg_start) {
                    if (c.seg > 0) mma_commit(&sm.q_empty[(c.seg - 1) & 1]);
                    if (!mbar_wait(&sm.q_full[c.seg & 1], (c.seg >> 1) & 1, abort_flag, p.status))
                        break;
                }
                const int stage = n % C::kStages, acc = n % kAcc;
                if (!mbar_wait(&sm.acc_empty[acc], ((n / kAcc) & 1) ^ 1, abort_flag, p.status))
                    break;
                if (!mbar_wait(&sm.full[stage], (n / C::kStages) & 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t keys = smem_u32(sm.keys[stage]);
                const uint32_t qs = smem_u32(sm.q[c.seg & 1]);
                const uint32_t d = tmem + acc * kHeads;
                // 32 bytes of K per instruction: four per 128-byte chunk (the
                // descriptor address counts 16-byte units)
#pragma unroll
                for (int kk = 0; kk < C::kMmas; ++kk) {
                    const int ch = kk / 4, w = kk % 4;
                    const uint64_t adesc = desc_kmajor_sw128(keys + ch * (kKeys * kAtom)) + 2 * w;
                    const uint64_t bdesc = desc_kmajor_sw128(qs + ch * (kHeads * kAtom)) + 2 * w;
                    if (kBf16)
                        mma_bf16(d, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
                    else
                        mma_f8(d, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sm.empty[stage]);
                mma_commit(&sm.acc_full[acc]);
                seg_start = c.next(a.tile_end);
            }
            // every issued MMA has landed before TMEM is released
            mma_commit(&sm.done);
            mbar_wait(&sm.done, 0, abort_flag, p.status);
        }
    } else {
        // --------------------------------------------------- epilogue ---
        // Two groups of four warps take alternate tiles, so two tiles' chains
        // (scale wait, accumulator wait, TMEM loads, weighted ReLU sum, score
        // store, histogram) run side by side.  Within a group, warp w reads
        // TMEM lanes 32 (w % 4) .. +31: one key row per thread.  The loop
        // never leaves early: after a failed (timed-out) wait it carries on
        // without waiting, so a group's warps meet at the same named barriers.
        const int g = (warp - 2) >> 2;          // epilogue group
        const int quad = warp & 3;              // TMEM lanes this warp may read
        const int row = quad * 32 + lane;       // key row of the tile
        const int ea = threadIdx.x - 64;        // 0..255 over both groups
        const int et = ea - 128 * g;            // 0..127 within the group
        const int bar = 2 + g;                  // the group's named barrier (1: both groups)
        const bool histo = a.hist != nullptr;
        float *wq = sm.wq[g];
        if (histo) {
            for (int b = ea; b < kHistBins; b += 256) sm.hist[b] = 0;
            named_barrier(1, 256);
        }
        // add the CTA's counts of query t to the global histogram, then clear;
        // both groups walk every tile, so they get here at the same query change
        auto flush = [&](int32_t t) {
            named_barrier(1, 256);
            uint32_t *gh = a.hist + (int64_t)t * kHistBins;
            for (int b = ea; b < kHistBins; b += 256) {
                const uint32_t v = sm.hist[b];
                if (v != 0) {
                    atomicAdd(gh + b, v);
                    sm.hist[b] = 0;
                }
            }
            named_barrier(1, 256);
        };
        TileCursor c;
        c.init_at(a.tile_end, sm.start_t, sm.start_i, k0, k1);
        bool ok = true;
        int32_t V = 0, t_cur = -1;
        for (int n = 0; c.valid(); ++n, c.next(a.tile_end)) {
            if (c.t != t_cur) {  // a new query: both groups see it at the same tile
                if (histo && t_cur >= 0) flush(t_cur);
                named_barrier(bar, 128);  // the old weights are no longer read
                t_cur = c.t;
                V = a.vis[c.t];
                if (et < kHeads)
                    wq[et] = __ldg(p.w + (int64_t)c.t * kHeads + et) *
                             (kBf16 ? 1.f : __ldg(p.q_index_scale + (int64_t)c.t * kHeads + et));
                named_barrier(bar, 128);
            }
            if ((n & 1) != g) continue;  // the other group's tile
            const int64_t s = (int64_t)c.i * kKeys + row;
            // key scales and page validity have a ring of their own
            const int slot = n % kScaleSlots;
            if (ok)
                ok = warp_wait(&sm.sc_full[slot], (n / kScaleSlots) & 1, abort_flag, p.status);
            const bool page_ok = ok && sm.page_ok[slot][row >> 6] != 0;
            const float kscale = ok ? (kBf16 ? 1.f : sm.kscale[slot][row]) : 0.f;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.sc_empty[slot]);
            if (ok && s < V && !page_ok) report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_PAGE);
            const int acc = n % kAcc;
            if (ok) ok = warp_wait(&sm.acc_full[acc], (n / kAcc) & 1, abort_flag, p.status);
            float sum = 0.f;
            if (ok) {
                tc_fence_after();
                const uint32_t taddr =
                    tmem + (static_cast<uint32_t>(quad * 32) << 16) + acc * kHeads;
                float v[32], u[32];
                tmem_ld32(taddr, v);
                tmem_ld32(taddr + 32, u);
                tmem_wait_ld();
                const float4 *w4 = reinterpret_cast<const float4 *>(wq);
                float part[4] = {0.f, 0.f, 0.f, 0.f};  // four independent chains
#pragma unroll
                for (int j4 = 0; j4 < 8; ++j4) {
                    const float4 wa = w4[j4], wb = w4[8 + j4];
                    part[0] = fmaf(wa.x, relu_keep_nan(v[4 * j4]), part[0]);
                    part[1] = fmaf(wa.y, relu_keep_nan(v[4 * j4 + 1]), part[1]);
                    part[2] = fmaf(wa.z, relu_keep_nan(v[4 * j4 + 2]), part[2]);
                    part[3] = fmaf(wa.w, relu_keep_nan(v[4 * j4 + 3]), part[3]);
                    part[0] = fmaf(wb.x, relu_keep_nan(u[4 * j4]), part[0]);
                    part[1] = fmaf(wb.y, relu_keep_nan(u[4 * j4 + 1]), part[1]);
                    part[2] = fmaf(wb.z, relu_keep_nan(u[4 * j4 + 2]), part[2]);
                    part[3] = fmaf(wb.w, relu_keep_nan(u[4 * j4 + 3]), part[3]);
                }
                sum = (part[0] + part[1]) + (part[2] + part[3]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acc_empty[acc]);
            if (s < V) {
                const float score = page_ok ? sum * kscale : -INFINITY;
                a.scores[(int64_t)c.t * a.ld + s] = score;
                if (histo) atomicAdd(&sm.hist[order_key(score) >> (32 - kHistBits)], 1u);
            }
        }
        if (histo && t_cur >= 0) flush(t_cur);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool indexer_mma_supported(const PathParams &p) {
    return (p.index_dtype == SA_E4M3 || p.index_dtype == SA_BF16) && p.h_index == kHeads &&
           p.d_index == kDim;
}

namespace {

template <bool kBf16>
cudaError_t launch_indexer_mma_t(const PathParams &p, const int32_t *vis, const int32_t *tile_end,
                                 float *scores, int64_t ld, uint32_t *hist, cudaStream_t s) {
    using C = IxCfg<kBf16>;
    CUtensorMap tk, tq;
    if (!encode_tmap_2d(&tk, C::kElem, p.k_index, kDim, (uint64_t)p.num_pages * 64,
                        kDim * C::kElem, C::kChunkElems, 64, true) ||
        !encode_tmap_2d(&tq, C::kElem, p.q_index, kDim, (uint64_t)p.n_q * kHeads,
                        kDim * C::kElem, C::kChunkElems, kHeads, true))
        return cudaErrorInvalidValue;
    IndexerArgs a{p, vis, tile_end, scores, ld, hist};
    const int64_t max_tiles = (int64_t)p.n_q * ceil_div(p.max_visible, kKeys);
    const int64_t grid = std::min<int64_t>((int64_t)C::kCtasPerSm * num_sms(), max_tiles);
    const size_t smem = sizeof(IndexerSmem<kBf16>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(indexer_mma_kernel<kBf16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    return launch_pdl(indexer_mma_kernel<kBf16>, dim3(static_cast<unsigned>(grid)),
                      dim3(kThreads), smem, s, tk, tq, a);
}

}  // namespace

cudaError_t launch_indexer_mma(const PathParams &p, const int32_t *vis, const int32_t *tile_end,
                               float *scores, int64_t ld, uint32_t *hist, cudaStream_t s) {
    if (p.n_q == 0) return cudaSuccess;
    return p.index_dtype == SA_BF16
               ? launch_indexer_mma_t<true>(p, vis, tile_end, scores, ld, hist, s)
               : launch_indexer_mma_t<false>(p, vis, tile_end, scores, ld, hist, s);
}

}  // namespace sa
