// indexer_mma.cu -- lightning indexer on the 5th-generation tensor cores.
//
// Scores every visible cached position of every query ("Optimizing Next-Gen
// LLM Inference" §3.1: relevance scoring, head-weight weighting, and its two
// numerical paths; §4: index keys quantised to 8-bit floats):
//     I[t,s] = ks[s] * sum_j (w[t,j] * qs[t,j]) * max(0, q8[t,j,:] . k8[s,:])
// which equals sum_j w * max(0, q_I . k_I) because the scales are positive;
// on the BF16 path ("Inference Acceleration for New Large Model Architectures"
// §3.1) the query and keys are unscaled bf16 and ks = qs = 1.  On the MXFP8
// path (the index query and keys with one power-of-two scale per group of 32
// values: "Long-Context LLM Inference Optimization", Layered Quantization;
// "Inference Acceleration for New Large Model Architectures" §4.1) the group
// scales cannot leave the ReLU -- they differ inside one dot product -- so the
// tensor cores apply them: tcgen05.mma kind::mxf8f6f4.block_scale multiplies
// each 32-wide slice of a key row and of a query row by its E8M0 scale inside
// the MMA, and the epilogue sees q_I . k_I directly.
//
// The contraction of 64 heads x 128 dims against every key is a dense GEMM
// (M = 128 keys of a two-page tile, N = 64 heads, K = 128), so it runs as
// tcgen05.mma kind::f8f6f4 (e4m3 x e4m3 -> fp32 in TMEM), or kind::f16 with
// bf16 operands.  In chunked prefill, consecutive queries of one sequence see
// (nearly) the same keys ("Inference Acceleration for New Large Model
// Architectures" §5.2: the causal index load grows with position), so groups
// of four of them share every key tile: N = 4 x 64 heads, one full-rate
// M = 128, N = 256 MMA per 32-wide K step, each key tile read once per group.  A bf16 key row is 256 bytes, two 128-byte swizzle atoms
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
constexpr int kScaleSlots = 8;  // key-scale ring: the epilogue frees these, not the key stages
constexpr uint32_t kAtom = 128;  // bytes of a row in one 128-byte swizzle atom

// Numerical paths: e4m3 codes with one fp32 scale per key and per (query,
// head); unscaled bf16; e4m3 codes with one E8M0 scale byte per 32 values.
enum IxMode : int { kModeE4m3 = 0, kModeBf16 = 1, kModeMx = 2 };

// MXFP8 scale factors in tensor memory (columns past the accumulators): the
// block-scaled MMA reads the scale of row r of a 128-row operand for K-block
// kb from lane r % 32 (of every 32-lane subpartition), column r / 32, byte kb
// -- the layout tcgen05.cp 32x128b.warpx4 produces from 32 rows of 16 bytes.
constexpr uint32_t kMxGroup = 32;
constexpr uint32_t kColSfa = 192;  // key scales: 4 columns per accumulator in flight
constexpr uint32_t kColSfb = 208;  // query scales: 4 columns per query buffer

// Storage of one index element type.  A row of kDim elements is kChunks
// 128-byte column chunks; a tile stores chunk c of all 128 keys contiguously
// (16 KB, page h at + 8 KB * h), the query chunk c of its 64 heads likewise.
// kQb: queries sharing each key tile (1, or 4 for chunked prefill, e4m3 only).
template <int kMode, int kQb = 1>
struct IxCfg {
    static constexpr bool kBf16 = kMode == kModeBf16;
    static constexpr bool kMx = kMode == kModeMx;
    static constexpr int kElem = kBf16 ? 2 : 1;
    static constexpr int kChunks = kDim * kElem / kAtom;
    static constexpr int kChunkElems = kAtom / kElem;              // TMA box width
    static constexpr uint32_t kPageBytes = 64 * kDim * kElem;
    static constexpr uint32_t kTileBytes = 2 * kPageBytes;
    static constexpr uint32_t kQBytes = kHeads * kDim * kElem;
    static constexpr int kKPerMma = 32 / kElem;                      // K of one instruction
    static constexpr int kMmas = kDim / kKPerMma;
    static constexpr int kCtasPerSm = (kBf16 || kQb > 1) ? 1 : 2;
    static constexpr int kN = kHeads * kQb;                            // MMA N
    // key stages in flight per CTA: 2 x 4 x 16 KB (e4m3) or 4 x 32 KB (bf16) per SM
    // (a fifth bf16 stage measured no faster)
    static constexpr int kStages = 4;
    // TMEM accumulators (kN columns each); MXFP8 keeps three, leaving room
    // for the scale factors; query groups keep two of 256 columns
    static constexpr int kAcc = kMx ? 3 : (kQb > 1 ? 2 : 4);
    static constexpr uint32_t kTmemCols = kQb > 1 ? 512 : 256;
    // epilogue warp groups: two take alternate tiles; with query groups two
    // more share the tiles, each group summing half of the unit's queries
    static constexpr int kSplit = kQb > 1 ? 2 : 1;
    static constexpr int kEpiGroups = 2 * kSplit;
    static constexpr int kQPerGroup = kQb / kSplit;
    static constexpr int kEpiThreads = 128 * kEpiGroups;
    static constexpr int kThreads = 64 + kEpiThreads;
};

template <int kMode, int kQb = 1>
struct IndexerSmem {
    using C = IxCfg<kMode, kQb>;
    uint8_t keys[C::kStages][C::kTileBytes];  // 1024-byte aligned (swizzle atoms)
    uint32_t hist[kQb][kHistBins];            // score-key histograms of the current queries
    uint8_t q[2][kQb * C::kQBytes];           // 1024-byte aligned like the key stages
    float wq[C::kEpiGroups][C::kQPerGroup * kHeads];  // head weights x query scales, per group
    // key scales of the staged pages: one fp32 per key (e4m3), or four E8M0
    // bytes per key (MXFP8), 512 bytes a slot either way
    alignas(16) float kscale[kScaleSlots][kKeys];
    int32_t page_ok[kScaleSlots][2];    // 1 when the staged page id was valid
    // MXFP8: query scale bytes as loaded, and both operands' scales in the
    // 32 x 16-byte row order the copy into tensor memory takes
    alignas(16) uint8_t q_sf[2][kHeads * (kDim / kMxGroup)];
    alignas(128) uint8_t sfa[4][512];
    alignas(128) uint8_t sfb[2][512];
    uint64_t full[C::kStages], empty[C::kStages];
    uint64_t sc_full[kScaleSlots], sc_empty[kScaleSlots];
    uint64_t acc_full[C::kAcc], acc_empty[C::kAcc];
    uint64_t q_full[2], q_empty[2];
    uint64_t done;
    uint32_t tmem_base;
    int32_t start_t, start_i;           // this CTA's first tile (query or group, tile in it)
    int abort;
};

using PrefillSmem = IndexerSmem<kModeE4m3, 4>;
static_assert(offsetof(IndexerSmem<kModeE4m3>, q) % 1024 == 0 &&
                  offsetof(IndexerSmem<kModeBf16>, q) % 1024 == 0 &&
                  offsetof(IndexerSmem<kModeMx>, q) % 1024 == 0 &&
                  offsetof(PrefillSmem, q) % 1024 == 0,
              "128-byte-swizzled Q tiles need 1024-byte alignment");
static_assert(sizeof(PrefillSmem) + 1024 <= 232448, "query groups: one CTA per SM");
static_assert(offsetof(IndexerSmem<kModeE4m3>, wq) % 16 == 0 &&
                  offsetof(IndexerSmem<kModeBf16>, wq) % 16 == 0,
              "head weights are read as float4");
static_assert(2 * (sizeof(IndexerSmem<kModeE4m3>) + 2048) <= 233472, "e4m3: two CTAs per SM");
static_assert(2 * (sizeof(IndexerSmem<kModeMx>) + 2048) <= 233472, "mxfp8: two CTAs per SM");
static_assert(sizeof(IndexerSmem<kModeBf16>) + 1024 <= 232448, "bf16: one CTA per SM");
static_assert(IxCfg<kModeMx>::kAcc * kHeads <= kColSfa && kColSfa + 4 * 4 <= kColSfb &&
                  kColSfb + 2 * 4 <= IxCfg<kModeMx>::kTmemCols,
              "MXFP8 scale columns sit past the accumulators");

struct IndexerArgs {
    PathParams p;
    const int32_t *vis;       // [n_q] visible length (0 = invalid query)
    const int32_t *tile_end;  // [n_units] inclusive prefix of the units' tile counts
    int32_t n_units;          // queries, or groups of kQb queries
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

// Copy a 32-row x 16-byte shared-memory matrix (rows 16 bytes apart) into
// tensor memory lanes 0-31 of every subpartition, four 32-bit columns.
__device__ __forceinline__ void tmem_cp_32x128b(uint32_t taddr, const void *smem) {
    // no-swizzle K-major descriptor: 8-row core matrices of 16-byte rows, 128
    // bytes apart (one core matrix wide in K)
    const uint32_t a = smem_u32(smem);
    const uint64_t desc = (uint64_t)((a >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) |
                          ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc)
                 : "memory");
}

// D (+)= (A x its block scales) (B x its block scales)^T, e4m3 operands with
// one E8M0 scale per 32 K-values; sfa / sfb are tensor-memory addresses with
// the scale byte (the K-block) in their top two bits.
__device__ __forceinline__ void mma_mxf8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Instruction descriptor of the block-scaled MMA: e4m3 x e4m3, fp32
// accumulation, E8M0 scales; scale byte `kb` of both operands.
__host__ __device__ constexpr uint32_t mx_instr_desc(uint32_t m, uint32_t n, uint32_t kb) {
    return (kb << 4) | ((n >> 3) << 17) | (1u << 23) | ((m >> 4) << 24) | (kb << 29);
}

template <int kMode, int kQb>
__global__ void __launch_bounds__(IxCfg<kMode, kQb>::kThreads, IxCfg<kMode, kQb>::kCtasPerSm)
indexer_mma_kernel(const __grid_constant__ CUtensorMap tm_keys,
                   const __grid_constant__ CUtensorMap tm_q, const IndexerArgs a) {
    using C = IxCfg<kMode, kQb>;
    constexpr bool kBf16 = C::kBf16, kMx = C::kMx;
    constexpr int kAcc = C::kAcc;
    static_assert(kQb == 1 || kMode == kModeE4m3, "query groups: e4m3 keys only");
    static_assert(C::kMmas * C::kKPerMma == kDim, "the MMA K steps cover the index dimension");
    pdl_wait();
    extern __shared__ uint8_t smem_raw[];
    IndexerSmem<kMode, kQb> &sm =
        *reinterpret_cast<IndexerSmem<kMode, kQb> *>(align1024(smem_raw));
    const PathParams &p = a.p;
    const int warp = warp_id(), lane = lane_id();
    const int64_t total = a.n_units > 0 ? a.tile_end[a.n_units - 1] : 0;
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
            // the four warps of each epilogue group on the tile (and the MMA
            // warp, which reads the MXFP8 scale bytes)
            mbar_init(&sm.sc_empty[s], 4 * C::kSplit + (kMx ? 1 : 0));
        }
        for (int c = 0; c < kAcc; ++c) {
            mbar_init(&sm.acc_full[c], 1);
            mbar_init(&sm.acc_empty[c], 4 * C::kSplit);
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
        int lo = 0, hi = a.n_units - 1;
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
        tmem_alloc(&sm.tmem_base, C::kTmemCols);
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
            const uint64_t key_policy = l2_evict_first_policy();
            // a unit's keys: its (first) query's sequence, up to its longest query
            auto unit_vis = [&](int32_t u) {
                int32_t v = 0;
#pragma unroll
                for (int j = 0; j < kQb; ++j)
                    if (kQb * u + j < p.n_q) v = max(v, a.vis[kQb * u + j]);
                return v;
            };
            int32_t seq = p.q_seq[kQb * c.t], V = unit_vis(c.t);
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
                        nseq = p.q_seq[kQb * nx.t];
                        nV = unit_vis(nx.t);
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
                    constexpr uint32_t kQSfBytes = kHeads * (kDim / kMxGroup);
                    const int nq = min(kQb, p.n_q - kQb * c.t);  // queries of the unit
                    mbar_arrive_expect_tx(&sm.q_full[b],
                                          nq * C::kQBytes + (kMx ? kQSfBytes : 0u));
                    for (int j = 0; j < nq; ++j) {
#pragma unroll
                        for (int ch = 0; ch < C::kChunks; ++ch)
                            tma_load_2d(sm.q[b] + j * C::kQBytes + ch * (kQb * kHeads * kAtom),
                                        &tm_q, ch * C::kChunkElems, (kQb * c.t + j) * kHeads,
                                        &sm.q_full[b]);
                    }
                    if (kMx)
                        bulk_load(sm.q_sf[b],
                                  reinterpret_cast<const uint8_t *>(p.q_index_scale) +
                                      (int64_t)c.t * kQSfBytes,
                                  kQSfBytes, &sm.q_full[b]);
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
                        for (int ch = 0; ch < C::kChunks; ++ch) {
                            void *dst = sm.keys[stage] + ch * (kKeys * kAtom) + h * (64 * kAtom);
                            // one query per tile: its keys are read once, so they
                            // leave L2 first (the scores and the rows the next
                            // kernels read stay); query groups share key tiles
                            if constexpr (kQb == 1)
                                tma_load_2d_hint(dst, &tm_keys, ch * C::kChunkElems, rows[h],
                                                 &sm.full[stage], key_policy);
                            else
                                tma_load_2d(dst, &tm_keys, ch * C::kChunkElems, rows[h],
                                            &sm.full[stage]);
                        }
                        // 256 bytes a page either way: 64 fp32 scales, or 64 x 4
                        // E8M0 bytes (MXFP8, [num_pages, 64, 4] in memory)
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
        if constexpr (kMx) {
            // The whole warp: it reorders the scale bytes of each tile (and of
            // each query) into the 32 x 16-byte rows that tcgen05.cp copies to
            // tensor memory -- row r holds the four K-block scales of operand
            // rows r, r + 32, r + 64, r + 96 -- then lane 0 copies them and
            // issues the four block-scaled MMAs (one per 32-wide K-block).
            TileCursor c;
            c.init_at(a.tile_end, sm.start_t, sm.start_i, k0, k1);
            bool seg_start = true;
            for (int n = 0; c.valid(); ++n) {
                const int b = c.seg & 1;
                if (seg_start) {
                    if (c.seg > 0 && lane == 0) mma_commit(&sm.q_empty[(c.seg - 1) & 1]);
                    if (!warp_wait(&sm.q_full[b], (c.seg >> 1) & 1, abort_flag, p.status)) break;
                    // heads 0-63: row r = heads r and r + 32 (4 bytes each), padded
                    const uint32_t *qsf = reinterpret_cast<const uint32_t *>(sm.q_sf[b]);
                    *reinterpret_cast<uint4 *>(sm.sfb[b] + 16 * lane) =
                        make_uint4(qsf[lane], qsf[lane + 32], 0x7F7F7F7Fu, 0x7F7F7F7Fu);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tc_fence_after();
                        tmem_cp_32x128b(tmem + kColSfb + 4 * b, sm.sfb[b]);
                    }
                }
                const int stage = n % C::kStages, acc = n % kAcc, slot = n % kScaleSlots;
                if (!warp_wait(&sm.acc_empty[acc], ((n / kAcc) & 1) ^ 1, abort_flag, p.status))
                    break;
                if (!warp_wait(&sm.sc_full[slot], (n / kScaleSlots) & 1, abort_flag, p.status))
                    break;
                // keys 0-127 of the tile: row r = keys r, r + 32, r + 64, r + 96
                const uint32_t *ksf = reinterpret_cast<const uint32_t *>(sm.kscale[slot]);
                *reinterpret_cast<uint4 *>(sm.sfa[acc] + 16 * lane) =
                    make_uint4(ksf[lane], ksf[lane + 32], ksf[lane + 64], ksf[lane + 96]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.sc_empty[slot]);
                if (!warp_wait(&sm.full[stage], (n / C::kStages) & 1, abort_flag, p.status)) break;
                if (lane == 0) {
                    tc_fence_after();
                    tmem_cp_32x128b(tmem + kColSfa + 4 * acc, sm.sfa[acc]);
                    const uint32_t keys = smem_u32(sm.keys[stage]);
                    const uint32_t qs = smem_u32(sm.q[b]);
                    const uint32_t d = tmem + acc * kHeads;
#pragma unroll
                    for (int kb = 0; kb < 4; ++kb)  // 32 bytes of K (one scale block) each
                        mma_mxf8(d, desc_kmajor_sw128(keys) + 2 * kb, desc_kmajor_sw128(qs) + 2 * kb,
                                 mx_instr_desc(kKeys, kHeads, kb),
                                 (tmem + kColSfa + 4 * acc) | ((uint32_t)kb << 30),
                                 (tmem + kColSfb + 4 * b) | ((uint32_t)kb << 30), kb > 0 ? 1u : 0u);
                    mma_commit(&sm.empty[stage]);
                    mma_commit(&sm.acc_full[acc]);
                }
                __syncwarp();
                seg_start = c.next(a.tile_end);
            }
            // every issued MMA has landed before TMEM is released
            if (lane == 0) {
                mma_commit(&sm.done);
                mbar_wait(&sm.done, 0, abort_flag, p.status);
            }
            __syncwarp();
        } else if (lane == 0) {
            // kind::f8f6f4 format 0 = e4m3; kind::f16 format 1 = bf16
            constexpr uint32_t idesc = instr_desc(kKeys, C::kN, kBf16 ? 1 : 0, 0, 0);
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
                const uint32_t d = tmem + acc * C::kN;
                // 32 bytes of K per instruction: four per 128-byte chunk (the
                // descriptor address counts 16-byte units)
#pragma unroll
                for (int kk = 0; kk < C::kMmas; ++kk) {
                    const int ch = kk / 4, w = kk % 4;
                    const uint64_t adesc = desc_kmajor_sw128(keys + ch * (kKeys * kAtom)) + 2 * w;
                    const uint64_t bdesc =
                        desc_kmajor_sw128(qs + ch * (kQb * kHeads * kAtom)) + 2 * w;
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
        // store, histogram) run side by side; with query groups a second pair
        // of groups shares the tiles, each group summing half of the unit's
        // queries, so every SM sub-partition has four epilogue warps to
        // interleave.  Within a group, warp w reads TMEM lanes 32 (w % 4) ..
        // +31: one key row per thread.  The loop never leaves early: after a
        // failed (timed-out) wait it carries on without waiting, so a group's
        // warps meet at the same named barriers.
        constexpr int kQg = C::kQPerGroup;
        const int g = (warp - 2) >> 2;          // epilogue group
        const int tp = g & 1;                   // the parity of the tiles it takes
        const int q0 = (g >> 1) * kQg;          // its first query within the unit
        const int quad = warp & 3;              // TMEM lanes this warp may read
        const int row = quad * 32 + lane;       // key row of the tile
        const int ea = threadIdx.x - 64;        // 0 .. kEpiThreads - 1 over all groups
        const int et = ea & 127;                // 0..127 within the group
        const int bar = 2 + g;                  // the group's named barrier (1: all groups)
        const bool histo = a.hist != nullptr;
        float *wq = sm.wq[g];
        if (histo) {
            for (int b = ea; b < kQb * kHistBins; b += C::kEpiThreads) (&sm.hist[0][0])[b] = 0;
            named_barrier(1, C::kEpiThreads);
        }
        // add the CTA's counts of unit u's queries to their global histograms,
        // then clear; every group walks every tile, so they all get here at
        // the same unit change
        auto flush = [&](int32_t u) {
            named_barrier(1, C::kEpiThreads);
            for (int j = 0; j < kQb; ++j) {
                const int32_t t = kQb * u + j;
                if (t >= p.n_q) break;
                uint32_t *gh = a.hist + (int64_t)t * kHistBins;
                for (int b = ea; b < kHistBins; b += C::kEpiThreads) {
                    const uint32_t v = sm.hist[j][b];
                    if (v != 0) {
                        atomicAdd(gh + b, v);
                        sm.hist[j][b] = 0;
                    }
                }
            }
            named_barrier(1, C::kEpiThreads);
        };
        TileCursor c;
        c.init_at(a.tile_end, sm.start_t, sm.start_i, k0, k1);
        bool ok = true;
        int32_t Vq[kQg];  // visible length of each of the group's queries (0: none)
#pragma unroll
        for (int j = 0; j < kQg; ++j) Vq[j] = 0;
        int32_t t_cur = -1;
        for (int n = 0; c.valid(); ++n, c.next(a.tile_end)) {
            if (c.t != t_cur) {  // a new unit: every group sees it at the same tile
                if (histo && t_cur >= 0) flush(t_cur);
                named_barrier(bar, 128);  // the old weights are no longer read
                t_cur = c.t;
#pragma unroll
                for (int j = 0; j < kQg; ++j) {
                    const int32_t t = kQb * c.t + q0 + j;
                    Vq[j] = t < p.n_q ? a.vis[t] : 0;
                }
                for (int i = et; i < kQg * kHeads; i += 128) {
                    const int32_t t = kQb * c.t + q0 + i / kHeads;
                    const int64_t wi = ((int64_t)kQb * c.t + q0) * kHeads + i;
                    wq[i] = t >= p.n_q ? 0.f
                                       : __ldg(p.w + wi) *
                                             ((kBf16 || kMx) ? 1.f : __ldg(p.q_index_scale + wi));
                }
                named_barrier(bar, 128);
            }
            if ((n & 1) != tp) continue;  // the other groups' tile
            const int64_t s = (int64_t)c.i * kKeys + row;
            int32_t V = 0;  // the longest visible length of the group's queries
#pragma unroll
            for (int j = 0; j < kQg; ++j) V = max(V, Vq[j]);
            // key scales and page validity have a ring of their own
            const int slot = n % kScaleSlots;
            if (ok)
                ok = warp_wait(&sm.sc_full[slot], (n / kScaleSlots) & 1, abort_flag, p.status);
            const bool page_ok = ok && sm.page_ok[slot][row >> 6] != 0;
            const float kscale = ok ? ((kBf16 || kMx) ? 1.f : sm.kscale[slot][row]) : 0.f;
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.sc_empty[slot]);
            if (ok && s < V && !page_ok) report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_PAGE);
            const int acc = n % kAcc;
            if (ok) ok = warp_wait(&sm.acc_full[acc], (n / kAcc) & 1, abort_flag, p.status);
            float sum[kQg];
#pragma unroll
            for (int j = 0; j < kQg; ++j) sum[j] = 0.f;
            if (ok) {
                tc_fence_after();
                const uint32_t tbase =
                    tmem + (static_cast<uint32_t>(quad * 32) << 16) + acc * C::kN + q0 * kHeads;
                // eight independent chains per query: heads 4i + {0, 1} and 4i +
                // {2, 3} of each 32-head half; the query-group kernel runs them
                // as packed fp32 FMAs (one half after the other), the
                // 2-CTA-per-SM kernels (96 registers) as scalar ones (halves
                // interleaved); both round the same products and sums in the same
                // order, so a query's scores do not depend on the kernel
                auto half_sum = [&](const float (&x)[32], const float4 *w4, float2 &p0,
                                    float2 &p1) {
#pragma unroll
                    for (int j4 = 0; j4 < 8; ++j4) {
                        const float4 w = w4[j4];
                        const float2 x0 = make_float2(relu_keep_nan(x[4 * j4]),
                                                      relu_keep_nan(x[4 * j4 + 1]));
                        const float2 x1 = make_float2(relu_keep_nan(x[4 * j4 + 2]),
                                                      relu_keep_nan(x[4 * j4 + 3]));
                        p0 = __ffma2_rn(make_float2(w.x, w.y), x0, p0);
                        p1 = __ffma2_rn(make_float2(w.z, w.w), x1, p1);
                    }
                };
                if constexpr (kQb > 1) {
                    // 2 kQg chunks of 32 columns (query j = i / 2, heads 32 (i % 2) ..):
                    // the load of chunk i + 1 is in flight while chunk i is summed
                    float ca[32], cb[32];
                    float2 part[4] = {};
                    tmem_ld32(tbase, ca);
                    tmem_wait_ld_keep(ca);
#pragma unroll
                    for (int i = 0; i < 2 * kQg; ++i) {
                        float(&cur)[32] = (i & 1) ? cb : ca;
                        float(&nxt)[32] = (i & 1) ? ca : cb;
                        if (i + 1 < 2 * kQg) tmem_ld32(tbase + 32 * (i + 1), nxt);
                        const int j = i >> 1, hf = i & 1;
                        const float4 *w4 = reinterpret_cast<const float4 *>(wq + j * kHeads) + 8 * hf;
                        half_sum(cur, w4, part[2 * hf], part[2 * hf + 1]);
                        if (hf == 1) {
                            sum[j] = ((part[0].x + part[0].y) + (part[1].x + part[1].y)) +
                                     ((part[2].x + part[2].y) + (part[3].x + part[3].y));
#pragma unroll
                            for (int c = 0; c < 4; ++c) part[c] = make_float2(0.f, 0.f);
                        }
                        if (i + 1 < 2 * kQg) tmem_wait_ld_keep(nxt);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < kQg; ++j) {
                        if (!__any_sync(0xffffffffu, s < Vq[j])) continue;  // nothing visible here
                        const uint32_t taddr = tbase + j * kHeads;
                        float v[32], u[32];
                        tmem_ld32(taddr, v);
                        tmem_ld32(taddr + 32, u);
                        tmem_wait_ld();
                        const float4 *w4 = reinterpret_cast<const float4 *>(wq + j * kHeads);
                        float2 part[4] = {};
#pragma unroll
                        for (int j4 = 0; j4 < 8; ++j4) {  // the two halves interleaved
                            const float4 wa = w4[j4], wb = w4[8 + j4];
                            part[0].x = fmaf(wa.x, relu_keep_nan(v[4 * j4]), part[0].x);
                            part[0].y = fmaf(wa.y, relu_keep_nan(v[4 * j4 + 1]), part[0].y);
                            part[1].x = fmaf(wa.z, relu_keep_nan(v[4 * j4 + 2]), part[1].x);
                            part[1].y = fmaf(wa.w, relu_keep_nan(v[4 * j4 + 3]), part[1].y);
                            part[2].x = fmaf(wb.x, relu_keep_nan(u[4 * j4]), part[2].x);
                            part[2].y = fmaf(wb.y, relu_keep_nan(u[4 * j4 + 1]), part[2].y);
                            part[3].x = fmaf(wb.z, relu_keep_nan(u[4 * j4 + 2]), part[3].x);
                            part[3].y = fmaf(wb.w, relu_keep_nan(u[4 * j4 + 3]), part[3].y);
                        }
                        sum[j] = ((part[0].x + part[0].y) + (part[1].x + part[1].y)) +
                                 ((part[2].x + part[2].y) + (part[3].x + part[3].y));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.acc_empty[acc]);
#pragma unroll
            for (int j = 0; j < kQg; ++j) {
                if (s < Vq[j]) {
                    const float score = page_ok ? sum[j] * kscale : -INFINITY;
                    a.scores[(int64_t)(kQb * c.t + q0 + j) * a.ld + s] = score;
                    if (histo)
                        atomicAdd(&sm.hist[q0 + j][order_key(score) >> (32 - kHistBits)], 1u);
                }
            }
        }
        if (histo && t_cur >= 0) flush(t_cur);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace

bool indexer_mma_supported(const PathParams &p) {
    return (p.index_dtype == SA_E4M3 || p.index_dtype == SA_BF16 ||
            p.index_dtype == SA_MXFP8) &&
           p.h_index == kHeads && p.d_index == kDim;
}

namespace {

template <int kMode, int kQb>
cudaError_t launch_indexer_mma_t(const PathParams &p, const int32_t *vis, const int32_t *tile_end,
                                 float *scores, int64_t ld, uint32_t *hist, cudaStream_t s) {
    using C = IxCfg<kMode, kQb>;
    CUtensorMap tk, tq;
    if (!encode_tmap_2d(&tk, C::kElem, p.k_index, kDim, (uint64_t)p.num_pages * 64,
                        kDim * C::kElem, C::kChunkElems, 64, true) ||
        !encode_tmap_2d(&tq, C::kElem, p.q_index, kDim, (uint64_t)p.n_q * kHeads,
                        kDim * C::kElem, C::kChunkElems, kHeads, true))
        return cudaErrorInvalidValue;
    const int32_t n_units = static_cast<int32_t>(ceil_div(p.n_q, kQb));
    IndexerArgs a{p, vis, tile_end, n_units, scores, ld, hist};
    const int64_t max_tiles = (int64_t)n_units * ceil_div(p.max_visible, kKeys);
    const int64_t grid = std::min<int64_t>((int64_t)C::kCtasPerSm * num_sms(), max_tiles);
    const size_t smem = sizeof(IndexerSmem<kMode, kQb>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(indexer_mma_kernel<kMode, kQb>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    return launch_pdl(indexer_mma_kernel<kMode, kQb>, dim3(static_cast<unsigned>(grid)),
                      dim3(C::kThreads), smem, s, tk, tq, a);
}

}  // namespace

int32_t indexer_query_group(const PathParams &p) {
    return (p.q_group == 4 && p.index_dtype == SA_E4M3 && p.n_q >= 4) ? 4 : 1;
}

cudaError_t launch_indexer_mma(const PathParams &p, const int32_t *vis, const int32_t *tile_end,
                               float *scores, int64_t ld, uint32_t *hist, cudaStream_t s) {
    if (p.n_q == 0) return cudaSuccess;
    if (p.index_dtype == SA_BF16)
        return launch_indexer_mma_t<kModeBf16, 1>(p, vis, tile_end, scores, ld, hist, s);
    if (p.index_dtype == SA_MXFP8)
        return launch_indexer_mma_t<kModeMx, 1>(p, vis, tile_end, scores, ld, hist, s);
    if (indexer_query_group(p) == 4)
        return launch_indexer_mma_t<kModeE4m3, 4>(p, vis, tile_end, scores, ld, hist, s);
    return launch_indexer_mma_t<kModeE4m3, 1>(p, vis, tile_end, scores, ld, hist, s);
}

}  // namespace sa
