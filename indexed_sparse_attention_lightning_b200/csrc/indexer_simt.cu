// indexer_simt.cu -- CUDA-core indexer for any (h_index, d_index) shape.
//
// Computes I[t,s] = sum_j w[t,j] * max(0, q_I[t,j,:] . k_I[s,:]) for every
// visible position ("Optimizing Next-Gen LLM Inference" §3.1, relevance scoring
// plus head-weight weighting; fp32, the BF16 path or e4m3 inputs).  With e4m3
// inputs the positive per-(token, head)
// query scale and per-token key scale factor out of the ReLU:
//     I[t,s] = ks[s] * sum_j (w[t,j] * qs[t,j]) * max(0, q8[t,j,:] . k8[s,:]).
// With MXFP8 inputs (one E8M0 scale per 32 values) the scales differ inside a
// dot product, so both sides are dequantised first (exact in fp32: an e4m3
// value times a power of two).  This kernel serves the small fp32
// configuration and any shape the tensor-core indexer does not take; one
// thread owns one position.
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kThreads = 256;
constexpr int kHeadBlock = 16;  // head dot products kept in registers at once

template <int kFmt>  // sa_dtype of the index query and keys
__global__ void __launch_bounds__(kThreads)
indexer_simt_kernel(const PathParams p, float *__restrict__ scores, int64_t ld) {
    constexpr bool kE4M3 = kFmt == SA_E4M3, kBF16 = kFmt == SA_BF16, kMX = kFmt == SA_MXFP8;
    pdl_wait();
    pdl_trigger();
    extern __shared__ float smem[];
    const int32_t H = p.h_index, d = p.d_index;
    float *q_s = smem;          // [H][d] query codes as floats (scale folded into w)
    float *w_s = smem + H * d;  // [H] w * qs
    const int32_t t = blockIdx.y;

    for (int i = threadIdx.x; i < H * d; i += kThreads) {
        if (kE4M3 || kMX) {
            const uint8_t *qb = static_cast<const uint8_t *>(p.q_index) + (int64_t)t * H * d;
            q_s[i] = e4m3x2_to_float2(qb[i]).x;
            if (kMX) {  // [n_q, H, d / 32] scale bytes: element i of the row block
                const uint8_t *qsf = reinterpret_cast<const uint8_t *>(p.q_index_scale);
                q_s[i] *= e8m0_to_float(qsf[((int64_t)t * H * d + i) / 32]);
            }
        } else if (kBF16) {
            q_s[i] = bf16_bits_to_float(
                static_cast<const uint16_t *>(p.q_index)[(int64_t)t * H * d + i]);
        } else {
            q_s[i] = static_cast<const float *>(p.q_index)[(int64_t)t * H * d + i];
        }
    }
    for (int j = threadIdx.x; j < H; j += kThreads) {
        float wj = p.w[(int64_t)t * H + j];
        w_s[j] = kE4M3 ? wj * p.q_index_scale[(int64_t)t * H + j] : wj;
    }
    __syncthreads();

    const int32_t V = visible_len(p, t);
    const int64_t s = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (s >= V) return;
    const int32_t seq = p.q_seq[t];
    const int64_t row = phys_row(p.page_table, p.max_pages, p.num_pages, seq, s);
    if (row < 0) {
        report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_PAGE);
        return;
    }

    float total = 0.f;
    for (int j0 = 0; j0 < H; j0 += kHeadBlock) {
        float acc[kHeadBlock];
#pragma unroll
        for (int jj = 0; jj < kHeadBlock; ++jj) acc[jj] = 0.f;
        for (int d0 = 0; d0 < d; d0 += 16) {
            float k[16];
            if (kE4M3 || kMX) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(
                    static_cast<const uint8_t *>(p.k_index) + row * d + d0);
                const uint32_t words[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float2 lo = e4m3x2_to_float2(static_cast<uint16_t>(words[i] & 0xffffu));
                    float2 hi = e4m3x2_to_float2(static_cast<uint16_t>(words[i] >> 16));
                    k[4 * i + 0] = lo.x;
                    k[4 * i + 1] = lo.y;
                    k[4 * i + 2] = hi.x;
                    k[4 * i + 3] = hi.y;
                }
                if (kMX) {  // the key's scale for these 16 values (one 32-value group)
                    const float ks = e8m0_to_float(
                        reinterpret_cast<const uint8_t *>(p.k_index_scale)[(row * d + d0) / 32]);
#pragma unroll
                    for (int i = 0; i < 16; ++i) k[i] *= ks;
                }
            } else if (kBF16) {
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    static_cast<const uint16_t *>(p.k_index) + row * d + d0);
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const uint4 v = src[i];
                    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        k[8 * i + 2 * j] = __uint_as_float(words[j] << 16);
                        k[8 * i + 2 * j + 1] = __uint_as_float(words[j] & 0xffff0000u);
                    }
                }
            } else {
                const float4 *src = reinterpret_cast<const float4 *>(
                    static_cast<const float *>(p.k_index) + row * d + d0);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float4 v = src[i];
                    k[4 * i + 0] = v.x;
                    k[4 * i + 1] = v.y;
                    k[4 * i + 2] = v.z;
                    k[4 * i + 3] = v.w;
                }
            }
#pragma unroll
            for (int jj = 0; jj < kHeadBlock; ++jj) {
                if (j0 + jj < H) {
                    const float *qj = q_s + (j0 + jj) * d + d0;
#pragma unroll
                    for (int i = 0; i < 16; ++i) acc[jj] = fmaf(qj[i], k[i], acc[jj]);
                }
            }
        }
#pragma unroll
        for (int jj = 0; jj < kHeadBlock; ++jj)
            if (j0 + jj < H) total = fmaf(w_s[j0 + jj], relu_keep_nan(acc[jj]), total);
    }
    if (kE4M3) total *= p.k_index_scale[row];
    scores[(int64_t)t * ld + s] = total;
}

}  // namespace

cudaError_t launch_indexer_simt(const PathParams &p, float *scores, int64_t ld, cudaStream_t s) {
    if (p.n_q == 0 || p.max_visible == 0) return cudaSuccess;
    dim3 grid(static_cast<unsigned>(ceil_div(p.max_visible, kThreads)), p.n_q);
    size_t smem = sizeof(float) * ((size_t)p.h_index * p.d_index + p.h_index);
    auto go = [&](auto kernel) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        count_launch();
        return launch_pdl(kernel, grid, dim3(kThreads), smem, s, p, scores, ld);
    };
    if (p.index_dtype == SA_E4M3) return go(indexer_simt_kernel<SA_E4M3>);
    if (p.index_dtype == SA_MXFP8) return go(indexer_simt_kernel<SA_MXFP8>);
    if (p.index_dtype == SA_BF16) return go(indexer_simt_kernel<SA_BF16>);
    return go(indexer_simt_kernel<SA_F32>);
}

}  // namespace sa
