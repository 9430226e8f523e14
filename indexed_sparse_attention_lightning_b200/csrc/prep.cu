// prep.cu -- input preparation before the indexer: FP8 quantisation of the
// indexer query and the append of new tokens to the paged caches
// ("Optimizing Next-Gen LLM Inference", §3.2 and the §4 table; "Inference
// Acceleration for New Large Model Architectures", §3.3 and §4.1-4.2).
//
// Dynamic FP8 quantisation, per group of values, in fp32:
//     amax = max |x|,  scale = amax / 448 (1 for an all-zero group),
//     code = e4m3(x / scale), round to nearest even, saturated to +-448,
// so the largest magnitude of a group lands on e4m3's largest finite value.
// The division is IEEE round-to-nearest (__fdiv_rn): the codes depend on it.
//
// Both kernels are memory-bound: one warp per quantised row of the query
// (d_index values), one CTA per appended token.
#include "common.cuh"
#include "internal.h"
#include "prep.h"

namespace sa {
namespace {

constexpr float kE4m3Max = 448.0f;
constexpr int kAppendThreads = 128;
constexpr int kMaxGroups = 32;  // latent groups per token: d_latent <= 512, group >= 16

__device__ __forceinline__ float fp8_scale(float amax) {
    return amax > 0.0f ? __fdiv_rn(amax, kE4m3Max) : 1.0f;
}

__device__ __forceinline__ uint8_t to_e4m3(float x, float scale) {
    return static_cast<uint8_t>(
        __nv_cvt_float_to_fp8(__fdiv_rn(x, scale), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ float load_value(const void *base, int64_t i, bool bf16) {
    return bf16 ? bf16_bits_to_float(static_cast<const uint16_t *>(base)[i])
                : static_cast<const float *>(base)[i];
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// ---------------------------------------------------------------------------
// Query quantisation.  Rows of d = 32 * C values: lane l holds values
// [l*C, l*C + C) (one 8- or 16-byte load for bf16, one or two 16-byte loads
// for fp32) and stores its C codes with one 4- or 8-byte store.
// ---------------------------------------------------------------------------
template <int C, bool BF16>
__global__ void __launch_bounds__(256) quantize_rows_vec_kernel(const void *__restrict__ in,
                                                                int64_t n_rows,
                                                                uint8_t *__restrict__ codes,
                                                                float *__restrict__ scales) {
    static_assert(C == 4 || C == 8, "4 or 8 values per lane");
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n_rows;
         r += warps) {
        const int64_t base = r * (32 * C) + (int64_t)lane * C;
        float v[C];
        if constexpr (BF16) {
            const uint16_t *src = static_cast<const uint16_t *>(in) + base;
            uint32_t w[C / 2];
            if constexpr (C == 4) {
                const uint2 u = __ldg(reinterpret_cast<const uint2 *>(src));
                w[0] = u.x, w[1] = u.y;
            } else {
                const uint4 u = __ldg(reinterpret_cast<const uint4 *>(src));
                w[0] = u.x, w[1] = u.y, w[2] = u.z, w[3] = u.w;
            }
#pragma unroll
            for (int j = 0; j < C / 2; j++) {
                v[2 * j] = __uint_as_float(w[j] << 16);
                v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
            }
        } else {
            const float *src = static_cast<const float *>(in) + base;
#pragma unroll
            for (int j = 0; j < C; j += 4) {
                const float4 f = __ldg(reinterpret_cast<const float4 *>(src + j));
                v[j] = f.x, v[j + 1] = f.y, v[j + 2] = f.z, v[j + 3] = f.w;
            }
        }
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < C; j++) amax = fmaxf(amax, fabsf(v[j]));
        const float scale = fp8_scale(warp_max(amax));
        uint32_t packed[C / 4];
#pragma unroll
        for (int j = 0; j < C / 4; j++) {
            packed[j] = 0;
#pragma unroll
            for (int b = 0; b < 4; b++)
                packed[j] |= static_cast<uint32_t>(to_e4m3(v[4 * j + b], scale)) << (8 * b);
        }
        if constexpr (C == 4) {
            *reinterpret_cast<uint32_t *>(codes + base) = packed[0];
        } else {
            *reinterpret_cast<uint2 *>(codes + base) = make_uint2(packed[0], packed[1]);
        }
        if (lane == 0) scales[r] = scale;
    }
}

// Any row length: lanes stride over the row (coalesced), two passes.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const void *__restrict__ in,
                                                            int32_t bf16, int64_t n_rows,
                                                            int32_t d,
                                                            uint8_t *__restrict__ codes,
                                                            float *__restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n_rows;
         r += warps) {
        const int64_t base = r * d;
        float amax = 0.0f;
        for (int32_t i = lane; i < d; i += 32)
            amax = fmaxf(amax, fabsf(load_value(in, base + i, bf16 != 0)));
        const float scale = fp8_scale(warp_max(amax));
        for (int32_t i = lane; i < d; i += 32)
            codes[base + i] = to_e4m3(load_value(in, base + i, bf16 != 0), scale);
        if (lane == 0) scales[r] = scale;
    }
}

// ---------------------------------------------------------------------------
// Append.  One CTA per new token (grid-stride); group maxima go through
// shared-memory atomics on the bit patterns of |x| (non-negative floats order
// like their bits).
// ---------------------------------------------------------------------------

// n values starting at element s0 of src -> codes at dst[0..n) and one scale
// per group of g values at scl[0..n/g).  Every thread of the CTA calls it.
__device__ void quantize_groups(const void *src, int64_t s0, bool bf16, int32_t n, int32_t g,
                                uint8_t *dst, float *scl, int32_t *gmax) {
    const int32_t groups = n / g;
    for (int32_t i = threadIdx.x; i < groups; i += blockDim.x) gmax[i] = 0;
    __syncthreads();
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x)
        atomicMax(&gmax[i / g], __float_as_int(fabsf(load_value(src, s0 + i, bf16))));
    __syncthreads();
    for (int32_t i = threadIdx.x; i < n; i += blockDim.x)
        dst[i] = to_e4m3(load_value(src, s0 + i, bf16), fp8_scale(__int_as_float(gmax[i / g])));
    for (int32_t i = threadIdx.x; i < groups; i += blockDim.x)
        scl[i] = fp8_scale(__int_as_float(gmax[i]));
    __syncthreads();  // gmax is reused by the next call
}

__device__ __forceinline__ uint16_t to_bf16_bits(const void *src, int64_t i, bool bf16) {
    if (bf16) return static_cast<const uint16_t *>(src)[i];
    return __bfloat16_as_ushort(__float2bfloat16_rn(static_cast<const float *>(src)[i]));
}

__global__ void __launch_bounds__(kAppendThreads) append_kernel(const AppendParams p) {
    __shared__ int32_t gmax[kMaxGroups];
    const bool bf16 = p.in_bf16 != 0;
    for (int32_t t = blockIdx.x; t < p.n_new; t += gridDim.x) {
        const int32_t seq = __ldg(p.seq + t), pos = __ldg(p.pos + t);
        if (seq < 0 || seq >= p.batch || pos < 0 || (pos >> 6) >= p.max_pages) {
            if (threadIdx.x == 0) report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_POSITION);
            continue;  // uniform over the CTA
        }
        const int64_t row = phys_row(p.page_table, p.max_pages, p.num_pages, seq, pos);
        if (row < 0) {
            if (threadIdx.x == 0) report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_PAGE);
            continue;
        }
        if (p.k_new != nullptr) {
            const int64_t s0 = (int64_t)t * p.d_index;
            if (p.index_dtype == SA_E4M3) {
                quantize_groups(p.k_new, s0, bf16, p.d_index, p.d_index,
                                static_cast<uint8_t *>(p.k_index) + row * p.d_index,
                                p.k_index_scale + row, gmax);
            } else if (p.index_dtype == SA_BF16) {
                uint16_t *dst = static_cast<uint16_t *>(p.k_index) + row * p.d_index;
                for (int32_t i = threadIdx.x; i < p.d_index; i += blockDim.x)
                    dst[i] = to_bf16_bits(p.k_new, s0 + i, bf16);
            } else {
                float *dst = static_cast<float *>(p.k_index) + row * p.d_index;
                for (int32_t i = threadIdx.x; i < p.d_index; i += blockDim.x)
                    dst[i] = load_value(p.k_new, s0 + i, bf16);
            }
        }
        if (p.kv_new != nullptr) {
            const int32_t D = p.d_latent + p.d_rope;
            const int64_t s0 = (int64_t)t * D;
            if (p.kv_dtype == SA_E4M3) {
                const int32_t groups = p.d_latent / p.kv_scale_dims;
                quantize_groups(p.kv_new, s0, bf16, p.d_latent, p.kv_scale_dims,
                                static_cast<uint8_t *>(p.kv) + row * p.d_latent,
                                p.kv_scale + row * groups, gmax);
                uint16_t *rope = static_cast<uint16_t *>(p.kv_rope) + row * p.d_rope;
                for (int32_t i = threadIdx.x; i < p.d_rope; i += blockDim.x)
                    rope[i] = to_bf16_bits(p.kv_new, s0 + p.d_latent + i, bf16);
            } else if (p.kv_dtype == SA_BF16) {
                uint16_t *dst = static_cast<uint16_t *>(p.kv) + row * D;
                for (int32_t i = threadIdx.x; i < D; i += blockDim.x)
                    dst[i] = to_bf16_bits(p.kv_new, s0 + i, bf16);
            } else {
                float *dst = static_cast<float *>(p.kv) + row * D;
                for (int32_t i = threadIdx.x; i < D; i += blockDim.x)
                    dst[i] = load_value(p.kv_new, s0 + i, bf16);
            }
        }
    }
}

}  // namespace

cudaError_t launch_quantize_rows(const void *in, sa_dtype in_dtype, int64_t n_rows, int32_t d,
                                 uint8_t *codes, float *scales, cudaStream_t s) {
    if (n_rows <= 0) return cudaSuccess;
    constexpr int kThreads = 256, kWarps = kThreads / 32;
    const int64_t want = (n_rows + kWarps - 1) / kWarps;
    const int grid = (int)std::min<int64_t>(want, (int64_t)num_sms() * 16);
    const bool bf16 = in_dtype == SA_BF16;
    count_launch();
    if (d == 128) {
        if (bf16)
            quantize_rows_vec_kernel<4, true><<<grid, kThreads, 0, s>>>(in, n_rows, codes, scales);
        else
            quantize_rows_vec_kernel<4, false><<<grid, kThreads, 0, s>>>(in, n_rows, codes, scales);
    } else if (d == 256) {
        if (bf16)
            quantize_rows_vec_kernel<8, true><<<grid, kThreads, 0, s>>>(in, n_rows, codes, scales);
        else
            quantize_rows_vec_kernel<8, false><<<grid, kThreads, 0, s>>>(in, n_rows, codes, scales);
    } else {
        quantize_rows_kernel<<<grid, kThreads, 0, s>>>(in, bf16 ? 1 : 0, n_rows, d, codes, scales);
    }
    return cudaGetLastError();
}

cudaError_t launch_append(const AppendParams &p, cudaStream_t s) {
    if (p.n_new <= 0) return cudaSuccess;
    const int grid = std::min(p.n_new, num_sms() * 16);
    count_launch();
    append_kernel<<<grid, kAppendThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace sa
