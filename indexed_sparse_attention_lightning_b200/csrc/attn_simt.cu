// attn_simt.cu -- CUDA-core sparse MLA attention for any shape.
//
// For query t and head h, over the selected rows s of the latent cache
// ("Optimizing Next-Gen LLM Inference" §3.3: attention on the selected
// positions only, reading the cache by index):
//     z_s = sm_scale * q[t,h,:] . kv[s,:],   out = sum_s softmax(z)_s kv[s,0:dl]
// An e4m3 latent is dequantised with its page-tile scale while it is staged
// ("Optimizing Next-Gen LLM Inference" §4: dequantisation fused into attention,
// no dequantised cache is materialised).  Rows are staged through shared
// memory 32 at a time and shared by a group of heads; softmax is online in
// fp32.  This kernel serves the small fp32 configuration and shapes the
// tensor-core kernel does not take.
#include "common.cuh"
#include "internal.h"

namespace sa {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 32;     // rows staged per step
constexpr int kMaxOut = 2;    // output columns per thread: d_latent <= 512

__device__ __forceinline__ float load_q(const PathParams &p, int64_t i) {
    if (p.q_dtype == SA_BF16) return bf16_bits_to_float(static_cast<const uint16_t *>(p.q)[i]);
    return static_cast<const float *>(p.q)[i];
}

__device__ __forceinline__ float load_kv(const PathParams &p, int64_t row, int dd) {
    const int D = p.d_latent + p.d_rope;
    switch (p.kv_dtype) {
    case SA_F32: return static_cast<const float *>(p.kv)[row * D + dd];
    case SA_BF16: return bf16_bits_to_float(static_cast<const uint16_t *>(p.kv)[row * D + dd]);
    default:
        if (dd < p.d_latent) {
            uint8_t c = static_cast<const uint8_t *>(p.kv)[row * p.d_latent + dd];
            return e4m3x2_to_float2(c).x * kv_scale_at(p, row, dd);
        }
        return bf16_bits_to_float(
            static_cast<const uint16_t *>(p.kv_rope)[row * p.d_rope + (dd - p.d_latent)]);
    }
}

template <int HG>
__global__ void __launch_bounds__(kThreads)
attn_simt_kernel(const PathParams p, const int32_t *__restrict__ idx, int32_t K, void *out,
                 int32_t out_dtype, float *__restrict__ lse) {
    pdl_wait();
    pdl_trigger();
    extern __shared__ float smem[];
    const int D = p.d_latent + p.d_rope, dl = p.d_latent, ldr = D + 1;
    float *q_s = smem;                      // [HG][D]
    float *rows_s = q_s + HG * D;           // [kRows][D + 1]
    float *p_s = rows_s + kRows * ldr;      // [HG][kRows]
    float *m_s = p_s + HG * kRows;          // [HG]
    float *l_s = m_s + HG;                  // [HG]
    float *corr_s = l_s + HG;               // [HG]
    int64_t *row_s = reinterpret_cast<int64_t *>(
        (reinterpret_cast<uintptr_t>(corr_s + HG) + 7) & ~static_cast<uintptr_t>(7));  // [kRows]

    const int t = blockIdx.y, h0 = blockIdx.x * HG, tid = threadIdx.x;
    const int32_t V = visible_len(p, t);
    const int32_t seq = p.q_seq[t];

    for (int i = tid; i < HG * D; i += kThreads)
        q_s[i] = load_q(p, ((int64_t)t * p.heads + h0) * D + i);
    if (tid < HG) {
        m_s[tid] = -INFINITY;
        l_s[tid] = 0.f;
    }
    float acc[HG][kMaxOut];
#pragma unroll
    for (int h = 0; h < HG; ++h)
#pragma unroll
        for (int c = 0; c < kMaxOut; ++c) acc[h][c] = 0.f;
    __syncthreads();

    for (int k0 = 0; k0 < K; k0 += kRows) {
        if (tid < kRows) {
            int64_t row = -1;
            if (k0 + tid < K) {
                int32_t s = idx[(int64_t)t * K + k0 + tid];
                if (s >= V) {
                    report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_INDEX);
                } else if (s >= 0) {
                    row = phys_row(p.page_table, p.max_pages, p.num_pages, seq, s);
                    if (row < 0) report(p.status, SA_ERR_DEVICE_FAULT, SA_DETAIL_BAD_PAGE);
                }
            }
            row_s[tid] = row;
        }
        __syncthreads();
        for (int e = tid; e < kRows * D; e += kThreads) {
            const int r = e / D, dd = e - r * D;
            const int64_t row = row_s[r];
            rows_s[r * ldr + dd] = row >= 0 ? load_kv(p, row, dd) : 0.f;
        }
        __syncthreads();
        for (int pr = tid; pr < HG * kRows; pr += kThreads) {
            const int h = pr / kRows, r = pr - h * kRows;
            float z = -INFINITY;
            if (row_s[r] >= 0) {
                float dot = 0.f;
                const float *qh = q_s + h * D, *kr = rows_s + r * ldr;
                for (int dd = 0; dd < D; ++dd) dot = fmaf(qh[dd], kr[dd], dot);
                z = p.sm_scale * dot;
            }
            p_s[h * kRows + r] = z;
        }
        __syncthreads();
        if (tid < HG) {
            float *z = p_s + tid * kRows;
            float m_old = m_s[tid], m_new = m_old;
            for (int r = 0; r < kRows; ++r) m_new = fmaxf(m_new, z[r]);
            float corr = 1.f, sum = 0.f;
            if (m_new != -INFINITY) {
                corr = __expf(m_old - m_new);  // m_old == -inf gives 0
                for (int r = 0; r < kRows; ++r) {
                    float e = z[r] == -INFINITY ? 0.f : __expf(z[r] - m_new);
                    z[r] = e;
                    sum += e;
                }
            } else {
                for (int r = 0; r < kRows; ++r) z[r] = 0.f;
            }
            l_s[tid] = l_s[tid] * corr + sum;
            m_s[tid] = m_new;
            corr_s[tid] = corr;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < kMaxOut; ++c) {
            const int dv = tid + c * kThreads;
            if (dv < dl) {
#pragma unroll
                for (int h = 0; h < HG; ++h) {
                    float a = acc[h][c] * corr_s[h];
                    for (int r = 0; r < kRows; ++r) a = fmaf(p_s[h * kRows + r], rows_s[r * ldr + dv], a);
                    acc[h][c] = a;
                }
            }
        }
        __syncthreads();
    }

#pragma unroll
    for (int c = 0; c < kMaxOut; ++c) {
        const int dv = tid + c * kThreads;
        if (dv < dl) {
#pragma unroll
            for (int h = 0; h < HG; ++h) {
                const float l = l_s[h];
                const float v = l > 0.f ? acc[h][c] / l : 0.f;
                const int64_t o = ((int64_t)t * p.heads + h0 + h) * dl + dv;
                if (out_dtype == SA_BF16)
                    static_cast<__nv_bfloat16 *>(out)[o] = __float2bfloat16_rn(v);
                else
                    static_cast<float *>(out)[o] = v;
            }
        }
    }
    if (lse != nullptr && tid < HG) {
        const float l = l_s[tid];
        lse[(int64_t)t * p.heads + h0 + tid] = l > 0.f ? m_s[tid] + logf(l) : -INFINITY;
    }
}

template <int HG>
cudaError_t launch_hg(const PathParams &p, const int32_t *idx, int32_t K, void *out,
                      int32_t out_dtype, float *lse, cudaStream_t s) {
    const int D = p.d_latent + p.d_rope;
    size_t smem = sizeof(float) * ((size_t)HG * D + (size_t)kRows * (D + 1) + HG * kRows + 4 * HG) +
                  sizeof(int64_t) * (kRows + 2);
    const cudaError_t e = cudaFuncSetAttribute(
        attn_simt_kernel<HG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.heads / HG, p.n_q);
    count_launch();
    return launch_pdl(attn_simt_kernel<HG>, grid, dim3(kThreads), smem, s, p, idx, K, out,
                      out_dtype, lse);
}

}  // namespace

cudaError_t launch_attn_simt(const PathParams &p, const int32_t *idx, int32_t top_k, void *out,
                             int32_t out_dtype, float *lse, cudaStream_t s) {
    if (p.n_q == 0) return cudaSuccess;
    if (p.heads % 16 == 0) return launch_hg<16>(p, idx, top_k, out, out_dtype, lse, s);
    if (p.heads % 4 == 0) return launch_hg<4>(p, idx, top_k, out, out_dtype, lse, s);
    return launch_hg<1>(p, idx, top_k, out, out_dtype, lse, s);
}

}  // namespace sa
