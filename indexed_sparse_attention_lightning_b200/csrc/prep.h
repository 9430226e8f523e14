// prep.h -- launchers of the input-preparation kernels (prep.cu): FP8
// quantisation of the indexer query and the append of new tokens to the paged
// caches.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sa.h"

namespace sa {

// Rows of `d` values (bf16 or fp32) -> e4m3 codes + one fp32 scale per row.
cudaError_t launch_quantize_rows(const void *in, sa_dtype in_dtype, int64_t n_rows, int32_t d,
                                 uint8_t *codes, float *scales, cudaStream_t s);

// Everything the append kernel reads and writes.
struct AppendParams {
    // paging
    const int32_t *page_table;
    int32_t batch, max_pages, num_pages;
    // new tokens
    int32_t n_new;
    const int32_t *seq, *pos;
    int32_t in_bf16;  // 1: inputs are bf16, 0: fp32
    const void *k_new;  // [n_new, d_index] or null
    const void *kv_new;  // [n_new, d_latent + d_rope] or null
    // index key pool
    void *k_index;
    float *k_index_scale;
    int32_t d_index;
    int32_t index_dtype;  // sa_dtype of the pool
    // latent pool
    void *kv;
    void *kv_rope;
    float *kv_scale;
    int32_t d_latent, d_rope;
    int32_t kv_dtype;  // sa_dtype
    int32_t kv_scale_dims;  // e4m3: latent dims per scale (one token per scale)
    // status word
    int32_t *status;
};

cudaError_t launch_append(const AppendParams &p, cudaStream_t s);

}  // namespace sa
