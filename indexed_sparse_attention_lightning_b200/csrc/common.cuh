// common.cuh -- device helpers shared by the sa kernels (storage formats,
// paged addressing, status reporting, order-preserving score keys).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sa.h"

namespace sa {

// ---------------------------------------------------------------------------
// Status word at the start of every workspace: {code, detail, spare...}.
// The first error wins; later ones are dropped.
// ---------------------------------------------------------------------------
constexpr size_t kStatusBytes = 256;

__device__ __forceinline__ void report(int32_t *status, int32_t code, int32_t detail) {
    if (status != nullptr && atomicCAS(status, 0, code) == 0) {
        atomicExch(status + 1, detail);
    }
}

// ---------------------------------------------------------------------------
// Storage formats
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Two e4m3 codes (low byte first) -> two floats, exact (every e4m3 value is a
// half value); uses the hardware conversion.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
    __half2 hh = *reinterpret_cast<__half2 *>(&h);
    return __half22float2(hh);
}

// E8M0 scale byte (OCP MX) -> its value 2^(b - 127), exactly; 255 is NaN.
__device__ __forceinline__ float e8m0_to_float(uint32_t b) {
    if (b == 255u) return __int_as_float(0x7FC00000);
    return b == 0u ? __int_as_float(0x00400000) : __int_as_float(static_cast<int>(b << 23));
}

// ---------------------------------------------------------------------------
// Order-preserving map float -> uint32: a > b as floats (no NaN) iff
// key(a) > key(b) as unsigned integers, and a == b iff the keys are equal.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;  // -0 and +0 compare equal, so they share a key
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Radix buckets of the score histogram built by the indexer for top-K: the
// top kHistBits bits of order_key().
constexpr int kHistBits = 12;
constexpr int kHistBins = 1 << kHistBits;

// ReLU that lets a NaN through, so a poisoned slot stays visible.
// max(x, 0) that keeps NaN (a poisoned key must not turn into a finite
// score): one max.NaN instruction instead of a compare and a select.
__device__ __forceinline__ float relu_keep_nan(float x) {
    float y;
    asm("max.NaN.f32 %0, %1, 0f00000000;" : "=f"(y) : "f"(x));
    return y;
}

// ---------------------------------------------------------------------------
// Paged addressing: physical row of logical position s of sequence seq, or -1
// when the page id is outside [0, num_pages) or the slot is past max_pages.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int64_t phys_row(const int32_t *page_table, int32_t max_pages,
                                            int32_t num_pages, int32_t seq, int64_t s) {
    int64_t slot = s >> 6;  // page size 64
    if (slot >= max_pages) return -1;
    int32_t page = __ldg(page_table + (int64_t)seq * max_pages + slot);
    if (page < 0 || page >= num_pages) return -1;
    return (int64_t)page * 64 + (s & 63);
}

// Programmatic dependent launch.  pdl_wait: block until the kernel before
// this one in the stream has completed and its writes are visible (a no-op
// when launched without the attribute).  pdl_trigger: let the next kernel in
// the stream start launching; its blocks still stop in their pdl_wait.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ constexpr int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

}  // namespace sa
