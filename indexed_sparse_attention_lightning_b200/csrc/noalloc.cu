// noalloc.cu -- the fused decode for callers that cannot allocate device memory.
//
// sa_decode needs a caller-provided workspace.  Some callers cannot get one:
// code running under a host application or framework that owns every device
// allocation (a plugin, or a pool with a hard cap that this library may not
// grow), and latency-critical loops where a cudaMalloc -- which can
// synchronise the device -- is not allowed.  sa_decode_noalloc gives them the
// same path with its scratch in a statically sized device array owned by this
// library, so the call itself allocates nothing.
//
// Facts a caller must know:
//  - The array holds SA_NOALLOC_SCRATCH_BYTES on every device that loads this
//    library, for the life of the process.
//  - The first call on a device looks up the array's device address with that
//    device current (cudaGetSymbolAddress); make that first call before any
//    stream capture.  The address is remembered per device together with the
//    CUDA context it was taken in: after cudaDeviceReset the next call finds a
//    new context and looks the address up again.
//  - Every call on a device shares the one array and leaves its contents
//    behind; the call clears what must start at zero (the status word) itself.
//    Calls whose GPU work overlaps (e.g. on two streams without ordering)
//    race on the array and must not be issued.
//  - A request whose workspace would exceed the array is rejected with
//    SA_ERR_WORKSPACE before anything is launched.
//  - Bad data the kernels meet on the device (a page id, a query position, a
//    bounded wait that gave up) is recorded in the status word at the start of
//    the array, as sa_decode records it in its workspace; sa_noalloc_status
//    reads it back.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"
#include "sa.h"

namespace {

constexpr size_t kScratchBytes = SA_NOALLOC_SCRATCH_BYTES;

// The scratch itself.  In host code `g_scratch` only names the symbol; its
// device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 128;
std::mutex g_mutex;
void *g_device_addr[kMaxDevices];
CUcontext g_device_ctx[kMaxDevices];

// cuCtxGetCurrent through the driver entry point (no link-time dependency on
// libcuda), looked up once.
PFN_cuCtxGetCurrent_v4000 ctx_get_current() {
    static const PFN_cuCtxGetCurrent_v4000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        return static_cast<PFN_cuCtxGetCurrent_v4000>(nullptr);
    }();
    return fn;
}

// Device address of g_scratch on the current device, looked up once per
// device and context (a device reset replaces the context, and the module --
// with the array -- is loaded again at a possibly different address).
sa_status scratch_address(void **addr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SA_ERR_UNSUPPORTED;
    const PFN_cuCtxGetCurrent_v4000 get_ctx = ctx_get_current();
    if (get_ctx == nullptr) return SA_ERR_CUDA;
    // null until the runtime first uses this device in this thread
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return SA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (ctx == nullptr || g_device_addr[dev] == nullptr || g_device_ctx[dev] != ctx) {
        void *p = nullptr;  // the lookup also makes the device's context current
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr)
            return SA_ERR_CUDA;
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return SA_ERR_CUDA;
        g_device_addr[dev] = p;
        g_device_ctx[dev] = ctx;
    }
    *addr = g_device_addr[dev];
    return SA_OK;
}

}  // namespace

extern "C" sa_status sa_decode_noalloc(const sa_cache *cache, const sa_query *query,
                                       int32_t top_k, int32_t *idx_out, void *out,
                                       sa_dtype out_dtype, float *lse, void *stream) {
    const size_t need = sa_workspace_size(cache, query, top_k, SA_WS_DECODE);
    if (need > kScratchBytes) return SA_ERR_WORKSPACE;
    void *scratch = nullptr;
    sa_status st = scratch_address(&scratch);
    if (st != SA_OK) return st;
    // need == 0 means invalid arguments: sa_decode returns the precise code
    // before it touches the scratch.
    return sa_decode(cache, query, top_k, idx_out, out, out_dtype, lse, scratch, kScratchBytes,
                     stream);
}

extern "C" sa_status sa_noalloc_status(void *stream, int32_t *detail) {
    void *scratch = nullptr;
    const sa_status st = scratch_address(&scratch);
    if (st != SA_OK) return st;
    return sa_device_status(scratch, kScratchBytes, stream, detail);
}
