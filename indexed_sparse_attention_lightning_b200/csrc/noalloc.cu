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
//    stream capture.
//  - Every call on a device shares the one array and leaves its contents
//    behind; the call clears what must start at zero (the status word) itself.
//    Calls whose GPU work overlaps (e.g. on two streams without ordering)
//    race on the array and must not be issued.
//  - A request whose workspace would exceed the array is rejected with
//    SA_ERR_WORKSPACE before anything is launched.
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

// Device address of g_scratch on the current device, looked up once per device.
sa_status scratch_address(void **addr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_device_addr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr)
            return SA_ERR_CUDA;
        g_device_addr[dev] = p;
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
