// lmoe_forward_noalloc: the layer forward on a workspace that lives in the
// library itself, for callers that cannot call cudaMalloc.
//
// Some callers have no way to allocate device memory at the point where they
// run the layer: code recorded into a CUDA graph whose capture forbids
// allocation, an embedding runtime whose allocator is owned by someone else,
// or a hot path that must not take the allocator's locks.  For them this file
// reserves a fixed scratch area as a file-scope device array: the driver
// allocates it when the library's module is loaded on a device, and every GPU
// that loads the library keeps it until the process exits.
//
// Limits and rules:
//  - The area holds LMOE_NOALLOC_WORKSPACE_BYTES (64 MiB).  A call whose
//    lmoe_workspace_size(h, T) exceeds it returns LMOE_ERR_WORKSPACE and
//    launches nothing.
//  - In host code the array's name is only a host-side stand-in; its device
//    address is obtained once per device with cudaGetSymbolAddress, with that
//    device current, the first time the entry point runs there.  Make that
//    first call before any stream capture.
//  - Every call on a device shares the one area, and the area keeps whatever
//    the previous call left in it.  The forward resets the parts that must
//    start at zero (its status word and per-block expert counts) itself.
//    Calls that overlap on the GPU (different streams, or different handles on
//    the same device without ordering) race on the area: order them.
//  - The handle's device must be current (the area of another device would
//    hold none of its data); otherwise the call returns LMOE_ERR_INVALID_ARG.
//  - lmoe_check_device and lmoe_qb_histogram given a NULL workspace read the
//    area, so the status word and the router statistics of this entry point
//    stay reachable.
//  - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "lmoe_internal.cuh"

namespace {

constexpr size_t kNoallocBytes = LMOE_NOALLOC_WORKSPACE_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_workspace[kNoallocBytes];

std::mutex g_noalloc_mutex;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of the area on the current device (set up on first use).
lmoe_status noalloc_area(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return LMOE_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_workspace);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return LMOE_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return LMOE_OK;
}

}  // namespace

lmoe_status lmoe::noalloc_area_for(const lmoe_handle *h, void **area, size_t *bytes)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return lmoe::report_error(LMOE_ERR_CUDA, "cudaGetDevice failed");
    }
    if (dev != lmoe::handle_device(h))
        return lmoe::report_error(LMOE_ERR_INVALID_ARG,
                                  "the current device is not the one the handle was created on: make the "
                                  "handle's device current before using the built-in scratch area");
    const lmoe_status st = noalloc_area(area);
    if (st != LMOE_OK) return lmoe::report_error(st, "cudaGetSymbolAddress of the built-in scratch area failed");
    *bytes = kNoallocBytes;
    return LMOE_OK;
}

extern "C" lmoe_status lmoe_forward_noalloc(lmoe_handle *h, const void *x, int64_t T, void *output,
                                            int32_t *selected_experts, void *mixture_weights,
                                            void *latent_routed_aggregate, void *stream)
{
    if (!h) return lmoe::report_error(LMOE_ERR_INVALID_ARG, "handle is NULL");
    if (T < 0) return lmoe::report_error(LMOE_ERR_INVALID_ARG, "T < 0");
    if (T == 0) return LMOE_OK;
    size_t need = 0;
    lmoe_status st = lmoe_workspace_size(h, T, &need);
    if (st != LMOE_OK) return st;
    if (need > kNoallocBytes)
        return lmoe::report_error(LMOE_ERR_WORKSPACE,
                                  "T tokens need more scratch than the built-in area of LMOE_NOALLOC_WORKSPACE_BYTES "
                                  "(64 MiB): use lmoe_forward with a caller workspace, or fewer tokens per call");
    void *area = nullptr;
    size_t area_bytes = 0;
    st = lmoe::noalloc_area_for(h, &area, &area_bytes);
    if (st != LMOE_OK) return st;
    return lmoe_forward(h, x, T, output, selected_experts, mixture_weights, latent_routed_aggregate, area,
                        kNoallocBytes, stream);
}
