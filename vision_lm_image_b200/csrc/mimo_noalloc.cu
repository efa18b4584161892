// mimo_noalloc.cu -- the fixed device staging area behind
// mimo_preprocess_batch_host_noalloc (include/mimo.h).
//
// Some callers cannot allocate device memory at all: code running where the
// device allocator is owned by someone else (a host application that hands
// the GPU to a framework with its own pool), or where an allocation may not
// happen at that point in time. For them the host-to-host path can stage its
// images and rows in this statically sized array instead of caller-provided
// buffers. The array belongs to the library image: every GPU that loads the
// library holds MIMO_NOALLOC_STAGING_BYTES of it until the process exits.
#include <cuda_runtime.h>

#include <mutex>

#include "mimo.h"
#include "mimo_internal.h"

namespace mimo {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_stage[MIMO_NOALLOC_STAGING_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_stage_ptr[kMaxDevices] = {};

}  // namespace

// Device address of the staging array on the current device. In host code
// the array's name is only a host-side handle, so the address is looked up
// once per device, with that device current, and kept for later calls.
int noalloc_staging(void **dev_ptr, size_t *bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MIMO_ECUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_stage_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_stage) != cudaSuccess || p == nullptr) return MIMO_ECUDA;
        g_stage_ptr[dev] = p;
    }
    *dev_ptr = g_stage_ptr[dev];
    *bytes = MIMO_NOALLOC_STAGING_BYTES;
    return MIMO_OK;
}

}  // namespace mimo
