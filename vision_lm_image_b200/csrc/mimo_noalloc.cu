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

#include "mimo.h"
#include "mimo_internal.h"

namespace mimo {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_stage[MIMO_NOALLOC_STAGING_BYTES];

}  // namespace

// Device address of the staging array in the current device's context. In
// host code the array's name is only a host-side handle, so the address is
// looked up with the device current. It is looked up on every call rather
// than cached: a cudaDeviceReset or a new primary context loads the module
// again, and the array can then sit at another address. The lookup is a
// runtime table query, small beside the copies of a call.
int noalloc_staging(void **dev_ptr, size_t *bytes) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_stage) != cudaSuccess || p == nullptr) return MIMO_ECUDA;
    *dev_ptr = p;
    *bytes = MIMO_NOALLOC_STAGING_BYTES;
    return MIMO_OK;
}

}  // namespace mimo
