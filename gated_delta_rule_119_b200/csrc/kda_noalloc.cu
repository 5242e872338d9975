// The fixed device scratch buffer behind kda_chunk_fwd_noalloc.  See include/kda.h.
//
// Some callers must not take device memory while a call runs.  A serving process may
// have reserved almost all of HBM for its state and KV caches at start-up, so that any
// further allocation can fail or evict; a runtime may need its device footprint fixed
// and known before the first request; a latency-critical host thread may have to stay
// clear of allocator state (pool growth, its locks, the synchronisation that a
// non-stream-ordered allocator can imply).  For such callers the tensor-core prefill
// takes its workspace from this buffer, which is part of the library's device image:
// the CUDA runtime reserves it on a device when it loads this module there, and no
// call allocates or frees it.
#include <mutex>

#include "../../include/kda.h"
#include "kda_common.cuh"

namespace {

constexpr int kMaxDevices = 64;

// One buffer per device.  Nothing in it has to start at zero: each call's kernels write
// every byte they later read.
static __device__ __align__(256) unsigned char g_kda_scratch[KDA_NOALLOC_SCRATCH_BYTES];

std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

}  // namespace

// Looks the buffer's address up once per device, with that device current (the
// caller's current device), and remembers it.
cudaError_t kda_noalloc_scratch(void **ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_kda_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = p;
    }
    *ptr = g_addr[dev];
    return cudaSuccess;
}
