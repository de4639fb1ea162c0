// Stream-ordered scratch memory for the library's temporary buffers (query tables, gathered
// queries, the dense encoder's residual workspace).
//
// The buffers come from a memory pool the library owns, one per device, that keeps up to
// kScratchKeepBytes of freed memory across synchronisations: with the default pool (whose
// release threshold is 0) every synchronisation hands the memory back and the next call
// pays for a fresh device allocation.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "internal.h"

namespace tq {
namespace {

constexpr uint64_t kScratchKeepBytes = 1ull << 30;
std::mutex g_pool_mu;
cudaMemPool_t g_pools[kMaxDevices] = {};

}  // namespace

int scratch_alloc(void** p, size_t bytes, void* stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (int)e;
    if (dev < 0 || dev >= kMaxDevices) return (int)cudaErrorInvalidDevice;
    cudaMemPool_t pool = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_pool_mu);
        if (!g_pools[dev]) {
            cudaMemPoolProps props = {};
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            cudaMemPool_t created = nullptr;
            e = cudaMemPoolCreate(&created, &props);
            if (e != cudaSuccess) return (int)e;
            uint64_t keep = kScratchKeepBytes;
            e = cudaMemPoolSetAttribute(created, cudaMemPoolAttrReleaseThreshold, &keep);
            if (e != cudaSuccess) {
                cudaMemPoolDestroy(created);
                return (int)e;
            }
            g_pools[dev] = created;
        }
        pool = g_pools[dev];
    }
    return (int)cudaMallocFromPoolAsync(p, bytes, pool, (cudaStream_t)stream);
}

int scratch_free(void* p, void* stream) { return (int)cudaFreeAsync(p, (cudaStream_t)stream); }

}  // namespace tq
