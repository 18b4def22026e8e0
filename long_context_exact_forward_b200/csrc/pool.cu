// pool.cu -- scratch memory of the entry points that allocate (no caller workspace).
//
// Those entry points allocate stream-ordered and free at the end of the call.  From the device's
// default memory pool, whose release threshold is 0, that memory may go back to the driver at every
// synchronisation and be mapped anew by the next call -- for the zigzag layout 3 x B*S*H*D bf16
// (3.2 GB on the 128K-token workload) per call.  The library therefore allocates from a pool of its
// own, one per device, whose release threshold is the largest value: what a call frees stays
// reserved in the process for the next call, and other users of the default pool are unaffected.
// A stream that is being captured into a CUDA graph allocates from the default pool as before
// (graph memory nodes belong to the graph).
#include <cuda_runtime.h>

#include <map>
#include <mutex>

#include "ra_internal.cuh"

namespace ra {

cudaError_t scratch_alloc(void** ptr, size_t bytes, cudaStream_t stream) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return e;
    if (cap != cudaStreamCaptureStatusNone) return cudaMallocAsync(ptr, bytes, stream);
    static std::mutex mu;
    static std::map<int, cudaMemPool_t> pools;
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    cudaMemPool_t pool = nullptr;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = pools.find(dev);
        if (it == pools.end()) {
            cudaMemPoolProps props{};
            props.allocType = cudaMemAllocationTypePinned;
            props.location.type = cudaMemLocationTypeDevice;
            props.location.id = dev;
            if ((e = cudaMemPoolCreate(&pool, &props)) != cudaSuccess) return e;
            uint64_t keep = ~uint64_t(0);
            if ((e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep)) != cudaSuccess) {
                cudaMemPoolDestroy(pool);
                return e;
            }
            it = pools.emplace(dev, pool).first;
        }
        pool = it->second;
    }
    return cudaMallocFromPoolAsync(ptr, bytes, pool, stream);
}

}  // namespace ra
