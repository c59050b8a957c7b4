// launch_cache.cu -- per-device launch facts of the kernels (host code): the dynamic shared-memory attribute and
// the resident-CTA grid of the persistent kernels.
#include "kernels.h"

namespace gdr {

cudaError_t LaunchCache::allow_smem(int smem) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool rec = dev >= 0 && dev < kMaxDevices;
    std::lock_guard<std::mutex> lock(mu_);
    if (rec && smem <= smem_[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(func_, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess && rec) smem_[dev] = smem;
    return e;
}

cudaError_t LaunchCache::resident_grid(int threads, int smem, int *grid) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool rec = dev >= 0 && dev < kMaxDevices;
    const int key = (threads << 20) | smem;  // threads <= 1024 and smem < 1 MB
    std::lock_guard<std::mutex> lock(mu_);
    if (rec && grid_key_[dev] == key) {
        *grid = grid_[dev];
        return cudaSuccess;
    }
    int nsm = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, func_, threads, (size_t)smem);
    if (e != cudaSuccess) return e;
    const int g = nsm * (per_sm > 0 ? per_sm : 1);
    *grid = g > 0 ? g : 1;
    if (rec) {
        grid_key_[dev] = key;
        grid_[dev] = *grid;
    }
    return cudaSuccess;
}

}  // namespace gdr
