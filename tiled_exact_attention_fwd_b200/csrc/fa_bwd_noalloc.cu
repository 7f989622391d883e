// fa_bwd_noalloc.cu -- the fixed device buffer behind fa_bwd_noalloc: the backward pass's
// delta workspace (rowsum(dO * O), fp32, one value per (batch, head, row)) as a file-scope
// device array instead of a caller-owned buffer. Nothing here allocates: the array is part of
// this compilation unit's module image and its address is looked up once per device.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "fa_internal.h"

namespace fa {

static __device__ __align__(256) float g_bwd_delta_scratch[kNoallocDeltaFloats];

cudaError_t noalloc_delta_buffer(float **ptr) {
    static std::atomic<float *> addr[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    float *a = addr[dev].load(std::memory_order_acquire);
    if (!a) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_bwd_delta_scratch);  // loads this module on the device
        if (e != cudaSuccess) return e;
        a = static_cast<float *>(p);
        addr[dev].store(a, std::memory_order_release);
    }
    *ptr = a;
    return cudaSuccess;
}

}  // namespace fa
