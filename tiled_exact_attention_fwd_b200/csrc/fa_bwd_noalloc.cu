// fa_bwd_noalloc.cu -- the fixed device buffer behind fa_bwd_noalloc: the backward pass's
// delta workspace (rowsum(dO * O), fp32, one value per (batch, head, row)) as a file-scope
// device array instead of a caller-owned buffer. Nothing here allocates: the array is part of
// this compilation unit's module image, present on every device that loads the library until
// the process exits.
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa_internal.h"

namespace fa {

static __device__ __align__(256) float g_bwd_delta_scratch[kNoallocDeltaFloats];

// In host code the array's name only stands for the symbol; its device address on the
// current device comes from the runtime. The lookup runs on every call: the first one on a
// device loads this module there, later ones are a table lookup, and a context that was
// reset and created again gets its new address instead of a stale one.
cudaError_t noalloc_delta_buffer(float **ptr) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_bwd_delta_scratch);
    if (e != cudaSuccess) return e;
    *ptr = static_cast<float *>(p);
    return cudaSuccess;
}

}  // namespace fa
