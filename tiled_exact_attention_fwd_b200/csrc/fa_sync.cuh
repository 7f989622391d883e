// fa_sync.cuh -- the device error word and the bounded mbarrier wait shared by the kernels.
// Each compilation unit that includes this header gets its own error word (static device
// variables); device_error_addrs gives its device addresses, which the status query reads
// and clears on the caller's stream.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa.h"
#include "fa_ptx.cuh"

namespace fa {

static __device__ int g_err_code;
static __device__ int g_err_where;

static __device__ __noinline__ void record_error(int code, int where) {
    if (atomicCAS(&g_err_code, 0, code) == 0) atomicExch(&g_err_where, where);
}

// Wait for phase `parity` of `bar`, giving up after limit_ns or when another role aborted.
__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                             uint64_t limit_ns, int where) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
#pragma unroll 1
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                record_error(FA_ERR_TIMEOUT, where);
                return false;
            }
        }
    }
}

// The same with cluster-scope acquire, for barriers that the other CTA of a pair (its threads
// or its MMA commits) completes.
__device__ __forceinline__ bool wait_bounded_cluster(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                     uint64_t limit_ns, int where) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
#pragma unroll 1
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if ((it & 31u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                record_error(FA_ERR_TIMEOUT, where);
                return false;
            }
        }
    }
}

// Device addresses (on the current device) of this compilation unit's error word.
static cudaError_t device_error_addrs(int **code, int **where) {
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(code), g_err_code);
    if (e != cudaSuccess) return e;
    return cudaGetSymbolAddress(reinterpret_cast<void **>(where), g_err_where);
}

}  // namespace fa
