// fa_padding.cu -- unpad (row gather) and pad (row scatter with zero fill) kernels.
//
// Page "IAW 模型 FA2 vs FA3 实测": section 1 describes the packed path -- unpad drops the
// padding tokens of a (B, total_len, H, D) tensor by taking rows by `indices`, pad puts
// the compact rows back by `indices`; section 2 shows pad as a zero fill followed by an
// index put. Here both are pure byte movement: one warp moves one row with 16-byte
// vectors (several loads in flight per lane), and pad writes every output row exactly
// once (copy when some index names it, zeros otherwise) instead of a fill plus a scatter;
// the index searches are done by whole warps (32 probes per dependent load).
#include <cuda_runtime.h>
#include <stdint.h>

#include "fa.h"
#include "fa_internal.h"

namespace fa {

static __device__ int g_pad_err_code;
static __device__ int g_pad_err_where;

__device__ __noinline__ void pad_record_error(int code, int where) {
    if (atomicCAS(&g_pad_err_code, 0, code) == 0) atomicExch(&g_pad_err_where, where);
}

template <typename T>
__device__ __forceinline__ T zero_of();
template <>
__device__ __forceinline__ uint4 zero_of<uint4>() { return make_uint4(0, 0, 0, 0); }
template <>
__device__ __forceinline__ uint8_t zero_of<uint8_t>() { return 0; }

template <typename T>
__device__ __forceinline__ T ld_stream(const T *p) { return __ldg(p); }

// Copy one row of `n` elements of T with the lanes of a warp, 4 vectors in flight per lane.
template <typename T>
__device__ __forceinline__ void warp_copy_row(const T *__restrict__ src, T *__restrict__ dst,
                                              int64_t n, int lane) {
    int64_t c = lane;
    for (; c + 96 < n; c += 128) {
        const T a = ld_stream(src + c), b = ld_stream(src + c + 32);
        const T d = ld_stream(src + c + 64), e = ld_stream(src + c + 96);
        dst[c] = a;
        dst[c + 32] = b;
        dst[c + 64] = d;
        dst[c + 96] = e;
    }
    for (; c < n; c += 32) dst[c] = ld_stream(src + c);
}

template <typename T>
__device__ __forceinline__ void warp_zero_row(T *__restrict__ dst, int64_t n, int lane) {
    const T z = zero_of<T>();
    for (int64_t c = lane; c < n; c += 32) dst[c] = z;
}

// out[r] = x[indices[r]]: one warp per compact row r, grid-stride over rows.
template <typename T>
__global__ void __launch_bounds__(256) unpad_kernel(const T *__restrict__ x, const int64_t *__restrict__ idx,
                                                    int64_t nnz, int64_t total_rows, int64_t per_row,
                                                    T *__restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t wpb = blockDim.x >> 5;
    const int64_t nw = gridDim.x * wpb;
    for (int64_t r = blockIdx.x * wpb + (threadIdx.x >> 5); r < nnz; r += nw) {
        const int64_t src = __ldg(idx + r);
        T *o = out + r * per_row;
        if (src < 0 || src >= total_rows) {
            warp_zero_row(o, per_row, lane);
            if (lane == 0) pad_record_error(FA_ERR_INDEX, 1);
            continue;
        }
        warp_copy_row(x + src * per_row, o, per_row, lane);
    }
}

// The three gathers of the packed path (q, k, v share one index list) in one launch: each
// warp moves row r of all three tensors, so three rows' loads are in flight together.
template <typename T>
__global__ void __launch_bounds__(256) unpad3_kernel(const T *__restrict__ x0, const T *__restrict__ x1,
                                                     const T *__restrict__ x2, const int64_t *__restrict__ idx,
                                                     int64_t nnz, int64_t total_rows, int64_t per_row,
                                                     T *__restrict__ o0, T *__restrict__ o1, T *__restrict__ o2) {
    const int lane = threadIdx.x & 31;
    const int64_t wpb = blockDim.x >> 5;
    const int64_t nw = gridDim.x * wpb;
    for (int64_t r = blockIdx.x * wpb + (threadIdx.x >> 5); r < nnz; r += nw) {
        const int64_t src = __ldg(idx + r);
        const int64_t dst = r * per_row;
        if (src < 0 || src >= total_rows) {
            warp_zero_row(o0 + dst, per_row, lane);
            warp_zero_row(o1 + dst, per_row, lane);
            warp_zero_row(o2 + dst, per_row, lane);
            if (lane == 0) pad_record_error(FA_ERR_INDEX, 3);
            continue;
        }
        const int64_t so = src * per_row;
        int64_t c = lane;
        for (; c + 32 < per_row; c += 64) {
            const T a0 = ld_stream(x0 + so + c), a1 = ld_stream(x1 + so + c), a2 = ld_stream(x2 + so + c);
            const T b0 = ld_stream(x0 + so + c + 32), b1 = ld_stream(x1 + so + c + 32), b2 = ld_stream(x2 + so + c + 32);
            o0[dst + c] = a0;
            o1[dst + c] = a1;
            o2[dst + c] = a2;
            o0[dst + c + 32] = b0;
            o1[dst + c + 32] = b1;
            o2[dst + c + 32] = b2;
        }
        for (; c < per_row; c += 32) {
            const T a0 = ld_stream(x0 + so + c), a1 = ld_stream(x1 + so + c), a2 = ld_stream(x2 + so + c);
            o0[dst + c] = a0;
            o1[dst + c] = a1;
            o2[dst + c] = a2;
        }
    }
}

// First position r in the sorted idx[0, nnz) with idx[r] >= key, found by the 32 lanes of a
// warp together: each round probes 32 evenly spaced entries at once, so the dependent-load
// chain is log32(nnz) long instead of log2(nnz).
__device__ __forceinline__ int64_t warp_lower_bound(const int64_t *__restrict__ idx, int64_t nnz, int64_t key,
                                                    int lane) {
    int64_t lo = 0, hi = nnz;  // answer in [lo, hi]
    while (hi - lo > 32) {
        const int64_t step = (hi - lo + 31) / 32;
        const int64_t p = lo + lane * step;
        const bool less = p < hi && __ldg(idx + p) < key;
        const int c = __popc(__ballot_sync(0xffffffffu, less));  // probes below key form a prefix
        const int64_t new_lo = (c == 0) ? lo : lo + (c - 1) * step + 1;
        hi = min(hi, lo + c * step);
        lo = new_lo;
    }
    const int64_t p = lo + lane;
    const bool less = p < hi && __ldg(idx + p) < key;
    return lo + __popc(__ballot_sync(0xffffffffu, less));
}

// Output rows [t0, t0 + 16) per block (8 warps, 2 rows each): copy x[r] if indices[r] == t for
// some r, zeros otherwise. With strictly increasing indices, the r of row t lies in
// [r0, r0 + (t - t0)] with r0 = lower_bound(indices, t0), so one 32-wide load of
// indices[r0 .. r0 + 31] answers every row of the block with a ballot (ROWS <= 32).
template <typename T>
__global__ void __launch_bounds__(256) pad_kernel(const T *__restrict__ x, const int64_t *__restrict__ idx,
                                                  int64_t nnz, int64_t total_rows, int64_t per_row,
                                                  T *__restrict__ out) {
    constexpr int ROWS = 16;
    const int lane = threadIdx.x & 31;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * ROWS;
    if (t0 >= total_rows) return;
    const int64_t r0 = warp_lower_bound(idx, nnz, t0, lane);
    const int64_t cand = (r0 + lane < nnz) ? __ldg(idx + r0 + lane) : -1;
    for (int k = threadIdx.x >> 5; k < ROWS; k += blockDim.x >> 5) {
        const int64_t t = t0 + k;
        if (t >= total_rows) break;
        const unsigned hit = __ballot_sync(0xffffffffu, cand == t);
        T *o = out + t * per_row;
        if (hit)
            warp_copy_row(x + (r0 + __ffs(hit) - 1) * per_row, o, per_row, lane);
        else
            warp_zero_row(o, per_row, lane);
    }
}

static int num_sms() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
            sms = n;
        else
            return 148;
    }
    return sms;
}

static bool vec16_ok(const void *a, const void *b, int64_t row_bytes) {
    return (row_bytes % 16) == 0 && (reinterpret_cast<uintptr_t>(a) % 16) == 0 &&
           (reinterpret_cast<uintptr_t>(b) % 16) == 0;
}

cudaError_t launch_unpad(const void *x, const int64_t *indices, int64_t nnz, int64_t total_rows,
                         int64_t row_bytes, void *out, cudaStream_t st) {
    if (nnz == 0) return cudaSuccess;
    const int64_t want = (nnz + 7) / 8;
    const int blocks = static_cast<int>(want < int64_t(num_sms()) * 8 ? want : int64_t(num_sms()) * 8);
    if (vec16_ok(x, out, row_bytes))
        unpad_kernel<uint4><<<blocks, 256, 0, st>>>(static_cast<const uint4 *>(x), indices, nnz, total_rows,
                                                    row_bytes / 16, static_cast<uint4 *>(out));
    else
        unpad_kernel<uint8_t><<<blocks, 256, 0, st>>>(static_cast<const uint8_t *>(x), indices, nnz,
                                                      total_rows, row_bytes, static_cast<uint8_t *>(out));
    return cudaGetLastError();
}

cudaError_t launch_unpad3(const void *const x[3], const int64_t *indices, int64_t nnz, int64_t total_rows,
                          int64_t row_bytes, void *const out[3], cudaStream_t st) {
    if (nnz == 0) return cudaSuccess;
    const int64_t want = (nnz + 7) / 8;
    const int blocks = static_cast<int>(want < int64_t(num_sms()) * 8 ? want : int64_t(num_sms()) * 8);
    bool vec = true;
    for (int i = 0; i < 3; ++i) vec = vec && vec16_ok(x[i], out[i], row_bytes);
    if (vec)
        unpad3_kernel<uint4><<<blocks, 256, 0, st>>>(
            static_cast<const uint4 *>(x[0]), static_cast<const uint4 *>(x[1]), static_cast<const uint4 *>(x[2]),
            indices, nnz, total_rows, row_bytes / 16, static_cast<uint4 *>(out[0]), static_cast<uint4 *>(out[1]),
            static_cast<uint4 *>(out[2]));
    else
        unpad3_kernel<uint8_t><<<blocks, 256, 0, st>>>(
            static_cast<const uint8_t *>(x[0]), static_cast<const uint8_t *>(x[1]), static_cast<const uint8_t *>(x[2]),
            indices, nnz, total_rows, row_bytes, static_cast<uint8_t *>(out[0]), static_cast<uint8_t *>(out[1]),
            static_cast<uint8_t *>(out[2]));
    return cudaGetLastError();
}

cudaError_t launch_pad(const void *x, const int64_t *indices, int64_t nnz, int64_t total_rows,
                       int64_t row_bytes, void *out, cudaStream_t st) {
    if (total_rows == 0) return cudaSuccess;
    const int64_t blocks = (total_rows + 15) / 16;
    if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
    if (vec16_ok(x ? x : out, out, row_bytes))
        pad_kernel<uint4><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
            static_cast<const uint4 *>(x), indices, nnz, total_rows, row_bytes / 16, static_cast<uint4 *>(out));
    else
        pad_kernel<uint8_t><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
            static_cast<const uint8_t *>(x), indices, nnz, total_rows, row_bytes, static_cast<uint8_t *>(out));
    return cudaGetLastError();
}

cudaError_t pad_error_addrs(int **code, int **where) {
    cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(code), g_pad_err_code);
    if (e != cudaSuccess) return e;
    return cudaGetSymbolAddress(reinterpret_cast<void **>(where), g_pad_err_where);
}

}  // namespace fa
