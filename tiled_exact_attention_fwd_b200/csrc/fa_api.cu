// fa_api.cu -- the C ABI declared in include/fa.h: argument validation, TMA tensor-map
// encoding and kernel dispatch. No entry point allocates, synchronises (except
// fa_device_status, which waits for the caller's stream) or touches host copies of tensor
// data.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include <atomic>

#include "fa.h"
#include "fa_internal.h"

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load(std::memory_order_acquire);
    if (!f) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess && p) {
            f = reinterpret_cast<EncodeTiledFn>(p);
            fn.store(f, std::memory_order_release);
        }
    }
    return f;
}

uint64_t wait_limit_ns() {
    static std::atomic<uint64_t> lim{0};
    uint64_t v = lim.load(std::memory_order_relaxed);
    if (v == 0) {
        v = 2000000000ull;  // 2 s: every wait inside a CTA normally lasts microseconds
        if (const char *e = getenv("FA_WAIT_LIMIT_NS")) {
            const unsigned long long x = strtoull(e, nullptr, 10);
            if (x > 0) v = x;
        }
        lim.store(v, std::memory_order_relaxed);
    }
    return v;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Streaming multiprocessors of the current device (looked up once per device).
int sm_count() {
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return -1;
    if (dev >= 64) {
        int n = 0;
        return cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? n : -1;
    }
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return -1;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

bool head_dim_ok(int D) { return D == 32 || D == 64 || D == 128 || D == 256; }

// Token-major (N, H, D) 16-bit tensor seen by TMA as dims (D, H, N); one box is
// `inner` elements of one head of `rows` consecutive tokens (a [rows][inner] tile).
bool encode_map(CUtensorMap *m, const void *base, bool bf16, int D, int H, int64_t N, int inner, int rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                                static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(inner), 1, static_cast<cuuint32_t>(rows)};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapSwizzle sw = (inner * 2 == 128) ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const CUresult r = f(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                         const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct Paging {
    const int32_t *block_table;
    int max_blocks, page_size, num_pages;
};

fa_status run_fwd(const void *q, const void *k, const void *v, void *out, float *lse,
                  const int32_t *cu_seqlens, int num_seqs, int seqlen, int64_t N, int H, int D,
                  float scale, int causal, fa_dtype dtype, void *stream,
                  const int64_t *gather = nullptr, int64_t padded_rows = 0, const Paging *paging = nullptr) {
    const bool bf16 = dtype == FA_BF16;
    const int inner = fa::fwd_box_inner_elems(D);
    CUtensorMap tq, tk, tv;
    // fused path: maps over the padded tensors with 32-row boxes (one box per run of 32
    // consecutive padded rows; other rows are copied by threads)
    const int64_t map_rows = gather ? padded_rows : N;
    const int64_t kv_rows = paging ? static_cast<int64_t>(paging->num_pages) * paging->page_size : map_rows;
    const int q_box = gather ? fa::fwd_gather_run_rows() : fa::fwd_tile_rows();
    // dense D = 256 runs in CTA pairs: each CTA loads 64 key rows of K_j and 128 columns of V_j
    const bool pair = fa::fwd_pair_mode(D) && !paging && !cu_seqlens;
    const int k_box = paging ? fa::fwd_paged_k_box_rows(D, paging->page_size)
                             : (gather ? fa::fwd_gather_run_rows() : (pair ? 64 : fa::fwd_kv_tile_rows(D)));
    const int v_box = paging ? fa::fwd_paged_v_box_rows(D, paging->page_size)
                             : (gather ? fa::fwd_gather_run_rows() : (pair ? 128 : fa::fwd_v_box_rows(D)));
    if (!encode_map(&tq, q, bf16, D, H, map_rows, inner, q_box) ||
        !encode_map(&tk, k, bf16, D, H, kv_rows, inner, k_box) ||
        !encode_map(&tv, v, bf16, D, H, kv_rows, inner, v_box))
        return FA_ERR_CUDA;
    if (!(scale > 0.f)) scale = 1.0f / sqrtf(static_cast<float>(D));
    fa::FwdParams p;
    p.queue = nullptr;  // set by the launcher where the item queue applies
    p.out = out;
    p.lse = lse;
    p.cu_seqlens = cu_seqlens;
    p.num_seqs = num_seqs;
    p.gather = gather;
    p.padded_rows = padded_rows;
    p.q = q;
    p.k = k;
    p.v = v;
    p.seqlen = seqlen;
    p.H = H;
    p.total_tokens = static_cast<int>(N);
    p.scale_log2 = scale * 1.4426950408889634f;
    p.timeout_ns = wait_limit_ns();
    p.block_table = paging ? paging->block_table : nullptr;
    p.max_blocks = paging ? paging->max_blocks : 0;
    p.page_size = paging ? paging->page_size : 0;
    p.page_shift = 0;
    while (paging && (1 << p.page_shift) < paging->page_size) ++p.page_shift;
    p.num_pages = paging ? paging->num_pages : 0;
    const int rows = fa::fwd_tile_rows();
    dim3 grid;
    p.batch = num_seqs;
    p.out_align32 = (reinterpret_cast<uintptr_t>(out) % 32) == 0;
    p.npairs = 0;
    p.num_items = 0;
    p.head_group = p.num_groups = p.group_rounds = 0;
    if (cu_seqlens) {
        // packed: one CTA per tiles_per_cta x 128 consecutive tokens of the packed tensor
        const int64_t span = static_cast<int64_t>(rows) * fa::fwd_tiles_per_cta(D);
        grid = dim3(static_cast<unsigned>(H), static_cast<unsigned>((N + span - 1) / span), 1);
    } else {
        // dense: persistent, one CTA per SM (at most one per work item)
        const int qtiles = (seqlen + rows - 1) / rows;
        const int per_cta = pair ? 2 : fa::fwd_tiles_per_cta(D);  // query tiles per work item
        p.npairs = (qtiles + per_cta - 1) / per_cta;
        const int64_t items = static_cast<int64_t>(num_seqs) * H * p.npairs;
        if (items > INT32_MAX) return FA_ERR_SHAPE;
        p.num_items = static_cast<int>(items);
        const int sms = sm_count();
        if (sms <= 0) return FA_ERR_CUDA;
        if (pair) {
            const int clusters = sms / 2;  // CTA pairs: one cluster of two per two SMs
            grid = dim3(2u * static_cast<unsigned>(p.num_items < clusters ? p.num_items : clusters), 1, 1);
        } else {
            grid = dim3(static_cast<unsigned>(p.num_items < sms ? p.num_items : sms), 1, 1);
        }
        // Causal items run longest first across all heads; when the K/V of all (batch entry,
        // head) pairs exceeds 64 MB (half of L2), they are dealt in groups of heads whose K/V
        // takes ~32 MB, each group at least 1.5 rounds of the grid (so the rounds stay balanced).
        const int bh = num_seqs * H, G = static_cast<int>(pair ? grid.x / 2 : grid.x);
        int hg = bh;
        const double per_bh = static_cast<double>(seqlen) * D * 4.0;  // K and V bytes of one pair
        if (causal && !pair && per_bh * bh > 64.0 * 1024 * 1024) {
            hg = static_cast<int>(32.0 * 1024 * 1024 / per_bh);
            if (hg < 1) hg = 1;
            while (hg < bh && 2LL * hg * p.npairs < 3LL * G) hg *= 2;
            if (hg > bh) hg = bh;
        }
        p.head_group = hg;
        p.num_groups = (bh + hg - 1) / hg;
        p.group_rounds = static_cast<int>((static_cast<int64_t>(hg) * p.npairs + G - 1) / G);
    }
    const cudaError_t e = paging ? fa::launch_fwd_paged(D, bf16, causal != 0, tq, tk, tv, p, grid,
                                                        static_cast<cudaStream_t>(stream))
                                 : fa::launch_fwd(D, bf16, causal != 0, tq, tk, tv, p, grid,
                                                  static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

fa_status fa_fwd(const void *q, const void *k, const void *v, void *out, float *lse, int B, int H, int S,
                 int D, float scale, int causal, fa_dtype dtype, void *stream) {
    if (!q || !k || !v || !out) return FA_ERR_NULL;
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (!head_dim_ok(D)) return FA_ERR_HEADDIM;
    if (B <= 0 || H <= 0 || S <= 0) return FA_ERR_SHAPE;
    const int64_t N = static_cast<int64_t>(B) * S;
    if (N > INT32_MAX || B > 65535 || (S + 127) / 128 > 65535) return FA_ERR_SHAPE;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4))
        return FA_ERR_ALIGN;
    return run_fwd(q, k, v, out, lse, nullptr, B, S, N, H, D, scale, causal, dtype, stream);
}

fa_status fa_fwd_paged(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
                       int max_blocks_per_seq, int page_size, int num_pages, void *out, float *lse, int B, int H,
                       int S, int D, float scale, int causal, fa_dtype dtype, void *stream) {
    if (!q || !k_cache || !v_cache || !block_table || !out) return FA_ERR_NULL;
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (!head_dim_ok(D)) return FA_ERR_HEADDIM;
    if (B <= 0 || H <= 0 || S <= 0 || num_pages <= 0 || max_blocks_per_seq <= 0) return FA_ERR_SHAPE;
    // a power of two of at least 16 rows: a page is a whole number of 16-row boxes, and a
    // 128-row key tile either holds whole pages or lies inside one
    if (page_size < 16 || page_size > (1 << 20) || (page_size & (page_size - 1)) != 0) return FA_ERR_SHAPE;
    if (static_cast<int64_t>(max_blocks_per_seq) * page_size < S) return FA_ERR_SHAPE;
    if (static_cast<int64_t>(num_pages) * page_size > INT32_MAX) return FA_ERR_SHAPE;
    const int64_t N = static_cast<int64_t>(B) * S;
    if (N > INT32_MAX || B > 65535 || (S + 127) / 128 > 65535) return FA_ERR_SHAPE;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
        !aligned(lse, 4) || !aligned(block_table, 4))
        return FA_ERR_ALIGN;
    const Paging paging{block_table, max_blocks_per_seq, page_size, num_pages};
    return run_fwd(q, k_cache, v_cache, out, lse, nullptr, B, S, N, H, D, scale, causal, dtype, stream, nullptr, 0,
                   &paging);
}

}  // extern "C"

namespace {

// Shared by the dense and packed backward entry points: N token rows; cu_seqlens null for
// dense (B sequences of S) or the packed offsets (B = 1, S = N).
fa_status run_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
                  void *dq, void *dk, void *dv, float *delta, const int32_t *cu_seqlens, int num_seqs, int B, int H,
                  int S, int D, float scale, int causal, fa_dtype dtype, void *stream) {
    const int64_t N = static_cast<int64_t>(B) * S;
    const bool bf16 = dtype == FA_BF16;
    const int inner = fa::fwd_box_inner_elems(D);
    CUtensorMap tq, tk, tv, tdo;
    const int box_rows = (D == 256) ? 64 : 128;  // D = 256 streams 64-row half tiles
    if (!encode_map(&tq, q, bf16, D, H, N, inner, box_rows) || !encode_map(&tk, k, bf16, D, H, N, inner, box_rows) ||
        !encode_map(&tv, v, bf16, D, H, N, inner, box_rows) || !encode_map(&tdo, dout, bf16, D, H, N, inner, box_rows))
        return FA_ERR_CUDA;
    if (!(scale > 0.f)) scale = 1.0f / sqrtf(static_cast<float>(D));
    fa::BwdParams p;
    p.out = out;
    p.dout = dout;
    p.lse = lse;
    p.delta = delta;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.B = B;
    p.H = H;
    p.seqlen = S;
    p.cu_seqlens = cu_seqlens;
    p.num_seqs = num_seqs;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.timeout_ns = wait_limit_ns();
    const cudaError_t e = fa::launch_bwd(D, bf16, causal != 0, tq, tk, tv, tdo, p, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

bool bwd_aligned(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
                 const void *dq, const void *dk, const void *dv, const float *delta) {
    return aligned(q, 16) && aligned(k, 16) && aligned(v, 16) && aligned(out, 16) && aligned(dout, 16) &&
           aligned(dq, 16) && aligned(dk, 16) && aligned(dv, 16) && aligned(lse, 4) && aligned(delta, 4);
}

// The error words of the kernel families (one per compilation unit), read and cleared in one
// launch on the caller's stream; the first nonzero code wins.
constexpr int kErrorWords = 5;
struct ErrorWords {
    int *code[kErrorWords];
    int *where[kErrorWords];
};

__device__ int g_status_out[2];

__global__ void status_collect_kernel(ErrorWords w) {
    int code = 0, where = 0;
    for (int i = 0; i < kErrorWords; ++i) {
        const int c = atomicExch(w.code[i], 0), wh = atomicExch(w.where[i], 0);
        if (c != 0 && code == 0) {
            code = c;
            where = wh;
        }
    }
    g_status_out[0] = code;
    g_status_out[1] = where;
}

}  // namespace

extern "C" {

fa_status fa_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout, const float *lse,
                 void *dq, void *dk, void *dv, float *delta, int B, int H, int S, int D, float scale, int causal,
                 fa_dtype dtype, void *stream) {
    if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !delta) return FA_ERR_NULL;
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (!head_dim_ok(D)) return FA_ERR_HEADDIM;
    if (B <= 0 || H <= 0 || S <= 0) return FA_ERR_SHAPE;
    const int64_t N = static_cast<int64_t>(B) * S;
    if (N > INT32_MAX || B > 65535 || (S + 127) / 128 > 65535) return FA_ERR_SHAPE;
    if (!bwd_aligned(q, k, v, out, dout, lse, dq, dk, dv, delta)) return FA_ERR_ALIGN;
    return run_bwd(q, k, v, out, dout, lse, dq, dk, dv, delta, nullptr, 0, B, H, S, D, scale, causal, dtype, stream);
}

fa_status fa_varlen_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout,
                        const float *lse, const int32_t *cu_seqlens, int num_seqs, int max_seqlen, int total,
                        void *dq, void *dk, void *dv, float *delta, int H, int D, float scale, int causal,
                        fa_dtype dtype, void *stream) {
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (!head_dim_ok(D)) return FA_ERR_HEADDIM;
    if (num_seqs < 0 || total < 0 || max_seqlen < 0 || H <= 0) return FA_ERR_SHAPE;
    if (total == 0 || num_seqs == 0) return FA_OK;  // no rows, nothing to launch
    if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !delta || !cu_seqlens) return FA_ERR_NULL;
    if (max_seqlen == 0) return FA_ERR_SHAPE;
    if ((static_cast<int64_t>(total) + 127) / 128 > 65535) return FA_ERR_SHAPE;
    if (!bwd_aligned(q, k, v, out, dout, lse, dq, dk, dv, delta) || !aligned(cu_seqlens, 4)) return FA_ERR_ALIGN;
    return run_bwd(q, k, v, out, dout, lse, dq, dk, dv, delta, cu_seqlens, num_seqs, 1, H, total, D, scale, causal,
                   dtype, stream);
}

fa_status fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *out, const void *dout,
                         const float *lse, void *dq, void *dk, void *dv, int B, int H, int S, int D, float scale,
                         int causal, fa_dtype dtype, void *stream) {
    // the fixed delta buffer holds B * H * S floats at most; larger problems are refused
    if (B > 0 && H > 0 && S > 0 && static_cast<int64_t>(B) * H * S > fa::kNoallocDeltaFloats) return FA_ERR_SHAPE;
    if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv) return FA_ERR_NULL;
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (!head_dim_ok(D)) return FA_ERR_HEADDIM;
    if (B <= 0 || H <= 0 || S <= 0) return FA_ERR_SHAPE;
    float *delta = nullptr;
    if (fa::noalloc_delta_buffer(&delta) != cudaSuccess) return FA_ERR_CUDA;
    return fa_bwd(q, k, v, out, dout, lse, dq, dk, dv, delta, B, H, S, D, scale, causal, dtype, stream);
}

fa_status fa_varlen_fwd(const void *q, const void *k, const void *v, const int32_t *cu_seqlens, int num_seqs,
                        int max_seqlen, int total, void *out, float *lse, int H, int D, float scale, int causal,
                        fa_dtype dtype, void *stream) {
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (!head_dim_ok(D)) return FA_ERR_HEADDIM;
    if (num_seqs < 0 || total < 0 || max_seqlen < 0 || H <= 0) return FA_ERR_SHAPE;
    if (total == 0 || num_seqs == 0) return FA_OK;  // no rows, nothing to launch
    if (!q || !k || !v || !out || !cu_seqlens) return FA_ERR_NULL;
    if (max_seqlen == 0) return FA_ERR_SHAPE;
    if ((static_cast<int64_t>(total) + 127) / 128 > 65535) return FA_ERR_SHAPE;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
        !aligned(cu_seqlens, 4))
        return FA_ERR_ALIGN;
    return run_fwd(q, k, v, out, lse, cu_seqlens, num_seqs, max_seqlen, total, H, D, scale, causal, dtype,
                   stream);
}

fa_status fa_varlen_fwd_padded(const void *q, const void *k, const void *v, const int64_t *indices,
                               const int32_t *cu_seqlens, int num_seqs, int max_seqlen, int total,
                               int64_t padded_rows, void *out, float *lse, int H, int D, float scale, int causal,
                               fa_dtype dtype, void *stream) {
    if (dtype != FA_FP16 && dtype != FA_BF16) return FA_ERR_DTYPE;
    if (!head_dim_ok(D)) return FA_ERR_HEADDIM;
    if (num_seqs < 0 || total < 0 || max_seqlen < 0 || H <= 0 || padded_rows < 0) return FA_ERR_SHAPE;
    if (total > padded_rows || padded_rows > INT32_MAX) return FA_ERR_SHAPE;
    if (padded_rows == 0) return FA_OK;
    if (!out) return FA_ERR_NULL;
    if (!aligned(out, 16)) return FA_ERR_ALIGN;
    if (total == 0 || num_seqs == 0) {
        // no valid token: the padded output is all zeros
        const size_t bytes = static_cast<size_t>(padded_rows) * H * D * 2;
        return cudaMemsetAsync(out, 0, bytes, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    }
    if (!q || !k || !v || !cu_seqlens || !indices) return FA_ERR_NULL;
    if (max_seqlen == 0) return FA_ERR_SHAPE;
    if ((static_cast<int64_t>(total) + 127) / 128 > 65535) return FA_ERR_SHAPE;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(lse, 4) || !aligned(cu_seqlens, 4) ||
        !aligned(indices, 8))
        return FA_ERR_ALIGN;
    return run_fwd(q, k, v, out, lse, cu_seqlens, num_seqs, max_seqlen, total, H, D, scale, causal, dtype, stream,
                   indices, padded_rows);
}

fa_status fa_unpad(const void *x, const int64_t *indices, int64_t nnz, int64_t total_rows, int64_t row_bytes,
                   void *out, void *stream) {
    if (nnz < 0 || total_rows < 0 || row_bytes <= 0) return FA_ERR_SHAPE;
    if (nnz == 0) return FA_OK;
    if (!x || !indices || !out) return FA_ERR_NULL;
    if (!aligned(indices, 8)) return FA_ERR_ALIGN;
    const cudaError_t e = fa::launch_unpad(x, indices, nnz, total_rows, row_bytes, out,
                                           static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_unpad_qkv(const void *q, const void *k, const void *v, const int64_t *indices, int64_t nnz,
                       int64_t total_rows, int64_t row_bytes, void *q_out, void *k_out, void *v_out, void *stream) {
    if (nnz < 0 || total_rows < 0 || row_bytes <= 0) return FA_ERR_SHAPE;
    if (nnz == 0) return FA_OK;
    if (!q || !k || !v || !indices || !q_out || !k_out || !v_out) return FA_ERR_NULL;
    if (!aligned(indices, 8)) return FA_ERR_ALIGN;
    const void *const x[3] = {q, k, v};
    void *const o[3] = {q_out, k_out, v_out};
    const cudaError_t e = fa::launch_unpad3(x, indices, nnz, total_rows, row_bytes, o, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_pad(const void *x, const int64_t *indices, int64_t nnz, int64_t total_rows, int64_t row_bytes,
                 void *out, void *stream) {
    if (nnz < 0 || total_rows < 0 || row_bytes <= 0 || nnz > total_rows) return FA_ERR_SHAPE;
    if (total_rows == 0) return FA_OK;
    if (!out || (nnz > 0 && (!x || !indices))) return FA_ERR_NULL;
    if (!aligned(indices, 8)) return FA_ERR_ALIGN;
    const cudaError_t e = fa::launch_pad(x, indices, nnz, total_rows, row_bytes, out,
                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

fa_status fa_device_status(int *where, void *stream) {
    // every kernel family keeps its own word; one kernel on the caller's stream reads and
    // clears them all, one copy brings the result back, and only that stream is waited for
    ErrorWords w;
    if (fa::fwd_error_addrs(&w.code[0], &w.where[0]) != cudaSuccess ||
        fa::fwd_paged_error_addrs(&w.code[1], &w.where[1]) != cudaSuccess ||
        fa::bwd_error_addrs(&w.code[2], &w.where[2]) != cudaSuccess ||
        fa::pad_error_addrs(&w.code[3], &w.where[3]) != cudaSuccess ||
        fa::bwd256_error_addrs(&w.code[4], &w.where[4]) != cudaSuccess)
        return FA_ERR_CUDA;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    status_collect_kernel<<<1, 1, 0, st>>>(w);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    int res[2] = {0, 0};
    if (cudaMemcpyFromSymbolAsync(res, g_status_out, sizeof(res), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return FA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return FA_ERR_CUDA;
    if (where) *where = res[1];
    return static_cast<fa_status>(res[0]);
}

fa_status fa_selftest_bounded_wait(uint64_t limit_ns, void *stream) {
    if (limit_ns == 0 || limit_ns > 10000000000ull) return FA_ERR_SHAPE;
    return fa::launch_selftest_wait(limit_ns, static_cast<cudaStream_t>(stream)) == cudaSuccess ? FA_OK
                                                                                                : FA_ERR_CUDA;
}

const char *fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "FA_OK";
        case FA_ERR_NULL: return "FA_ERR_NULL: a required pointer is NULL";
        case FA_ERR_SHAPE: return "FA_ERR_SHAPE: unsupported or inconsistent sizes";
        case FA_ERR_DTYPE: return "FA_ERR_DTYPE: dtype must be FA_FP16 or FA_BF16";
        case FA_ERR_HEADDIM: return "FA_ERR_HEADDIM: head dim must be 32, 64, 128 or 256";
        case FA_ERR_ALIGN: return "FA_ERR_ALIGN: tensors must be 16-byte aligned (lse 4-byte)";
        case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA call failed";
        case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a kernel's bounded wait ran out";
        case FA_ERR_INDEX: return "FA_ERR_INDEX: an index was out of range";
        default: return "unknown fa_status";
    }
}

const char *fa_version(void) { return "fa-b200 0.1 (sm_100a: tcgen05 + TMEM + TMA)"; }

}  // extern "C"
