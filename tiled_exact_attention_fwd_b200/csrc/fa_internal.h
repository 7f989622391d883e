// fa_internal.h -- declarations shared by the C-ABI layer and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// Kernel parameters of the attention forward (passed by value).
struct FwdParams {
    void *out;                  // token-major (N, H, D) output
    float *lse;                 // dense: (B, H, S); packed: (H, total); may be null
    const int32_t *cu_seqlens;  // null for dense (uniform sequences of `seqlen`)
    int num_seqs;               // packed: entries of cu_seqlens minus one
    const int64_t *gather;      // fused packed path: padded row of every packed token (else null);
                                // q/k/v/out are then padded (padded_rows, H, D) and read by threads
    int64_t padded_rows;
    const void *q, *k, *v;      // the inputs (used by the fused path's copy threads)
    int seqlen;                 // dense sequence length
    int H;                      // heads
    int total_tokens;           // N = rows of the token-major tensors
    float scale_log2;           // scale * log2(e)
    uint64_t timeout_ns;        // bound of every pipeline wait
    // Paged K/V (dense queries only; null otherwise): k and v are pools of num_pages pages of
    // page_size token rows, (num_pages * page_size, H, D); key position pos of batch entry b
    // lives in page block_table[b * max_blocks + pos / page_size], row pos % page_size.
    const int32_t *block_table;
    int max_blocks;
    int page_size;   // a power of two
    int page_shift;  // log2(page_size)
    int num_pages;
    // Dense inputs (persistent grid): batch entries, groups of fwd_tiles_per_cta(D) query tiles
    // per sequence, and work items batch * H * npairs.
    int batch, npairs, num_items;
    // The items are dealt in groups of head_group (batch entry, head) pairs (num_groups groups,
    // group_rounds rounds of one item per CTA each), so that the CTAs running at a time read the
    // K/V of a few heads; head_group = batch * H (one group) unless K/V would not fit in L2.
    int head_group, num_groups, group_rounds;
    int out_align32;  // out is 32-byte aligned (the persistent epilogue then stores 32 bytes per lane)
    // Dense inputs over more than one round (contiguous K/V, D <= 128): {next item index, CTAs
    // done} in device memory, zero at launch; the CTAs take their items from it in the rounds'
    // order instead of round by round, and the last CTA to finish zeroes it again. Else null.
    int *queue;
};

// Attention forward. Dense: a persistent grid of min(num_items, SMs) CTAs; a work item is
// fwd_tiles_per_cta(D) consecutive 128-row query tiles of one head of one sequence. Packed:
// grid (H, ceil(total / (128 * tiles_per_cta)), 1), a CTA owns that many consecutive packed
// tokens.
cudaError_t launch_fwd(int D, bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const FwdParams &p, dim3 grid, cudaStream_t st);
// The same with p.block_table set (paged K/V; maps tk/tv cover the page pools).
cudaError_t launch_fwd_paged(int D, bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                             const CUtensorMap &tv, const FwdParams &p, dim3 grid, cudaStream_t st);
int fwd_tile_rows();
int fwd_tiles_per_cta(int D);
// Dense (not paged, not packed) inputs of head dim D run in 2-CTA clusters: each work item is two
// consecutive query tiles, one per CTA, and the grid is twice the number of clusters.
bool fwd_pair_mode(int D);
int fwd_box_inner_elems(int D);
int fwd_kv_tile_rows(int D);
// Rows of one V box the producer copies (a V tile may move as several row parts).
int fwd_v_box_rows(int D);
// Fused packed path: rows of one TMA box (a run of consecutive padded rows).
int fwd_gather_run_rows();
// Paged K/V: rows per K box / V box for a page size (a box never crosses a page).
int fwd_paged_k_box_rows(int D, int page_size);
int fwd_paged_v_box_rows(int D, int page_size);
cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t st);
// Device addresses of each kernel family's error word (code, location) on the current device.
cudaError_t fwd_error_addrs(int **code, int **where);
cudaError_t fwd_paged_error_addrs(int **code, int **where);

// Attention backward (fa_bwd.cu): dQ, dK, dV from q, k, v, out, dout and the forward's LSE.
struct BwdParams {
    const void *out, *dout;  // (B, S, H, D), read by the delta kernel
    const float *lse;        // (B, H, S) from the forward (packed: (H, total))
    float *delta;            // (B, H, S) workspace: rowsum(dO * O) (packed: (H, total))
    void *dq, *dk, *dv;      // (B, S, H, D) gradients
    int B, H, seqlen;        // packed: B = 1, seqlen = total tokens
    const int32_t *cu_seqlens;  // packed (total, H, D) tensors: sequence offsets (else null)
    int num_seqs;
    float scale;             // softmax scale
    float scale_log2;        // scale * log2(e)
    uint64_t timeout_ns;     // bound of every pipeline wait
};
// tq, tk, tv, tdo: TMA maps of q, k, v, dout as for the forward (128-row boxes; 64 at D = 256).
cudaError_t launch_bwd(int D, bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const CUtensorMap &tdo, const BwdParams &p, cudaStream_t st);
cudaError_t bwd_error_addrs(int **code, int **where);
// D = 256 (fa_bwd256.cu): dV, dK and dQ kernels after the delta kernel; tq, tk, tv, tdo with
// 64-row boxes.
cudaError_t launch_bwd256(bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                          const CUtensorMap &tdo, const BwdParams &p, cudaStream_t st);
cudaError_t bwd256_error_addrs(int **code, int **where);
// The fixed delta buffer of fa_bwd_noalloc: kNoallocDeltaFloats floats (64 MiB) in device
// memory that belongs to the library's module image; its address on the current device.
constexpr int64_t kNoallocDeltaFloats = int64_t(1) << 24;
cudaError_t noalloc_delta_buffer(float **ptr);

// Unpad / pad (row gather / scatter + zero fill).
cudaError_t launch_unpad(const void *x, const int64_t *indices, int64_t nnz, int64_t total_rows,
                         int64_t row_bytes, void *out, cudaStream_t st);
cudaError_t launch_unpad3(const void *const x[3], const int64_t *indices, int64_t nnz, int64_t total_rows,
                          int64_t row_bytes, void *const out[3], cudaStream_t st);
cudaError_t launch_pad(const void *x, const int64_t *indices, int64_t nnz, int64_t total_rows,
                       int64_t row_bytes, void *out, cudaStream_t st);
cudaError_t pad_error_addrs(int **code, int **where);

}  // namespace fa
