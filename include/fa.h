/*
 * fa.h -- C ABI of libfa: exact attention forward computed tile by tile on one
 * NVIDIA B200 (sm_100a), dense, packed and with paged K/V; the unpad gather and pad
 * scatter of the packed path (also fused into the forward); and the backward pass by
 * recomputation.
 *
 * Every entry point is asynchronous on the caller's CUDA stream, allocates no
 * device memory, never synchronises, and takes plain device pointers that the
 * caller allocates and owns. Arguments are validated on the host before any
 * launch; a rejected call launches nothing and returns a negative status.
 *
 * Definitions followed (pages are cited by title and section):
 *   - standard attention, page "昇腾CANN跑大模型，FlashAttention这个算子你得认识一下",
 *     section "传统实现到底慢在哪": O = softmax(Q K^T * scale) V, scale = 1/sqrt(d_k);
 *   - tiling and the online softmax (running row max and row sum, correction of the
 *     earlier partial output), same page, section "分块计算，这事没那么简单";
 *   - causal masking fused with skipping of masked blocks, same page, section
 *     "昇腾NPU上做了什么特殊优化";
 *   - the packed path unpad -> flash_attn_varlen_func -> pad, page
 *     "IAW 模型 FA2 vs FA3 实测", sections 1 and 2.
 *
 * Layouts (all contiguous, row-major, element type fp16 or bf16 unless stated):
 *   dense  q, k, v, out : (B, S, H, D)         lse : (B, H, S)   float32
 *   packed q, k, v, out : (total, H, D)        lse : (H, total)  float32
 *   lse is the natural log of sum_j exp(scale * q.k_j) over the keys the row sees.
 *
 * Supported: D in {32, 64, 128, 256} (forward and backward); q, k, v, out 16-byte
 * aligned; lse 4-byte aligned (may be NULL to skip it in the forward). Causal masking is
 * aligned at the first token of each sequence (query and key lengths are equal per
 * sequence). The header is plain C99.
 */
#ifndef FA_H_
#define FA_H_

#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_NULL = -1,     /* a required pointer is NULL */
    FA_ERR_SHAPE = -2,    /* a size is negative, zero where it must not be, or overflows */
    FA_ERR_DTYPE = -3,    /* dtype is not FA_FP16 / FA_BF16 */
    FA_ERR_HEADDIM = -4,  /* D is not 32, 64, 128 or 256 */
    FA_ERR_ALIGN = -5,    /* a pointer or row size breaks the alignment rule */
    FA_ERR_CUDA = -6,     /* a CUDA runtime/driver call failed (launch, tensor map) */
    FA_ERR_TIMEOUT = -7,  /* a kernel's bounded wait ran out (reported by fa_device_status) */
    FA_ERR_INDEX = -8     /* an index was out of range (reported by fa_device_status) */
} fa_status;

typedef enum { FA_FP16 = 0, FA_BF16 = 1 } fa_dtype;

/*
 * Dense attention forward.
 *   q, k, v   (B, S, H, D) inputs, element type `dtype`.
 *   out       (B, S, H, D) output, same type; every element is written.
 *   lse       (B, H, S) float32 log-sum-exp, or NULL.
 *   scale     score scale; <= 0 selects 1/sqrt(D).
 *   causal    nonzero: query i sees keys 0..i only; fully masked key tiles are skipped.
 *   stream    a cudaStream_t (NULL = the legacy default stream).
 * B, H, S >= 1 (S may be any length; a ragged last tile is masked).
 */
FA_API fa_status fa_fwd(const void *q, const void *k, const void *v, void *out, float *lse,
                 int B, int H, int S, int D, float scale, int causal, fa_dtype dtype,
                 void *stream);

/*
 * Dense attention forward with K and V in a paged pool (the PagedAttention layout that page
 * mooersco.com "FlashAttention 的“加速玄学”", section 5, recommends for long contexts; the
 * page gives no layout, so this one is the common block-table form). Same result as
 * fa_fwd on the contiguous K/V that the block table describes.
 *   q            (B, S, H, D) queries, element type `dtype`.
 *   k_cache,
 *   v_cache      pools (num_pages, page_size, H, D): page n holds page_size consecutive token
 *                rows of some sequence.
 *   block_table  device int32 (B, max_blocks_per_seq): key position pos of batch entry b is
 *                row pos % page_size of page block_table[b * max_blocks_per_seq + pos / page_size].
 *                Entries past ceil(S / page_size) are never read. An entry outside
 *                [0, num_pages) is not dereferenced: page 0 is read instead (that output is
 *                wrong) and FA_ERR_INDEX is left for fa_device_status.
 *   page_size    a power of two, 16 <= page_size <= 2^20; max_blocks_per_seq * page_size >= S;
 *                num_pages * page_size < 2^31.
 *   out, lse     as fa_fwd: (B, S, H, D) and (B, H, S) float32 or NULL.
 * Queries and keys have the same length S per batch entry (causal masks key j > query i).
 * The caller owns every buffer; nothing is allocated; asynchronous on `stream`.
 */
FA_API fa_status fa_fwd_paged(const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *block_table, int max_blocks_per_seq, int page_size,
                              int num_pages, void *out, float *lse, int B, int H, int S, int D,
                              float scale, int causal, fa_dtype dtype, void *stream);

/*
 * Dense attention backward: the gradients of out = softmax(scale * q k^T) v (causal mask as
 * in fa_fwd) with respect to q, k and v, by recomputation from the forward's LSE (page
 * "昇腾CANN跑大模型，FlashAttention这个算子你得认识一下", section "分块计算，这事没那么简单",
 * second pitfall: the scores are not stored, the backward pass computes them again).
 *   q, k, v, out   (B, S, H, D) forward inputs and output, element type `dtype`.
 *   dout           (B, S, H, D) gradient of the loss with respect to out.
 *   lse            (B, H, S) float32 log-sum-exp written by fa_fwd for the same inputs.
 *   dq, dk, dv     (B, S, H, D) outputs, element type `dtype`; every element is written.
 *   delta          (B, H, S) float32 caller-owned workspace; on return it holds
 *                  rowsum(dout * out), the per-row term of the softmax derivative.
 *   scale          <= 0 selects 1/sqrt(D); must be the value the forward used.
 * D in {32, 64, 128, 256}. Launches on `stream`: delta, then dK/dV and dQ (D <= 128, where
 * the dK and dV accumulators of a 128-key tile fit in TMEM side by side) or dV, dK and dQ
 * (D = 256, one accumulator per kernel); nothing is allocated.
 */
FA_API fa_status fa_bwd(const void *q, const void *k, const void *v, const void *out, const void *dout,
                        const float *lse, void *dq, void *dk, void *dv, float *delta, int B, int H, int S,
                        int D, float scale, int causal, fa_dtype dtype, void *stream);

/*
 * Packed variable-length attention backward (the backward of fa_varlen_fwd): gradients of
 * every sequence's attention, sequence s owning rows [cu_seqlens[s], cu_seqlens[s+1]).
 *   q, k, v, out, dout   (total, H, D) packed inputs, output and output gradient.
 *   lse                  (H, total) float32 from fa_varlen_fwd.
 *   dq, dk, dv           (total, H, D) outputs; every element is written.
 *   delta                (H, total) float32 caller-owned workspace (rowsum(dout * out)).
 *   cu_seqlens, num_seqs, max_seqlen, total, scale, causal: as fa_varlen_fwd.
 * D in {32, 64, 128, 256}. Work is split into tiles of 128 consecutive packed tokens whatever
 * sequences they hold. total == 0 is a successful no-op.
 */
FA_API fa_status fa_varlen_bwd(const void *q, const void *k, const void *v, const void *out,
                               const void *dout, const float *lse, const int32_t *cu_seqlens,
                               int num_seqs, int max_seqlen, int total, void *dq, void *dk, void *dv,
                               float *delta, int H, int D, float scale, int causal, fa_dtype dtype,
                               void *stream);

/*
 * fa_bwd without the caller's delta workspace: the same computation and results, with the
 * workspace taken from a fixed device array that is part of the library (64 MiB, room for
 * B * H * S <= 2^24 rows; larger problems return FA_ERR_SHAPE before any launch). The pages
 * have no counterpart to this entry point. It is for callers that cannot allocate device
 * memory at the point where they run the backward pass: a runtime whose caching allocator
 * already owns the device's free memory (a cudaMalloc there fails or breaks the allocator's
 * accounting), or an engine that plans all of its memory ahead of time and forbids
 * allocation inside a step. Nothing here calls cudaMalloc, cudaFree or any allocating routine.
 *   Device: the array lives on every device that loads the library, until the process exits;
 *   the call uses the copy on the current device, which must be the operands' device.
 *   Set-up: the first call on each device looks the array's address up, which loads the
 *   library's module on that device; make that first call before any stream capture.
 *   Nothing has to start at zero: every call overwrites the rows it reads.
 *   Calls that overlap on the GPU (different streams, or concurrent graph nodes) share the
 *   one array and race; serialise them.
 * Arguments as fa_bwd, minus `delta`.
 */
FA_API fa_status fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *out, const void *dout,
                                const float *lse, void *dq, void *dk, void *dv, int B, int H, int S, int D,
                                float scale, int causal, fa_dtype dtype, void *stream);

/*
 * Packed variable-length attention forward (the flash_attn_varlen_func step).
 *   q, k, v      (total, H, D) packed inputs; sequence s owns rows
 *                [cu_seqlens[s], cu_seqlens[s+1]) and attends only inside itself.
 *   cu_seqlens   device int32 array of num_seqs+1 non-decreasing offsets, cu_seqlens[0] = 0,
 *                cu_seqlens[num_seqs] = total (read on the device; not checked on the host).
 *   max_seqlen   the longest sequence (>= 1 when total > 0); kept for the interface of
 *                flash_attn_varlen_func, the launch is sized by total.
 *   out          (total, H, D); lse (H, total) float32 or NULL.
 * Zero-length sequences are allowed and produce no rows. total may be 0 (no launch);
 * total <= 65535 * 128. Work is split into tiles of 128 consecutive packed tokens, whatever
 * sequences they hold (short sequences share a tile; each row only sees its own sequence).
 */
FA_API fa_status fa_varlen_fwd(const void *q, const void *k, const void *v, const int32_t *cu_seqlens,
                        int num_seqs, int max_seqlen, int total, void *out, float *lse, int H,
                        int D, float scale, int causal, fa_dtype dtype, void *stream);

/*
 * The whole packed path in one launch (unpad -> packed attention -> pad): the same result as
 * fa_unpad of q, k, v, then fa_varlen_fwd, then fa_pad of the output, without the compact
 * copies. Page "IAW 模型 FA2 vs FA3 实测", section 6, counts the separate gathers, fill and
 * pads as ~18 us of a 118 us call; here the attention kernel gathers its Q/K/V tiles from
 * the padded tensors and scatters O to the padded rows itself.
 *   q, k, v      padded (padded_rows, H, D) inputs (e.g. (B * total_len, H, D)).
 *   indices      device int64 [total]: padded row of packed token r, strictly increasing.
 *   cu_seqlens   device int32 [num_seqs + 1] over the packed tokens (as in fa_varlen_fwd).
 *   out          padded (padded_rows, H, D): row indices[r] receives token r's output, every
 *                other row is zero.
 *   lse          (H, total) float32 in packed order, or NULL.
 * padded_rows < 2^31; total <= padded_rows. total == 0 writes an all-zero out.
 */
FA_API fa_status fa_varlen_fwd_padded(const void *q, const void *k, const void *v, const int64_t *indices,
                                      const int32_t *cu_seqlens, int num_seqs, int max_seqlen, int total,
                                      int64_t padded_rows, void *out, float *lse, int H, int D, float scale,
                                      int causal, fa_dtype dtype, void *stream);

/*
 * Unpad (gather): out[r, :] = x[indices[r], :] for r < nnz, rows of `row_bytes` bytes.
 *   x        (total_rows, row_bytes) padded input, e.g. (B*total_len, H*D*elt).
 *   indices  device int64 [nnz], each in [0, total_rows).
 *   out      (nnz, row_bytes).
 * Bit-exact byte copy, so one call serves every dtype. Rows whose index is out of range
 * are written as zeros and flag FA_ERR_INDEX for fa_device_status. 16-byte vectors are
 * used when row_bytes and both pointers are 16-byte aligned; otherwise a byte loop.
 */
FA_API fa_status fa_unpad(const void *x, const int64_t *indices, int64_t nnz, int64_t total_rows,
                   int64_t row_bytes, void *out, void *stream);

/*
 * Unpad of q, k and v in one launch: q_out[r] = q[indices[r]], k_out[r] = k[indices[r]],
 * v_out[r] = v[indices[r]] for r < nnz. The packed path of page "IAW 模型 FA2 vs FA3 实测"
 * (sections 1 and 6) gathers the three tensors with the same indices; one launch moves
 * all three. Same argument rules and error behaviour as fa_unpad (all six pointers
 * required; the 16-byte path needs all of them 16-byte aligned).
 */
FA_API fa_status fa_unpad_qkv(const void *q, const void *k, const void *v, const int64_t *indices,
                              int64_t nnz, int64_t total_rows, int64_t row_bytes, void *q_out,
                              void *k_out, void *v_out, void *stream);

/*
 * Pad (scatter + zero fill): out[indices[r], :] = x[r, :] for r < nnz and every other
 * row of out (total_rows, row_bytes) is zero. Each output row is written exactly once.
 *   indices  device int64 [nnz], strictly increasing, each in [0, total_rows)
 *            (the order a nonzero() over a padding mask produces). Entries that break
 *            this rule leave the affected rows unspecified but never cause an access
 *            outside the buffers.
 */
FA_API fa_status fa_pad(const void *x, const int64_t *indices, int64_t nnz, int64_t total_rows,
                 int64_t row_bytes, void *out, void *stream);

/*
 * Device-side status of earlier launches: returns FA_OK or the first FA_ERR_TIMEOUT /
 * FA_ERR_INDEX that a kernel of this library recorded on the current device since the last
 * call, and clears it. `where` (may be NULL) receives a kernel-specific location code.
 * One small kernel and one 8-byte copy run on `stream` (NULL = the legacy default stream),
 * and the call then waits for that stream only: every launch queued on `stream` before the
 * call is covered; work on other streams is covered once it has finished. Returns
 * FA_ERR_CUDA if the stream reports an error (for example a fault of an earlier kernel).
 */
FA_API fa_status fa_device_status(int *where, void *stream);

/*
 * Self-test of the bounded wait used by every pipeline wait in the attention kernel:
 * launches one CTA that waits on a barrier nothing ever completes, with a limit of
 * `limit_ns` nanoseconds. The kernel gives up, records FA_ERR_TIMEOUT and returns, so
 * fa_device_status must then report FA_ERR_TIMEOUT.
 */
FA_API fa_status fa_selftest_bounded_wait(uint64_t limit_ns, void *stream);

/* Human-readable name of a status code (static storage). */
FA_API const char *fa_status_string(int status);

/* Library version string (static storage). */
FA_API const char *fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
