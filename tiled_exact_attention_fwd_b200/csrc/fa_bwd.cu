// fa_bwd.cu -- attention backward on sm_100a: gradients dQ, dK, dV of O = softmax(Z) V,
// Z = scale * Q K^T, by recomputation (page "昇腾CANN跑大模型，FlashAttention这个算子你得认识一下",
// section "分块计算，这事没那么简单", second pitfall: the score matrix is never stored, the
// backward pass recomputes it from Q, K and the saved log-sum-exp).
//
// Per (batch, head), with P = exp(Z - lse) recomputed tile by tile:
//   delta_i = sum_d dO_id O_id                    (bwd_delta_kernel; equals rowsum(P * dP))
//   dV = P^T dO,  dP = dO V^T,  dZ = P * (dP - delta),  dQ = scale dZ K,  dK = scale dZ^T Q
//
// Two tcgen05 kernels, one template (no atomics, no accumulation workspace):
//   dK/dV: a CTA owns one 128-row key tile j (K_j, V_j stay in shared memory) and streams the
//          query tiles i >= j (causal) or all of them through a two-stage TMA ring, each in
//          two half-steps of 64 query rows:
//            S^T  = K_j Q_i^T, dP^T = V_j dO_i^T        (SS MMAs, N = 64, fp32 in TMEM)
//            P^T, dZ^T (16-bit) over S^T, dP^T in TMEM  (elementwise warps, thread = key)
//            dV  += P^T dO_i,  dK += dZ^T Q_i           (TS MMAs, A from TMEM, K = 64)
//          S^T and dP^T of consecutive half-steps alternate between two 128-column TMEM
//          buffers, so the tensor core computes the next half-step's S^T and dP^T (and the
//          previous one's accumulator updates) while the elementwise warps work on the
//          current one: TMEM holds both buffers and the two accumulators (2 x 128 + 2 x D <=
//          512 columns), which whole 128-row steps could not.
//   dQ:    a CTA owns one 128-row query tile i (Q_i, dO_i stay) and streams key tiles j <= i
//          in whole steps (an N = 64 MMA takes nearly as long as an N = 128 one, and the dQ
//          kernel has one accumulator to overlap with, not two):
//            S = Q_i K_j^T, dP = dO_i V_j^T;  dZ over S;  dQ += dZ K_j
// Warps 0-7 do the elementwise work (two threads per TMEM lane = row, each on half of the
// columns), warp 8 lane 0 issues the TMA loads, warp 9 allocates TMEM and lane 0 issues
// every MMA. Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <type_traits>

#include "fa.h"
#include "fa_internal.h"
#include "fa_ptx.cuh"
#include "fa_seq.cuh"
#include "fa_sync.cuh"

namespace fa {
namespace {

template <int D>
struct BwdCfg {
    static constexpr int BM = 128;                           // rows of every tile
    static constexpr int SW = (2 * D >= 128) ? 128 : 2 * D;  // swizzle span in bytes
    static constexpr int SWE = SW / 2;                       // 16-bit elements per swizzle row
    static constexpr int NBLK = D / SWE;                     // column blocks per tile row
    static constexpr int TILE_BYTES = BM * D * 2;
    static constexpr uint32_t LAYOUT = (SW == 128) ? kLayoutSw128 : kLayoutSw64;
    // warps 0-7 elementwise (warp w: TMEM lanes 32*(w%4).., columns half w/4), 8 TMA, 9 MMA
    static constexpr int NUM_EW = 256;
    static constexpr int NUM_THREADS = NUM_EW + 64;
    static constexpr int WARP_TMA = 8, WARP_MMA = 9;
    // shared memory: fixed tiles A0, A1; ring stages s = 0, 1 holding tiles B0, B1;
    // per-column statistics (dK/dV kernel) in two slots; barriers; misc
    static constexpr int OFF_FIX = 0;
    static constexpr int OFF_RING = 2 * TILE_BYTES;
    static constexpr int OFF_STAT = OFF_RING + 4 * TILE_BYTES;  // [slot][-lse*log2e | -delta][128]
    static constexpr int OFF_BAR = OFF_STAT + 2 * 2 * BM * 4;
    // fix_full, ring_full[2], ring_empty[2], s_full[2], p_ready[2], done, drain, stats_ready[2]
    static constexpr int NUM_BARS = 13;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int USED = OFF_MISC + 16;
    static constexpr int MIN_SMEM = 120 * 1024;  // one CTA (and one TMEM allocation) per SM
    static constexpr int SMEM_BYTES = (USED + 1024 > MIN_SMEM) ? USED + 1024 : MIN_SMEM;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int COL_ACC0 = 256, COL_ACC1 = 256 + D;  // accumulators
    static_assert(USED + 1024 <= 227 * 1024, "shared memory budget");
    static_assert(COL_ACC1 + D <= (int)TMEM_COLS, "TMEM budget (dK and dV accumulators)");
    static_assert(TILE_BYTES % 1024 == 0, "tile alignment");
};

// Steps of the streamed loop: STEP streamed rows each, S/dP buffers used in turn (buffer b at
// TMEM column 128 b: S in [0, STEP), dP in [STEP, 2 STEP)).
template <bool DKDV>
struct BwdStep {
    static constexpr int STEP = DKDV ? 64 : 128;  // streamed rows per step
    static constexpr int NBUF = DKDV ? 2 : 1;     // S/dP buffers
    static constexpr int PER_TILE = 128 / STEP;
    static constexpr int COL_BUF = 128, COL_DP = STEP;
};

// Loads of one 128-row tile of a token-major (N, H, D) tensor: NBLK boxes side by side.
template <int D>
__device__ __forceinline__ void load_tile(uint8_t *dst, const CUtensorMap *map, uint64_t *bar, int h, int row,
                                          uint64_t pol) {
    using C = BwdCfg<D>;
#pragma unroll
    for (int b = 0; b < C::NBLK; ++b) tma_load_3d(dst + b * C::BM * C::SW, map, bar, b * C::SWE, h, row, pol);
}

// D_out = A B_u^T over the head dimension: A a K-major 128-row tile in shared memory, B_u rows
// [STEP u, STEP u + STEP) of another (N = STEP).
template <int D, bool BF16, int STEP>
__device__ __forceinline__ void mma_rows_step(uint32_t d_tmem, const uint8_t *a, const uint8_t *b, int u) {
    using C = BwdCfg<D>;
    constexpr uint32_t idesc = idesc_f16(C::BM, STEP, BF16, false);
    const uint32_t a0 = smem_u32(a), b0 = smem_u32(b) + u * STEP * C::SW;
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
        const uint32_t blk = (k * 32) / C::SW, off = (k * 32) % C::SW;
        umma_ss(d_tmem, smem_desc(a0 + blk * C::BM * C::SW + off, 16, 8 * C::SW, C::LAYOUT),
                smem_desc(b0 + blk * C::BM * C::SW + off, 16, 8 * C::SW, C::LAYOUT), idesc, k > 0 ? 1u : 0u);
    }
}

// D_out (+)= A_tmem B_u over STEP rows: A (128 x STEP, 16-bit) in TMEM, B_u rows
// [STEP u, STEP u + STEP) of a 128-row tile read MN-major (its D columns are the output
// columns). A's first STEP/2 elements sit packed at a_tmem + [0, STEP/4) and the others at
// a_tmem + [STEP/2, 3 STEP/4): each half was written by its own thread over the fp32
// columns it had read.
template <int D, bool BF16, int STEP>
__device__ __forceinline__ void mma_acc_step(uint32_t d_tmem, uint32_t a_tmem, const uint8_t *b, int u,
                                             bool accumulate) {
    using C = BwdCfg<D>;
    constexpr uint32_t idesc = idesc_f16(C::BM, D, BF16, true);
    const uint32_t b0 = smem_u32(b) + u * STEP * C::SW;
#pragma unroll
    for (int k = 0; k < STEP / 16; ++k)
        umma_ts(d_tmem, a_tmem + k * 8 + (k >= STEP / 32 ? STEP / 4 : 0),
                smem_desc(b0 + k * 16 * C::SW, C::BM * C::SW, 8 * C::SW, C::LAYOUT), idesc,
                (accumulate || k > 0) ? 1u : 0u);
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2b(float lo, float hi) {
    return BF16 ? pack2_bf16(lo, hi) : pack2_f16(lo, hi);
}

// One row of a TMEM accumulator (D fp32 columns) times `mul` -> 16-bit -> global; the two
// threads of a row take alternate 32-column chunks (half = 0, 1).
template <int D, bool BF16>
__device__ __forceinline__ void store_row(uint32_t taddr, float mul, uint8_t *grow, bool store, int half) {
#pragma unroll 1
    for (int cc = half; cc < D / 32; cc += 2) {
        uint32_t o[32];
        tmem_ld32(taddr + cc * 32, o);
        tmem_ld_wait();
        tmem_reg_fence<32>(o);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = pack2b<BF16>(__uint_as_float(o[2 * i]) * mul, __uint_as_float(o[2 * i + 1]) * mul);
        if (store) {
            uint4 *g = reinterpret_cast<uint4 *>(grow) + cc * 4;
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) g[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
        }
    }
}

// DKDV: the CTA owns key tile j = blockIdx.y; fixed A0 = K_j, A1 = V_j; ring B0 = Q_i, B1 = dO_i.
// !DKDV: the CTA owns query tile i (longest first); fixed A0 = Q_i, A1 = dO_i; ring B0 = K_j, B1 = V_j.
// PACKED: (total, H, D) tensors with cu_seqlens; tiles are 128 consecutive tokens whatever
// sequences they hold (p.B = 1, p.seqlen = total), the streamed windows cover the tokens of
// the owned tile's sequences, and every element is masked to its own sequence.
template <int D, bool BF16, bool CAUSAL, bool DKDV, bool PACKED>
__global__ void __launch_bounds__(BwdCfg<D>::NUM_THREADS, 1)
fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
              const BwdParams p) {
    using C = BwdCfg<D>;
    constexpr int BM = C::BM;
    const int h = blockIdx.x, b = blockIdx.z, S = p.seqlen;  // packed: S = total tokens
    const int ntiles = (S + BM - 1) / BM;
    const int own = (DKDV || PACKED) ? static_cast<int>(blockIdx.y) : ntiles - 1 - static_cast<int>(blockIdx.y);
    const int own_start = own * BM;  // position of the owned tile's first row
    // Streamed windows t = 0..n-1 start at positions ws + t*BM.
    int ws, n;
    if constexpr (PACKED) {
        const int lane_ = threadIdx.x & 31;
        const int last = min(own_start + BM, S) - 1;
        const int s_first = warp_seq_of_token(p.cu_seqlens, p.num_seqs, own_start, lane_);
        const int s_last = warp_seq_of_token(p.cu_seqlens, p.num_seqs, last, lane_);
        const int seq_lo = __ldg(p.cu_seqlens + s_first), seq_hi = __ldg(p.cu_seqlens + s_last + 1);
        // dK/dV: queries of the tile's sequences (from the first key on, when causal);
        // dQ: keys of the tile's sequences (up to the last query, when causal)
        ws = (DKDV && CAUSAL) ? own_start : seq_lo;
        const int we = (!DKDV && CAUSAL) ? min(seq_hi, last + 1) : seq_hi;
        n = (we - ws + BM - 1) / BM;
    } else {
        const int t0 = (DKDV && CAUSAL) ? own : 0;
        const int t1 = (!DKDV && CAUSAL) ? own + 1 : ntiles;
        ws = t0 * BM;
        n = t1 - t0;
    }
    const int64_t row0 = static_cast<int64_t>(b) * S;  // first token row of this batch entry

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *fixA0 = smem + C::OFF_FIX, *fixA1 = fixA0 + C::TILE_BYTES;
    float *stats = reinterpret_cast<float *>(smem + C::OFF_STAT);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *fix_full = bars, *ring_full = bars + 1, *ring_empty = bars + 3, *s_full = bars + 5,
             *p_ready = bars + 7, *done = bars + 9, *drain = bars + 10, *stats_ready = bars + 11;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    const uint64_t lim = p.timeout_ns;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto ring_tile = [&](int stage, int which) { return smem + C::OFF_RING + (2 * stage + which) * C::TILE_BYTES; };

    if (threadIdx.x == 0) {
        mbar_init(fix_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&ring_full[s], 1);
            mbar_init(&ring_empty[s], 1);
            mbar_init(&stats_ready[s], BM);  // the column-half-0 threads publish 128 columns
            mbar_init(&s_full[s], 1);
            mbar_init(&p_ready[s], C::NUM_EW);
        }
        mbar_init(done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == C::WARP_TMA && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        tma_prefetch_desc(&tm_do);
    }
    if (warp == C::WARP_MMA) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == C::WARP_TMA) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n > 0) {
            const uint64_t pol_fix = l2_policy_evict_first();
            const uint64_t pol_ring = l2_policy_evict_last();
            const CUtensorMap *fa0 = DKDV ? &tm_k : &tm_q, *fa1 = DKDV ? &tm_v : &tm_do;
            const CUtensorMap *rb0 = DKDV ? &tm_q : &tm_k, *rb1 = DKDV ? &tm_do : &tm_v;
            mbar_arrive_expect_tx(fix_full, 2 * C::TILE_BYTES);
            load_tile<D>(fixA0, fa0, fix_full, h, static_cast<int>(row0 + own_start), pol_fix);
            load_tile<D>(fixA1, fa1, fix_full, h, static_cast<int>(row0 + own_start), pol_fix);
            int issued = 0;
            for (int t = 0; t < n; ++t) {
                const int s = t & 1;
                if (t >= 2 && !wait_bounded(&ring_empty[s], ((t >> 1) - 1) & 1, abort_flag, lim, 400 + s)) break;
                mbar_arrive_expect_tx(&ring_full[s], 2 * C::TILE_BYTES);
                const int row = static_cast<int>(row0 + ws + t * BM);
                load_tile<D>(ring_tile(s, 0), rb0, &ring_full[s], h, row, pol_ring);
                load_tile<D>(ring_tile(s, 1), rb1, &ring_full[s], h, row, pol_ring);
                issued = t + 1;
            }
            if (*abort_flag) {
                // let the copies already issued land before shared memory goes away
                const uint64_t g0 = global_timer_ns();
                while (!mbar_try_wait(fix_full, 0) && global_timer_ns() - g0 < lim) {
                }
                for (int t = (issued > 2 ? issued - 2 : 0); t < issued; ++t) {
                    const uint64_t g1 = global_timer_ns();
                    while (!mbar_try_wait(&ring_full[t & 1], (t >> 1) & 1) && global_timer_ns() - g1 < lim) {
                    }
                }
            }
        }
    } else if (warp == C::WARP_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n > 0) {
            ok = wait_bounded(fix_full, 0, abort_flag, lim, 410);
            if (ok) tc_fence_after_sync();
            // Step k: streamed tile t = k / PER_TILE, rows [STEP u, STEP u + STEP) with
            // u = k % PER_TILE, TMEM buffer k % NBUF. With two buffers the issue order is
            // S/dP(k+1), then (once the elementwise warps are done with k) the accumulator
            // updates of k; the tensor core runs them in that order, so S/dP(k+2) overwrite
            // buffer k % 2 only after the updates of k have read it. With one buffer S/dP(k+1)
            // follow the updates of k.
            using St = BwdStep<DKDV>;
            const int nk = n * St::PER_TILE;
            auto issue_sdp = [&](int k) -> bool {
                const int t = k / St::PER_TILE, u = k % St::PER_TILE, s = t & 1;
                if (u == 0) {
                    if (!wait_bounded(&ring_full[s], (t >> 1) & 1, abort_flag, lim, 420 + s)) return false;
                    tc_fence_after_sync();
                }
                const uint32_t buf = tmem + (k % St::NBUF) * St::COL_BUF;
                mma_rows_step<D, BF16, St::STEP>(buf, fixA0, ring_tile(s, 0), u);               // S (or S^T)
                mma_rows_step<D, BF16, St::STEP>(buf + St::COL_DP, fixA1, ring_tile(s, 1), u);  // dP (or dP^T)
                umma_commit(&s_full[k % St::NBUF]);
                return true;
            };
            if (ok) ok = issue_sdp(0);
            for (int k = 0; ok && k < nk; ++k) {
                if (St::NBUF == 2 && k + 1 < nk && !(ok = issue_sdp(k + 1))) break;
                if (!(ok = wait_bounded(&p_ready[k % St::NBUF], (k / St::NBUF) & 1, abort_flag, lim,
                                        430 + k % St::NBUF)))
                    break;
                tc_fence_after_sync();
                const int t = k / St::PER_TILE, u = k % St::PER_TILE, s = t & 1;
                const uint32_t buf = tmem + (k % St::NBUF) * St::COL_BUF;
                if (DKDV) {
                    mma_acc_step<D, BF16, St::STEP>(tmem + C::COL_ACC0, buf, ring_tile(s, 1), u, k > 0);  // dV += P^T dO
                    mma_acc_step<D, BF16, St::STEP>(tmem + C::COL_ACC1, buf + St::COL_DP, ring_tile(s, 0), u,
                                                    k > 0);  // dK += dZ^T Q
                } else {
                    mma_acc_step<D, BF16, St::STEP>(tmem + C::COL_ACC0, buf, ring_tile(s, 0), u, k > 0);  // dQ += dZ K
                }
                if (u == St::PER_TILE - 1) umma_commit(&ring_empty[s]);  // every step of tile t has read it
                if (St::NBUF == 1 && k + 1 < nk && !(ok = issue_sdp(k + 1))) break;
            }
            if (ok) umma_commit(done);
            umma_commit(drain);  // every MMA issued above has finished once this arrives
            const uint64_t g0 = global_timer_ns();
            while (!mbar_try_wait(drain, 0) && global_timer_ns() - g0 < lim) {
            }
        }
    } else {
        // ------------------------------------------------------------ elementwise warps 0-7
        const int quarter = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
        const int r = quarter * 32 + lane;                // TMEM lane = row of the owned tile
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const int own_pos = own_start + r;  // position of this row (key or query)
        // the positions this row may pair with: its sequence (packed) or [0, S)
        int row_lo = 0, row_hi = S;
        if constexpr (PACKED) {
            const int tok = min(own_pos, S - 1);
            const int s0 = warp_seq_of_token(p.cu_seqlens, p.num_seqs, min(own_start + quarter * 32, S - 1), lane);
            const int sq = lane_seq_of_token(p.cu_seqlens, p.num_seqs, s0, tok, lane);
            row_lo = __ldg(p.cu_seqlens + sq);
            row_hi = __ldg(p.cu_seqlens + sq + 1);
            if (own_pos >= S) row_lo = row_hi = 0;  // past the last token: pairs with nothing
        }
        const float sl2 = p.scale_log2;
        constexpr float kLog2e = 1.4426950408889634f;
        const int64_t stat_base = (static_cast<int64_t>(b) * p.H + h) * S;
        // statistics of a query position: -lse*log2(e) and -delta (0 past the sequence end, which
        // makes every weight of that query exactly 0)
        auto query_stats = [&](int qpos, float &nl, float &nd) {
            if (qpos < S) {
                nl = -__ldg(p.lse + stat_base + qpos) * kLog2e;
                nd = -__ldg(p.delta + stat_base + qpos);
            } else {
                nl = -INFINITY;
                nd = 0.f;
            }
        };
        const bool publisher = DKDV && half == 0;  // publishes the statistics of query column r
        float my_nl = 0.f, my_nd = 0.f;  // dQ: this row's statistics; dK/dV: prefetched column stats
        if (publisher) {
            if (n > 0) query_stats(ws + r, my_nl, my_nd);
        } else if (!DKDV) {
            query_stats(own_pos, my_nl, my_nd);
        }
        // P (or P^T) and dZ for the 32 columns [col0, col0 + 32) of TMEM buffer `buf`, whose
        // column c is streamed position w0 + c; MASK applies the causal diagonal and the
        // sequence bounds.
        auto chunk = [&](auto mask_c, uint32_t buf, int col0, const float *snl, const float *snd, int w0) {
            constexpr bool MASK = decltype(mask_c)::value;
            uint32_t sv[32], dv[32];
            tmem_ld32(buf + lane_base + col0, sv);
            tmem_ld32(buf + lane_base + BwdStep<DKDV>::COL_DP + col0, dv);
            tmem_ld_wait();
            tmem_reg_fence<32>(sv);
            tmem_reg_fence<32>(dv);
            uint32_t pk[16], zk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int col = col0 + 2 * i;
                float nl0, nl1, nd0, nd1;
                if (DKDV) {
                    const float2 a = *reinterpret_cast<const float2 *>(snl + col);
                    const float2 c2 = *reinterpret_cast<const float2 *>(snd + col);
                    nl0 = a.x, nl1 = a.y, nd0 = c2.x, nd1 = c2.y;
                } else {
                    nl0 = nl1 = my_nl;
                    nd0 = nd1 = my_nd;
                }
                const uint64_t x2 = ffma2(f2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])),
                                          f2(sl2, sl2), f2(nl0, nl1));
                float x0, x1;
                f2_split(x2, x0, x1);
                float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                if constexpr (MASK) {
                    // a pair weighs 0 unless the column lies in the row's sequence (or [0, S))
                    // and, when causal, the key position is not past the query position (dK/dV
                    // rows are keys and columns queries, dQ the other way round)
                    const int c0 = w0 + col, c1 = c0 + 1;
                    if (c0 < row_lo || c0 >= row_hi || (CAUSAL && (DKDV ? c0 < own_pos : c0 > own_pos))) p0 = 0.f;
                    if (c1 < row_lo || c1 >= row_hi || (CAUSAL && (DKDV ? c1 < own_pos : c1 > own_pos))) p1 = 0.f;
                }
                const uint64_t z2 = fmul2(f2(p0, p1), fadd2(f2(__uint_as_float(dv[2 * i]), __uint_as_float(dv[2 * i + 1])),
                                                            f2(nd0, nd1)));
                float z0, z1;
                f2_split(z2, z0, z1);
                pk[i] = pack2b<BF16>(p0, p1);
                zk[i] = pack2b<BF16>(z0, z1);
            }
            // packed columns of this thread start at its own first column (STEP/2 * half), so
            // neither thread of the row overwrites columns the other one has yet to read
            constexpr int HS = BwdStep<DKDV>::STEP / 2;  // columns per thread and step
            const int pcol = half * HS + (col0 - half * HS) / 2;
            if (DKDV) {
                tmem_st16(buf + lane_base + pcol, pk);                             // P^T over S^T
                tmem_st16(buf + lane_base + BwdStep<DKDV>::COL_DP + pcol, zk);  // dZ^T over dP^T
            } else {
                tmem_st16(buf + lane_base + pcol, zk);  // dZ over S
            }
        };
        using St = BwdStep<DKDV>;
        for (int k = 0; ok && k < n * St::PER_TILE; ++k) {
            const int t = k / St::PER_TILE, u = k % St::PER_TILE;  // streamed tile, part
            const int w0 = ws + t * BM + u * St::STEP;              // position of the step's first streamed row
            const int slot = t & 1;
            const float *snl = stats + slot * 2 * BM + u * St::STEP, *snd = snl + BM;
            if (DKDV && u == 0) {
                if (publisher) {
                    // publish this thread's query column statistics, prefetch the next tile's
                    stats[slot * 2 * BM + r] = my_nl;
                    stats[slot * 2 * BM + BM + r] = my_nd;
                    mbar_arrive(&stats_ready[slot]);
                    if (t + 1 < n) query_stats(w0 + BM + r, my_nl, my_nd);
                }
                if (!(ok = __all_sync(0xffffffffu, wait_bounded(&stats_ready[slot], (t >> 1) & 1, abort_flag, lim, 440))))
                    break;
            }
            if (!(ok = __all_sync(0xffffffffu, wait_bounded(&s_full[k % St::NBUF], (k / St::NBUF) & 1, abort_flag,
                                                            lim, 450 + k % St::NBUF))))
                break;
            tc_fence_after_sync();
            // does any pair of this warp's rows with the step's positions need a mask?
            const bool row_partial = w0 < row_lo || w0 + St::STEP > row_hi ||
                                     (CAUSAL && (DKDV ? w0 < own_pos : w0 + St::STEP - 1 > own_pos));
            const bool masked = __any_sync(0xffffffffu, row_partial);
            // this thread's STEP/2 columns [STEP/2 * half, ...) of the step, 32 at a time; the
            // results are stored over columns this thread has already read
            const uint32_t buf = tmem + (k % St::NBUF) * St::COL_BUF;
#pragma unroll 1
            for (int c = 0; c < St::STEP / 64; ++c) {
                const int col0 = half * (St::STEP / 2) + c * 32;
                if (masked)
                    chunk(std::integral_constant<bool, true>{}, buf, col0, snl, snd, w0);
                else
                    chunk(std::integral_constant<bool, false>{}, buf, col0, snl, snd, w0);
            }
            tmem_st_wait();
            tc_fence_before_sync();
            mbar_arrive(&p_ready[k % St::NBUF]);
        }
        if (ok && n > 0) ok = __all_sync(0xffffffffu, wait_bounded(done, 0, abort_flag, lim, 460));
        if (ok) {
            tc_fence_after_sync();
            const bool store = own_pos < S;
            const int64_t grow = (row0 + own_pos) * p.H + h;  // token row, head
            if (DKDV) {
                store_row<D, BF16>(tmem + lane_base + C::COL_ACC0, 1.f, static_cast<uint8_t *>(p.dv) + grow * D * 2,
                                   store, half);
                store_row<D, BF16>(tmem + lane_base + C::COL_ACC1, p.scale, static_cast<uint8_t *>(p.dk) + grow * D * 2,
                                   store, half);
            } else {
                store_row<D, BF16>(tmem + lane_base + C::COL_ACC0, p.scale, static_cast<uint8_t *>(p.dq) + grow * D * 2,
                                   store, half);
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// delta[b, h, s] = sum_d dO[b, s, h, d] * O[b, s, h, d] in fp32: D/8 lanes per (row, head),
// 16-byte loads, a shuffle reduction. Warps stride over groups of 32/(D/8) consecutive
// (row, head) items, so every lane of a warp runs the same number of iterations.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const void *out, const void *dout, float *delta, int64_t rows,
                                                        int H, int S) {
    constexpr int LPH = D / 8;           // lanes per (row, head)
    constexpr int PER_WARP = 32 / LPH;   // items per warp and iteration
    const int64_t items = rows * H;
    const int lane = threadIdx.x & 31, sub = lane % LPH;
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * blockDim.x / 32;
    for (int64_t base = warp0 * PER_WARP; base < items; base += nwarps * PER_WARP) {
        const int64_t it = base + lane / LPH;
        const bool live = it < items;
        float acc = 0.f;
        if (live) {
            const uint4 o4 = ld_nc_v4(static_cast<const uint8_t *>(out) + (it * D + sub * 8) * 2);
            const uint4 g4 = ld_nc_v4(static_cast<const uint8_t *>(dout) + (it * D + sub * 8) * 2);
            const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w}, gw[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float2 of, gf;
                if (BF16) {
                    of = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&ow[i]));
                    gf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&gw[i]));
                } else {
                    of = __half22float2(*reinterpret_cast<const __half2 *>(&ow[i]));
                    gf = __half22float2(*reinterpret_cast<const __half2 *>(&gw[i]));
                }
                acc = fmaf(of.x, gf.x, acc);
                acc = fmaf(of.y, gf.y, acc);
            }
        }
#pragma unroll
        for (int off = LPH / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (live && sub == 0) {
            const int64_t row = it / H;  // token row b*S + s
            const int hh = static_cast<int>(it % H);
            const int64_t bb = row / S, ss = row % S;
            delta[(bb * H + hh) * S + ss] = acc;
        }
    }
}

template <int D, bool BF16, bool CAUSAL, bool DKDV, bool PACKED>
cudaError_t launch_bwd_t(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tdo,
                         const BwdParams &p, dim3 grid, cudaStream_t st) {
    using C = BwdCfg<D>;
    auto kern = fa_bwd_kernel<D, BF16, CAUSAL, DKDV, PACKED>;
    static uint64_t attr_set_mask = 0;  // per-device shared-memory opt-in done
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = uint64_t(1) << (dev & 63);
    if (!(__atomic_load_n(&attr_set_mask, __ATOMIC_ACQUIRE) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        __atomic_fetch_or(&attr_set_mask, bit, __ATOMIC_RELEASE);
    }
    kern<<<grid, C::NUM_THREADS, C::SMEM_BYTES, st>>>(tq, tk, tv, tdo, p);
    return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t launch_bwd_d(bool causal, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                         const CUtensorMap &tdo, const BwdParams &p, cudaStream_t st) {
    const int rows = p.B * p.seqlen;
    const int64_t items = static_cast<int64_t>(rows) * p.H;
    const int threads = 256;
    int64_t blocks = (items * (D / 8) + threads - 1) / threads;  // one (row, head) per D/8 lanes
    if (blocks > 148 * 16) blocks = 148 * 16;
    bwd_delta_kernel<D, BF16><<<static_cast<unsigned>(blocks), threads, 0, st>>>(p.out, p.dout, p.delta, rows, p.H,
                                                                                 p.seqlen);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int ntiles = (p.seqlen + 127) / 128;
    const dim3 grid(static_cast<unsigned>(p.H), static_cast<unsigned>(ntiles), static_cast<unsigned>(p.B));
    if (p.cu_seqlens) {
        e = causal ? launch_bwd_t<D, BF16, true, true, true>(tq, tk, tv, tdo, p, grid, st)
                   : launch_bwd_t<D, BF16, false, true, true>(tq, tk, tv, tdo, p, grid, st);
        if (e != cudaSuccess) return e;
        return causal ? launch_bwd_t<D, BF16, true, false, true>(tq, tk, tv, tdo, p, grid, st)
                      : launch_bwd_t<D, BF16, false, false, true>(tq, tk, tv, tdo, p, grid, st);
    }
    e = causal ? launch_bwd_t<D, BF16, true, true, false>(tq, tk, tv, tdo, p, grid, st)
               : launch_bwd_t<D, BF16, false, true, false>(tq, tk, tv, tdo, p, grid, st);
    if (e != cudaSuccess) return e;
    return causal ? launch_bwd_t<D, BF16, true, false, false>(tq, tk, tv, tdo, p, grid, st)
                  : launch_bwd_t<D, BF16, false, false, false>(tq, tk, tv, tdo, p, grid, st);
}

}  // namespace

cudaError_t launch_bwd(int D, bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const CUtensorMap &tdo, const BwdParams &p, cudaStream_t st) {
    switch (D) {
        case 32: return bf16 ? launch_bwd_d<32, true>(causal, tq, tk, tv, tdo, p, st)
                             : launch_bwd_d<32, false>(causal, tq, tk, tv, tdo, p, st);
        case 64: return bf16 ? launch_bwd_d<64, true>(causal, tq, tk, tv, tdo, p, st)
                             : launch_bwd_d<64, false>(causal, tq, tk, tv, tdo, p, st);
        case 128: return bf16 ? launch_bwd_d<128, true>(causal, tq, tk, tv, tdo, p, st)
                              : launch_bwd_d<128, false>(causal, tq, tk, tv, tdo, p, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t bwd_take_device_error(int *code, int *where) { return take_device_error(code, where); }

}  // namespace fa
