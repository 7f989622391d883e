// fa_bwd256.cu -- attention backward at head dim 256 on sm_100a: dQ, dK, dV by recomputation
// (page "昇腾CANN跑大模型，FlashAttention这个算子你得认识一下", section "分块计算，这事没那么简单",
// second pitfall: the scores are recomputed from Q, K and the saved log-sum-exp, never stored).
// Same arithmetic as the D <= 128 kernels of fa_bwd.cu:
//   P = exp(Z - lse), Z = scale Q K^T;  dV = P^T dO;  dP = dO V^T;  dZ = P * (dP - delta);
//   dQ = scale dZ K;  dK = scale dZ^T Q   (delta = rowsum(dO * O), from bwd_delta_kernel).
//
// Why other kernels at D = 256: a 128-row tile is 64 KB, and one accumulator of a 128-row
// tile takes 256 of the 512 TMEM columns. The dK and dV accumulators of one key tile no
// longer fit beside each other (2 x 256 columns, nothing left for the scores), so each of the
// three gradients gets a kernel of its own, all from one template. A CTA owns a 128-row tile
// (key tile j for dV and dK, query tile i for dQ), keeps it (and its partner) in shared
// memory, and streams the other side in 64-row half tiles:
//   dV:  X = K_j Q_u^T (S^T);                       P^T over X;   dV += P^T dO_u
//   dK:  X = K_j Q_u^T, Y = V_j dO_u^T (dP^T);       dZ^T over X;  dK += dZ^T Q_u
//   dQ:  X = Q_i K_u^T (S),  Y = dO_i V_u^T (dP);    dZ over X;    dQ += dZ K_u
// X and Y are N = 64 SS MMAs over the 256 head columns (16 k-steps); the update is one TS MMA
// (A = the 16-bit step from TMEM, B = the streamed half tile read MN-major, N = 256, K = 64).
// TMEM: two 128-column buffers (X at +0, Y at +64) used by alternate steps, so the next step's
// products run while the elementwise warps work on this one, and the accumulator at column
// 256. In dK and dQ the MMA warp issues X(k+1), the update of k, then Y(k+1), so that Y covers
// the refill of the slot the update frees (see the issue loop).
// Shared memory: the fixed tile(s) (64 KB each), the half tiles read by X in a two-slot ring,
// the other stream in a one-slot ring (dK, dQ: Y is its only reader, so the slot is free once
// Y completes, long before the next step needs it) or a three-slot ring (dV: read by the
// update, whose slot is refilled two steps ahead), and the streamed queries' statistics (dV,
// dK) in three slots. The three kernels do
// 8 score-sized products per tile pair where the D <= 128 kernels do 7 (S^T is recomputed by
// dV and dK).
// Warps 0-7 are elementwise (two threads per TMEM lane = row, 32 columns each), warp 8 lane 0
// issues the TMA loads, warp 9 allocates TMEM and issues every MMA. Every wait is bounded.
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

enum { KIND_DV = 0, KIND_DK = 1, KIND_DQ = 2 };

struct B256 {
    static constexpr int D = 256;
    static constexpr int BM = 128;    // rows of the owned tile
    static constexpr int STEP = 64;   // streamed rows per step
    static constexpr int SW = 128;    // swizzle span in bytes
    static constexpr int SWE = 64;    // 16-bit elements per swizzle row
    static constexpr int NBLK = 4;    // column blocks per row
    static constexpr int FIX_BYTES = BM * D * 2;
    static constexpr int HALF_BYTES = STEP * D * 2;
    static constexpr int NUM_EW = 256;
    static constexpr int NUM_THREADS = NUM_EW + 64;
    static constexpr int WARP_TMA = 8, WARP_MMA = 9;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int COL_ACC = 256;
};

template <int KIND>
struct B256Kind {
    using C = B256;
    static constexpr bool HAS_Y = KIND != KIND_DV;      // a second score-sized product (dP)
    static constexpr bool COL_STATS = KIND != KIND_DQ;  // statistics belong to the streamed rows
    static constexpr int NFIX = HAS_Y ? 2 : 1;
    static constexpr int R0_SLOTS = 2;                  // read by X (and, dK / dQ, the update)
    static constexpr int R1_SLOTS = HAS_Y ? 1 : 3;      // read by Y (dK, dQ) or the update (dV)
    static constexpr int STAT_SLOTS = 3;
    static constexpr int OFF_R0 = NFIX * C::FIX_BYTES;
    static constexpr int OFF_R1 = OFF_R0 + R0_SLOTS * C::HALF_BYTES;
    static constexpr int OFF_STAT = OFF_R1 + R1_SLOTS * C::HALF_BYTES;  // [slot][-lse*log2e | -delta][64]
    static constexpr int OFF_BAR = OFF_STAT + (COL_STATS ? STAT_SLOTS * 2 * C::STEP * 4 : 0);
    // fix_full, r0_full[2], r0_empty[2], r1_full[3], r1_empty[3], s_full[2], p_ready[2],
    // stats_ready[3], done, drain
    static constexpr int NUM_BARS = 20;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int USED = OFF_MISC + 16;
    static constexpr int SMEM_BYTES = USED + 1024;  // + alignment of the base to 1024 bytes
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

template <bool BF16>
__device__ __forceinline__ uint32_t pack2x(float lo, float hi) {
    return BF16 ? pack2_bf16(lo, hi) : pack2_f16(lo, hi);
}

// The owned 128-row tile: per column block, two 64-row boxes (the maps have 64-row boxes);
// the 128B swizzle repeats every 8 rows, so they land exactly as one 128-row box would.
__device__ __forceinline__ void load_fixed(uint8_t *dst, const CUtensorMap *map, uint64_t *bar, int h, int row,
                                           uint64_t pol) {
    using C = B256;
#pragma unroll
    for (int b = 0; b < C::NBLK; ++b) {
        tma_load_3d(dst + b * C::BM * C::SW, map, bar, b * C::SWE, h, row, pol);
        tma_load_3d(dst + b * C::BM * C::SW + C::STEP * C::SW, map, bar, b * C::SWE, h, row + C::STEP, pol);
    }
}

// A streamed 64-row half tile: one box per column block.
__device__ __forceinline__ void load_half(uint8_t *dst, const CUtensorMap *map, uint64_t *bar, int h, int row,
                                          uint64_t pol) {
    using C = B256;
#pragma unroll
    for (int b = 0; b < C::NBLK; ++b) tma_load_3d(dst + b * C::STEP * C::SW, map, bar, b * C::SWE, h, row, pol);
}

// d = F R^T over the 256 head columns: F the owned 128-row tile, R a 64-row half tile, both
// K-major (M = 128, N = 64, 16 k-steps of 16 columns; column block k / 4 of each).
template <bool BF16>
__device__ __forceinline__ void mma_scores(uint32_t d_tmem, const uint8_t *f, const uint8_t *r) {
    using C = B256;
    constexpr uint32_t idesc = idesc_f16(C::BM, C::STEP, BF16, false);
    constexpr uint32_t hi = smem_desc_hi(8 * C::SW, kLayoutSw128);
    const uint32_t f_lo = smem_desc_lo(smem_u32(f), 16), r_lo = smem_desc_lo(smem_u32(r), 16);
#pragma unroll
    for (int k = 0; k < C::D / 16; ++k) {
        const uint32_t blk = (k * 32) / C::SW, off = (k * 32) % C::SW;
        umma_ss_elect(d_tmem, f_lo + ((blk * C::BM * C::SW + off) >> 4), r_lo + ((blk * C::STEP * C::SW + off) >> 4),
                      hi, idesc, k > 0 ? 1u : 0u);
    }
}

// acc (+)= Z R: Z (128 x 64, 16-bit) in TMEM, R a 64-row half tile read MN-major (its 256
// columns are the output columns; LBO = the distance between its column blocks). Z's first
// 32 elements sit packed at z_tmem + [0, 16), the other 32 at z_tmem + [32, 48): each half
// was written by its own thread over the fp32 columns it had read.
template <bool BF16>
__device__ __forceinline__ void mma_update(uint32_t acc_tmem, uint32_t z_tmem, const uint8_t *r, bool accumulate) {
    using C = B256;
    constexpr uint32_t idesc = idesc_f16(C::BM, C::D, BF16, true);
    constexpr uint32_t hi = smem_desc_hi(8 * C::SW, kLayoutSw128);
    const uint32_t r_lo = smem_desc_lo(smem_u32(r), C::STEP * C::SW);
#pragma unroll
    for (int k = 0; k < C::STEP / 16; ++k)
        umma_ts_elect(acc_tmem, z_tmem + k * 8 + (k >= 2 ? 16 : 0), r_lo + ((k * 16 * C::SW) >> 4), hi, idesc,
                      (accumulate || k > 0) ? 1u : 0u);
}

// One row of the accumulator times `mul` -> 16-bit -> global; the two threads of a row take
// alternate 32-column chunks.
template <bool BF16>
__device__ __forceinline__ void store_acc_row(uint32_t taddr, float mul, uint8_t *grow, bool store, int half) {
#pragma unroll 1
    for (int cc = half; cc < B256::D / 32; cc += 2) {
        uint32_t o[32];
        tmem_ld32(taddr + cc * 32, o);
        tmem_ld_wait();
        tmem_reg_fence<32>(o);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) w[i] = pack2x<BF16>(__uint_as_float(o[2 * i]) * mul, __uint_as_float(o[2 * i + 1]) * mul);
        if (store) {
            uint4 *g = reinterpret_cast<uint4 *>(grow) + cc * 4;
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) g[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
        }
    }
}

// Heads per group in the order the CTAs are dealt out (as in the D <= 128 kernels).
constexpr int B256_HEAD_GROUP = 8;

// KIND_DV / KIND_DK: the CTA owns key tile j (fixed K_j [, V_j]); streamed Q_u [, dO_u].
// KIND_DQ: the CTA owns query tile i (longest first when causal; fixed Q_i, dO_i); streamed
// K_u, V_u. PACKED: (total, H, D) tensors with cu_seqlens, tiles of 128 consecutive tokens,
// every pair masked to its own sequence.
template <bool BF16, bool CAUSAL, int KIND, bool PACKED>
__global__ void __launch_bounds__(B256::NUM_THREADS, 1)
fa_bwd256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                 const BwdParams p) {
    using C = B256;
    using Kd = B256Kind<KIND>;
    constexpr bool KEYS = KIND != KIND_DQ;  // the owned rows are keys
    constexpr int BM = C::BM, STEP = C::STEP;
    const int b = blockIdx.z, S = p.seqlen;  // packed: S = total tokens
    const int ntiles = (S + BM - 1) / BM;
    int h, tile;
    {
        const int lin = static_cast<int>(blockIdx.x) + p.H * static_cast<int>(blockIdx.y);
        const int g0 = (lin / (B256_HEAD_GROUP * ntiles)) * B256_HEAD_GROUP;
        const int gsize = min(B256_HEAD_GROUP, p.H - g0);
        const int idx = lin - g0 * ntiles;
        tile = idx / gsize;
        h = g0 + idx % gsize;
    }
    const int own = (KEYS || PACKED) ? tile : ntiles - 1 - tile;
    const int own_start = own * BM;
    // Streamed positions [ws, we), in steps of STEP rows.
    int ws, we;
    if constexpr (PACKED) {
        const int lane_ = threadIdx.x & 31;
        const int last = min(own_start + BM, S) - 1;
        const int s_first = warp_seq_of_token(p.cu_seqlens, p.num_seqs, own_start, lane_);
        const int s_last = warp_seq_of_token(p.cu_seqlens, p.num_seqs, last, lane_);
        const int seq_lo = __ldg(p.cu_seqlens + s_first), seq_hi = __ldg(p.cu_seqlens + s_last + 1);
        ws = (KEYS && CAUSAL) ? own_start : seq_lo;
        we = (!KEYS && CAUSAL) ? min(seq_hi, last + 1) : seq_hi;
    } else {
        ws = (KEYS && CAUSAL) ? own_start : 0;
        we = (!KEYS && CAUSAL) ? min(S, own_start + BM) : S;
    }
    const int n = (we - ws + STEP - 1) / STEP;  // streamed steps
    const int64_t row0 = static_cast<int64_t>(b) * S;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *fix0 = smem, *fix1 = smem + C::FIX_BYTES;
    float *stats = reinterpret_cast<float *>(smem + Kd::OFF_STAT);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Kd::OFF_BAR);
    uint64_t *fix_full = bars, *r0_full = bars + 1, *r0_empty = bars + 3, *r1_full = bars + 5, *r1_empty = bars + 8;
    uint64_t *s_full = bars + 11, *p_ready = bars + 13, *stats_ready = bars + 15, *done = bars + 18, *drain = bars + 19;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Kd::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Kd::OFF_MISC + 4);
    const uint64_t lim = p.timeout_ns;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto r0_tile = [&](int slot) { return smem + Kd::OFF_R0 + slot * C::HALF_BYTES; };
    auto r1_tile = [&](int slot) { return smem + Kd::OFF_R1 + slot * C::HALF_BYTES; };

    if (threadIdx.x == 0) {
        mbar_init(fix_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&r0_full[s], 1);
            mbar_init(&r0_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&p_ready[s], C::NUM_EW);
        }
        for (int s = 0; s < 3; ++s) {
            mbar_init(&r1_full[s], 1);
            mbar_init(&r1_empty[s], 1);
        }
        for (int s = 0; s < Kd::STAT_SLOTS; ++s) mbar_init(&stats_ready[s], STEP);  // 64 publishing threads
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

    // fixed tiles and streams of this kind
    const CUtensorMap *mf0 = KEYS ? &tm_k : &tm_q, *mf1 = KEYS ? &tm_v : &tm_do;
    const CUtensorMap *mr0 = KEYS ? &tm_q : &tm_k;
    const CUtensorMap *mr1 = (KIND == KIND_DQ) ? &tm_v : &tm_do;

    if (warp == C::WARP_TMA) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0 && n > 0) {
            const uint64_t pol_fix = l2_policy_evict_first();
            const uint64_t pol_ring = l2_policy_evict_last();
            mbar_arrive_expect_tx(fix_full, Kd::NFIX * C::FIX_BYTES);
            load_fixed(fix0, mf0, fix_full, h, static_cast<int>(row0 + own_start), pol_fix);
            if (Kd::NFIX == 2) load_fixed(fix1, mf1, fix_full, h, static_cast<int>(row0 + own_start), pol_fix);
            int i0 = 0, i1 = 0;  // half tiles issued per stream
            for (int k = 0; k < n; ++k) {
                const int row = static_cast<int>(row0 + ws + k * STEP);
                const int s0 = k & 1;
                if (k >= 2 && !wait_bounded(&r0_empty[s0], ((k >> 1) - 1) & 1, abort_flag, lim, 500 + s0)) break;
                mbar_arrive_expect_tx(&r0_full[s0], C::HALF_BYTES);
                load_half(r0_tile(s0), mr0, &r0_full[s0], h, row, pol_ring);
                i0 = k + 1;
                const int s1 = k % Kd::R1_SLOTS;
                if (k >= Kd::R1_SLOTS &&
                    !wait_bounded(&r1_empty[s1], ((k / Kd::R1_SLOTS) - 1) & 1, abort_flag, lim, 502 + s1))
                    break;
                mbar_arrive_expect_tx(&r1_full[s1], C::HALF_BYTES);
                load_half(r1_tile(s1), mr1, &r1_full[s1], h, row, pol_ring);
                i1 = k + 1;
            }
            if (*abort_flag) {
                // let the copies already issued land before shared memory goes away
                auto settle = [&](uint64_t *bar, uint32_t ph) {
                    const uint64_t g1 = global_timer_ns();
                    while (!mbar_try_wait(bar, ph) && global_timer_ns() - g1 < lim) {
                    }
                };
                settle(fix_full, 0);
                for (int k = (i0 > 2 ? i0 - 2 : 0); k < i0; ++k) settle(&r0_full[k & 1], (k >> 1) & 1);
                for (int k = (i1 > Kd::R1_SLOTS ? i1 - Kd::R1_SLOTS : 0); k < i1; ++k)
                    settle(&r1_full[k % Kd::R1_SLOTS], (k / Kd::R1_SLOTS) & 1);
            }
        }
    } else if (warp == C::WARP_MMA) {
        // ------------------------------------------------------------ MMA issuer
        auto wait_all = [&](uint64_t *bar, uint32_t ph, int where) {
            return __all_sync(0xffffffffu, wait_bounded(bar, ph, abort_flag, lim, where));
        };
        if (n > 0) {
            ok = wait_all(fix_full, 0, 510);
            if (ok) tc_fence_after_sync();
            // X and Y of step k go into TMEM buffer k % 2; the update of step k reads it once the
            // elementwise warps are done with k. Issue order, dV: X(k+1), then the update of k.
            // dK and dQ: X(k+1), the update of k, then Y(k+1) — the update frees the slot of the
            // stream X and the update read (step k's), whose refill for X(k+2) is a 32 KB load, and
            // Y(k+1) runs while it lands (issued before the update, X(k+2) would wait for it in
            // the tensor pipe on every step). The tensor core runs MMAs in issue order, so X/Y
            // of step k+2 overwrite buffer k % 2 only after the update of k has read it.
            auto issue_x = [&](int k) -> bool {
                const int s0 = k & 1;
                if (!wait_all(&r0_full[s0], (k >> 1) & 1, 520 + s0)) return false;
                tc_fence_after_sync();
                mma_scores<BF16>(tmem + (k & 1) * 128, fix0, r0_tile(s0));
                if constexpr (!Kd::HAS_Y) {
                    umma_commit_elect(&r0_empty[s0]);  // X was the slot's only reader
                    umma_commit_elect(&s_full[k & 1]);
                }
                return true;
            };
            auto issue_y = [&](int k) -> bool {
                if (!wait_all(&r1_full[0], k & 1, 524)) return false;
                tc_fence_after_sync();
                mma_scores<BF16>(tmem + (k & 1) * 128 + STEP, fix1, r1_tile(0));
                umma_commit_elect(&r1_empty[0]);  // Y was the slot's only reader
                umma_commit_elect(&s_full[k & 1]);
                return true;
            };
            if (ok) ok = issue_x(0) && (!Kd::HAS_Y || issue_y(0));
            for (int k = 0; ok && k < n; ++k) {
                if (k + 1 < n && !(ok = issue_x(k + 1))) break;
                if (!(ok = wait_all(&p_ready[k & 1], (k >> 1) & 1, 530 + (k & 1)))) break;
                tc_fence_after_sync();
                const uint32_t zbuf = tmem + (k & 1) * 128;
                if constexpr (Kd::HAS_Y) {
                    mma_update<BF16>(tmem + C::COL_ACC, zbuf, r0_tile(k & 1), k > 0);  // dK += dZ^T Q / dQ += dZ K
                    umma_commit_elect(&r0_empty[k & 1]);
                    if (k + 1 < n && !(ok = issue_y(k + 1))) break;
                } else {
                    const int s1 = k % Kd::R1_SLOTS;
                    if (!(ok = wait_all(&r1_full[s1], (k / Kd::R1_SLOTS) & 1, 526 + s1))) break;
                    tc_fence_after_sync();
                    mma_update<BF16>(tmem + C::COL_ACC, zbuf, r1_tile(s1), k > 0);  // dV += P^T dO
                    umma_commit_elect(&r1_empty[s1]);
                }
            }
            if (ok) umma_commit_elect(done);
            umma_commit_elect(drain);  // every MMA issued above has finished once this arrives
            const uint64_t g0 = global_timer_ns();
            while (!mbar_try_wait(drain, 0) && global_timer_ns() - g0 < lim) {
            }
        }
    } else {
        // ------------------------------------------------------------ elementwise warps 0-7
        const int quarter = warp & 3, half = warp >> 2;  // TMEM lane quarter, column half
        const int r = quarter * 32 + lane;                // TMEM lane = row of the owned tile
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const int own_pos = own_start + r;
        int row_lo = 0, row_hi = S;  // the positions this row may pair with
        if constexpr (PACKED) {
            const int tok = min(own_pos, S - 1);
            const int s0 = warp_seq_of_token(p.cu_seqlens, p.num_seqs, min(own_start + quarter * 32, S - 1), lane);
            const int sq = lane_seq_of_token(p.cu_seqlens, p.num_seqs, s0, tok, lane);
            row_lo = __ldg(p.cu_seqlens + sq);
            row_hi = __ldg(p.cu_seqlens + sq + 1);
            if (own_pos >= S) row_lo = row_hi = 0;
        }
        const float sl2 = p.scale_log2;
        constexpr float kLog2e = 1.4426950408889634f;
        const int64_t stat_base = (static_cast<int64_t>(b) * p.H + h) * S;
        // -lse*log2(e) and -delta of a query position (-inf and 0 past the end: weight 0)
        auto query_stats = [&](int qpos, float &nl, float &nd) {
            if (qpos < S) {
                nl = -__ldg(p.lse + stat_base + qpos) * kLog2e;
                nd = Kd::HAS_Y ? -__ldg(p.delta + stat_base + qpos) : 0.f;
            } else {
                nl = -INFINITY;
                nd = 0.f;
            }
        };
        // dV, dK: warps 0 and 1 (column half 0, lanes 0..63) publish the statistics of the
        // step's streamed query r; dQ: each row's own statistics
        const bool publisher = Kd::COL_STATS && half == 0 && quarter < 2;
        float my_nl = 0.f, my_nd = 0.f;
        if (publisher) {
            if (n > 0) query_stats(ws + r, my_nl, my_nd);
        } else if (!Kd::COL_STATS) {
            query_stats(own_pos, my_nl, my_nd);
        }
        // this thread's 32 columns [32 half, +32) of step k (X at x_col, Y at x_col + 64):
        // P (dV) or dZ (dK, dQ) packed to 16-bit over the X columns it has read
        auto chunk = [&](auto mask_c, uint32_t x_col, const float *snl, const float *snd, int w0) {
            constexpr bool MASK = decltype(mask_c)::value;
            const int col0 = half * 32;
            uint32_t sv[32], dv[32];
            tmem_ld32(x_col + lane_base + col0, sv);
            if (Kd::HAS_Y) tmem_ld32(x_col + STEP + lane_base + col0, dv);
            tmem_ld_wait();
            tmem_reg_fence<32>(sv);
            if (Kd::HAS_Y) tmem_reg_fence<32>(dv);
            uint32_t zk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int col = col0 + 2 * i;
                float nl0, nl1, nd0 = 0.f, nd1 = 0.f;
                if (Kd::COL_STATS) {
                    const float2 a = *reinterpret_cast<const float2 *>(snl + col);
                    nl0 = a.x, nl1 = a.y;
                    if (Kd::HAS_Y) {
                        const float2 c2 = *reinterpret_cast<const float2 *>(snd + col);
                        nd0 = c2.x, nd1 = c2.y;
                    }
                } else {
                    nl0 = nl1 = my_nl;
                    nd0 = nd1 = my_nd;
                }
                const uint64_t x2 = ffma2(f2(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), f2(sl2, sl2),
                                          f2(nl0, nl1));
                float x0, x1;
                f2_split(x2, x0, x1);
                float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                if constexpr (MASK) {
                    // a pair weighs 0 unless the column lies in the row's sequence (or [0, S))
                    // and, when causal, the key is not past the query
                    const int c0 = w0 + col, c1 = c0 + 1;
                    if (c0 < row_lo || c0 >= row_hi || (CAUSAL && (KEYS ? c0 < own_pos : c0 > own_pos))) p0 = 0.f;
                    if (c1 < row_lo || c1 >= row_hi || (CAUSAL && (KEYS ? c1 < own_pos : c1 > own_pos))) p1 = 0.f;
                }
                if constexpr (Kd::HAS_Y) {
                    const uint64_t z2 = fmul2(f2(p0, p1), fadd2(f2(__uint_as_float(dv[2 * i]), __uint_as_float(dv[2 * i + 1])),
                                                                f2(nd0, nd1)));
                    f2_split(z2, p0, p1);
                }
                zk[i] = pack2x<BF16>(p0, p1);
            }
            tmem_st16(x_col + lane_base + col0, zk);
        };
        for (int k = 0; ok && k < n; ++k) {
            const int w0 = ws + k * STEP;  // position of the step's first streamed row
            const int slot = k % Kd::STAT_SLOTS;
            const float *snl = stats + slot * 2 * STEP, *snd = snl + STEP;
            if (Kd::COL_STATS) {
                // Slot k % 3 was last read at step k - 3; this thread has seen X of step k - 1,
                // issued only after every elementwise thread finished step k - 3.
                if (publisher) {
                    stats[slot * 2 * STEP + r] = my_nl;
                    stats[slot * 2 * STEP + STEP + r] = my_nd;
                    mbar_arrive(&stats_ready[slot]);
                    if (k + 1 < n) query_stats(w0 + STEP + r, my_nl, my_nd);
                }
                if (!(ok = __all_sync(0xffffffffu, wait_bounded(&stats_ready[slot], (k / Kd::STAT_SLOTS) & 1,
                                                                abort_flag, lim, 540 + slot))))
                    break;
            }
            if (!(ok = __all_sync(0xffffffffu, wait_bounded(&s_full[k & 1], (k >> 1) & 1, abort_flag, lim, 550 + (k & 1)))))
                break;
            tc_fence_after_sync();
            const bool row_partial = w0 < row_lo || w0 + STEP > row_hi ||
                                     (CAUSAL && (KEYS ? w0 < own_pos : w0 + STEP - 1 > own_pos));
            const bool masked = __any_sync(0xffffffffu, row_partial);
            const uint32_t x_col = tmem + (k & 1) * 128;
            if (masked)
                chunk(std::integral_constant<bool, true>{}, x_col, snl, snd, w0);
            else
                chunk(std::integral_constant<bool, false>{}, x_col, snl, snd, w0);
            tmem_st_wait();
            tc_fence_before_sync();
            mbar_arrive(&p_ready[k & 1]);
        }
        if (ok && n > 0) ok = __all_sync(0xffffffffu, wait_bounded(done, 0, abort_flag, lim, 560));
        if (ok && n > 0) {
            tc_fence_after_sync();
            const bool store = own_pos < S;
            const int64_t grow = (row0 + own_pos) * p.H + h;  // token row, head
            void *dst = (KIND == KIND_DV) ? p.dv : (KIND == KIND_DK) ? p.dk : p.dq;
            store_acc_row<BF16>(tmem + lane_base + C::COL_ACC, KIND == KIND_DV ? 1.f : p.scale,
                                static_cast<uint8_t *>(dst) + grow * C::D * 2, store, half);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <bool BF16, bool CAUSAL, int KIND, bool PACKED>
cudaError_t launch_kind(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tdo,
                        const BwdParams &p, dim3 grid, cudaStream_t st) {
    using Kd = B256Kind<KIND>;
    auto kern = fa_bwd256_kernel<BF16, CAUSAL, KIND, PACKED>;
    static uint64_t attr_set_mask = 0;  // per-device shared-memory opt-in done
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = uint64_t(1) << (dev & 63);
    if (!(__atomic_load_n(&attr_set_mask, __ATOMIC_ACQUIRE) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Kd::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        __atomic_fetch_or(&attr_set_mask, bit, __ATOMIC_RELEASE);
    }
    kern<<<grid, B256::NUM_THREADS, Kd::SMEM_BYTES, st>>>(tq, tk, tv, tdo, p);
    return cudaGetLastError();
}

template <bool BF16, bool CAUSAL, bool PACKED>
cudaError_t launch_all(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tdo,
                       const BwdParams &p, cudaStream_t st) {
    const int ntiles = (p.seqlen + B256::BM - 1) / B256::BM;
    const dim3 grid(static_cast<unsigned>(p.H), static_cast<unsigned>(ntiles), static_cast<unsigned>(p.B));
    cudaError_t e = launch_kind<BF16, CAUSAL, KIND_DV, PACKED>(tq, tk, tv, tdo, p, grid, st);
    if (e != cudaSuccess) return e;
    e = launch_kind<BF16, CAUSAL, KIND_DK, PACKED>(tq, tk, tv, tdo, p, grid, st);
    if (e != cudaSuccess) return e;
    return launch_kind<BF16, CAUSAL, KIND_DQ, PACKED>(tq, tk, tv, tdo, p, grid, st);
}

}  // namespace

cudaError_t launch_bwd256(bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                          const CUtensorMap &tdo, const BwdParams &p, cudaStream_t st) {
    const bool packed = p.cu_seqlens != nullptr;
    if (bf16) {
        if (packed)
            return causal ? launch_all<true, true, true>(tq, tk, tv, tdo, p, st)
                          : launch_all<true, false, true>(tq, tk, tv, tdo, p, st);
        return causal ? launch_all<true, true, false>(tq, tk, tv, tdo, p, st)
                      : launch_all<true, false, false>(tq, tk, tv, tdo, p, st);
    }
    if (packed)
        return causal ? launch_all<false, true, true>(tq, tk, tv, tdo, p, st)
                      : launch_all<false, false, true>(tq, tk, tv, tdo, p, st);
    return causal ? launch_all<false, true, false>(tq, tk, tv, tdo, p, st)
                  : launch_all<false, false, false>(tq, tk, tv, tdo, p, st);
}

cudaError_t bwd256_error_addrs(int **code, int **where) { return device_error_addrs(code, where); }

}  // namespace fa
