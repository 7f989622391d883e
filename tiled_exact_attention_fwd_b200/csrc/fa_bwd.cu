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
//          in whole steps (an N = 64 MMA takes nearly as long as an N = 128 one):
//            S = Q_i K_j^T, dP = dO_i V_j^T;  dZ over S;  dQ += dZ K_j
//          S alternates between two TMEM buffers (2 x 128 + dP 128 + dQ D <= 512 columns):
//          S_{j+1} is computed while the elementwise warps work on step j, and after them
//          the tensor core runs dP_{j+1} first (the next step's last input), then dQ += dZ_j
//          K_j and S_{j+2}. K and V stream through separate rings (three K slots: K_j is read
//          from S_j until dQ's update two steps later; two V slots).
// Warps 0-7 do the elementwise work (two threads per TMEM lane = row, each on half of the
// columns), warp 8 lane 0 issues the TMA loads, warp 9 allocates TMEM and issues every MMA
// (the whole warp runs the loop and waits; elect.sync picks the lane that issues each MMA and
// commit). Every wait is bounded.
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
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(TILE_BYTES % 1024 == 0, "tile alignment");
};

// Shared memory and TMEM of one kernel kind. Shared: fixed tiles A0, A1, then
//   dK/dV: ring stages s = 0, 1 holding tiles B0 = Q_i, B1 = dO_i; per-column statistics in
//          two slots;
//   dQ:    K ring of three tiles, V ring of two;
// then barriers and misc. Steps: STEP streamed rows each, S in TMEM buffer k % 2 (column
// 128 (k % 2)); dP next to it (dK/dV: half-steps) or in its own columns (dQ); barriers for
// S-ready / P-ready in NBAR sets used in turn.
template <int D, bool DKDV>
struct BwdKind {
    using C = BwdCfg<D>;
    static constexpr int STEP = DKDV ? 64 : 128;  // streamed rows per step
    static constexpr int PER_TILE = 128 / STEP;
    static constexpr int NBAR = DKDV ? 2 : 1;
    static constexpr int COL_DP_DQ = 256;                         // dQ: dP columns
    static constexpr int COL_ACC0 = DKDV ? 256 : 384;             // dV (dK/dV) or dQ
    static constexpr int COL_ACC1 = 256 + D;                      // dK (dK/dV)
    static constexpr int K_SLOTS = 3, V_SLOTS = 2;                // dQ rings
    static constexpr int OFF_FIX = 0;
    static constexpr int OFF_RING = 2 * C::TILE_BYTES;
    static constexpr int RING_TILES = DKDV ? 4 : K_SLOTS + V_SLOTS;
    static constexpr int OFF_STAT = OFF_RING + RING_TILES * C::TILE_BYTES;  // [slot][-lse*log2e | -delta][128]
    static constexpr int OFF_BAR = OFF_STAT + (DKDV ? 2 * 2 * C::BM * 4 : 0);
    // dK/dV: fix_full, ring_full[2], ring_empty[2], s_full[2], p_ready[2], done, drain, stats_ready[2]
    // dQ:    fix_full, k_full[3], k_empty[3], v_full[2], v_empty[2], s_full, p_ready, done, drain
    static constexpr int NUM_BARS = 16;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int USED = OFF_MISC + 16;
    static constexpr int MIN_SMEM = 120 * 1024;  // one CTA (and one TMEM allocation) per SM
    static constexpr int SMEM_BYTES = (USED + 1024 > MIN_SMEM) ? USED + 1024 : MIN_SMEM;
    static_assert(USED + 1024 <= 227 * 1024, "shared memory budget");
    static_assert(DKDV ? (COL_ACC1 + D <= 512) : (COL_ACC0 + D <= 512), "TMEM budget");
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
    // descriptors as 32-bit words: a k-step adds its byte offset / 16 to the low word
    constexpr uint32_t hi = smem_desc_hi(8 * C::SW, C::LAYOUT);
    const uint32_t a_lo = smem_desc_lo(smem_u32(a), 16), b_lo = smem_desc_lo(smem_u32(b) + u * STEP * C::SW, 16);
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
        const uint32_t blk = (k * 32) / C::SW, off = (k * 32) % C::SW;
        const uint32_t o = (blk * C::BM * C::SW + off) >> 4;
        umma_ss_elect(d_tmem, a_lo + o, b_lo + o, hi, idesc, k > 0 ? 1u : 0u);
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
    constexpr uint32_t hi = smem_desc_hi(8 * C::SW, C::LAYOUT);
    const uint32_t b_lo = smem_desc_lo(smem_u32(b) + u * STEP * C::SW, C::BM * C::SW);
#pragma unroll
    for (int k = 0; k < STEP / 16; ++k)
        umma_ts_elect(d_tmem, a_tmem + k * 8 + (k >= STEP / 32 ? STEP / 4 : 0), b_lo + ((k * 16 * C::SW) >> 4), hi,
                      idesc, (accumulate || k > 0) ? 1u : 0u);
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

// Heads per group in the order the backward CTAs are dealt out (see fa_bwd_kernel).
constexpr int BWD_HEAD_GROUP = 8;

// DKDV: the CTA owns key tile j; fixed A0 = K_j, A1 = V_j; ring B0 = Q_i, B1 = dO_i.
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
    using Kd = BwdKind<D, DKDV>;
    constexpr int BM = C::BM;
    const int b = blockIdx.z, S = p.seqlen;  // packed: S = total tokens
    const int ntiles = (S + BM - 1) / BM;
    // Blocks start in linear order (x fastest), so the (head, tile) pairs are dealt in groups of
    // BWD_HEAD_GROUP heads, tile by tile inside a group (longest work first): the CTAs resident at
    // a time stream the tensors of a few heads, which then stay in L2, instead of those of all.
    int h, tile;
    {
        const int lin = static_cast<int>(blockIdx.x) + p.H * static_cast<int>(blockIdx.y);
        const int g0 = (lin / (BWD_HEAD_GROUP * ntiles)) * BWD_HEAD_GROUP;  // first head of the group
        const int gsize = min(BWD_HEAD_GROUP, p.H - g0);
        const int idx = lin - g0 * ntiles;
        tile = idx / gsize;
        h = g0 + idx % gsize;
    }
    const int own = (DKDV || PACKED) ? tile : ntiles - 1 - tile;
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
    uint8_t *fixA0 = smem + Kd::OFF_FIX, *fixA1 = fixA0 + C::TILE_BYTES;
    float *stats = reinterpret_cast<float *>(smem + Kd::OFF_STAT);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Kd::OFF_BAR);
    uint64_t *fix_full = bars;
    // dK/dV barriers
    uint64_t *ring_full = bars + 1, *ring_empty = bars + 3, *stats_ready = bars + 11;
    // dQ barriers
    uint64_t *k_full = bars + 1, *k_empty = bars + 4, *v_full = bars + 7, *v_empty = bars + 9;
    uint64_t *s_full = DKDV ? bars + 5 : bars + 11, *p_ready = DKDV ? bars + 7 : bars + 12;
    uint64_t *done = DKDV ? bars + 9 : bars + 13, *drain = DKDV ? bars + 10 : bars + 14;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Kd::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Kd::OFF_MISC + 4);
    const uint64_t lim = p.timeout_ns;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto ring_tile = [&](int stage, int which) { return smem + Kd::OFF_RING + (2 * stage + which) * C::TILE_BYTES; };
    auto k_tile = [&](int slot) { return smem + Kd::OFF_RING + slot * C::TILE_BYTES; };
    auto v_tile = [&](int slot) { return smem + Kd::OFF_RING + (Kd::K_SLOTS + slot) * C::TILE_BYTES; };

    if (threadIdx.x == 0) {
        mbar_init(fix_full, 1);
        if (DKDV) {
            for (int s = 0; s < 2; ++s) {
                mbar_init(&ring_full[s], 1);
                mbar_init(&ring_empty[s], 1);
                mbar_init(&stats_ready[s], BM);  // the column-half-0 threads publish 128 columns
                mbar_init(&s_full[s], 1);
                mbar_init(&p_ready[s], C::NUM_EW);
            }
        } else {
            for (int s = 0; s < Kd::K_SLOTS; ++s) {
                mbar_init(&k_full[s], 1);
                mbar_init(&k_empty[s], 1);
            }
            for (int s = 0; s < Kd::V_SLOTS; ++s) {
                mbar_init(&v_full[s], 1);
                mbar_init(&v_empty[s], 1);
            }
            mbar_init(s_full, 1);
            mbar_init(p_ready, C::NUM_EW);
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
            // (bounded) wait for phase `ph` of `bar` before shared memory goes away
            auto settle = [&](uint64_t *bar, uint32_t ph) {
                const uint64_t g1 = global_timer_ns();
                while (!mbar_try_wait(bar, ph) && global_timer_ns() - g1 < lim) {
                }
            };
            if constexpr (DKDV) {
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
                    settle(fix_full, 0);
                    for (int t = (issued > 2 ? issued - 2 : 0); t < issued; ++t) settle(&ring_full[t & 1], (t >> 1) & 1);
                }
            } else {
                // K_t is first read two steps before V_t: order K_0, K_1, V_0, K_2, V_1, ...
                int k_issued = 0, v_issued = 0;
                for (int t = 0; t <= n; ++t) {
                    if (t < n) {
                        const int ks = t % Kd::K_SLOTS;
                        if (t >= Kd::K_SLOTS &&
                            !wait_bounded(&k_empty[ks], ((t / Kd::K_SLOTS) - 1) & 1, abort_flag, lim, 400 + ks))
                            break;
                        mbar_arrive_expect_tx(&k_full[ks], C::TILE_BYTES);
                        load_tile<D>(k_tile(ks), rb0, &k_full[ks], h, static_cast<int>(row0 + ws + t * BM), pol_ring);
                        k_issued = t + 1;
                    }
                    if (t >= 1) {
                        const int tv = t - 1, vs = tv & 1;
                        if (tv >= Kd::V_SLOTS && !wait_bounded(&v_empty[vs], ((tv >> 1) - 1) & 1, abort_flag, lim, 404 + vs))
                            break;
                        mbar_arrive_expect_tx(&v_full[vs], C::TILE_BYTES);
                        load_tile<D>(v_tile(vs), rb1, &v_full[vs], h, static_cast<int>(row0 + ws + tv * BM), pol_ring);
                        v_issued = tv + 1;
                    }
                }
                if (*abort_flag) {
                    settle(fix_full, 0);
                    for (int t = (k_issued > Kd::K_SLOTS ? k_issued - Kd::K_SLOTS : 0); t < k_issued; ++t)
                        settle(&k_full[t % Kd::K_SLOTS], (t / Kd::K_SLOTS) & 1);
                    for (int t = (v_issued > Kd::V_SLOTS ? v_issued - Kd::V_SLOTS : 0); t < v_issued; ++t)
                        settle(&v_full[t & 1], (t >> 1) & 1);
                }
            }
        }
    } else if (warp == C::WARP_MMA) {
        // ------------------------------------------------------------ MMA issuer
        // (every wait below is taken by the whole warp: __all_sync keeps its control flow converged)
        auto wait_all = [&](uint64_t *bar, uint32_t ph, int where) {
            return __all_sync(0xffffffffu, wait_bounded(bar, ph, abort_flag, lim, where));
        };
        if (n > 0) {
            ok = wait_all(fix_full, 0, 410);
            if (ok) tc_fence_after_sync();
            if constexpr (DKDV) {
                // Half-step k: streamed tile t = k / 2, rows [64 u, 64 u + 64) with u = k % 2,
                // TMEM buffer k % 2. Issue order: S/dP(k+1), then (once the elementwise warps
                // are done with k) the accumulator updates of k; the tensor core runs them in
                // that order, so S/dP(k+2) overwrite buffer k % 2 only after the updates of k
                // have read it.
                const int nk = n * Kd::PER_TILE;
                auto issue_sdp = [&](int k) -> bool {
                    const int t = k / Kd::PER_TILE, u = k % Kd::PER_TILE, s = t & 1;
                    if (u == 0) {
                        if (!wait_all(&ring_full[s], (t >> 1) & 1, 420 + s)) return false;
                        tc_fence_after_sync();
                    }
                    const uint32_t buf = tmem + (k & 1) * 128;
                    mma_rows_step<D, BF16, Kd::STEP>(buf, fixA0, ring_tile(s, 0), u);             // S^T
                    mma_rows_step<D, BF16, Kd::STEP>(buf + Kd::STEP, fixA1, ring_tile(s, 1), u);  // dP^T
                    umma_commit_elect(&s_full[k & 1]);
                    return true;
                };
                if (ok) ok = issue_sdp(0);
                for (int k = 0; ok && k < nk; ++k) {
                    if (k + 1 < nk && !(ok = issue_sdp(k + 1))) break;
                    if (!(ok = wait_all(&p_ready[k & 1], (k >> 1) & 1, 430 + (k & 1)))) break;
                    tc_fence_after_sync();
                    const int t = k / Kd::PER_TILE, u = k % Kd::PER_TILE, s = t & 1;
                    const uint32_t buf = tmem + (k & 1) * 128;
                    mma_acc_step<D, BF16, Kd::STEP>(tmem + Kd::COL_ACC0, buf, ring_tile(s, 1), u, k > 0);  // dV += P^T dO
                    mma_acc_step<D, BF16, Kd::STEP>(tmem + Kd::COL_ACC1, buf + Kd::STEP, ring_tile(s, 0), u,
                                                    k > 0);                                        // dK += dZ^T Q
                    if (u == Kd::PER_TILE - 1) umma_commit_elect(&ring_empty[s]);  // both halves of tile t have read it
                }
            } else {
                // Step t: S_t in TMEM buffer t % 2, dP_t in its own columns. Issue order:
                // S_0, dP_0, S_1; then per step t, once the elementwise warps are done with it:
                // dP_{t+1}, dQ += dZ_t K_t, S_{t+2} (into buffer t % 2, after dQ has read dZ_t).
                auto issue_s = [&](int t) -> bool {
                    const int ks = t % Kd::K_SLOTS;
                    if (!wait_all(&k_full[ks], (t / Kd::K_SLOTS) & 1, 420 + ks)) return false;
                    tc_fence_after_sync();
                    mma_rows_step<D, BF16, 128>(tmem + (t & 1) * 128, fixA0, k_tile(ks), 0);  // S = Q K^T
                    return true;
                };
                auto issue_dp = [&](int t) -> bool {
                    const int vs = t & 1;
                    if (!wait_all(&v_full[vs], (t >> 1) & 1, 424 + vs)) return false;
                    tc_fence_after_sync();
                    mma_rows_step<D, BF16, 128>(tmem + Kd::COL_DP_DQ, fixA1, v_tile(vs), 0);  // dP = dO V^T
                    umma_commit_elect(&v_empty[vs]);
                    umma_commit_elect(s_full);  // step t's S and dP are done
                    return true;
                };
                if (ok) ok = issue_s(0) && issue_dp(0);
                if (ok && n > 1) ok = issue_s(1);
                for (int t = 0; ok && t < n; ++t) {
                    if (!(ok = wait_all(p_ready, t & 1, 430))) break;
                    tc_fence_after_sync();
                    if (t + 1 < n && !(ok = issue_dp(t + 1))) break;
                    mma_acc_step<D, BF16, 128>(tmem + Kd::COL_ACC0, tmem + (t & 1) * 128, k_tile(t % Kd::K_SLOTS), 0,
                                               t > 0);  // dQ += dZ K
                    umma_commit_elect(&k_empty[t % Kd::K_SLOTS]);
                    if (t + 2 < n && !(ok = issue_s(t + 2))) break;
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
        // P (or P^T) and dZ for the 32 columns [col0, col0 + 32) of the step (S at TMEM column
        // s_col, dP at dp_col), column c being streamed position w0 + c; MASK applies the
        // causal diagonal and the sequence bounds.
        auto chunk = [&](auto mask_c, uint32_t s_col, uint32_t dp_col, int col0, const float *snl, const float *snd,
                         int w0) {
            constexpr bool MASK = decltype(mask_c)::value;
            uint32_t sv[32], dv[32];
            tmem_ld32(s_col + lane_base + col0, sv);
            tmem_ld32(dp_col + lane_base + col0, dv);
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
            constexpr int HS = Kd::STEP / 2;  // columns per thread and step
            const int pcol = half * HS + (col0 - half * HS) / 2;
            if (DKDV) {
                tmem_st16(s_col + lane_base + pcol, pk);   // P^T over S^T
                tmem_st16(dp_col + lane_base + pcol, zk);  // dZ^T over dP^T
            } else {
                tmem_st16(s_col + lane_base + pcol, zk);  // dZ over S
            }
        };
        for (int k = 0; ok && k < n * Kd::PER_TILE; ++k) {
            const int t = k / Kd::PER_TILE, u = k % Kd::PER_TILE;  // streamed tile, part
            const int w0 = ws + t * BM + u * Kd::STEP;              // position of the step's first streamed row
            const int slot = t & 1;
            const float *snl = stats + slot * 2 * BM + u * Kd::STEP, *snd = snl + BM;
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
            if (!(ok = __all_sync(0xffffffffu, wait_bounded(&s_full[k % Kd::NBAR], (k / Kd::NBAR) & 1, abort_flag,
                                                            lim, 450 + k % Kd::NBAR))))
                break;
            tc_fence_after_sync();
            // does any pair of this warp's rows with the step's positions need a mask?
            const bool row_partial = w0 < row_lo || w0 + Kd::STEP > row_hi ||
                                     (CAUSAL && (DKDV ? w0 < own_pos : w0 + Kd::STEP - 1 > own_pos));
            const bool masked = __any_sync(0xffffffffu, row_partial);
            // this thread's STEP/2 columns [STEP/2 * half, ...) of the step, 32 at a time; the
            // results are stored over columns this thread has already read
            // S of step k in TMEM buffer k % 2; dP next to it (dK/dV) or in its own columns (dQ)
            const uint32_t s_col = tmem + (k & 1) * 128;
            const uint32_t dp_col = DKDV ? s_col + Kd::STEP : tmem + Kd::COL_DP_DQ;
#pragma unroll 1
            for (int c = 0; c < Kd::STEP / 64; ++c) {
                const int col0 = half * (Kd::STEP / 2) + c * 32;
                if (masked)
                    chunk(std::integral_constant<bool, true>{}, s_col, dp_col, col0, snl, snd, w0);
                else
                    chunk(std::integral_constant<bool, false>{}, s_col, dp_col, col0, snl, snd, w0);
            }
            tmem_st_wait();
            tc_fence_before_sync();
            mbar_arrive(&p_ready[k % Kd::NBAR]);
        }
        if (ok && n > 0) ok = __all_sync(0xffffffffu, wait_bounded(done, 0, abort_flag, lim, 460));
        if (ok) {
            tc_fence_after_sync();
            const bool store = own_pos < S;
            const int64_t grow = (row0 + own_pos) * p.H + h;  // token row, head
            if (DKDV) {
                store_row<D, BF16>(tmem + lane_base + Kd::COL_ACC0, 1.f, static_cast<uint8_t *>(p.dv) + grow * D * 2,
                                   store, half);
                store_row<D, BF16>(tmem + lane_base + Kd::COL_ACC1, p.scale, static_cast<uint8_t *>(p.dk) + grow * D * 2,
                                   store, half);
            } else {
                store_row<D, BF16>(tmem + lane_base + Kd::COL_ACC0, p.scale, static_cast<uint8_t *>(p.dq) + grow * D * 2,
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
    using Kd = BwdKind<D, DKDV>;
    auto kern = fa_bwd_kernel<D, BF16, CAUSAL, DKDV, PACKED>;
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
    kern<<<grid, C::NUM_THREADS, Kd::SMEM_BYTES, st>>>(tq, tk, tv, tdo, p);
    return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t launch_delta(const BwdParams &p, cudaStream_t st) {
    const int rows = p.B * p.seqlen;
    const int64_t items = static_cast<int64_t>(rows) * p.H;
    const int threads = 256;
    int64_t blocks = (items * (D / 8) + threads - 1) / threads;  // one (row, head) per D/8 lanes
    if (blocks > 148 * 16) blocks = 148 * 16;
    bwd_delta_kernel<D, BF16><<<static_cast<unsigned>(blocks), threads, 0, st>>>(p.out, p.dout, p.delta, rows, p.H,
                                                                                 p.seqlen);
    return cudaGetLastError();
}

template <int D, bool BF16>
cudaError_t launch_bwd_d(bool causal, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                         const CUtensorMap &tdo, const BwdParams &p, cudaStream_t st) {
    cudaError_t e = launch_delta<D, BF16>(p, st);
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
        case 256: {
            const cudaError_t e = bf16 ? launch_delta<256, true>(p, st) : launch_delta<256, false>(p, st);
            if (e != cudaSuccess) return e;
            return launch_bwd256(bf16, causal, tq, tk, tv, tdo, p, st);
        }
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t bwd_error_addrs(int **code, int **where) { return device_error_addrs(code, where); }

}  // namespace fa
