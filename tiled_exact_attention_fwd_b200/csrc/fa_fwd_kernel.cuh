// fa_fwd_kernel.cuh -- exact attention forward, tile by tile, on sm_100a: the kernel template
// and its launcher. Included by fa_fwd.cu (contiguous K/V) and fa_fwd_paged.cu (paged K/V),
// each instantiating one variant, so the two never share a compilation unit (register
// allocation of one variant stays independent of the other's code).
//
// What is computed (page "昇腾CANN跑大模型，FlashAttention这个算子你得认识一下"):
//   section "传统实现到底慢在哪": O = softmax(Q K^T * scale) V;
//   section "分块计算，这事没那么简单": Q, K, V are cut into tiles that stay on chip and
//     only O is written back; each row keeps a running max m and sum l, and a new key
//     tile updates (m, l) and corrects the partial output computed so far;
//   section "昇腾NPU上做了什么特殊优化": the causal mask is fused, key tiles that are fully
//     masked are never loaded or multiplied.
// The packed case (page "IAW 模型 FA2 vs FA3 实测", section 1) is the same loop run inside
// each sequence of cu_seqlens.
//
// B200 design. One CTA owns up to two 128-row query tiles (A, B) of one head of one
// sequence that share every K/V tile it loads (one tile when D = 256, where two O
// accumulators do not fit in TMEM), which halves the K/V bytes moved per MMA flop:
//   warps 0-7   two softmax warpgroups, warpgroup t for tile t; thread (warp w, lane l)
//               owns row 32*(w%4)+l of its tile, the TMEM lane its warp may access. It
//               reads its S row with tcgen05.ld, masks, updates (m, l) with exp2 of scores
//               pre-multiplied by scale*log2(e), writes P (16-bit) over S in TMEM (D <= 64:
//               into its own TMEM columns, so the next S can be computed meanwhile), and
//               when its max grew by more than 2^8 rescales its O row in TMEM (lazy
//               rescale: between rescales every exponent uses the same stale max, which the
//               final 1/l cancels exactly). At the end: O/l -> fp16/bf16 -> global, and the
//               LSE.
//   warp 8      TMA producer: Q tiles once, then K_0, V_0, K_1, V_1, ... through an
//               NS-stage shared-memory ring guarded by full/empty mbarriers. Fused unpad:
//               warps 8, 10 and 11 copy the K/V rows with cp.async instead, each softmax
//               warp copies its own Q rows, 32-row runs of consecutive padded rows move as
//               TMA boxes, and warps 8, 10 and 11 clear the output's padding rows once their
//               copies are issued. Pages under 64 rows: warp 8 moves Q and K by TMA while
//               warps 10 and 11 copy V with cp.async.
//   epilogue    each softmax warp stages its 32 O rows in its tile's Q buffer (free once
//               the tile's MMAs are done) and writes them out as whole rows.
//   warp 9      allocates TMEM; one thread issues every tcgen05.mma:
//                 S_t = Q_t K_j^T   (A = Q_t, B = K_j, both K-major in SMEM, 128B swizzle)
//                 O_t += P_t V_j    (A = P_t read from TMEM, B = V_j MN-major in SMEM)
//               in the ping-pong order QK_A0, QK_B0, PV_A0, QK_A1, PV_B0, QK_B1, ..., so the
//               tensor core works on one tile while the other tile's softmax runs. With a
//               single tile the two S buffers are used alternately by that tile instead
//               (order QK_0, QK_1, PV_0, QK_2, PV_1, ...). A single issuing thread is slower
//               than the tensor core unless each MMA costs it a few instructions, so the
//               operand descriptors are kept as 32-bit words and a k-step adds its offset.
//
// Every pipeline wait is bounded: after `timeout_ns` the waiting thread records
// FA_ERR_TIMEOUT in a device word, raises a CTA-wide abort flag, and all roles drain
// their in-flight copies/MMAs (again with a bound) before TMEM is released.
#pragma once
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
#include "fa_sync.cuh"
#include "fa_seq.cuh"

namespace fa {

template <int D>
struct Cfg {
    static constexpr int BM = 128;                           // query rows per tile (MMA M)
    static constexpr int BN = 128;                           // key rows per tile
    static constexpr int MAXQ = (D == 256) ? 1 : 2;          // query tiles per CTA
    static constexpr int SW = (2 * D >= 128) ? 128 : 2 * D;  // swizzle span in bytes
    static constexpr int SWE = SW / 2;                       // 16-bit elements per swizzle row
    static constexpr int NBLK = D / SWE;                     // column blocks per tile row
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int KV_BYTES = BN * D * 2;
    // The K/V ring moves tiles in UNITS parts (D = 256: 64 KB tiles in two 32 KB parts, so
    // the ring keeps 5 stages): part u of K_j holds column blocks [u*NBLK/UNITS, ...) of all
    // rows, part u of V_j rows [u*BN/UNITS, ...) of all column blocks.
    static constexpr int UNITS = (D == 256) ? 2 : 1;
    static constexpr int UNIT_BYTES = KV_BYTES / UNITS;
    static constexpr int KBLK_PER_UNIT = NBLK / UNITS;   // K column blocks per part
    static constexpr int VROWS_PER_UNIT = BN / UNITS;    // V rows per part
    static constexpr uint32_t LAYOUT = (SW == 128) ? kLayoutSw128 : kLayoutSw64;
    static constexpr uint32_t TMEM_COLS = 512;
    // TMEM columns: S0 at 0, S1 at BN. With D <= 64 two separate P buffers fit (P_COL + 64t)
    // so a tile's next S = QK^T can be computed while its softmax still works on the last
    // one ("decoupled"); otherwise P overwrites the first half of its S buffer.
    static constexpr bool DECOUPLED = (MAXQ == 2) && (D <= 64);
    static constexpr uint32_t P_COL = 2 * BN;
    static constexpr uint32_t O_COL = 2 * BN + (DECOUPLED ? 128 : 0);  // O_A, O_B
    static constexpr int NUM_SOFTMAX_WARPS = 4 * MAXQ;
    static constexpr int WARP_TMA = NUM_SOFTMAX_WARPS;
    static constexpr int WARP_MMA = NUM_SOFTMAX_WARPS + 1;
    // A full last warpgroup (two idle warps) so that per-warpgroup register limits apply.
    static constexpr int NUM_THREADS = 32 * (NUM_SOFTMAX_WARPS + 4);
    // Register split (two query tiles): 384 threads launch with LAUNCH_REGS each; the
    // producer/MMA warpgroup drops to REGS_LOW and the softmax warpgroups rise to REGS_HIGH.
    // The host refuses to launch unless the pool covers the split (it would otherwise wait).
    static constexpr int LAUNCH_REGS = 168;
    static constexpr int REGS_LOW = 56;
    static constexpr int REGS_HIGH = 224;

    static constexpr bool SPLIT_REGS = (MAXQ == 2);
    static_assert(!SPLIT_REGS || 128 * REGS_LOW + 256 * REGS_HIGH <= NUM_THREADS * LAUNCH_REGS, "register split");
    // Column pairs (out of every 4) whose exp2 runs on the FMA pipe instead of MUFU.
    static constexpr int EMU_PAIRS_OF_4 = 0;
    // shared memory map (offsets from a 1024-byte aligned base)
    static constexpr int SMEM_LIMIT = 227 * 1024;
    static constexpr int RESERVED = 1024 /*alignment*/ + 512 /*barriers, misc*/;
    static constexpr int NS_FIT = (SMEM_LIMIT - RESERVED - MAXQ * Q_BYTES) / UNIT_BYTES;
    static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = MAXQ * Q_BYTES;
    static constexpr int OFF_BAR = OFF_KV + NS * UNIT_BYTES;
    // q_full[2], kv_full[NS], kv_empty[NS], s_full[2], p_full[2], pv_done[2], drain, s_free[2], tail
    static constexpr int NUM_BARS = 2 + 2 * NS + 2 + 2 + 2 + 1 + 2 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // TMEM address, abort flag
    static constexpr int USED = OFF_MISC + 16;
    // More than half of the SM's shared memory, so exactly one CTA (and one 512-column
    // TMEM allocation) lives on an SM.
    static constexpr int MIN_SMEM = 120 * 1024;
    static constexpr int SMEM_BYTES = (USED + 1024 > MIN_SMEM) ? USED + 1024 : MIN_SMEM;
    static_assert(NS >= 3, "K/V ring too shallow");
    static_assert(O_COL + MAXQ * D <= TMEM_COLS, "TMEM budget");
    static_assert(USED + 1024 <= SMEM_LIMIT, "shared memory budget");
    static_assert(NUM_BARS * 8 + 16 <= 512, "barrier area");
    static_assert(Q_BYTES % 1024 == 0 && UNIT_BYTES % 1024 == 0, "tile alignment");
    // The MMA thread waits for K_{j+1} while V_j is still held: the ring needs both, plus a part.
    static_assert(NS >= 2 * UNITS + 1, "K/V ring too shallow");
};

// Single-tile order of MMA steps: K0, K1, V0, K2, V1, ..., V_{n-1} (QK runs one tile ahead).
__device__ __forceinline__ void decode_step(int idx, int n, bool &is_v, int &j) {
    if (idx == 0) { is_v = false; j = 0; }
    else if (idx == 2 * n - 1) { is_v = true; j = n - 1; }
    else if (idx & 1) { is_v = false; j = (idx + 1) >> 1; }
    else { is_v = true; j = (idx >> 1) - 1; }
}

template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    return BF16 ? pack2_bf16(lo, hi) : pack2_f16(lo, hi);
}

// 2^x for a pair of scores, evaluated on the FMA pipe instead of the MUFU unit. Cody-Waite
// style reduction x = n + f with n = round(x) taken from the 1.5*2^23 shifter and f in
// [-1/2, 1/2]; 2^f by a degree-3 polynomial fitted with the Remez algorithm for minimax
// relative error (7.5e-5, below the 2^-11 rounding of the 16-bit P it feeds;
// gen_exp2_poly.py); 2^n is added to the exponent field. The float arithmetic runs two
// lanes at a time (add/fma .f32x2). Inputs below -126 are clamped (the result is then ~1e-38
// instead of a smaller number, irrelevant next to the row sum, which is at least 1); it is
// only used on tiles without masked (-inf) scores.
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float &y0, float &y1) {
    constexpr float c3 = 5.517166853e-02f, c2 = 2.426111251e-01f, c1 = 6.932609677e-01f, c0 = 9.999280572e-01f;
    constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
    const uint64_t x2 = f2(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
    const uint64_t t2 = fadd2(x2, f2(kShift, kShift));
    const uint64_t n2 = fadd2(t2, f2(-kShift, -kShift));
    const uint64_t r2 = ffma2(n2, f2(-1.0f, -1.0f), x2);  // x - n, exact
    uint64_t p2 = ffma2(f2(c3, c3), r2, f2(c2, c2));
    p2 = ffma2(p2, r2, f2(c1, c1));
    p2 = ffma2(p2, r2, f2(c0, c0));
    float t0, t1, p0, p1;
    f2_split(t2, t0, t1);
    f2_split(p2, p0, p1);
    y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
    y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// Maximum of an S row held in registers: 8 independent chains of three-input maxima.
template <int BN>
__device__ __forceinline__ float row_max(const uint32_t *sr) {
    float mm[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) mm[k] = fmaxf(__uint_as_float(sr[k]), __uint_as_float(sr[k + 8]));
#pragma unroll
    for (int i = 16; i < BN; i += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mm[k] = fmax3(mm[k], __uint_as_float(sr[i + k]), __uint_as_float(sr[i + 8 + k]));
    return fmaxf(fmax3(mm[0], mm[1], mm[2]), fmax3(fmax3(mm[3], mm[4], mm[5]), mm[6], mm[7]));
}

// For each 64-column chunk of an S row (in registers): p = 2^(s*c + neg_m) (scaling done two
// lanes at a time with fma.f32x2), row sum in four fp32x2 partial sums, pairs packed to
// 16 bits and the chunk stored to TMEM at p_addr. Of every 4 column pairs, EMU use
// exp2_poly, the rest the MUFU ex2. Returns the row sum of this tile.
template <int BN, bool BF16, int EMU>
__device__ __forceinline__ float softmax_chunk_store(const uint32_t *sr, float c, float neg_m, uint32_t p_addr) {
    const uint64_t c2 = f2(c, c), nm2 = f2(neg_m, neg_m);
    uint64_t acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
    for (int cc = 0; cc < BN / 64; ++cc) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int e = cc * 64 + 2 * i;
            const uint64_t x2 = ffma2(f2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), c2, nm2);
            float x0, x1;
            f2_split(x2, x0, x1);
            float p0, p1;
            if ((i & 3) >= 4 - EMU) {
                exp2_poly2(x0, x1, p0, p1);
            } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
            }
            acc[i & 3] = fadd2(acc[i & 3], f2(p0, p1));
            pk[i] = pack2<BF16>(p0, p1);
        }
        tmem_st32(p_addr + cc * 32, pk);
    }
    const uint64_t s2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
    float lo, hi;
    f2_split(s2, lo, hi);
    return lo + hi;
}

// A whole S row (in registers) to packed 16-bit P in registers pk[BN/2]:
// p = 2^(s*c + neg_m), scaling two lanes at a time; returns the row sum.
template <int BN, bool BF16, int EMU>
__device__ __forceinline__ float softmax_row_to_regs(const uint32_t *sr, float c, float neg_m, uint32_t *pk) {
    const uint64_t c2 = f2(c, c), nm2 = f2(neg_m, neg_m);
    uint64_t acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
    for (int i = 0; i < BN / 2; ++i) {
        const uint64_t x2 = ffma2(f2(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), c2, nm2);
        float x0, x1;
        f2_split(x2, x0, x1);
        float p0, p1;
        if ((i & 3) >= 4 - EMU) {
            exp2_poly2(x0, x1, p0, p1);
        } else {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
        }
        acc[i & 3] = fadd2(acc[i & 3], f2(p0, p1));
        pk[i] = pack2<BF16>(p0, p1);
    }
    const uint64_t s2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
    float lo, hi;
    f2_split(s2, lo, hi);
    return lo + hi;
}

// Shared state of one CTA: shared-memory buffers, barriers, TMEM base and the plan.
template <int D>
struct Cta {
    using C = Cfg<D>;
    uint8_t *sQ, *sKV;
    uint64_t *q_full, *kv_full, *kv_empty, *s_full, *p_full, *pv_done, *drain, *s_free;
    uint64_t *tail;  // paged K/V: the one V part that straddles the sequence end lands here first
    volatile int *abort_flag;
    uint32_t tmem;
    uint64_t lim;
    // Tile A visits key tiles [0, nA), tile B [jB0, nB) (nB = 0 when B is absent); key tile j
    // covers tokens kvbase + [j*BN, (j+1)*BN). In dense sequences jB0 = 0; in packed ones
    // B may begin a later sequence. Always jB0 <= nA <= nB, so the two ranges leave no gap.
    int nA, nB, jB0;
    __device__ __forceinline__ int j0(int t) const { return t ? jB0 : 0; }
    __device__ __forceinline__ bool uses(int t, int j) const { return t ? (j >= jB0 && j < nB) : (j < nA); }
    bool two;      // two query tiles (ping-pong) or one (S double-buffered)
    bool dec;      // two tiles with separate P buffers (Cfg::DECOUPLED)
    bool fused;    // Q/K/V tiles written by threads (cp.async), not TMA: fence before the MMA reads them
    // S/P buffer and barrier phase used by tile t at key step j
    __device__ __forceinline__ int buf(int t, int j) const { return two ? t : (j & 1); }
    __device__ __forceinline__ uint32_t sphase(int j) const { return two ? (j & 1) : ((j >> 1) & 1); }
};

// One MMA step of the issuing thread. Returns false when a wait gave up.
template <int D, bool BF16>
// S_t = Q_t K_j^T for key tile j (tile-local step jj = j - j0(t)).
__device__ __forceinline__ bool mma_qk(const Cta<D> &c, int t, int j, bool first_use, bool last_use) {
    using C = Cfg<D>;
    constexpr int BM = C::BM, BN = C::BN, SW = C::SW, NS = C::NS;
    constexpr uint32_t idesc = idesc_f16(BM, BN, BF16, false);
    const int jj = j - c.j0(t);
    if (jj == 0) {
        if (!wait_bounded(&c.q_full[t], 0, c.abort_flag, c.lim, 200 + t)) return false;
        tc_fence_after_sync();
        if (c.fused) fence_proxy_async_smem();
    } else if (c.dec) {
        // S_t is overwritten: the softmax warps must have read the previous S_t
        if (!wait_bounded(&c.s_free[t], (jj - 1) & 1, c.abort_flag, c.lim, 240 + t)) return false;
        tc_fence_after_sync();
    }
    constexpr int UK = D / 16 / C::UNITS;  // k-steps per K part
    // Operand descriptors as 32-bit words: the low word of each tile base, to which a k-step
    // adds its byte offset / 16, and the high word shared by Q and K (one add per operand
    // and k-step keeps the single issuing thread's work per MMA short).
    constexpr uint32_t dhi = smem_desc_hi(8 * SW, C::LAYOUT);
    const uint32_t q_lo = smem_desc_lo(smem_u32(c.sQ + t * C::Q_BYTES), 16);
    const int b = c.buf(t, jj);
    const uint32_t d_tmem = c.tmem + b * BN;
#pragma unroll
    for (int u = 0; u < C::UNITS; ++u) {
        const int U = 2 * j * C::UNITS + u, stage = U % NS;  // ring part holding K_j part u
        if (first_use) {
            if (!wait_bounded(&c.kv_full[stage], (U / NS) & 1, c.abort_flag, c.lim, 220 + stage)) return false;
            tc_fence_after_sync();
            if (c.fused) fence_proxy_async_smem();
        }
        const uint32_t k_lo = smem_desc_lo(smem_u32(c.sKV + stage * C::UNIT_BYTES), 16);
#pragma unroll
        for (int kk = 0; kk < UK; ++kk) {
            const int k = u * UK + kk;
            const uint32_t blk = (k * 32) / SW, off = (k * 32) % SW;
            const uint32_t lb = blk - u * C::KBLK_PER_UNIT;  // column block inside the part
            umma_ss_w(d_tmem, q_lo + ((blk * BM * SW + off) >> 4), k_lo + ((lb * BN * SW + off) >> 4), dhi, idesc,
                      k > 0 ? 1u : 0u);
        }
        if (u + 1 < C::UNITS) {
            if (last_use) umma_commit(&c.kv_empty[stage]);  // release this part early
        } else {
            umma_commit(&c.s_full[b]);  // the softmax waits on S first
            if (last_use) umma_commit(&c.kv_empty[stage]);
        }
    }
    return true;
}

template <int D, bool BF16>
// O_t += P_t V_j for key tile j (tile-local step jj = j - j0(t)).
__device__ __forceinline__ bool mma_pv(const Cta<D> &c, int t, int j, bool first_use, bool last_use) {
    using C = Cfg<D>;
    constexpr int BM = C::BM, BN = C::BN, SW = C::SW, NS = C::NS;
    constexpr uint32_t idesc = idesc_f16(BM, D, BF16, true);
    const int jj = j - c.j0(t);
    const int b = c.buf(t, jj);
    if (!wait_bounded(&c.p_full[b], c.sphase(jj), c.abort_flag, c.lim, 210 + t)) return false;
    tc_fence_after_sync();
    constexpr int UV = BN / 16 / C::UNITS;  // k-steps per V part
    constexpr uint32_t dhi = smem_desc_hi(8 * SW, C::LAYOUT);  // high descriptor word of V
    const uint32_t a_tmem = c.tmem + (c.dec ? C::P_COL + 64 * t : b * BN);
    const uint32_t o_tmem = c.tmem + C::O_COL + t * D;
#pragma unroll
    for (int u = 0; u < C::UNITS; ++u) {
        const int U = (2 * j + 1) * C::UNITS + u, stage = U % NS;  // ring part holding V_j part u
        if (first_use) {
            if (!wait_bounded(&c.kv_full[stage], (U / NS) & 1, c.abort_flag, c.lim, 230 + stage)) return false;
            tc_fence_after_sync();
            if (c.fused) fence_proxy_async_smem();
        }
        const uint32_t v_lo = smem_desc_lo(smem_u32(c.sKV + stage * C::UNIT_BYTES), C::VROWS_PER_UNIT * SW);
#pragma unroll
        for (int kk = 0; kk < UV; ++kk) {
            const int k = u * UV + kk;
            umma_ts_w(o_tmem, a_tmem + k * 8, v_lo + ((kk * 16 * SW) >> 4), dhi, idesc, (jj > 0 || k > 0) ? 1u : 0u);
        }
        if (u + 1 < C::UNITS) {
            if (last_use) umma_commit(&c.kv_empty[stage]);
        } else {
            umma_commit(&c.pv_done[t]);
            if (last_use) umma_commit(&c.kv_empty[stage]);
        }
    }
    return true;
}

// Fused packed path: padded rows of the 32-row groups g0 and g0 + 3 of a copy job over tokens
// [tok0, tok0 + rows), one row per lane; rows past the job or the tokens, and indices outside
// the padded tensor, read as row 0 (never outside q/k/v; the masks ignore such rows).
__device__ __forceinline__ void fused_group_rows(const FwdParams &p, int tok0, int rows, int g0, int lane,
                                                 int64_t (&pr)[2]) {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int g = g0 + 3 * k;
        const int tok = tok0 + g * 32 + lane;
        int64_t r = (g * 32 < rows && tok >= 0 && tok < p.total_tokens) ? __ldg(p.gather + tok) : 0;
        if (r < 0 || r >= p.padded_rows) r = 0;
        pr[k] = r;
    }
}

// Fused packed path: one warp copies the 32-row group g of a tile laid out [NB][rows][SW]
// (the swizzled layout the TMA would produce) with 16-byte cp.async; tile row g*32 + i is
// source row pr of lane i, whose column blocks [b0, b0 + NB) start at src + b0 * SW.
template <int NB, int SW, int D>
__device__ __forceinline__ void copy_group(uint32_t dst, int rows, int g, int64_t pr, const void *src, int b0,
                                           int H, int h, int lane) {
    constexpr int CPB = SW / 16;      // 16-byte chunks per swizzle row (column block)
    constexpr int CPR = NB * CPB;     // chunks per tile row
    const uint8_t *srow = static_cast<const uint8_t *>(src) + b0 * SW;
#pragma unroll 4
    for (int i = 0; i < CPR; ++i) {
        const int idx = i * 32 + lane;
        const int rr = idx / CPR, ch = idx % CPR;
        const int64_t prow = __shfl_sync(0xffffffffu, pr, rr);
        const int r = g * 32 + rr;
        const int blk = ch / CPB, cc = ch % CPB;
        const int swz = (SW == 128) ? (r & 7) : ((r >> 1) & 3);
        cp_async_16(dst + blk * rows * SW + r * SW + ((cc ^ swz) << 4),
                    srow + (prow * H + h) * static_cast<int64_t>(D) * 2 + ch * 16);
    }
}

// Fused packed path: the 32-row group g of a [NB][rows][SW] tile whose row g*32 + i comes from
// padded row pr of lane i. When the 32 padded rows are consecutive (one sequence's tokens in
// a right-padded batch) the group moves as NB TMA boxes of 32 rows, its bytes counted on
// `bar` before this warp's arrivals; otherwise as 16-byte cp.async copies.
template <int NB, int SW, int D>
__device__ __forceinline__ void fetch_group(uint8_t *tile, int rows, int g, int64_t pr, const void *src,
                                            const CUtensorMap *map, int b0, int H, int h, int lane, uint64_t *bar,
                                            uint64_t pol) {
    const int64_t pr0 = __shfl_sync(0xffffffffu, pr, 0);
    if (__all_sync(0xffffffffu, pr == pr0 + lane)) {
        if (lane == 0) {
            mbar_expect_tx(bar, 32 * NB * SW);
#pragma unroll
            for (int b = 0; b < NB; ++b)
                tma_load_3d(tile + (b * rows + g * 32) * SW, map, bar, (b0 + b) * (SW / 2), h, static_cast<int>(pr0), pol);
        }
    } else {
        copy_group<NB, SW, D>(smem_u32(tile), rows, g, pr, src, b0, H, h, lane);
    }
}

// PAGED: K/V read through p.block_table (a separate instantiation, so the producer code of
// the contiguous path stays as small as its register budget wants).
template <int D, bool BF16, bool CAUSAL, bool PAGED>
__global__ void __launch_bounds__(Cfg<D>::NUM_THREADS, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = Cfg<D>;
    constexpr int BM = C::BM, BN = C::BN, SW = C::SW, NS = C::NS;

    const int h = blockIdx.x;
    // Rows of the CTA are tokens qbase + t*128 + r; keys are addressed from token kvbase.
    //  dense : blockIdx.z is the batch entry; the CTA owns query tiles `pair` (two of them
    //          when MAXQ = 2) of that sequence, longest (causal) tiles launched first.
    //  packed: the CTA owns the 128 consecutive packed tokens of tile blockIdx.y, whatever
    //          sequences they belong to; its keys are the union of those sequences' keys
    //          (the device walks cu_seqlens), and each row is masked to its own sequence.
    const bool packed = p.cu_seqlens != nullptr;
    int seq_start = 0, seqlen = 0, q0 = 0, qbase, kvbase, kv_end_A, kv_end_B = 0, kv_start_B = 0;
    bool two = false;
    if (!packed) {
        const int pair = gridDim.y - 1 - blockIdx.y;
        seq_start = blockIdx.z * p.seqlen;
        seqlen = p.seqlen;
        q0 = pair * C::MAXQ * BM;
        if (q0 >= seqlen) return;  // uniform over the CTA, before any barrier exists
        two = (C::MAXQ == 2) && (q0 + BM < seqlen);
        qbase = seq_start + q0;
        kvbase = seq_start;
        kv_end_A = CAUSAL ? min(seqlen, q0 + BM) : seqlen;
        if (two) kv_end_B = CAUSAL ? min(seqlen, q0 + 2 * BM) : seqlen;
    } else {
        qbase = blockIdx.y * C::MAXQ * BM;
        if (qbase >= p.total_tokens) return;
        two = (C::MAXQ == 2) && (qbase + BM < p.total_tokens);
        const int ln = threadIdx.x & 31;
        // With fewer than 64 sequences every warp holds all of cu_seqlens (two entries per
        // lane), so the lookups below are ballots and shuffles after one round of loads;
        // otherwise each lookup is a search with dependent loads.
        const CuWindow win(p.cu_seqlens, p.num_seqs, ln);
        auto seq_of = [win, ln, &p](int tok) {
            return win.ok ? win.seq(tok, ln) : warp_seq_of_token(p.cu_seqlens, p.num_seqs, tok, ln);
        };
        auto cu_at = [win, &p](int s) { return win.ok ? win.at(s) : p.cu_seqlens[s]; };
        const int s_first = seq_of(qbase);
        kvbase = cu_at(s_first);
        // keys of a tile end with its last row's sequence (or the causal limit)
        auto kv_end = [&](int tlast) {
            const int s_last = seq_of(tlast);
            return (CAUSAL ? min(cu_at(s_last + 1), tlast + 1) : cu_at(s_last + 1)) - kvbase;
        };
        kv_end_A = kv_end(min(qbase + BM, p.total_tokens) - 1);
        if (two) {
            kv_end_B = kv_end(min(qbase + 2 * BM, p.total_tokens) - 1);
            kv_start_B = cu_at(seq_of(qbase + BM)) - kvbase;
        }
    }

    Cta<D> c;
    c.two = two;
    c.dec = C::DECOUPLED && c.two;
    // Fused path: stage contents are written by cp.async copies, whose writer cannot fence
    // after they land, so the MMA thread fences the async proxy after its waits. (The paged
    // path's zeroed page tails are fenced by the writing thread itself before it releases
    // the stage.)
    // Paged K/V in pages under 64 rows: TMA boxes that small move too few bytes per SM, so
    // the V parts go by cp.async copies beside the TMA's K parts (the same fence applies).
    const bool copy_pages = PAGED && p.page_size < 64;
    c.fused = p.gather != nullptr || copy_pages;
    c.nA = (kv_end_A + BN - 1) / BN;
    c.nB = c.two ? (kv_end_B + BN - 1) / BN : 0;
    c.jB0 = c.two ? kv_start_B / BN : 0;
    const int n_all = max(c.nA, c.nB);  // key tiles this CTA loads

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    c.sQ = smem + C::OFF_Q;
    c.sKV = smem + C::OFF_KV;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    c.q_full = bars;
    c.kv_full = bars + 2;
    c.kv_empty = c.kv_full + NS;
    c.s_full = c.kv_empty + NS;
    c.p_full = c.s_full + 2;
    c.pv_done = c.p_full + 2;
    c.drain = c.pv_done + 2;
    c.s_free = c.drain + 1;
    c.tail = c.s_free + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    c.abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    c.lim = p.timeout_ns;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int pw = (warp == C::WARP_TMA) ? 0 : warp - C::WARP_MMA;  // copy producer warp 0..2 (8, 10, 11)
    // Fused packed path: the copy warps read the padded rows of their groups of the first key
    // part now, so that load overlaps the barrier and TMEM set-up.
    int64_t first_rows[2] = {0, 0};
    if (p.gather && (warp == C::WARP_TMA || warp > C::WARP_MMA)) fused_group_rows(p, kvbase, BN, pw, lane, first_rows);

    if (threadIdx.x == 0) {
        // ring barriers: one arrival (the TMA lane's), or per copy thread: fused packed path 96
        // (warps 8, 10, 11); pages under 64 rows 65 (the TMA lane + warps 10, 11). Query tiles: the
        // TMA lane's, or the 128 threads of the softmax warpgroup (fused packed path).
        const int fill_arrivals = p.gather ? 96 : (copy_pages ? 65 : 1);
        const int q_arrivals = p.gather ? 128 : 1;
        for (int t = 0; t < 2; ++t) {
            mbar_init(&c.q_full[t], q_arrivals);
            mbar_init(&c.s_full[t], 1);
            mbar_init(&c.p_full[t], 128);
            mbar_init(&c.pv_done[t], 1);
            mbar_init(&c.s_free[t], 4);  // one arrival per softmax warp
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&c.kv_full[s], fill_arrivals);
            mbar_init(&c.kv_empty[s], 1);
        }
        mbar_init(c.drain, 1);
        mbar_init(c.tail, 1);
        *c.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == C::WARP_TMA && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == C::WARP_MMA) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    c.tmem = *tmem_slot;

    if (warp >= C::NUM_SOFTMAX_WARPS) {
        // producer / MMA warpgroup (its two remaining warps idle unless they copy rows)
        if constexpr (C::SPLIT_REGS) regs_dec<C::REGS_LOW>();
        if (warp == C::WARP_TMA || (c.fused && warp > C::WARP_MMA)) {
            // ------------------------------------------------------------ TMA producer
            // (fused packed path and pages under 64 rows: warps 10 and 11 copy rows too)
            const int nq = c.two ? 2 : 1;
            const int loads = 2 * n_all * C::UNITS;  // parts of K_0, V_0, K_1, V_1, ...
            int issued = 0;
            bool tail_issued = false;
            if (PAGED && copy_pages) {
                // Paged K/V in small pages: two engines share the bytes. Warp 8 (lane 0) moves
                // the query tiles and the K parts by TMA, one box per page chunk (chunks wholly
                // past the sequence end are boxes at a negative row: zeros); warps 10 and 11
                // copy the V parts row by row with 16-byte cp.async into the swizzled layout,
                // zero-filling positions past the sequence end (no page is read for them). A
                // ring barrier takes 65 arrivals per part: the TMA lane's (with the K bytes, or
                // a plain arrival on a V part) and one per copy thread (plain on a K part, or
                // once its V copies have landed).
                const int32_t *bt = p.block_table + static_cast<int64_t>(blockIdx.z) * p.max_blocks;
                bool bad_page = false;
                auto page_row = [&](int pos) {  // physical row of key position pos (< seqlen)
                    int pg = __ldg(bt + (pos >> p.page_shift));
                    if (pg < 0 || pg >= p.num_pages) {
                        bad_page = true;
                        pg = 0;
                    }
                    return (static_cast<int64_t>(pg) << p.page_shift) + (pos & (p.page_size - 1));
                };
                if (warp == C::WARP_TMA) {
                    if (lane == 0) {
                        const uint64_t pol_q = l2_policy_evict_first();
                        const uint64_t pol_kv = l2_policy_evict_last();
                        for (int t = 0; t < nq; ++t) {
                            mbar_arrive_expect_tx(&c.q_full[t], C::Q_BYTES);
#pragma unroll
                            for (int b = 0; b < C::NBLK; ++b)
                                tma_load_3d(c.sQ + t * C::Q_BYTES + b * BM * SW, &tm_q, &c.q_full[t], b * C::SWE, h,
                                            qbase + t * BM, pol_q);
                        }
                        const int box = min(p.page_size, BN);
                        for (int U = 0; U < loads; ++U) {
                            const int stage = U % NS;
                            if (U >= NS &&
                                !wait_bounded(&c.kv_empty[stage], ((U / NS) - 1) & 1, c.abort_flag, c.lim, 100 + stage))
                                break;
                            const int L = U / C::UNITS, u = U % C::UNITS, j = L >> 1;
                            if (L & 1) {
                                mbar_arrive(&c.kv_full[stage]);  // V part: copied by warps 10 and 11
                            } else {
                                uint8_t *dst = c.sKV + stage * C::UNIT_BYTES;
                                const int pos0 = j * BN;
                                const int part_valid = seqlen - pos0;
                                mbar_arrive_expect_tx(&c.kv_full[stage], C::UNIT_BYTES);
                                for (int r = 0; r < BN; r += box) {
                                    const int prow = (r < part_valid) ? static_cast<int>(page_row(pos0 + r)) : -box;
                                    for (int b = 0; b < C::KBLK_PER_UNIT; ++b)
                                        tma_load_3d(dst + (b * BN + r) * SW, &tm_k, &c.kv_full[stage],
                                                    (u * C::KBLK_PER_UNIT + b) * C::SWE, h, prow, pol_kv);
                                }
                            }
                            issued = U + 1;
                        }
                    }
                } else {
                    constexpr int CPB = SW / 16;
                    constexpr int CPR = C::NBLK * CPB;  // 16-byte chunks per V row
                    const int w = pw - 1;                // copy warp 0, 1
                    for (int U = 0; U < loads; ++U) {
                        const int stage = U % NS;
                        if (U >= NS &&
                            !wait_bounded(&c.kv_empty[stage], ((U / NS) - 1) & 1, c.abort_flag, c.lim, 100 + stage))
                            break;
                        const int L = U / C::UNITS, u = U % C::UNITS, j = L >> 1;
                        if (!(L & 1)) {
                            mbar_arrive(&c.kv_full[stage]);  // K part: moved by the TMA
                            continue;
                        }
                        // V part u of tile j: rows [pos0, pos0 + VROWS_PER_UNIT), every column block
                        const int pos0 = j * BN + u * C::VROWS_PER_UNIT;
                        const uint32_t dst_u32 = smem_u32(c.sKV + stage * C::UNIT_BYTES);
                        for (int g = w; g * 32 < C::VROWS_PER_UNIT; g += 2) {
                            const int pos = pos0 + g * 32 + lane;
                            const bool valid = pos < seqlen;
                            const int64_t prow = valid ? page_row(pos) : 0;
#pragma unroll 4
                            for (int i = 0; i < CPR; ++i) {
                                const int idx = i * 32 + lane;
                                const int rr = idx / CPR, ch = idx % CPR;
                                const int64_t pr = __shfl_sync(0xffffffffu, prow, rr);
                                const bool ok_row = __shfl_sync(0xffffffffu, valid, rr);
                                const int r = g * 32 + rr;
                                const int blk = ch / CPB, cc = ch % CPB;
                                const int swz = (SW == 128) ? (r & 7) : ((r >> 1) & 3);
                                cp_async_16_zfill(dst_u32 + blk * C::VROWS_PER_UNIT * SW + r * SW + ((cc ^ swz) << 4),
                                                  static_cast<const uint8_t *>(p.v) +
                                                      (pr * p.H + h) * static_cast<int64_t>(D) * 2 + ch * 16,
                                                  ok_row ? 16u : 0u);
                            }
                        }
                        cp_async_mbar_arrive(&c.kv_full[stage]);  // arrives once this thread's copies have landed
                    }
                    cp_async_wait_all();  // nothing of this thread is left in flight at exit
                }
                if (bad_page) record_error(FA_ERR_INDEX, 151);
            } else if (p.gather) {
                // Fused packed path: warps 8, 10 and 11 (96 threads) copy every K/V row from the
                // padded tensor (row = padded row of the packed token; rows past the last token
                // read row 0, which the masks then ignore) with 16-byte cp.async into the same
                // swizzled layout the TMA would produce; each thread's copies arrive on the part's
                // barrier when they land, and the MMA thread fences the async proxy. (The softmax
                // warps copy the query tiles.) The 32-row groups of the ring parts are dealt to
                // the three warps in one running order (group G to warp G % 3), so each warp moves
                // a third of the bytes and holds at most two groups of a part. A warp reads the
                // padded rows of its next part's groups (one coalesced load per group) before it
                // issues this part's copies, so index loads never wait in line.
                auto part_rows = [&](int U, int &tok0, int &rows) {
                    const int L = U / C::UNITS, u = U % C::UNITS, j = L >> 1;
                    tok0 = kvbase + j * BN + ((L & 1) ? u * C::VROWS_PER_UNIT : 0);
                    rows = (L & 1) ? C::VROWS_PER_UNIT : BN;
                };
                const uint64_t pol_kv = l2_policy_evict_last();
                int64_t cur[2], nxt[2] = {first_rows[0], first_rows[1]};  // part 0's rows: read at set-up
                int gU = 0;                                                // running index of part U's first group
                for (int U = 0; U < loads; ++U) {
                    int tok0, rows;
                    part_rows(U, tok0, rows);
                    const int g0 = (pw + 3 - gU % 3) % 3;
                    gU += rows / 32;
                    cur[0] = nxt[0];
                    cur[1] = nxt[1];
                    if (U + 1 < loads) {
                        int tok1, rows1;
                        part_rows(U + 1, tok1, rows1);
                        fused_group_rows(p, tok1, rows1, (pw + 3 - gU % 3) % 3, lane, nxt);
                    }
                    const int stage = U % NS;
                    if (U >= NS &&
                        !wait_bounded(&c.kv_empty[stage], ((U / NS) - 1) & 1, c.abort_flag, c.lim, 100 + stage))
                        break;
                    uint8_t *dst = c.sKV + stage * C::UNIT_BYTES;
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int g = g0 + 3 * k;
                        if (g * 32 >= rows) continue;
                        if ((U / C::UNITS) & 1)
                            fetch_group<C::NBLK, SW, D>(dst, rows, g, cur[k], p.v, &tm_v, 0, p.H, h, lane,
                                                        &c.kv_full[stage], pol_kv);
                        else
                            fetch_group<C::KBLK_PER_UNIT, SW, D>(dst, rows, g, cur[k], p.k, &tm_k,
                                                                 (U % C::UNITS) * C::KBLK_PER_UNIT, p.H, h, lane,
                                                                 &c.kv_full[stage], pol_kv);
                    }
                    cp_async_mbar_arrive(&c.kv_full[stage]);  // arrives once this thread's copies have landed
                    issued = U + 1;
                }
                if (!*c.abort_flag) {
                    // Fused pad, while the attention runs: the packed tokens of this CTA go in
                    // groups of 32 over the three warps; a group owns the padded rows from just
                    // after the previous token's row up to its last token's row (through the end
                    // of the tensor for the last token, from row 0 for the first). Of those, the
                    // rows no token maps to become 0 (the others receive O). Candidates go 32 at
                    // a time; the ones to clear are written whole, several rows per instruction.
                    constexpr int RB = D * 2;                // bytes of one row of one head
                    constexpr int CH = RB / 16;              // 16-byte chunks per row
                    constexpr int LPR = CH < 32 ? CH : 32;  // lanes per row
                    constexpr int RPI = 32 / LPR;            // rows per store instruction
                    const int ch = lane % LPR;
                    uint8_t *const zbase = static_cast<uint8_t *>(p.out) + static_cast<int64_t>(h) * RB + ch * 16;
                    for (int gi = pw; gi < C::MAXQ * 4; gi += 3) {
                        const int64_t tw0 = static_cast<int64_t>(qbase) + gi * 32;
                        if (tw0 >= p.total_tokens) break;
                        const int64_t tw1 = min(tw0 + 32, static_cast<int64_t>(p.total_tokens)) - 1;
                        // padded rows of the group's tokens, sorted (lanes past the last token: +inf)
                        const int64_t g_lane = (tw0 + lane <= tw1) ? __ldg(p.gather + tw0 + lane) : INT64_MAX;
                        const int64_t lo_row = max(int64_t(0), (tw0 == 0) ? int64_t(0) : __ldg(p.gather + tw0 - 1) + 1);
                        const int64_t hi_row =
                            min(p.padded_rows, (tw1 == p.total_tokens - 1) ? p.padded_rows : __ldg(p.gather + tw1));
                        for (int64_t base = lo_row; base < hi_row; base += 32) {
                            const int64_t pr = base + lane;
                            // is pr one of the 32 mapped rows? binary search over the lanes' sorted values
                            int lo = 0;
#pragma unroll
                            for (int step = 16; step >= 1; step >>= 1) {
                                const int64_t v = __shfl_sync(0xffffffffu, g_lane, lo + step - 1);
                                if (v < pr) lo += step;
                            }
                            const bool mapped = __shfl_sync(0xffffffffu, g_lane, lo & 31) == pr;
                            unsigned z = __ballot_sync(0xffffffffu, pr < hi_row && !mapped);  // rows to clear
                            while (z) {
                                int mine = -1;  // the candidate this lane's row slot takes
#pragma unroll
                                for (int sl = 0; sl < RPI; ++sl) {
                                    const int bit = z ? __ffs(z) - 1 : -1;
                                    z &= z - 1;
                                    if (lane / LPR == sl) mine = bit;
                                }
                                if (mine >= 0)
                                    *reinterpret_cast<uint4 *>(zbase + (base + mine) * p.H * RB) = make_uint4(0, 0, 0, 0);
                            }
                        }
                    }
                }
                cp_async_wait_all();  // nothing of this thread is left in flight at exit
                issued = 0;
            } else if (lane == 0) {
                const uint64_t pol_q = l2_policy_evict_first();
                const uint64_t pol_kv = l2_policy_evict_last();
                for (int t = 0; t < nq; ++t) {
                    mbar_arrive_expect_tx(&c.q_full[t], C::Q_BYTES);
#pragma unroll
                    for (int b = 0; b < C::NBLK; ++b)
                        tma_load_3d(c.sQ + t * C::Q_BYTES + b * BM * SW, &tm_q, &c.q_full[t], b * C::SWE, h,
                                    qbase + t * BM, pol_q);
                }
                // Paged K/V: physical row of key position pos (< seqlen) of this batch entry. A
                // page index outside the pool is reported and replaced by page 0 (the result is
                // then wrong, but nothing outside the pool is read).
                const int32_t *bt = PAGED ? p.block_table + static_cast<int64_t>(blockIdx.z) * p.max_blocks : nullptr;
                bool bad_page = false;  // reported once, after the loads
                auto paged_row = [&](int pos) {
                    int pg = __ldg(bt + (pos >> p.page_shift));
                    if (pg < 0 || pg >= p.num_pages) {
                        bad_page = true;
                        pg = 0;
                    }
                    return (pg << p.page_shift) + (pos & (p.page_size - 1));
                };
                for (int U = 0; U < loads; ++U) {
                    const int stage = U % NS;
                    if (U >= NS &&
                        !wait_bounded(&c.kv_empty[stage], ((U / NS) - 1) & 1, c.abort_flag, c.lim, 100 + stage))
                        break;
                    const int L = U / C::UNITS, u = U % C::UNITS, j = L >> 1;
                    uint8_t *dst = c.sKV + stage * C::UNIT_BYTES;
                    if constexpr (PAGED) {
                        // One box per (column block, page-sized row chunk) of the part. Rows of a
                        // sequence's last page past its end hold whatever the pool holds there:
                        // for K they are masked (their scores become -inf), but in V a NaN would
                        // survive P = 0, so the V part that straddles the end lands on `tail`
                        // first, its stray rows are zeroed, and only then is the stage released.
                        const bool is_v = L & 1;
                        const int rows = is_v ? C::VROWS_PER_UNIT : BN;
                        const int box = min(p.page_size, rows);
                        const int pos0 = j * BN + (is_v ? u * C::VROWS_PER_UNIT : 0);
                        const int part_valid = p.seqlen - pos0;  // rows of the part inside the sequence
                        const bool straddles = is_v && part_valid > 0 && part_valid < rows && part_valid % box != 0;
                        uint64_t *bar = straddles ? c.tail : &c.kv_full[stage];
                        tail_issued |= straddles;
                        mbar_arrive_expect_tx(bar, C::UNIT_BYTES);
                        for (int r = 0; r < rows; r += box) {
                            // a chunk wholly past the sequence end (its table entry need not
                            // exist) is a box at a negative row: all fill value (zeros)
                            const int prow = (r < part_valid) ? paged_row(pos0 + r) : -box;
                            if (is_v) {
                                for (int b = 0; b < C::NBLK; ++b)
                                    tma_load_3d(dst + (b * C::VROWS_PER_UNIT + r) * SW, &tm_v, bar, b * C::SWE, h,
                                                prow, pol_kv);
                            } else {
                                for (int b = 0; b < C::KBLK_PER_UNIT; ++b)
                                    tma_load_3d(dst + (b * BN + r) * SW, &tm_k, bar, (u * C::KBLK_PER_UNIT + b) * C::SWE,
                                                h, prow, pol_kv);
                            }
                        }
                        if (straddles) {
                            // at most one such part per CTA (the last V tile): phase 0 of `tail`
                            if (!wait_bounded(c.tail, 0, c.abort_flag, c.lim, 160)) break;
                            const int r1 = min(rows, (part_valid + box - 1) / box * box);  // end of the ragged chunk
                            for (int b = 0; b < C::NBLK; ++b)
                                for (int r = part_valid; r < r1; ++r) {
                                    uint4 *row = reinterpret_cast<uint4 *>(dst + (b * C::VROWS_PER_UNIT + r) * SW);
#pragma unroll
                                    for (int i = 0; i < SW / 16; ++i) row[i] = make_uint4(0u, 0u, 0u, 0u);
                                }
                            fence_proxy_async_smem();  // the zeros, before the tensor core reads them
                            mbar_arrive(&c.kv_full[stage]);
                        }
                    } else {
                        mbar_arrive_expect_tx(&c.kv_full[stage], C::UNIT_BYTES);
                        if (L & 1) {
                            // V part u: rows [u*VROWS_PER_UNIT, ...) of the tile, every column block
#pragma unroll
                            for (int b = 0; b < C::NBLK; ++b)
                                tma_load_3d(dst + b * C::VROWS_PER_UNIT * SW, &tm_v, &c.kv_full[stage], b * C::SWE,
                                            h, kvbase + j * BN + u * C::VROWS_PER_UNIT, pol_kv);
                        } else {
                            // K part u: column blocks [u*KBLK_PER_UNIT, ...) of every tile row
#pragma unroll
                            for (int b = 0; b < C::KBLK_PER_UNIT; ++b)
                                tma_load_3d(dst + b * BN * SW, &tm_k, &c.kv_full[stage],
                                            (u * C::KBLK_PER_UNIT + b) * C::SWE, h, kvbase + j * BN, pol_kv);
                        }
                    }
                    issued = U + 1;
                }
                if (PAGED && bad_page) record_error(FA_ERR_INDEX, 150);
            }
            if (warp == C::WARP_TMA && lane == 0 && *c.abort_flag) {
                // Let the copies already issued land before the CTA's shared memory goes away.
                for (int t = 0; t < nq; ++t) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(&c.q_full[t], 0) && global_timer_ns() - t0 < c.lim) {
                    }
                }
                for (int U = (issued > NS ? issued - NS : 0); U < issued; ++U) {
                    const int stage = U % NS;
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(&c.kv_full[stage], (U / NS) & 1) && global_timer_ns() - t0 < c.lim) {
                    }
                }
                if (tail_issued) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(c.tail, 0) && global_timer_ns() - t0 < c.lim) {
                    }
                }
            }
        } else if (warp == C::WARP_MMA) {
            // ------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                bool ok = true;
                if (!c.two) {
                    const int n = c.nA;
                    for (int idx = 0; ok && idx < 2 * n; ++idx) {
                        bool is_v;
                        int j;
                        decode_step(idx, n, is_v, j);
                        ok = is_v ? mma_pv<D, BF16>(c, 0, j, true, true) : mma_qk<D, BF16>(c, 0, j, true, true);
                    }
                } else if (c.dec) {
                    // Separate P buffers: QK_t(j+1) only waits until the softmax warps have read
                    // S_t(j), so it runs while they compute P_t(j). Order per key tile j:
                    // QK_A(j+1), QK_B(j+1), PV_A(j), PV_B(j), each when that tile uses key tile j.
                    const int nB = c.nB;
                    if (c.uses(0, 0)) ok = mma_qk<D, BF16>(c, 0, 0, true, !c.uses(1, 0));
                    if (ok && c.uses(1, 0)) ok = mma_qk<D, BF16>(c, 1, 0, !c.uses(0, 0), true);
                    for (int j = 0; ok && j < nB; ++j) {
                        const bool a1 = c.uses(0, j + 1), b1 = c.uses(1, j + 1), a0 = c.uses(0, j), b0 = c.uses(1, j);
                        if (a1) ok = mma_qk<D, BF16>(c, 0, j + 1, true, !b1);
                        if (ok && b1) ok = mma_qk<D, BF16>(c, 1, j + 1, !a1, true);
                        if (ok && a0) ok = mma_pv<D, BF16>(c, 0, j, true, !b0);
                        if (ok && b0) ok = mma_pv<D, BF16>(c, 1, j, !a0, true);
                    }
                } else {
                    // Ping-pong over key tiles j: PV_A(j-1), QK_A(j), PV_B(j-1), QK_B(j). A key or
                    // value tile is waited for at its first use and released after its last.
                    const int nB = c.nB;
                    if (c.uses(0, 0)) ok = mma_qk<D, BF16>(c, 0, 0, true, !c.uses(1, 0));
                    if (ok && c.uses(1, 0)) ok = mma_qk<D, BF16>(c, 1, 0, !c.uses(0, 0), true);
                    for (int j = 1; ok && j <= nB; ++j) {
                        const bool ap = c.uses(0, j - 1), bp = c.uses(1, j - 1), ac = c.uses(0, j), bc = c.uses(1, j);
                        if (ap) ok = mma_pv<D, BF16>(c, 0, j - 1, true, !bp);
                        if (ok && ac) ok = mma_qk<D, BF16>(c, 0, j, true, !bc);
                        if (ok && bp) ok = mma_pv<D, BF16>(c, 1, j - 1, !ap, true);
                        if (ok && bc) ok = mma_qk<D, BF16>(c, 1, j, !ac, true);
                    }
                }
                // Every MMA issued above has finished once `drain` completes.
                umma_commit(c.drain);
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(c.drain, 0) && global_timer_ns() - t0 < c.lim) {
                }
            }
    }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        if constexpr (C::SPLIT_REGS) regs_inc<C::REGS_HIGH>();
        const int t = warp >> 2;                      // query tile of this warpgroup
        const int n = t ? c.nB - c.jB0 : c.nA;  // key tiles this warpgroup visits
        const int j0 = c.j0(t);
        const int quarter = warp & 3;                 // TMEM lanes this warp may access
        const int r = quarter * 32 + lane;            // row of the tile == TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        // This row's token and its visible keys [klo, khi), counted from kvbase.
        const int64_t tok = static_cast<int64_t>(qbase) + t * BM + r;
        if (p.gather && (t == 0 || c.two)) {
            // Fused packed path: each warp copies its own 32 rows of query tile t from their
            // padded rows (rows past the last token read row 0); the warpgroup's 128 threads
            // arrive on q_full[t] as their copies land.
            int64_t pr = (tok < p.total_tokens) ? __ldg(p.gather + tok) : 0;
            if (pr < 0 || pr >= p.padded_rows) pr = 0;  // never read outside q
            fetch_group<C::NBLK, SW, D>(c.sQ + t * C::Q_BYTES, BM, quarter, pr, p.q, &tm_q, 0, p.H, h, lane,
                                        &c.q_full[t], l2_policy_evict_first());
            cp_async_mbar_arrive(&c.q_full[t]);
        }
        int klo = 0, khi = 1;
        bool row_ok;
        if (!packed) {
            const int row_pos = q0 + t * BM + r;  // position inside the sequence
            row_ok = row_pos < seqlen;
            khi = CAUSAL ? min(seqlen, row_pos + 1) : seqlen;
        } else {
            row_ok = tok < p.total_tokens;
            const int tw0 = qbase + t * BM + quarter * 32;  // this warp's first token
            int s_lane = 0;
            if (tw0 < p.total_tokens) {  // warp-uniform
                const int s_w = warp_seq_of_token(p.cu_seqlens, p.num_seqs, tw0, lane);
                s_lane = lane_seq_of_token(p.cu_seqlens, p.num_seqs, s_w,
                                           static_cast<int>(min(tok, static_cast<int64_t>(p.total_tokens - 1))), lane);
            }
            if (row_ok) {
                const int s_r = s_lane;
                klo = p.cu_seqlens[s_r] - kvbase;
                khi = (CAUSAL ? min(p.cu_seqlens[s_r + 1], static_cast<int>(tok) + 1) : p.cu_seqlens[s_r + 1]) - kvbase;
            }
        }
        const uint32_t o_col = C::O_COL + t * D;
        const float sc = p.scale_log2;
        float m = -INFINITY;  // running max of scaled scores, log2 units (possibly stale)
        float l = 0.f;        // running sum of 2^(s*sc - m)
        bool ok = n > 0;
        if (c.dec) {
            // Separate P buffer: S_t is released right after it is read, so QK_t(j+1) overlaps
            // this step's exponentials; P_t(j) is written once PV_t(j-1) has consumed P_t(j-1).
            const uint32_t p_addr = c.tmem + lane_base + C::P_COL + 64 * t;
            for (int jj = 0; jj < n; ++jj) {
                const int j = j0 + jj;  // key tile
                if (!__all_sync(0xffffffffu, wait_bounded(&c.s_full[t], jj & 1, c.abort_flag, c.lim, 330 + t))) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                uint32_t sr[BN];
#pragma unroll
                for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32(c.tmem + lane_base + t * BN + cc * 32, sr + cc * 32);
                tmem_ld_wait();
                tmem_reg_fence<BN>(sr);
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&c.s_free[t]);
                const int lo = klo - j * BN, hi = khi - j * BN;  // visible columns of this tile
                const bool need_mask = __any_sync(0xffffffffu, lo > 0 || hi < BN);
                if (need_mask) {
#pragma unroll
                    for (int i = 0; i < BN; ++i)
                        if (i < lo || i >= hi) sr[i] = __float_as_uint(-INFINITY);
                }
                const float m_cand = row_max<BN>(sr) * sc;
                const bool grow = m_cand > m + 8.0f;
                float alpha = 1.f;
                if (grow) {
                    alpha = ex2_approx(m - m_cand);
                    m = m_cand;
                }
                const bool warp_grow = __any_sync(0xffffffffu, grow);
                uint32_t pk[BN / 2];
                // a packed row may not have met any visible key yet (m = -inf): its P is 0
                const float neg_m = (m == -INFINITY) ? 0.f : -m;
                const float rs = need_mask ? softmax_row_to_regs<BN, BF16, 0>(sr, sc, neg_m, pk)
                                           : softmax_row_to_regs<BN, BF16, C::EMU_PAIRS_OF_4>(sr, sc, neg_m, pk);
                l = fmaf(l, alpha, rs);
                if (jj > 0) {
                    if (!__all_sync(0xffffffffu, wait_bounded(&c.pv_done[t], (jj - 1) & 1, c.abort_flag, c.lim, 340 + t))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    if (warp_grow) {
                        const uint64_t a2 = f2(alpha, alpha);
#pragma unroll 1
                        for (int cc = 0; cc < D / 32; ++cc) {
                            uint32_t o[32];
                            tmem_ld32(c.tmem + lane_base + o_col + cc * 32, o);
                            tmem_ld_wait();
                            tmem_reg_fence<32>(o);
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                float lo, hi;
                                f2_split(fmul2(f2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), a2), lo, hi);
                                o[2 * i] = __float_as_uint(lo);
                                o[2 * i + 1] = __float_as_uint(hi);
                            }
                            tmem_st32(c.tmem + lane_base + o_col + cc * 32, o);
                        }
                    }
                }
#pragma unroll
                for (int cc = 0; cc < BN / 64; ++cc) tmem_st32(p_addr + cc * 32, pk + cc * 32);
                tmem_st_wait();
                tc_fence_before_sync();
                mbar_arrive(&c.p_full[t]);
            }
        } else
        for (int jj = 0; jj < n; ++jj) {
            const int j = j0 + jj;  // key tile
            const int b = c.buf(t, jj);
            if (!__all_sync(0xffffffffu, wait_bounded(&c.s_full[b], c.sphase(jj), c.abort_flag, c.lim, 300 + t))) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            uint32_t sr[BN];
#pragma unroll
            for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32(c.tmem + lane_base + b * BN + cc * 32, sr + cc * 32);
            tmem_ld_wait();
            tmem_reg_fence<BN>(sr);
            const int lo = klo - j * BN, hi = khi - j * BN;  // visible columns of this tile
            const bool need_mask = __any_sync(0xffffffffu, lo > 0 || hi < BN);
            if (need_mask) {
#pragma unroll
                for (int i = 0; i < BN; ++i)
                    if (i < lo || i >= hi) sr[i] = __float_as_uint(-INFINITY);
            }
            const float mx = row_max<BN>(sr);
            const float m_cand = mx * sc;
            const bool grow = m_cand > m + 8.0f;
            float alpha = 1.f;
            if (grow) {
                alpha = ex2_approx(m - m_cand);
                m = m_cand;
            }
            const bool warp_grow = __any_sync(0xffffffffu, grow);
            // P = 2^(s*sc - m): written back to TMEM over S, 64 columns at a time.
            // a packed row may not have met any visible key yet (m = -inf): its P is 0
            const float neg_m = (m == -INFINITY) ? 0.f : -m;
            const uint32_t p_addr = c.tmem + lane_base + b * BN;
            const float rs = need_mask ? softmax_chunk_store<BN, BF16, 0>(sr, sc, neg_m, p_addr)  // -inf -> exactly 0
                                       : softmax_chunk_store<BN, BF16, C::EMU_PAIRS_OF_4>(sr, sc, neg_m, p_addr);
            l = fmaf(l, alpha, rs);
            tmem_st_wait();
            if (jj > 0) {
                // O must hold PV(j-1) before it is rescaled. With two tiles, PV_t(j-1) was
                // issued before QK_t(j), and the commit behind s_full only fires once every
                // earlier MMA of the issuing thread has completed, so it is done already. With
                // one tile QK(j) precedes PV(j-1): wait for it (on every step, so this thread
                // never falls two phases behind on pv_done). The final wait after the loop
                // always targets the newest phase, which is correct either way.
                if (!c.two &&
                    !__all_sync(0xffffffffu, wait_bounded(&c.pv_done[t], (jj - 1) & 1, c.abort_flag, c.lim, 310 + t))) {
                    ok = false;
                    break;
                }
                if (warp_grow) {
                    // O holds sum_{j' < j} P_j' V_j'; bring it to the new running max.
                    tc_fence_after_sync();
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t o[32];
                        tmem_ld32(c.tmem + lane_base + o_col + cc * 32, o);
                        tmem_ld_wait();
                        tmem_reg_fence<32>(o);
                        const uint64_t a2 = f2(alpha, alpha);
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float lo, hi;
                            f2_split(fmul2(f2(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1])), a2), lo, hi);
                            o[2 * i] = __float_as_uint(lo);
                            o[2 * i + 1] = __float_as_uint(hi);
                        }
                        tmem_st32(c.tmem + lane_base + o_col + cc * 32, o);
                    }
                    tmem_st_wait();
                }
            }
            tc_fence_before_sync();
            mbar_arrive(&c.p_full[b]);
        }
        if (ok) ok = __all_sync(0xffffffffu, wait_bounded(&c.pv_done[t], (n - 1) & 1, c.abort_flag, c.lim, 320 + t));
        if (ok) {
            tc_fence_after_sync();
            const float inv_l = 1.f / l;
            int64_t orow_idx = (p.gather && row_ok) ? __ldg(p.gather + tok) : tok;  // fused: padded row
            const bool store_ok = row_ok && (!p.gather || (orow_idx >= 0 && orow_idx < p.padded_rows));
            // O leaves through this tile's query buffer, unused now that every MMA of the tile
            // has completed: each warp stages its 32 rows there (a lane writes its row, 16-byte
            // chunk c of row r at chunk c ^ (r & 7), so eight lanes hit eight bank groups), then
            // writes whole rows to global memory, consecutive lanes on consecutive 16 bytes.
            constexpr int RB = D * 2;                // bytes of one row of one head
            constexpr int CH = RB / 16;              // 16-byte chunks per row
            constexpr int XM = (CH < 8 ? CH : 8) - 1;
            constexpr int LPR = CH < 32 ? CH : 32;  // lanes per row in the global stores
            constexpr int RPI = 32 / LPR;            // rows per store instruction
            const uint32_t stage = smem_u32(c.sQ + t * C::Q_BYTES) + quarter * 32 * RB;
            fence_proxy_async_smem();  // the tensor core's reads of Q come before these writes
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tmem_ld32(c.tmem + lane_base + o_col + cc * 32, o);
                tmem_ld_wait();
                tmem_reg_fence<32>(o);
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4)
                    st_shared_v4(stage + lane * RB + (((cc * 4 + v4) ^ (lane & XM)) << 4), w[4 * v4], w[4 * v4 + 1],
                                 w[4 * v4 + 2], w[4 * v4 + 3]);
            }
            __syncwarp();
            {
                const int ch = lane % LPR;
                uint8_t *const obase = static_cast<uint8_t *>(p.out) + static_cast<int64_t>(h) * RB + ch * 16;
#pragma unroll 4
                for (int r0 = 0; r0 < 32; r0 += RPI) {
                    const int rr = r0 + lane / LPR;
                    const int64_t orow_r = __shfl_sync(0xffffffffu, orow_idx, rr);
                    const bool ok_r = __shfl_sync(0xffffffffu, store_ok, rr);
                    const uint4 v = ld_shared_v4(stage + rr * RB + ((ch ^ (rr & XM)) << 4));
                    if (ok_r) *reinterpret_cast<uint4 *>(obase + orow_r * p.H * RB) = v;
                }
            }
            if (row_ok && p.lse) {
                const float lse = m * 0.6931471805599453f + logf(l);
                const int64_t li = packed ? static_cast<int64_t>(h) * p.total_tokens + tok
                                          : (static_cast<int64_t>(blockIdx.z) * p.H + h) * p.seqlen + (tok - seq_start);
                p.lse[li] = lse;
            }
        }
    }

    if (p.gather && warp < C::NUM_SOFTMAX_WARPS) cp_async_wait_all();  // the query copies (abort paths)
    tc_fence_before_sync();
    __syncthreads();
    if (warp == C::WARP_MMA) {
        tc_fence_after_sync();
        tmem_dealloc(c.tmem, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host launchers
template <int D, bool BF16, bool CAUSAL, bool PAGED>
static cudaError_t launch_t(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                            const FwdParams &p, dim3 grid, cudaStream_t st) {
    using C = Cfg<D>;
    auto kern = fa_fwd_kernel<D, BF16, CAUSAL, PAGED>;
    // The shared-memory opt-in is a per-device function attribute; setting it twice is harmless.
    static uint64_t attr_set_mask = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = uint64_t(1) << (dev & 63);
    if (!(__atomic_load_n(&attr_set_mask, __ATOMIC_ACQUIRE) & bit)) {
        if (C::SPLIT_REGS) {
            // The per-warpgroup register split draws on the registers the CTA launches with.
            cudaFuncAttributes fa_attr;
            e = cudaFuncGetAttributes(&fa_attr, kern);
            if (e != cudaSuccess) return e;
            if (fa_attr.numRegs * C::NUM_THREADS < 128 * C::REGS_LOW + 256 * C::REGS_HIGH)
                return cudaErrorInvalidConfiguration;
        }
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        __atomic_fetch_or(&attr_set_mask, bit, __ATOMIC_RELEASE);
    }
    kern<<<grid, C::NUM_THREADS, C::SMEM_BYTES, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace fa
