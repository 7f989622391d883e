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
//   warp 9      allocates TMEM and issues every tcgen05.mma (the whole warp runs the loop and
//               waits; elect.sync picks the lane that issues each MMA and commit):
//                 S_t = Q_t K_j^T   (A = Q_t, B = K_j, both K-major in SMEM, 128B swizzle)
//                 O_t += P_t V_j    (A = P_t read from TMEM, B = V_j MN-major in SMEM)
//               in the ping-pong order QK_A0, QK_B0, PV_A0, QK_A1, PV_B0, QK_B1, ..., so the
//               tensor core works on one tile while the other tile's softmax runs. With a
//               single tile the two S buffers are used alternately by that tile instead
//               (order QK_0, QK_1, PV_0, QK_2, PV_1, ...). The issuing lane is slower than the
//               tensor core unless each MMA costs it a few instructions, so the operand
//               descriptors are kept as 32-bit words and a k-step adds its offset.
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
    // producer/MMA warpgroup drops to regs_low and the softmax warpgroups rise to regs_high.
    // The persistent (dense) kernel keeps more state in its producer and MMA loops than the
    // packed one, so it moves 8 registers per softmax thread over to them.
    // The host refuses to launch unless the pool covers the split (it would otherwise wait).
    static constexpr int LAUNCH_REGS = 168;
    static constexpr int regs_low(bool packed) { return packed ? 56 : 72; }
    static constexpr int regs_high(bool packed) { return packed ? 224 : 216; }

    static constexpr bool SPLIT_REGS = (MAXQ == 2);
    static_assert(!SPLIT_REGS || 128 * regs_low(true) + 256 * regs_high(true) <= NUM_THREADS * LAUNCH_REGS,
                  "register split");
    static_assert(!SPLIT_REGS || 128 * regs_low(false) + 256 * regs_high(false) <= NUM_THREADS * LAUNCH_REGS,
                  "register split");
    // shared memory map (offsets from a 1024-byte aligned base)
    static constexpr int SMEM_LIMIT = 227 * 1024;
    static constexpr int RESERVED = 1024 /*alignment*/ + 512 /*barriers, misc*/;
    static constexpr int NS_FIT = (SMEM_LIMIT - RESERVED - MAXQ * Q_BYTES) / UNIT_BYTES;
    static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = MAXQ * Q_BYTES;
    static constexpr int OFF_BAR = OFF_KV + NS * UNIT_BYTES;
    // q_full[2], kv_full[NS], kv_empty[NS], s_full[2], p_full[2], pv_done[2], drain, s_free[2], tail, q_free[2],
    // q_peer, kv_peer[NS] (CTA pairs: the other CTA's copies have landed), item_full[QSLOTS],
    // item_empty[QSLOTS] (the item queue's ring)
    static constexpr int QSLOTS = 4;
    static constexpr int NUM_BARS = 2 + 2 * NS + 2 + 2 + 2 + 1 + 2 + 1 + 2 + 1 + NS + 2 * QSLOTS;
    // TMEM address, abort flag, the item queue's ring (QSLOTS item indices)
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int MISC_BYTES = 8 + 4 * QSLOTS;
    static constexpr int USED = OFF_MISC + MISC_BYTES;
    // More than half of the SM's shared memory, so exactly one CTA (and one 512-column
    // TMEM allocation) lives on an SM.
    static constexpr int MIN_SMEM = 120 * 1024;
    static constexpr int SMEM_BYTES = (USED + 1024 > MIN_SMEM) ? USED + 1024 : MIN_SMEM;
    static_assert(NS >= 3, "K/V ring too shallow");
    static_assert(O_COL + MAXQ * D <= TMEM_COLS, "TMEM budget");
    static_assert(USED + 1024 <= SMEM_LIMIT, "shared memory budget");
    static_assert(NUM_BARS * 8 + MISC_BYTES <= 512, "barrier area");
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
// lanes at a time with fma.f32x2, exp2 on the MUFU unit), row sum in four fp32x2 partial sums,
// pairs packed to 16 bits and the chunk stored to TMEM at p_addr. Returns the row sum of this
// tile.
template <int BN, bool BF16>
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
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
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
template <int BN, bool BF16>
__device__ __forceinline__ float softmax_row_to_regs(const uint32_t *sr, float c, float neg_m, uint32_t *pk) {
    const uint64_t c2 = f2(c, c), nm2 = f2(neg_m, neg_m);
    uint64_t acc[4] = {f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f), f2(0.f, 0.f)};
#pragma unroll
    for (int i = 0; i < BN / 2; ++i) {
        const uint64_t x2 = ffma2(f2(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), c2, nm2);
        float x0, x1;
        f2_split(x2, x0, x1);
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        acc[i & 3] = fadd2(acc[i & 3], f2(p0, p1));
        pk[i] = pack2<BF16>(p0, p1);
    }
    const uint64_t s2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
    float lo, hi;
    f2_split(s2, lo, hi);
    return lo + hi;
}

// Shared state of one CTA: shared-memory buffers, barriers, TMEM base, the current work item,
// and running counts that carry every barrier's phase from one work item to the next (a CTA
// of the dense path runs several items one after another).
template <int D>
struct Cta {
    using C = Cfg<D>;
    uint8_t *sQ, *sKV;
    uint64_t *q_full, *kv_full, *kv_empty, *s_full, *p_full, *pv_done, *drain, *s_free, *q_free;
    uint64_t *tail;  // paged K/V: the V part that straddles a sequence end lands here first
    uint64_t *q_peer, *kv_peer;  // CTA pairs (CTA 0): the other CTA's Q tile / ring part has landed
    uint64_t *item_full, *item_empty;  // item queue: a ring slot holds this CTA's next item / is free again
    volatile int *items;               // item queue: the ring of item indices (-1: no more items)
    volatile int *abort_flag;
    uint32_t tmem;
    uint64_t lim;
    bool dec;     // separate P buffers (Cfg::DECOUPLED)
    bool single;  // one query tile per CTA (Cfg::MAXQ == 1): its S alternates between two buffers
    bool fused;   // Q/K/V tiles written by threads (cp.async), not TMA: fence before the MMA reads them
    bool pair;    // one query tile in each CTA of a 2-CTA cluster, whose MMAs CTA 0 issues for both
    uint32_t rank;  // rank of this CTA in its pair
    // The current work item: query tiles A (and B) of head h; their rows are tokens qbase + t*128
    // + r, keys are addressed from token kvbase. Dense: batch entry b, rows from position q0 of
    // the sequence that starts at token seq_start. Tile A visits key tiles [0, nA), tile B
    // [jB0, nB) (nB = jB0 = 0 when B is absent); key tile j covers tokens kvbase + [j*BN,
    // (j+1)*BN). In dense sequences jB0 = 0; in packed ones B may begin a later sequence. Always
    // jB0 <= nA <= nB when B is present, so the two ranges leave no gap.
    int h, b, q0, seq_start, seqlen, qbase, kvbase;
    int nA, nB, jB0;
    bool two;  // tile B present
    // Items done so far: K/V ring parts loaded (u0), key steps of tile t (g0(t)), Q_t loads (nq(t)).
    // Scalars, not arrays: an array indexed by the runtime tile index would put the whole
    // struct in local memory.
    int u0, g0a, g0b, nqa, nqb;
    __device__ __forceinline__ int g0(int t) const { return t ? g0b : g0a; }
    __device__ __forceinline__ int nq(int t) const { return t ? nqb : nqa; }
    __device__ __forceinline__ int j0(int t) const { return t ? jB0 : 0; }
    __device__ __forceinline__ int steps(int t) const { return t ? nB - jB0 : nA; }
    __device__ __forceinline__ bool uses(int t, int j) const { return t ? (j >= jB0 && j < nB) : (j < nA); }
    // ring parts of the item (CTA pairs: half of K_j, then half of V_j, one part each)
    __device__ __forceinline__ int loads() const { return pair ? 2 * nA : 2 * max(nA, nB) * C::UNITS; }
    // S/P buffer of tile t at its running key step gs, and that buffer's barrier phase
    __device__ __forceinline__ int buf(int t, int gs) const { return single ? (gs & 1) : t; }
    __device__ __forceinline__ uint32_t sphase(int gs) const { return single ? ((gs >> 1) & 1) : (gs & 1); }
    __device__ __forceinline__ void advance() {
        u0 += loads();
        g0a += nA;
        g0b += nB - jB0;
        nqa += 1;
        nqb += two ? 1 : 0;
    }
};

// The dense work items: (batch entry, head, group of MAXQ query tiles), B*H*npairs in all, dealt
// to the G CTAs in rounds of one item each. The (batch entry, head) pairs form p.num_groups groups
// of p.head_group, each taking p.group_rounds rounds. Inside a group, causal items go longest
// first (query-tile group descending, all heads of the group at each step) and non-causal ones
// head by head (the groups of one head consecutive, so CTAs running together share its K/V in
// L2). Each round runs forward or backward over the CTAs (a snake, so that with longest-first
// items every CTA gets a similar total), and each group starts the snake a quarter of the grid
// further on. Returns false when CTA `cta` has no item in round rd. GROUPED: more than one group
// (a separate instantiation: the single-group arithmetic, which every role runs at every item,
// stays as short as it can be).
template <bool CAUSAL, bool GROUPED>
__device__ __forceinline__ bool dense_item_at(const FwdParams &p, int rd, int G, int cta, int &pair, int &bh) {
    if (!GROUPED) {
        const int w = rd * G + ((rd & 1) ? G - 1 - cta : cta);
        if (w >= p.num_items) return false;
        if (CAUSAL) {
            const int bhc = p.batch * p.H, q = w / bhc;
            pair = p.npairs - 1 - q;
            bh = w - q * bhc;
        } else {
            bh = w / p.npairs;
            pair = w - bh * p.npairs;
        }
        return true;
    }
    const int g = rd / p.group_rounds, r = rd - g * p.group_rounds;
    const int g0 = g * p.head_group;
    const int gb = min(p.head_group, p.batch * p.H - g0);  // pairs in this group
    const int slot = (cta + g * (G / 4)) % G;
    const int within = r * G + ((r & 1) ? G - 1 - slot : slot);
    if (within >= gb * p.npairs) return false;
    if (CAUSAL) {
        pair = p.npairs - 1 - within / gb;
        bh = g0 + within % gb;
    } else {
        pair = within % p.npairs;
        bh = g0 + within / p.npairs;
    }
    return true;
}

// PAIR: item `pair` is query tiles 2*pair (CTA 0) and 2*pair + 1 (CTA 1) of the head, run as
// one 256-row tile; both CTAs visit the key tiles of the longer one (CTA 0's rows mask the
// last one away when causal).
template <int D, bool CAUSAL, bool PAIR = false>
__device__ __forceinline__ void set_dense_item(Cta<D> &c, const FwdParams &p, int pair, int bh) {
    using C = Cfg<D>;
    c.b = bh / p.H;
    c.h = bh % p.H;
    c.seqlen = p.seqlen;
    c.seq_start = c.b * p.seqlen;
    c.q0 = PAIR ? (2 * pair + static_cast<int>(c.rank)) * C::BM : pair * C::MAXQ * C::BM;
    c.two = (C::MAXQ == 2) && (c.q0 + C::BM < p.seqlen);
    c.qbase = c.seq_start + c.q0;
    c.kvbase = c.seq_start;
    const int end_a = CAUSAL ? min(p.seqlen, (PAIR ? (2 * pair + 2) * C::BM : c.q0 + C::BM)) : p.seqlen;
    const int end_b = CAUSAL ? min(p.seqlen, c.q0 + 2 * C::BM) : p.seqlen;
    c.nA = (end_a + C::BN - 1) / C::BN;
    c.nB = c.two ? (end_b + C::BN - 1) / C::BN : 0;
    c.jB0 = 0;
}

// Head, batch entry, first query position and first query token of this CTA's item at round r
// (which must exist), derived afresh: packed inputs from the block index, dense ones as
// dense_item_at does. Keeps these out of the registers that live through an item's key steps.
template <int D, bool CAUSAL, bool GROUPED, bool PAIR = false>
__device__ __forceinline__ void item_coords(const FwdParams &p, int r, bool persistent, int &h, int &b, int &q0,
                                            int &qbase) {
    using C = Cfg<D>;
    if (!persistent) {
        h = blockIdx.x;
        b = 0;
        q0 = 0;
        qbase = blockIdx.y * C::MAXQ * C::BM;
        return;
    }
    int pair = 0, bh = 0;
    if (PAIR)
        dense_item_at<CAUSAL, GROUPED>(p, r, gridDim.x >> 1, blockIdx.x >> 1, pair, bh);
    else
        dense_item_at<CAUSAL, GROUPED>(p, r, gridDim.x, blockIdx.x, pair, bh);
    b = bh / p.H;
    h = bh % p.H;
    q0 = PAIR ? (2 * pair + static_cast<int>(cluster_ctarank())) * C::BM : pair * C::MAXQ * C::BM;
    qbase = b * p.seqlen + q0;
}

// Moves to this CTA's next work item at round r or later (r is advanced past rounds without
// one); false once there is none. Packed inputs: the one item set up front, at round 0. Called
// again with the same r it sets the same item.
template <int D, bool CAUSAL, bool GROUPED, bool PAIR = false>
__device__ __forceinline__ bool next_item(Cta<D> &c, const FwdParams &p, int &r, bool persistent) {
    if (!persistent) return r == 0;
    // pairs: the rounds deal items to the clusters of two CTAs
    const int G = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    const int cta = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int rounds = p.num_groups * p.group_rounds;
    for (; r < rounds; ++r) {
        int pair, bh;
        if (dense_item_at<CAUSAL, GROUPED>(p, r, G, cta, pair, bh)) {
            set_dense_item<D, CAUSAL, PAIR>(c, p, pair, bh);
            return true;
        }
    }
    return false;
}

// ------------------------------------------------------------------ item queue
// Dense inputs over more than one round (contiguous K/V, D <= 128) take their items from a
// counter in global memory instead of round by round: item index w runs over the order the
// rounds use (groups in turn; causal items longest first), and a CTA that finishes early takes
// the next index, so CTAs that run faster than others (their place on the chip, the L2 slices
// they read) end together. The producer's TMA lane takes each index when it needs it
// (atomicAdd) and puts it into a ring of QSLOTS slots in shared memory (item_full); the MMA and
// softmax warps read it from there and free the slot (item_empty, one arrival per warp) when
// they move on to their next item.

// (query-tile group, batch-entry-and-head) of item index w, in the rounds' order.
template <bool CAUSAL, bool GROUPED>
__device__ __forceinline__ void dense_item_of(const FwdParams &p, int w, int &pair, int &bh) {
    if (!GROUPED) {
        if (CAUSAL) {
            const int bhc = p.batch * p.H, q = w / bhc;
            pair = p.npairs - 1 - q;
            bh = w - q * bhc;
        } else {
            bh = w / p.npairs;
            pair = w - bh * p.npairs;
        }
        return;
    }
    const int per = p.head_group * p.npairs;  // items of a whole group
    const int g = w / per, within = w - g * per;
    const int g0 = g * p.head_group;
    const int gb = min(p.head_group, p.batch * p.H - g0);  // (batch entry, head) pairs of group g
    pair = p.npairs - 1 - within / gb;                     // head groups are causal only
    bh = g0 + within % gb;
}

// A reading warp's n-th item (whole warp): frees the slot of item n - 1, then waits for slot
// n % QSLOTS. False at the end of the items or when the wait gave up.
template <int D, bool CAUSAL, bool GROUPED>
__device__ __forceinline__ bool take_item(Cta<D> &c, const FwdParams &p, int n) {
    using C = Cfg<D>;
    if (n > 0) {
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(&c.item_empty[(n - 1) % C::QSLOTS]);
    }
    if (!wait_bounded(&c.item_full[n % C::QSLOTS], (n / C::QSLOTS) & 1, c.abort_flag, c.lim, 170)) return false;
    const int w = c.items[n % C::QSLOTS];
    if (w < 0) return false;
    int pair, bh;
    dense_item_of<CAUSAL, GROUPED>(p, w, pair, bh);
    set_dense_item<D, CAUSAL>(c, p, pair, bh);
    return true;
}

// The producer's TMA lane: takes this CTA's n-th item (its own index for the first, else the
// next index of the counter) and publishes it. The index is taken only now, when the lane has
// issued every load of the previous item (a few key steps before the CTA finishes it), not
// earlier: a CTA holding a reserved item while another one runs out of work is what unbalances
// the end of a launch. The lane is far enough ahead of the MMAs for the atomic's round trip.
template <int D, bool CAUSAL, bool GROUPED>
__device__ __forceinline__ bool fetch_item(Cta<D> &c, const FwdParams &p, int n) {
    using C = Cfg<D>;
    const int slot = n % C::QSLOTS;
    // the slot is free once every reading warp has moved past item n - QSLOTS
    if (n >= C::QSLOTS &&
        !wait_bounded(&c.item_empty[slot], ((n / C::QSLOTS) - 1) & 1, c.abort_flag, c.lim, 175))
        return false;
    // indices below gridDim.x are the CTAs' first items; the counter hands out the rest
    int w = (n == 0) ? static_cast<int>(blockIdx.x) : static_cast<int>(gridDim.x) + atomicAdd(p.queue, 1);
    if (w >= p.num_items) w = -1;
    c.items[slot] = w;
    mbar_arrive(&c.item_full[slot]);  // release: the readers see the index after their wait
    if (w < 0) return false;
    int pair, bh;
    dense_item_of<CAUSAL, GROUPED>(p, w, pair, bh);
    set_dense_item<D, CAUSAL>(c, p, pair, bh);
    return true;
}

// CTA pairs (D = 256): both CTAs of a cluster run the same items. CTA 0's producer lane takes
// them and publishes each to both rings (CTA 1's slot written through its shared::cluster
// address, then a release arrival on CTA 1's item_full); the reading warps of both CTAs free
// a slot on CTA 0's item_empty (remote arrivals from CTA 1). Every wait is cluster-scope.
template <int D, bool CAUSAL, bool GROUPED>
__device__ __forceinline__ bool fetch_item_pair(Cta<D> &c, const FwdParams &p, int n) {
    using C = Cfg<D>;
    const int slot = n % C::QSLOTS;
    if (n >= C::QSLOTS &&
        !wait_bounded_cluster(&c.item_empty[slot], ((n / C::QSLOTS) - 1) & 1, c.abort_flag, c.lim, 176))
        return false;
    // a cluster's first item is its own index; the counter hands out the rest
    const int clusters = static_cast<int>(gridDim.x >> 1);
    int w = (n == 0) ? static_cast<int>(blockIdx.x >> 1) : clusters + atomicAdd(p.queue, 1);
    if (w >= p.num_items) w = -1;
    c.items[slot] = w;
    mbar_arrive(&c.item_full[slot]);
    st_cluster_u32(mapa_shared(const_cast<int *>(c.items + slot), 1), static_cast<uint32_t>(w));
    mbar_arrive_cluster(mapa_shared(&c.item_full[slot], 1));  // release: orders the store above
    if (w < 0) return false;
    int pair, bh;
    dense_item_of<CAUSAL, GROUPED>(p, w, pair, bh);
    set_dense_item<D, CAUSAL, true>(c, p, pair, bh);
    return true;
}

// A reading role's n-th item in a CTA pair: a whole warp, or one lane (one_lane: the lane-0
// roles, CTA 1's producer and reporter).
template <int D, bool CAUSAL, bool GROUPED>
__device__ __forceinline__ bool take_item_pair(Cta<D> &c, const FwdParams &p, int n, bool one_lane) {
    using C = Cfg<D>;
    if (n > 0) {
        if (!one_lane) __syncwarp();
        if (one_lane || (threadIdx.x & 31) == 0) {
            uint64_t *bar = &c.item_empty[(n - 1) % C::QSLOTS];
            if (c.rank == 0)
                mbar_arrive(bar);
            else
                mbar_arrive_cluster(mapa_shared(bar, 0));
        }
    }
    if (!wait_bounded_cluster(&c.item_full[n % C::QSLOTS], (n / C::QSLOTS) & 1, c.abort_flag, c.lim, 171))
        return false;
    const int w = c.items[n % C::QSLOTS];
    if (w < 0) return false;
    int pair, bh;
    dense_item_of<CAUSAL, GROUPED>(p, w, pair, bh);
    set_dense_item<D, CAUSAL, true>(c, p, pair, bh);
    return true;
}

// S_t = Q_t K_j^T for key tile j (tile-local step jj = j - j0(t)); after the tile's last QK of
// the item, q_free[t] fires once the MMAs reading Q_t are done. Returns false when a wait gave up.
template <int D, bool BF16>
__device__ __forceinline__ bool mma_qk(const Cta<D> &c, int t, int j, bool first_use, bool last_use) {
    using C = Cfg<D>;
    constexpr int BM = C::BM, BN = C::BN, SW = C::SW, NS = C::NS;
    constexpr uint32_t idesc = idesc_f16(BM, BN, BF16, false);
    const int jj = j - c.j0(t);
    const int gs = c.g0(t) + jj;  // running key step of tile t
    if (jj == 0) {
        if (!__all_sync(0xffffffffu, wait_bounded(&c.q_full[t], c.nq(t) & 1, c.abort_flag, c.lim, 200 + t)))
            return false;
        tc_fence_after_sync();
        if (c.fused) fence_proxy_async_smem();
    }
    if (c.dec && gs > 0) {
        // S_t is overwritten: the softmax warps must have read the previous S_t
        if (!__all_sync(0xffffffffu, wait_bounded(&c.s_free[t], (gs - 1) & 1, c.abort_flag, c.lim, 240 + t)))
            return false;
        tc_fence_after_sync();
    }
    constexpr int UK = D / 16 / C::UNITS;  // k-steps per K part
    // Operand descriptors as 32-bit words: the low word of each tile base, to which a k-step
    // adds its byte offset / 16, and the high word shared by Q and K (one add per operand
    // and k-step keeps the issuing lane's work per MMA short).
    constexpr uint32_t dhi = smem_desc_hi(8 * SW, C::LAYOUT);
    const uint32_t q_lo = smem_desc_lo(smem_u32(c.sQ + t * C::Q_BYTES), 16);
    const int b = c.buf(t, gs);
    const uint32_t d_tmem = c.tmem + b * BN;
#pragma unroll
    for (int u = 0; u < C::UNITS; ++u) {
        const int U = c.u0 + 2 * j * C::UNITS + u, stage = U % NS;  // ring part holding K_j part u
        if (first_use) {
            if (!__all_sync(0xffffffffu,
                            wait_bounded(&c.kv_full[stage], (U / NS) & 1, c.abort_flag, c.lim, 220 + stage)))
                return false;
            tc_fence_after_sync();
            if (c.fused) fence_proxy_async_smem();
        }
        const uint32_t k_lo = smem_desc_lo(smem_u32(c.sKV + stage * C::UNIT_BYTES), 16);
#pragma unroll
        for (int kk = 0; kk < UK; ++kk) {
            const int k = u * UK + kk;
            const uint32_t blk = (k * 32) / SW, off = (k * 32) % SW;
            const uint32_t lb = blk - u * C::KBLK_PER_UNIT;  // column block inside the part
            umma_ss_elect(d_tmem, q_lo + ((blk * BM * SW + off) >> 4), k_lo + ((lb * BN * SW + off) >> 4), dhi, idesc,
                          k > 0 ? 1u : 0u);
        }
        if (u + 1 < C::UNITS) {
            if (last_use) umma_commit_elect(&c.kv_empty[stage]);  // release this part early
        } else {
            umma_commit_elect(&c.s_full[b]);  // the softmax waits on S first
            if (last_use) umma_commit_elect(&c.kv_empty[stage]);
        }
    }
    if (jj == c.steps(t) - 1) umma_commit_elect(&c.q_free[t]);  // Q_t may be reloaded for the next item
    return true;
}

// O_t += P_t V_j for key tile j (tile-local step jj = j - j0(t)).
template <int D, bool BF16>
__device__ __forceinline__ bool mma_pv(const Cta<D> &c, int t, int j, bool first_use, bool last_use) {
    using C = Cfg<D>;
    constexpr int BM = C::BM, BN = C::BN, SW = C::SW, NS = C::NS;
    constexpr uint32_t idesc = idesc_f16(BM, D, BF16, true);
    const int jj = j - c.j0(t);
    const int gs = c.g0(t) + jj;
    const int b = c.buf(t, gs);
    if (!__all_sync(0xffffffffu, wait_bounded(&c.p_full[b], c.sphase(gs), c.abort_flag, c.lim, 210 + t)))
        return false;
    tc_fence_after_sync();
    constexpr int UV = BN / 16 / C::UNITS;  // k-steps per V part
    constexpr uint32_t dhi = smem_desc_hi(8 * SW, C::LAYOUT);  // high descriptor word of V
    const uint32_t a_tmem = c.tmem + (c.dec ? C::P_COL + 64 * t : b * BN);
    const uint32_t o_tmem = c.tmem + C::O_COL + t * D;
#pragma unroll
    for (int u = 0; u < C::UNITS; ++u) {
        const int U = c.u0 + (2 * j + 1) * C::UNITS + u, stage = U % NS;  // ring part holding V_j part u
        if (first_use) {
            if (!__all_sync(0xffffffffu,
                            wait_bounded(&c.kv_full[stage], (U / NS) & 1, c.abort_flag, c.lim, 230 + stage)))
                return false;
            tc_fence_after_sync();
            if (c.fused) fence_proxy_async_smem();
        }
        const uint32_t v_lo = smem_desc_lo(smem_u32(c.sKV + stage * C::UNIT_BYTES), C::VROWS_PER_UNIT * SW);
#pragma unroll
        for (int kk = 0; kk < UV; ++kk) {
            const int k = u * UV + kk;
            umma_ts_elect(o_tmem, a_tmem + k * 8, v_lo + ((kk * 16 * SW) >> 4), dhi, idesc,
                          (jj > 0 || k > 0) ? 1u : 0u);
        }
        if (u + 1 < C::UNITS) {
            if (last_use) umma_commit_elect(&c.kv_empty[stage]);
        } else {
            umma_commit_elect(&c.pv_done[t]);
            if (last_use) umma_commit_elect(&c.kv_empty[stage]);
        }
    }
    return true;
}

// CTA pairs: a bounded wait taken by the whole MMA warp, cluster scope.
template <int D>
__device__ __forceinline__ bool pair_wait(const Cta<D> &c, uint64_t *bar, uint32_t parity, int where) {
    return __all_sync(0xffffffffu, wait_bounded_cluster(bar, parity, c.abort_flag, c.lim, where));
}
// CTA pairs: arrive on `bar` (same offset) in both CTAs once the pair MMAs issued so far complete.
__device__ __forceinline__ void pair_commit(uint64_t *bar) {
    umma_commit_pair_elect(smem_u32(bar));
    umma_commit_pair_elect(mapa_shared(bar, 1));
}

// CTA pairs, issued by CTA 0: S = Q K_j^T for the pair's 256 query rows (M = 256; CTA 0's query
// tile is rows 0-127, CTA 1's rows 128-255; N = 128 keys, rows [0, 64) of key tile j in CTA 0's
// ring part and [64, 128) in CTA 1's; K = D). The tile's S lands in each CTA's TMEM.
template <int D, bool BF16>
__device__ __forceinline__ bool mma_qk_pair(const Cta<D> &c, int j) {
    using C = Cfg<D>;
    constexpr int BM = C::BM, BN = C::BN, SW = C::SW, NS = C::NS;
    constexpr uint32_t idesc = idesc_f16(2 * BM, BN, BF16, false);
    const int gs = c.g0(0) + j;
    if (j == 0) {
        if (!pair_wait(c, &c.q_full[0], c.nq(0) & 1, 200) || !pair_wait(c, c.q_peer, c.nq(0) & 1, 201)) return false;
    }
    const int U = c.u0 + 2 * j, stage = U % NS;  // ring part holding this CTA's half of K_j
    if (!pair_wait(c, &c.kv_full[stage], (U / NS) & 1, 220 + stage) ||
        !pair_wait(c, &c.kv_peer[stage], (U / NS) & 1, 230 + stage))
        return false;
    tc_fence_after_sync();
    constexpr uint32_t dhi = smem_desc_hi(8 * SW, C::LAYOUT);
    const uint32_t q_lo = smem_desc_lo(smem_u32(c.sQ), 16);
    const uint32_t k_lo = smem_desc_lo(smem_u32(c.sKV + stage * C::UNIT_BYTES), 16);
    const int b = gs & 1;  // S buffer
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
        const uint32_t blk = (k * 32) / SW, off = (k * 32) % SW;  // column block of 64, byte offset inside
        umma_ss_pair_elect(c.tmem + b * BN, q_lo + ((blk * BM * SW + off) >> 4),
                           k_lo + ((blk * (BN / 2) * SW + off) >> 4), dhi, idesc, k > 0 ? 1u : 0u);
    }
    pair_commit(&c.s_full[b]);
    pair_commit(&c.kv_empty[stage]);
    if (j == c.nA - 1) pair_commit(&c.q_free[0]);  // the Q tiles may be reloaded for the next item
    return true;
}

// CTA pairs, issued by CTA 0: O += P V_j (M = 256, A = each CTA's P in its TMEM; N = D, columns
// [0, 128) of V_j in CTA 0's ring part and [128, 256) in CTA 1's, MN-major; K = 128 keys).
template <int D, bool BF16>
__device__ __forceinline__ bool mma_pv_pair(const Cta<D> &c, int j) {
    using C = Cfg<D>;
    constexpr int BM = C::BM, BN = C::BN, SW = C::SW, NS = C::NS;
    constexpr uint32_t idesc = idesc_f16(2 * BM, D, BF16, true);
    const int gs = c.g0(0) + j;
    const int b = gs & 1;
    if (!pair_wait(c, &c.p_full[b], (gs >> 1) & 1, 210)) return false;
    const int U = c.u0 + 2 * j + 1, stage = U % NS;  // ring part holding this CTA's half of V_j
    if (!pair_wait(c, &c.kv_full[stage], (U / NS) & 1, 220 + stage) ||
        !pair_wait(c, &c.kv_peer[stage], (U / NS) & 1, 230 + stage))
        return false;
    tc_fence_after_sync();
    constexpr uint32_t dhi = smem_desc_hi(8 * SW, C::LAYOUT);
    const uint32_t v_lo = smem_desc_lo(smem_u32(c.sKV + stage * C::UNIT_BYTES), BN * SW);
#pragma unroll
    for (int k = 0; k < BN / 16; ++k)
        umma_ts_pair_elect(c.tmem + C::O_COL, c.tmem + b * BN + k * 8, v_lo + ((k * 16 * SW) >> 4), dhi, idesc,
                           (j > 0 || k > 0) ? 1u : 0u);
    pair_commit(&c.pv_done[0]);
    pair_commit(&c.kv_empty[stage]);
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
// the contiguous path stays as small as its register budget wants). PACKED: packed sequences
// (cu_seqlens); a separate instantiation too, so that neither path's state takes registers in
// the other's loops.
//
// Dense inputs run persistently: the grid has one CTA per SM (at most one per work item), and
// each CTA takes its work items in rounds (dense_item_at) or, over more than one round with
// contiguous K/V and D <= 128, from the item queue in the same order. Every role loops over the
// same items;
// the producer loads an item's Q tiles as soon as the previous item's QKs on them are done, so
// the next item's loads and first QKs overlap the current item's last steps and epilogue.
// Packed inputs launch one CTA per 256 consecutive tokens (one item per CTA).
template <int D, bool BF16, bool CAUSAL, bool PAGED, bool PACKED, bool GROUPED>
__global__ void __launch_bounds__(Cfg<D>::NUM_THREADS, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = Cfg<D>;
    constexpr int BM = C::BM, BN = C::BN, SW = C::SW, NS = C::NS;

    static_assert(!(PAGED && PACKED), "paged K/V is for dense queries");
    static_assert(!GROUPED || (CAUSAL && !PACKED), "head groups order dense causal items");
    constexpr bool packed = PACKED;  // the host launches PACKED exactly when p.cu_seqlens is set
    constexpr bool persistent = !packed;
    // Dense D = 256 runs in 2-CTA clusters (the host launches them so): the pair's two query tiles
    // share every K/V tile, each CTA loading half of it, and CTA 0 issues M = 256 MMAs for both.
    constexpr bool PAIR = (D == 256) && !PAGED && !PACKED;
    // The item queue (dense inputs over contiguous K/V, more than one round; the host sets p.queue).
    constexpr bool QUEUE = persistent && !PAGED;
    const bool queued = QUEUE && p.queue != nullptr;
    Cta<D> c;
    c.dec = C::DECOUPLED;
    c.single = C::MAXQ == 1;
    c.pair = PAIR;
    c.rank = PAIR ? cluster_ctarank() : 0u;
    c.u0 = 0;
    c.g0a = c.g0b = 0;
    c.nqa = c.nqb = 0;
    if (packed) {
        // The CTA owns the 128 * MAXQ consecutive packed tokens of tile blockIdx.y, whatever
        // sequences they belong to; its keys are the union of those sequences' keys (the device
        // walks cu_seqlens), and each row is masked to its own sequence.
        c.h = blockIdx.x;
        c.b = 0;
        c.q0 = 0;
        c.seq_start = 0;
        c.seqlen = 0;
        c.qbase = blockIdx.y * C::MAXQ * BM;
        if (c.qbase >= p.total_tokens) return;  // uniform over the CTA, before any barrier exists
        c.two = (C::MAXQ == 2) && (c.qbase + BM < p.total_tokens);
        const int ln = threadIdx.x & 31;
        // With fewer than 64 sequences every warp holds all of cu_seqlens (two entries per
        // lane), so the lookups below are ballots and shuffles after one round of loads;
        // otherwise each lookup is a search with dependent loads.
        const CuWindow win(p.cu_seqlens, p.num_seqs, ln);
        auto seq_of = [win, ln, &p](int tok) {
            return win.ok ? win.seq(tok, ln) : warp_seq_of_token(p.cu_seqlens, p.num_seqs, tok, ln);
        };
        auto cu_at = [win, &p](int s) { return win.ok ? win.at(s) : p.cu_seqlens[s]; };
        const int s_first = seq_of(c.qbase);
        c.kvbase = cu_at(s_first);
        // keys of a tile end with its last row's sequence (or the causal limit)
        auto kv_end = [&](int tlast) {
            const int s_last = seq_of(tlast);
            return (CAUSAL ? min(cu_at(s_last + 1), tlast + 1) : cu_at(s_last + 1)) - c.kvbase;
        };
        const int end_a = kv_end(min(c.qbase + BM, p.total_tokens) - 1);
        c.nA = (end_a + BN - 1) / BN;
        c.nB = c.jB0 = 0;
        if (c.two) {
            const int end_b = kv_end(min(c.qbase + 2 * BM, p.total_tokens) - 1);
            c.nB = (end_b + BN - 1) / BN;
            c.jB0 = (cu_at(seq_of(c.qbase + BM)) - c.kvbase) / BN;
        }
    }
    // Fused path: stage contents are written by cp.async copies, whose writer cannot fence
    // after they land, so the MMA thread fences the async proxy after its waits. (The paged
    // path's zeroed page tails are fenced by the writing thread itself before it releases
    // the stage.)
    // Paged K/V in pages under 64 rows: TMA boxes that small move too few bytes per SM, so
    // the V parts go by cp.async copies beside the TMA's K parts (the same fence applies).
    const bool copy_pages = PAGED && p.page_size < 64;
    c.fused = p.gather != nullptr || copy_pages;
    // Separate P buffers and no copy warps: the MMAs are issued by two warps, warp 9 the
    // QKs and warp 10 the PVs, so that a tile's next S is computed as soon as its S buffer has
    // been read, never held up behind the other tile's PV (which waits for that tile's P).
    const bool split_issue = c.dec && !c.fused;
    // Every role runs `for (int rd = 0; next_item(...); ++rd) { ...; c.advance(); }` over this
    // CTA's work items (dense: the rounds of dense_item_at, or the queue: fetch_item in the TMA
    // lane, take_item in the MMA and softmax warps; packed: the one item set above), leaving the
    // loop early when a wait gives up.

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
    c.q_free = c.tail + 1;
    c.q_peer = c.q_free + 2;
    c.kv_peer = c.q_peer + 1;
    c.item_full = c.kv_peer + NS;
    c.item_empty = c.item_full + C::QSLOTS;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    c.abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    c.items = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);
    c.lim = p.timeout_ns;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int pw = (warp == C::WARP_TMA) ? 0 : warp - C::WARP_MMA;  // copy producer warp 0..2 (8, 10, 11)
    // Fused packed path: the copy warps read the padded rows of their groups of the first key
    // part now, so that load overlaps the barrier and TMEM set-up.
    int64_t first_rows[2] = {0, 0};
    if (p.gather && (warp == C::WARP_TMA || warp > C::WARP_MMA)) fused_group_rows(p, c.kvbase, BN, pw, lane, first_rows);

    if (threadIdx.x == 0) {
        // ring barriers: one arrival (the TMA lane's), or per copy thread: fused packed path 96
        // (warps 8, 10, 11); pages under 64 rows 65 (the TMA lane + warps 10, 11). Query tiles: the
        // TMA lane's, or the 128 threads of the softmax warpgroup (fused packed path).
        const int fill_arrivals = p.gather ? 96 : (copy_pages ? 65 : 1);
        const int q_arrivals = p.gather ? 128 : 1;
        for (int t = 0; t < 2; ++t) {
            mbar_init(&c.q_full[t], q_arrivals);
            mbar_init(&c.s_full[t], 1);
            mbar_init(&c.p_full[t], PAIR ? 256 : 128);  // pairs: CTA 0's barrier takes both CTAs' rows
            mbar_init(&c.pv_done[t], 1);
            mbar_init(&c.s_free[t], 4);  // one arrival per softmax warp
            mbar_init(&c.q_free[t], 1);
        }
        for (int s = 0; s < NS; ++s) {
            mbar_init(&c.kv_full[s], fill_arrivals);
            mbar_init(&c.kv_empty[s], 1);
        }
        mbar_init(c.drain, split_issue ? 2 : 1);  // one commit per issuing warp
        mbar_init(c.q_peer, 1);
        for (int s = 0; s < NS; ++s) mbar_init(&c.kv_peer[s], 1);
        mbar_init(c.tail, 1);
        for (int s = 0; s < C::QSLOTS; ++s) {
            mbar_init(&c.item_full[s], 1);
            // one arrival per reading warp: the softmax warps and the MMA-issuing warp(s); pairs
            // (CTA 0's barrier): CTA 0's MMA and softmax warps, CTA 1's producer and reporter
            // lanes and softmax warps
            mbar_init(&c.item_empty[s], PAIR ? 2 * C::NUM_SOFTMAX_WARPS + 3
                                             : C::NUM_SOFTMAX_WARPS + (split_issue ? 2 : 1));
        }
        *c.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == C::WARP_TMA && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == C::WARP_MMA) {
        if (PAIR) {
            tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, C::TMEM_COLS);
            tmem_relinquish();
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (PAIR) cluster_sync();  // both CTAs' barriers exist before either arrives on the other's
    tc_fence_after_sync();
    c.tmem = *tmem_slot;

    if (warp >= C::NUM_SOFTMAX_WARPS) {
        // producer / MMA warpgroup (its remaining warps idle unless they copy rows or issue PVs)
        if constexpr (C::SPLIT_REGS) regs_dec<C::regs_low(PACKED)>();
        if (warp == C::WARP_TMA || (c.fused && warp > C::WARP_MMA)) {
            // ------------------------------------------------------------ producer
            // (fused packed path and pages under 64 rows: warps 10 and 11 copy rows too)
            int issued = 0;                  // ring parts issued (running count)
            int q_issued_a = 0, q_issued_b = 0;  // Q_A, Q_B loads issued (running counts)
            int tail_uses = 0;               // paged: parts that went through `tail` (running count)
            int tail_pending = -1;           // phase of a `tail` use whose wait was cut short
            bool bad_page = false;           // reported once, after the loads
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last();
            // Q_t of the current item into its buffer, once the previous item's QKs on it are done.
            auto load_q = [&](int t) -> bool {
                if (c.nq(t) > 0 && !wait_bounded(&c.q_free[t], (c.nq(t) - 1) & 1, c.abort_flag, c.lim, 110 + t))
                    return false;
                mbar_arrive_expect_tx(&c.q_full[t], C::Q_BYTES);
#pragma unroll
                for (int b = 0; b < C::NBLK; ++b)
                    tma_load_3d(c.sQ + t * C::Q_BYTES + b * BM * SW, &tm_q, &c.q_full[t], b * C::SWE, c.h,
                                c.qbase + t * BM, pol_q);
                (t ? q_issued_b : q_issued_a) = c.nq(t) + 1;
                return true;
            };
            // Physical row of key position pos (< seqlen) of the item's batch entry. A page index
            // outside the pool is reported and replaced by page 0 (the result is then wrong, but
            // nothing outside the pool is read).
            auto page_row = [&](int pos) -> int64_t {
                const int32_t *bt = p.block_table + static_cast<int64_t>(c.b) * p.max_blocks;
                int pg = __ldg(bt + (pos >> p.page_shift));
                if (pg < 0 || pg >= p.num_pages) {
                    bad_page = true;
                    pg = 0;
                }
                return (static_cast<int64_t>(pg) << p.page_shift) + (pos & (p.page_size - 1));
            };
            if (PAGED && copy_pages) {
                // Paged K/V in small pages: two engines share the bytes. Warp 8 (lane 0) moves
                // the query tiles and the K parts by TMA, one box per page chunk (chunks wholly
                // past the sequence end are boxes at a negative row: zeros); warps 10 and 11
                // copy the V parts row by row with 16-byte cp.async into the swizzled layout,
                // zero-filling positions past the sequence end (no page is read for them). A
                // ring barrier takes 65 arrivals per part: the TMA lane's (with the K bytes, or
                // a plain arrival on a V part) and one per copy thread (plain on a K part, or
                // once its V copies have landed).
                if (warp == C::WARP_TMA) {
                    if (lane == 0) {
                        const int box = min(p.page_size, BN);
                        bool ok = true;
                        for (int rd = 0; ok && next_item<D, CAUSAL, GROUPED, PAIR>(c, p, rd, persistent); ++rd) {
                            ok = load_q(0);
                            const int loads = c.loads();
                            for (int L = 0; ok && L < loads; ++L) {
                                if (L == C::UNITS && c.two && !load_q(1)) {
                                    ok = false;
                                    break;
                                }
                                const int U = c.u0 + L, stage = U % NS;
                                if (U >= NS && !wait_bounded(&c.kv_empty[stage], ((U / NS) - 1) & 1, c.abort_flag,
                                                             c.lim, 100 + stage)) {
                                    ok = false;
                                    break;
                                }
                                const int Lk = L / C::UNITS, u = L % C::UNITS, j = Lk >> 1;
                                if (Lk & 1) {
                                    mbar_arrive(&c.kv_full[stage]);  // V part: copied by warps 10 and 11
                                } else {
                                    uint8_t *dst = c.sKV + stage * C::UNIT_BYTES;
                                    const int pos0 = j * BN;
                                    const int part_valid = c.seqlen - pos0;
                                    mbar_arrive_expect_tx(&c.kv_full[stage], C::UNIT_BYTES);
                                    for (int r = 0; r < BN; r += box) {
                                        const int prow = (r < part_valid) ? static_cast<int>(page_row(pos0 + r)) : -box;
                                        for (int b = 0; b < C::KBLK_PER_UNIT; ++b)
                                            tma_load_3d(dst + (b * BN + r) * SW, &tm_k, &c.kv_full[stage],
                                                        (u * C::KBLK_PER_UNIT + b) * C::SWE, c.h, prow, pol_kv);
                                    }
                                }
                                issued = U + 1;
                            }
                            c.advance();
                        }
                    }
                } else {
                    constexpr int CPB = SW / 16;
                    constexpr int CPR = C::NBLK * CPB;  // 16-byte chunks per V row
                    const int w = pw - 1;                // copy warp 0, 1
                    bool ok = true;
                    for (int rd = 0; ok && next_item<D, CAUSAL, GROUPED, PAIR>(c, p, rd, persistent); ++rd) {
                        const int loads = c.loads();
                        for (int L = 0; L < loads; ++L) {
                            const int U = c.u0 + L, stage = U % NS;
                            if (U >= NS && !wait_bounded(&c.kv_empty[stage], ((U / NS) - 1) & 1, c.abort_flag,
                                                         c.lim, 100 + stage)) {
                                ok = false;
                                break;
                            }
                            const int Lk = L / C::UNITS, u = L % C::UNITS, j = Lk >> 1;
                            if (!(Lk & 1)) {
                                mbar_arrive(&c.kv_full[stage]);  // K part: moved by the TMA
                                continue;
                            }
                            // V part u of tile j: rows [pos0, pos0 + VROWS_PER_UNIT), every column block
                            const int pos0 = j * BN + u * C::VROWS_PER_UNIT;
                            const uint32_t dst_u32 = smem_u32(c.sKV + stage * C::UNIT_BYTES);
                            for (int g = w; g * 32 < C::VROWS_PER_UNIT; g += 2) {
                                const int pos = pos0 + g * 32 + lane;
                                const bool valid = pos < c.seqlen;
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
                                                          (pr * p.H + c.h) * static_cast<int64_t>(D) * 2 + ch * 16,
                                                      ok_row ? 16u : 0u);
                                }
                            }
                            cp_async_mbar_arrive(&c.kv_full[stage]);  // arrives once this thread's copies have landed
                        }
                        c.advance();
                    }
                    cp_async_wait_all();  // nothing of this thread is left in flight at exit
                }
                if (bad_page) record_error(FA_ERR_INDEX, 151);
            } else if (p.gather) {
                // Fused packed path (one work item): warps 8, 10 and 11 (96 threads) copy every K/V
                // row from the padded tensor (row = padded row of the packed token; rows past the
                // last token read row 0, which the masks then ignore) with 16-byte cp.async into
                // the same swizzled layout the TMA would produce; each thread's copies arrive on
                // the part's barrier when they land, and the MMA thread fences the async proxy.
                // (The softmax warps copy the query tiles.) The 32-row groups of the ring parts
                // are dealt to the three warps in one running order (group G to warp G % 3), so
                // each warp moves a third of the bytes and holds at most two groups of a part. A
                // warp reads the padded rows of its next part's groups (one coalesced load per
                // group) before it issues this part's copies, so index loads never wait in line.
                q_issued_a = 1;
                q_issued_b = c.two ? 1 : 0;
                auto part_rows = [&](int U, int &tok0, int &rows) {
                    const int L = U / C::UNITS, u = U % C::UNITS, j = L >> 1;
                    tok0 = c.kvbase + j * BN + ((L & 1) ? u * C::VROWS_PER_UNIT : 0);
                    rows = (L & 1) ? C::VROWS_PER_UNIT : BN;
                };
                const int loads = c.loads();
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
                            fetch_group<C::NBLK, SW, D>(dst, rows, g, cur[k], p.v, &tm_v, 0, p.H, c.h, lane,
                                                        &c.kv_full[stage], pol_kv);
                        else
                            fetch_group<C::KBLK_PER_UNIT, SW, D>(dst, rows, g, cur[k], p.k, &tm_k,
                                                                 (U % C::UNITS) * C::KBLK_PER_UNIT, p.H, c.h, lane,
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
                    uint8_t *const zbase = static_cast<uint8_t *>(p.out) + static_cast<int64_t>(c.h) * RB + ch * 16;
                    for (int gi = pw; gi < C::MAXQ * 4; gi += 3) {
                        const int64_t tw0 = static_cast<int64_t>(c.qbase) + gi * 32;
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
            } else if (PAIR && lane == 0) {
                // CTA pairs: this CTA's query tile, then for each key tile j its half of K_j (key
                // rows [64 * rank, +64), all of D) and its half of V_j (columns [128 * rank, +128)),
                // each on this CTA's own barriers (CTA 1's reporter warp passes them on to CTA 0). The
                // ring slots and Q buffer are released by CTA 0's MMA commits.
                bool ok = true;
                for (int rd = 0;
                     ok && (queued ? (c.rank == 0 ? fetch_item_pair<D, CAUSAL, GROUPED>(c, p, rd)
                                                  : take_item_pair<D, CAUSAL, GROUPED>(c, p, rd, true))
                                   : next_item<D, CAUSAL, GROUPED, PAIR>(c, p, rd, persistent));
                     ++rd) {
                    if (c.nq(0) > 0 && !wait_bounded_cluster(&c.q_free[0], (c.nq(0) - 1) & 1, c.abort_flag, c.lim, 110)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&c.q_full[0], C::Q_BYTES);
#pragma unroll
                    for (int b = 0; b < C::NBLK; ++b)
                        tma_load_3d(c.sQ + b * BM * SW, &tm_q, &c.q_full[0], b * C::SWE, c.h, c.qbase, pol_q);
                    q_issued_a = c.nq(0) + 1;
                    const int loads = c.loads();
                    for (int L = 0; ok && L < loads; ++L) {
                        const int U = c.u0 + L, stage = U % NS, j = L >> 1;
                        if (U >= NS && !wait_bounded_cluster(&c.kv_empty[stage], ((U / NS) - 1) & 1, c.abort_flag,
                                                             c.lim, 100 + stage)) {
                            ok = false;
                            break;
                        }
                        uint8_t *dst = c.sKV + stage * C::UNIT_BYTES;
                        mbar_arrive_expect_tx(&c.kv_full[stage], C::UNIT_BYTES);
                        if (!(L & 1)) {
#pragma unroll
                            for (int b = 0; b < C::NBLK; ++b)
                                tma_load_3d(dst + b * (BN / 2) * SW, &tm_k, &c.kv_full[stage], b * C::SWE, c.h,
                                            c.kvbase + j * BN + static_cast<int>(c.rank) * (BN / 2), pol_kv);
                        } else {
#pragma unroll
                            for (int b = 0; b < C::NBLK / 2; ++b)
                                tma_load_3d(dst + b * BN * SW, &tm_v, &c.kv_full[stage],
                                            (static_cast<int>(c.rank) * (C::NBLK / 2) + b) * C::SWE, c.h, c.kvbase + j * BN,
                                            pol_kv);
                        }
                        issued = U + 1;
                    }
                    c.advance();
                }
            } else if (lane == 0) {
                bool ok = true;
                for (int rd = 0; ok && (queued ? fetch_item<D, CAUSAL, GROUPED>(c, p, rd)
                                               : next_item<D, CAUSAL, GROUPED, PAIR>(c, p, rd, persistent));
                     ++rd) {
                    ok = load_q(0);
                    const int loads = c.loads();
                    for (int L = 0; ok && L < loads; ++L) {
                        if (L == C::UNITS && c.two && !load_q(1)) {
                            ok = false;
                            break;
                        }
                        const int U = c.u0 + L, stage = U % NS;
                        if (U >= NS &&
                            !wait_bounded(&c.kv_empty[stage], ((U / NS) - 1) & 1, c.abort_flag, c.lim, 100 + stage)) {
                            ok = false;
                            break;
                        }
                        const int Lk = L / C::UNITS, u = L % C::UNITS, j = Lk >> 1;
                        uint8_t *dst = c.sKV + stage * C::UNIT_BYTES;
                        if constexpr (PAGED) {
                            // One box per (column block, page-sized row chunk) of the part. Rows of a
                            // sequence's last page past its end hold whatever the pool holds there:
                            // for K they are masked (their scores become -inf), but in V a NaN would
                            // survive P = 0, so the V part that straddles the end lands on `tail`
                            // first, its stray rows are zeroed, and only then is the stage released.
                            const bool is_v = Lk & 1;
                            const int rows = is_v ? C::VROWS_PER_UNIT : BN;
                            const int box = min(p.page_size, rows);
                            const int pos0 = j * BN + (is_v ? u * C::VROWS_PER_UNIT : 0);
                            const int part_valid = c.seqlen - pos0;  // rows of the part inside the sequence
                            const bool straddles = is_v && part_valid > 0 && part_valid < rows && part_valid % box != 0;
                            uint64_t *bar = straddles ? c.tail : &c.kv_full[stage];
                            mbar_arrive_expect_tx(bar, C::UNIT_BYTES);
                            for (int r = 0; r < rows; r += box) {
                                // a chunk wholly past the sequence end (its table entry need not
                                // exist) is a box at a negative row: all fill value (zeros)
                                const int prow = (r < part_valid) ? static_cast<int>(page_row(pos0 + r)) : -box;
                                if (is_v) {
                                    for (int b = 0; b < C::NBLK; ++b)
                                        tma_load_3d(dst + (b * C::VROWS_PER_UNIT + r) * SW, &tm_v, bar, b * C::SWE,
                                                    c.h, prow, pol_kv);
                                } else {
                                    for (int b = 0; b < C::KBLK_PER_UNIT; ++b)
                                        tma_load_3d(dst + (b * BN + r) * SW, &tm_k, bar,
                                                    (u * C::KBLK_PER_UNIT + b) * C::SWE, c.h, prow, pol_kv);
                                }
                            }
                            if (straddles) {
                                // at most one such part per item (its last V tile); `tail` phases
                                // count those parts over the items
                                if (!wait_bounded(c.tail, tail_uses & 1, c.abort_flag, c.lim, 160)) {
                                    tail_pending = tail_uses & 1;
                                    ok = false;
                                    break;
                                }
                                ++tail_uses;
                                tail_pending = -1;
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
                            issued = U + 1;
                        } else {
                            mbar_arrive_expect_tx(&c.kv_full[stage], C::UNIT_BYTES);
                            if (Lk & 1) {
                                // V part u: rows [u*VROWS_PER_UNIT, ...) of the tile, every column block
#pragma unroll
                                for (int b = 0; b < C::NBLK; ++b)
                                    tma_load_3d(dst + b * C::VROWS_PER_UNIT * SW, &tm_v, &c.kv_full[stage],
                                                b * C::SWE, c.h, c.kvbase + j * BN + u * C::VROWS_PER_UNIT, pol_kv);
                            } else {
                                // K part u: column blocks [u*KBLK_PER_UNIT, ...) of every tile row
#pragma unroll
                                for (int b = 0; b < C::KBLK_PER_UNIT; ++b)
                                    tma_load_3d(dst + b * BN * SW, &tm_k, &c.kv_full[stage],
                                                (u * C::KBLK_PER_UNIT + b) * C::SWE, c.h, c.kvbase + j * BN, pol_kv);
                            }
                            issued = U + 1;
                        }
                    }
                    c.advance();
                }
                if (PAGED && bad_page) record_error(FA_ERR_INDEX, 150);
            }
            if (warp == C::WARP_TMA && lane == 0 && *c.abort_flag) {
                // Let the copies already issued land before the CTA's shared memory goes away.
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const int qi = t ? q_issued_b : q_issued_a;
                    if (qi == 0) continue;
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(&c.q_full[t], (qi - 1) & 1) && global_timer_ns() - t0 < c.lim) {
                    }
                }
                for (int U = (issued > NS ? issued - NS : 0); U < issued; ++U) {
                    const int stage = U % NS;
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(&c.kv_full[stage], (U / NS) & 1) && global_timer_ns() - t0 < c.lim) {
                    }
                }
                if (tail_pending >= 0) {
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(c.tail, tail_pending) && global_timer_ns() - t0 < c.lim) {
                    }
                }
            }
        } else if (PAIR && warp == C::WARP_MMA + 1 && c.rank == 1) {
            // ------------------------------------------------------------ pair reporter (CTA 1)
            // Each of this CTA's Q tiles and ring parts, once landed, is reported to CTA 0
            // (q_peer, kv_peer), whose MMAs read it.
            if (lane == 0) {
                bool ok = true;
                const uint32_t q_peer0 = mapa_shared(c.q_peer, 0);
                for (int rd = 0; ok && (queued ? take_item_pair<D, CAUSAL, GROUPED>(c, p, rd, true)
                                               : next_item<D, CAUSAL, GROUPED, PAIR>(c, p, rd, persistent));
                     ++rd) {
                    if (!(ok = wait_bounded(&c.q_full[0], c.nq(0) & 1, c.abort_flag, c.lim, 120))) break;
                    mbar_arrive_cluster(q_peer0);
                    const int loads = c.loads();
                    for (int L = 0; ok && L < loads; ++L) {
                        const int U = c.u0 + L, stage = U % NS;
                        if (!(ok = wait_bounded(&c.kv_full[stage], (U / NS) & 1, c.abort_flag, c.lim, 125))) break;
                        mbar_arrive_cluster(mapa_shared(&c.kv_peer[stage], 0));
                    }
                    c.advance();
                }
            }
        } else if (PAIR && warp == C::WARP_MMA) {
            // ------------------------------------------------------------ pair MMA issuer (CTA 0)
            bool ok = true;
            if (c.rank == 0) {
                for (int rd = 0; ok && (queued ? take_item_pair<D, CAUSAL, GROUPED>(c, p, rd, false)
                                               : next_item<D, CAUSAL, GROUPED, PAIR>(c, p, rd, persistent));
                     ++rd) {
                    const int n = c.nA;
                    for (int idx = 0; ok && idx < 2 * n; ++idx) {
                        bool is_v;
                        int j;
                        decode_step(idx, n, is_v, j);
                        ok = is_v ? mma_pv_pair<D, BF16>(c, j) : mma_qk_pair<D, BF16>(c, j);
                    }
                    c.advance();
                }
                umma_commit_pair_elect(smem_u32(c.drain));
                const uint64_t t0 = global_timer_ns();
                while (!mbar_try_wait(c.drain, 0) && global_timer_ns() - t0 < c.lim) {
                }
            }
        } else if (warp == C::WARP_MMA || (split_issue && warp == C::WARP_MMA + 1)) {
            // ------------------------------------------------------------ MMA issuer(s)
            bool ok = true;
            const bool qk = !split_issue || warp == C::WARP_MMA;
            const bool pv = !split_issue || warp != C::WARP_MMA;
            for (int rd = 0; ok && (queued ? take_item<D, CAUSAL, GROUPED>(c, p, rd)
                                           : next_item<D, CAUSAL, GROUPED, PAIR>(c, p, rd, persistent));
                 ++rd) {
                const int nl = max(c.nA, c.nB);  // key tiles of the item
                if (c.single) {
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
                    // QK_A(j+1), QK_B(j+1), PV_A(j), PV_B(j), each when that tile uses key tile j;
                    // with two issuing warps each keeps its own half of that order (a key tile
                    // is released by the QK warp, a value tile by the PV warp).
                    if (qk && c.uses(0, 0)) ok = mma_qk<D, BF16>(c, 0, 0, true, !c.uses(1, 0));
                    if (qk && ok && c.uses(1, 0)) ok = mma_qk<D, BF16>(c, 1, 0, !c.uses(0, 0), true);
                    for (int j = 0; ok && j < nl; ++j) {
                        const bool a1 = c.uses(0, j + 1), b1 = c.uses(1, j + 1), a0 = c.uses(0, j), b0 = c.uses(1, j);
                        if (qk && a1) ok = mma_qk<D, BF16>(c, 0, j + 1, true, !b1);
                        if (qk && ok && b1) ok = mma_qk<D, BF16>(c, 1, j + 1, !a1, true);
                        if (pv && ok && a0) ok = mma_pv<D, BF16>(c, 0, j, true, !b0);
                        if (pv && ok && b0) ok = mma_pv<D, BF16>(c, 1, j, !a0, true);
                    }
                } else {
                    // Ping-pong over key tiles j: PV_A(j-1), QK_A(j), PV_B(j-1), QK_B(j). A key or
                    // value tile is waited for at its first use and released after its last.
                    if (c.uses(0, 0)) ok = mma_qk<D, BF16>(c, 0, 0, true, !c.uses(1, 0));
                    if (ok && c.uses(1, 0)) ok = mma_qk<D, BF16>(c, 1, 0, !c.uses(0, 0), true);
                    for (int j = 1; ok && j <= nl; ++j) {
                        const bool ap = c.uses(0, j - 1), bp = c.uses(1, j - 1), ac = c.uses(0, j), bc = c.uses(1, j);
                        if (ap) ok = mma_pv<D, BF16>(c, 0, j - 1, true, !bp);
                        if (ok && ac) ok = mma_qk<D, BF16>(c, 0, j, true, !bc);
                        if (ok && bp) ok = mma_pv<D, BF16>(c, 1, j - 1, !ap, true);
                        if (ok && bc) ok = mma_qk<D, BF16>(c, 1, j, !ac, true);
                    }
                }
                c.advance();
            }
            // Every MMA issued above has finished once `drain` completes.
            umma_commit_elect(c.drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(c.drain, 0) && global_timer_ns() - t0 < c.lim) {
            }
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        if constexpr (C::SPLIT_REGS) regs_inc<C::regs_high(PACKED)>();
        // pairs: S, P and O barriers are completed by CTA 0's MMA commits (cluster scope)
        auto swait = [&](uint64_t *bar, uint32_t ph, int where) {
            return PAIR ? wait_bounded_cluster(bar, ph, c.abort_flag, c.lim, where)
                        : wait_bounded(bar, ph, c.abort_flag, c.lim, where);
        };
        const int t = warp >> 2;                      // query tile of this warpgroup
        const int quarter = warp & 3;                 // TMEM lanes this warp may access
        const int r = quarter * 32 + lane;            // row of the tile == TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t o_col = C::O_COL + t * D;
        const float sc = p.scale_log2;
        bool ok = true;
        // Only the round and this tile's running key-step count stay live across an item's key
        // steps (the softmax warps are at their register limit there); the item is looked up
        // again for the epilogue.
        int gbase = 0;
        for (int rd = 0; ok && (queued ? (PAIR ? take_item_pair<D, CAUSAL, GROUPED>(c, p, rd, false)
                                               : take_item<D, CAUSAL, GROUPED>(c, p, rd))
                                       : next_item<D, CAUSAL, GROUPED, PAIR>(c, p, rd, persistent));
             ++rd) {
            const int n = c.steps(t);  // key tiles this warpgroup visits in the item
            if (n <= 0) continue;      // tile absent
            const int j0 = c.j0(t);
            // This row's token and its visible keys [klo, khi), counted from kvbase.
            const int64_t tok = static_cast<int64_t>(c.qbase) + t * BM + r;
            if (p.gather) {
                // Fused packed path: each warp copies its own 32 rows of query tile t from their
                // padded rows (rows past the last token read row 0); the warpgroup's 128 threads
                // arrive on q_full[t] as their copies land.
                int64_t pr = (tok < p.total_tokens) ? __ldg(p.gather + tok) : 0;
                if (pr < 0 || pr >= p.padded_rows) pr = 0;  // never read outside q
                fetch_group<C::NBLK, SW, D>(c.sQ + t * C::Q_BYTES, BM, quarter, pr, p.q, &tm_q, 0, p.H, c.h, lane,
                                            &c.q_full[t], l2_policy_evict_first());
                cp_async_mbar_arrive(&c.q_full[t]);
            }
            int klo = 0, khi = 1;
            bool row_ok;
            if (!packed) {
                const int row_pos = c.q0 + t * BM + r;  // position inside the sequence
                row_ok = row_pos < c.seqlen;
                khi = CAUSAL ? min(c.seqlen, row_pos + 1) : c.seqlen;
            } else {
                row_ok = tok < p.total_tokens;
                const int tw0 = c.qbase + t * BM + quarter * 32;  // this warp's first token
                int s_lane = 0;
                if (tw0 < p.total_tokens) {  // warp-uniform
                    const int s_w = warp_seq_of_token(p.cu_seqlens, p.num_seqs, tw0, lane);
                    s_lane = lane_seq_of_token(p.cu_seqlens, p.num_seqs, s_w,
                                               static_cast<int>(min(tok, static_cast<int64_t>(p.total_tokens - 1))), lane);
                }
                if (row_ok) {
                    const int s_r = s_lane;
                    klo = p.cu_seqlens[s_r] - c.kvbase;
                    khi = (CAUSAL ? min(p.cu_seqlens[s_r + 1], static_cast<int>(tok) + 1) : p.cu_seqlens[s_r + 1]) -
                          c.kvbase;
                }
            }
            float m = -INFINITY;  // running max of scaled scores, log2 units (possibly stale)
            float l = 0.f;        // running sum of 2^(s*sc - m)
            if (c.dec) {
                // Separate P buffer: S_t is released right after it is read, so QK_t(j+1) overlaps
                // this step's exponentials; P_t(j) is written once PV_t(j-1) has consumed P_t(j-1)
                // (at an item's first step, the previous item's epilogue has waited for its last PV).
                const uint32_t p_addr = c.tmem + lane_base + C::P_COL + 64 * t;
                for (int jj = 0; jj < n; ++jj) {
                    const int j = j0 + jj;       // key tile
                    const int gs = gbase + jj;  // running key step of this tile
                    if (!__all_sync(0xffffffffu, wait_bounded(&c.s_full[t], gs & 1, c.abort_flag, c.lim, 330 + t))) {
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
                    const float rs = softmax_row_to_regs<BN, BF16>(sr, sc, neg_m, pk);  // -inf -> exactly 0
                    l = fmaf(l, alpha, rs);
                    if (jj > 0) {
                        if (!__all_sync(0xffffffffu,
                                        wait_bounded(&c.pv_done[t], (gs - 1) & 1, c.abort_flag, c.lim, 340 + t))) {
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
            } else {
                for (int jj = 0; jj < n; ++jj) {
                    const int j = j0 + jj;       // key tile
                    const int gs = gbase + jj;  // running key step of this tile
                    const int b = c.buf(t, gs);
                    if (!__all_sync(0xffffffffu,
                                    swait(&c.s_full[b], c.sphase(gs), 300 + t))) {
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
                    const float rs = softmax_chunk_store<BN, BF16>(sr, sc, neg_m, p_addr);  // -inf -> exactly 0
                    l = fmaf(l, alpha, rs);
                    tmem_st_wait();
                    if (jj > 0) {
                        // O must hold PV(j-1) before it is rescaled. With two tiles, PV_t(j-1) was
                        // issued before QK_t(j), and the commit behind s_full only fires once every
                        // earlier MMA of the issuing thread has completed, so it is done already. With
                        // one tile QK(j) precedes PV(j-1): wait for it (on every step, so this thread
                        // never falls two phases behind on pv_done). The final wait after the loop
                        // always targets the newest phase, which is correct either way.
                        if (c.single && !__all_sync(0xffffffffu, swait(&c.pv_done[t], (gs - 1) & 1, 310 + t))) {
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
                    if (PAIR && c.rank != 0)
                        mbar_arrive_cluster(mapa_shared(&c.p_full[b], 0));  // CTA 0's MMA warp takes the pair's P
                    else
                        mbar_arrive(&c.p_full[b]);
                }
            }
            if (ok)
                ok = __all_sync(0xffffffffu, swait(&c.pv_done[t], (gbase + n - 1) & 1, 320 + t));
            if (!ok) break;
            gbase += n;
            tc_fence_after_sync();
            // the item's coordinates again, computed afresh rather than carried through the key steps
            int eh, eb, eq0, eqbase;
            if (queued) {
                // the item's slot is still this warp's: it is freed when the warp takes its next item
                int qpair, qbh;
                dense_item_of<CAUSAL, GROUPED>(p, c.items[rd % C::QSLOTS], qpair, qbh);
                eb = qbh / p.H;
                eh = qbh % p.H;
                eq0 = PAIR ? (2 * qpair + static_cast<int>(c.rank)) * BM : qpair * C::MAXQ * BM;
                eqbase = eb * p.seqlen + eq0;
            } else {
                item_coords<D, CAUSAL, GROUPED, PAIR>(p, rd, persistent, eh, eb, eq0, eqbase);
            }
            const int64_t otok = static_cast<int64_t>(eqbase) + t * BM + r;
            const bool orow_ok = packed ? otok < p.total_tokens : (eq0 + t * BM + r < p.seqlen);
            const float inv_l = 1.f / l;
            constexpr int RB = D * 2;  // bytes of one row of one head
            if (persistent) {
                // Each thread writes its own row straight from registers: the tile's query buffer
                // may already hold the next item's Q. Up to 128 columns of O come out of TMEM per
                // wait, and each lane stores 32 bytes at a time (whole sectors) when out allows.
                uint8_t *const orow = static_cast<uint8_t *>(p.out) + (otok * p.H + eh) * RB;
                constexpr int CW = (C::MAXQ == 1) ? 64 : (D < 128 ? D : 128);  // O columns per TMEM wave
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += CW) {
                    uint32_t o[CW];
#pragma unroll
                    for (int cc = 0; cc < CW / 32; ++cc) tmem_ld32(c.tmem + lane_base + o_col + c0 + cc * 32, o + cc * 32);
                    tmem_ld_wait();
                    tmem_reg_fence<CW>(o);
                    uint32_t w[CW / 2];
#pragma unroll
                    for (int i = 0; i < CW / 2; ++i)
                        w[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
                    if (orow_ok) {
                        if (p.out_align32) {
#pragma unroll
                            for (int v = 0; v < CW / 16; ++v)
                                asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                                                 orow + c0 * 2 + v * 32),
                                             "r"(w[8 * v]), "r"(w[8 * v + 1]), "r"(w[8 * v + 2]), "r"(w[8 * v + 3]),
                                             "r"(w[8 * v + 4]), "r"(w[8 * v + 5]), "r"(w[8 * v + 6]), "r"(w[8 * v + 7])
                                             : "memory");
                        } else {
#pragma unroll
                            for (int v4 = 0; v4 < CW / 8; ++v4)
                                *reinterpret_cast<uint4 *>(orow + c0 * 2 + v4 * 16) =
                                    make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
                        }
                    }
                }
            } else {
                int64_t orow_idx = (p.gather && orow_ok) ? __ldg(p.gather + otok) : otok;  // fused: padded row
                const bool store_ok = orow_ok && (!p.gather || (orow_idx >= 0 && orow_idx < p.padded_rows));
                // O leaves through this tile's query buffer, unused now that every MMA of the tile
                // has completed (one work item per CTA here): each warp stages its 32 rows there (a
                // lane writes its row, 16-byte chunk c of row r at chunk c ^ (r & 7), so eight
                // lanes hit eight bank groups), then writes whole rows to global memory,
                // consecutive lanes on consecutive 16 bytes.
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
                    uint8_t *const obase = static_cast<uint8_t *>(p.out) + static_cast<int64_t>(eh) * RB + ch * 16;
#pragma unroll 4
                    for (int r0 = 0; r0 < 32; r0 += RPI) {
                        const int rr = r0 + lane / LPR;
                        const int64_t orow_r = __shfl_sync(0xffffffffu, orow_idx, rr);
                        const bool ok_r = __shfl_sync(0xffffffffu, store_ok, rr);
                        const uint4 v = ld_shared_v4(stage + rr * RB + ((ch ^ (rr & XM)) << 4));
                        if (ok_r) *reinterpret_cast<uint4 *>(obase + orow_r * p.H * RB) = v;
                    }
                }
            }
            if (orow_ok && p.lse) {
                const float lse = m * 0.6931471805599453f + logf(l);
                const int64_t li = packed ? static_cast<int64_t>(eh) * p.total_tokens + otok
                                          : (static_cast<int64_t>(eb) * p.H + eh) * p.seqlen + (eq0 + t * BM + r);
                p.lse[li] = lse;
            }
        }
    }

    if (p.gather && warp < C::NUM_SOFTMAX_WARPS) cp_async_wait_all();  // the query copies (abort paths)
    tc_fence_before_sync();
    __syncthreads();
    if (queued && threadIdx.x == 0) {
        // Every index this CTA takes has been taken (the fetching lane used each one before the
        // barrier above); the last CTA to get here zeroes the counter for the next launch.
        __threadfence();
        if (atomicAdd(p.queue + 1, 1) == static_cast<int>(gridDim.x) - 1) {
            atomicExch(p.queue, 0);
            atomicExch(p.queue + 1, 0);
        }
    }
    // pairs: neither CTA leaves (and frees shared memory or TMEM) while the other's MMAs, which
    // read both CTAs' tiles, or its arrivals may still be running
    if (PAIR) cluster_sync();
    if (warp == C::WARP_MMA) {
        tc_fence_after_sync();
        if (PAIR)
            tmem_dealloc_pair(c.tmem, C::TMEM_COLS);
        else
            tmem_dealloc(c.tmem, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host launchers
template <int D, bool BF16, bool CAUSAL, bool PAGED, bool PACKED, bool GROUPED = false>
static cudaError_t launch_t(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                            const FwdParams &p, dim3 grid, cudaStream_t st) {
    using C = Cfg<D>;
    auto kern = fa_fwd_kernel<D, BF16, CAUSAL, PAGED, PACKED, GROUPED>;
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
            if (fa_attr.numRegs * C::NUM_THREADS < 128 * C::regs_low(PACKED) + 256 * C::regs_high(PACKED))
                return cudaErrorInvalidConfiguration;
        }
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        __atomic_fetch_or(&attr_set_mask, bit, __ATOMIC_RELEASE);
    }
    if constexpr (D == 256 && !PAGED && !PACKED) {
        // CTA pairs: clusters of two CTAs along x (the grid is an even number of CTAs)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(C::NUM_THREADS, 1, 1);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, p);
        if (e != cudaSuccess) return e;
        return cudaGetLastError();
    }
    kern<<<grid, C::NUM_THREADS, C::SMEM_BYTES, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace fa
