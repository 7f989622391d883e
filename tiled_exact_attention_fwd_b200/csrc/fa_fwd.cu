// fa_fwd.cu -- exact attention forward, tile by tile, on sm_100a.
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
// B200 design (one CTA = one 128-row query tile of one head of one sequence):
//   warp 0      TMA producer: Q once, then K_j / V_j tiles through an NS-stage ring of
//               shared-memory slots guarded by full/empty mbarriers, in the exact order
//               the MMA warp consumes them (K0, K1, V0, K2, V1, ..., V_last).
//   warp 1      allocates TMEM; one thread issues every tcgen05.mma:
//                 S_j = Q K_j^T    (A = Q, B = K_j, both K-major in SMEM, 128B swizzle)
//                 O  += P_j V_j    (A = P_j read from TMEM, B = V_j MN-major in SMEM)
//               S is double-buffered in TMEM so S_{j+1} is computed while the softmax
//               warps work on S_j; P_j (16-bit) overwrites the first half of S_j's columns.
//   warps 2-5   softmax: thread t owns query row t (TMEM lane t). It reads its S row
//               with tcgen05.ld, masks, updates (m, l) with exp2 of scores pre-multiplied
//               by scale*log2(e), writes P back to TMEM and, when its max grew by more than
//               2^8, rescales its O row in TMEM (lazy rescale: between rescales every
//               exponent uses the same stale max, which the final 1/l cancels exactly).
//               At the end it normalises O by 1/l, stores O (fp16/bf16) and the LSE.
//
// Every pipeline wait is bounded: after `timeout_ns` the waiting thread records
// FA_ERR_TIMEOUT in a device word, raises a CTA-wide abort flag, and all roles drain
// their in-flight copies/MMAs (again with a bound) before TMEM is released.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fa.h"
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {

static __device__ int g_err_code;
static __device__ int g_err_where;

__device__ __noinline__ void record_error(int code, int where) {
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

template <int D>
struct Cfg {
    static constexpr int BM = 128;                        // query rows per tile (MMA M)
    static constexpr int BN = (D == 256) ? 64 : 128;      // key rows per tile
    static constexpr int SW = (2 * D >= 128) ? 128 : 2 * D;  // swizzle span in bytes
    static constexpr int SWE = SW / 2;                    // 16-bit elements per swizzle row
    static constexpr int NBLK = D / SWE;                  // column blocks per tile row
    static constexpr int Q_BYTES = BM * D * 2;
    static constexpr int KV_BYTES = BN * D * 2;
    static constexpr int NS = (D == 32) ? 8 : (D == 64) ? 6 : (D == 128) ? 5 : 4;
    static constexpr uint32_t LAYOUT = (SW == 128) ? kLayoutSw128 : kLayoutSw64;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t O_COL = 2 * BN;            // S0 at col 0, S1 at col BN, O after
    static constexpr int NUM_THREADS = 192;
    // shared memory map (offsets from a 1024-byte aligned base)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = Q_BYTES;
    static constexpr int OFF_BAR = OFF_KV + NS * KV_BYTES;
    static constexpr int NUM_BARS = 1 + 2 * NS + 2 + 2 + 1 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int USED = OFF_MISC + 16;
    // Ask for more than half of the SM's shared memory so exactly one CTA (and one
    // 512-column TMEM allocation) lives on an SM.
    static constexpr int MIN_SMEM = 120 * 1024;
    static constexpr int SMEM_BYTES = (USED + 1024 > MIN_SMEM) ? USED + 1024 : MIN_SMEM;
    static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
    static_assert(USED + 1024 <= 227 * 1024, "shared memory budget");
    static_assert(Q_BYTES % 1024 == 0 && KV_BYTES % 1024 == 0, "tile alignment");
};

// Position of load/consume step `idx` in the sequence K0, K1, V0, K2, V1, ..., V_{n-1}.
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

template <int D, bool BF16, bool CAUSAL>
__global__ void __launch_bounds__(192, 1)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
    using C = Cfg<D>;
    constexpr int BM = C::BM, BN = C::BN, SW = C::SW, NS = C::NS;

    const int h = blockIdx.x;
    const int qt = gridDim.y - 1 - blockIdx.y;  // longest (causal) tiles first
    const int seq = blockIdx.z;
    int seq_start, seqlen;
    if (p.cu_seqlens) {
        seq_start = p.cu_seqlens[seq];
        seqlen = p.cu_seqlens[seq + 1] - seq_start;
    } else {
        seq_start = seq * p.seqlen;
        seqlen = p.seqlen;
    }
    const int q0 = qt * BM;
    if (q0 >= seqlen) return;  // uniform over the CTA, before any barrier exists
    const int kv_end = CAUSAL ? min(seqlen, q0 + BM) : seqlen;
    const int n_kv = (kv_end + BN - 1) / BN;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sKV = smem + C::OFF_KV;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars;
    uint64_t *kv_full = bars + 1;
    uint64_t *kv_empty = bars + 1 + NS;
    uint64_t *s_full = bars + 1 + 2 * NS;
    uint64_t *p_full = s_full + 2;
    uint64_t *pv_done = p_full + 2;
    uint64_t *drain = pv_done + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&p_full[b], 128);
        }
        mbar_init(pv_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint64_t lim = p.timeout_ns;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last();
            mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
            for (int b = 0; b < C::NBLK; ++b)
                tma_load_3d(sQ + b * BM * SW, &tm_q, q_full, b * C::SWE, h, seq_start + q0, pol_q);
            const int steps = 2 * n_kv;
            int issued = 0;
            for (int idx = 0; idx < steps; ++idx) {
                const int stage = idx % NS;
                if (idx >= NS &&
                    !wait_bounded(&kv_empty[stage], ((idx / NS) - 1) & 1, abort_flag, lim, 100 + stage))
                    break;
                bool is_v;
                int j;
                decode_step(idx, n_kv, is_v, j);
                uint8_t *dst = sKV + stage * C::KV_BYTES;
                mbar_arrive_expect_tx(&kv_full[stage], C::KV_BYTES);
                const CUtensorMap *map = is_v ? &tm_v : &tm_k;
#pragma unroll
                for (int b = 0; b < C::NBLK; ++b)
                    tma_load_3d(dst + b * BN * SW, map, &kv_full[stage], b * C::SWE, h,
                                seq_start + j * BN, pol_kv);
                issued = idx + 1;
            }
            if (*abort_flag) {
                // Let the copies already issued land before the CTA's shared memory goes away.
                wait_bounded(q_full, 0, abort_flag, lim, 190);
                for (int idx = (issued > NS ? issued - NS : 0); idx < issued; ++idx) {
                    const int stage = idx % NS;
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(&kv_full[stage], (idx / NS) & 1) &&
                           global_timer_ns() - t0 < lim) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_f16(BM, BN, BF16, false);
            constexpr uint32_t idesc_pv = idesc_f16(BM, D, BF16, true);
            bool ok = wait_bounded(q_full, 0, abort_flag, lim, 200);
            tc_fence_after_sync();
            const uint32_t q_addr = smem_u32(sQ);
            const int steps = 2 * n_kv;
            for (int idx = 0; ok && idx < steps; ++idx) {
                const int stage = idx % NS;
                bool is_v;
                int j;
                decode_step(idx, n_kv, is_v, j);
                if (is_v) {
                    if (!wait_bounded(&p_full[j & 1], (j >> 1) & 1, abort_flag, lim, 210)) break;
                    tc_fence_after_sync();
                }
                if (!wait_bounded(&kv_full[stage], (idx / NS) & 1, abort_flag, lim, 220 + stage)) break;
                tc_fence_after_sync();
                const uint32_t kv_addr = smem_u32(sKV + stage * C::KV_BYTES);
                if (!is_v) {
                    const uint32_t d_tmem = tmem + (j & 1) * BN;
#pragma unroll
                    for (int t = 0; t < D / 16; ++t) {
                        const uint32_t blk = (t * 32) / SW, off = (t * 32) % SW;
                        const uint64_t a = smem_desc(q_addr + blk * BM * SW + off, 16, 8 * SW, C::LAYOUT);
                        const uint64_t b = smem_desc(kv_addr + blk * BN * SW + off, 16, 8 * SW, C::LAYOUT);
                        umma_ss(d_tmem, a, b, idesc_qk, t > 0 ? 1u : 0u);
                    }
                    umma_commit(&kv_empty[stage]);
                    umma_commit(&s_full[j & 1]);
                } else {
                    const uint32_t a_tmem = tmem + (j & 1) * BN;
#pragma unroll
                    for (int t = 0; t < BN / 16; ++t) {
                        const uint64_t b = smem_desc(kv_addr + t * 16 * SW, BN * SW, 8 * SW, C::LAYOUT);
                        umma_ts(tmem + C::O_COL, a_tmem + t * 8, b, idesc_pv, (j > 0 || t > 0) ? 1u : 0u);
                    }
                    umma_commit(&kv_empty[stage]);
                    umma_commit(pv_done);
                }
            }
            // Every MMA issued above has finished once `drain` completes.
            umma_commit(drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < lim) {
            }
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int quarter = warp & 3;                 // TMEM lanes this warp may access
        const int r = quarter * 32 + lane;            // row of the tile == TMEM lane
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const int row_pos = q0 + r;                   // position inside the sequence
        const int row_lim = CAUSAL ? min(seqlen, row_pos + 1) : seqlen;  // keys [0, row_lim)
        const float c = p.scale_log2;
        float m = -INFINITY;  // running max of scaled scores, log2 units (possibly stale)
        float l = 0.f;        // running sum of 2^(t - m)
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            if (!__all_sync(0xffffffffu, wait_bounded(&s_full[j & 1], (j >> 1) & 1, abort_flag, lim, 300))) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            uint32_t sr[BN];
#pragma unroll
            for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32(tmem + lane_base + (j & 1) * BN + cc * 32, sr + cc * 32);
            tmem_ld_wait();
            tmem_reg_fence<BN>(sr);
            const int kv0 = j * BN;
            const bool need_mask = (kv0 + BN > seqlen) || (CAUSAL && kv0 + BN - 1 > q0);
            if (need_mask) {
                const int valid = row_lim - kv0;  // columns [0, valid) of this tile are visible
#pragma unroll
                for (int i = 0; i < BN; ++i)
                    if (i >= valid) sr[i] = __float_as_uint(-INFINITY);
            }
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < BN; ++i) mx = fmaxf(mx, __uint_as_float(sr[i]));
            const float m_cand = mx * c;
            const bool grow = m_cand > m + 8.0f;
            float alpha = 1.f;
            if (grow) {
                alpha = ex2_approx(m - m_cand);
                m = m_cand;
            }
            const bool warp_grow = __any_sync(0xffffffffu, grow);
            float rs = 0.f;
            uint32_t pk[BN / 2];
#pragma unroll
            for (int i = 0; i < BN / 2; ++i) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(sr[2 * i]), c, -m));
                const float p1 = ex2_approx(fmaf(__uint_as_float(sr[2 * i + 1]), c, -m));
                rs += p0 + p1;
                pk[i] = pack2<BF16>(p0, p1);
            }
            l = l * alpha + rs;
#pragma unroll
            for (int cc = 0; cc < BN / 64; ++cc) tmem_st32(tmem + lane_base + (j & 1) * BN + cc * 32, pk + cc * 32);
            tmem_st_wait();
            if (j > 0) {
                // PV_{j-1} is waited for on every tile (it has normally finished long before),
                // so this thread never falls two phases behind on pv_done.
                if (!__all_sync(0xffffffffu, wait_bounded(pv_done, (j - 1) & 1, abort_flag, lim, 310))) {
                    ok = false;
                    break;
                }
            }
            if (warp_grow && j > 0) {
                // O holds sum_{j' < j} P_j' V_j'; bring it to the new running max.
                tc_fence_after_sync();
#pragma unroll 1
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + C::O_COL + cc * 32, o);
                    tmem_ld_wait();
                    tmem_reg_fence<32>(o);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st32(tmem + lane_base + C::O_COL + cc * 32, o);
                }
                tmem_st_wait();
            }
            tc_fence_before_sync();
            mbar_arrive(&p_full[j & 1]);
        }
        if (ok) ok = __all_sync(0xffffffffu, wait_bounded(pv_done, (n_kv - 1) & 1, abort_flag, lim, 320));
        if (ok) {
            tc_fence_after_sync();
            const float inv_l = 1.f / l;
            const int64_t tok = static_cast<int64_t>(seq_start) + row_pos;
            const bool row_ok = row_pos < seqlen && tok < p.total_tokens;
            uint4 *orow = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(p.out) +
                                                    (tok * p.H + h) * static_cast<int64_t>(D) * 2);
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_base + C::O_COL + cc * 32, o);
                tmem_ld_wait();
                tmem_reg_fence<32>(o);
                uint32_t w[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack2<BF16>(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
                if (row_ok) {
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4)
                        orow[cc * 4 + v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
                }
            }
            if (row_ok && p.lse) {
                const float lse = m * 0.6931471805599453f + logf(l);
                const int64_t li = p.cu_seqlens ? static_cast<int64_t>(h) * p.total_tokens + tok
                                                : (static_cast<int64_t>(seq) * p.H + h) * p.seqlen + row_pos;
                p.lse[li] = lse;
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// One CTA waits on a barrier that nothing completes; the bounded wait must give up.
__global__ void fa_selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) wait_bounded(&bar, 0, &abort_flag, limit_ns, 900);
}

// ------------------------------------------------------------------ host launchers
template <int D, bool BF16, bool CAUSAL>
static cudaError_t launch_t(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                            const FwdParams &p, dim3 grid, cudaStream_t st) {
    using C = Cfg<D>;
    auto kern = fa_fwd_kernel<D, BF16, CAUSAL>;
    // The shared-memory opt-in is a per-device function attribute; setting it twice is harmless.
    static uint64_t attr_set_mask = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = uint64_t(1) << (dev & 63);
    if (!(__atomic_load_n(&attr_set_mask, __ATOMIC_ACQUIRE) & bit)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        __atomic_fetch_or(&attr_set_mask, bit, __ATOMIC_RELEASE);
    }
    kern<<<grid, C::NUM_THREADS, C::SMEM_BYTES, st>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

template <int D, bool BF16>
static cudaError_t launch_c(bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, const FwdParams &p, dim3 grid, cudaStream_t st) {
    return causal ? launch_t<D, BF16, true>(tq, tk, tv, p, grid, st)
                  : launch_t<D, BF16, false>(tq, tk, tv, p, grid, st);
}

template <int D>
static cudaError_t launch_d(bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, const FwdParams &p, dim3 grid, cudaStream_t st) {
    return bf16 ? launch_c<D, true>(causal, tq, tk, tv, p, grid, st)
                : launch_c<D, false>(causal, tq, tk, tv, p, grid, st);
}

cudaError_t launch_fwd(int D, bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const FwdParams &p, dim3 grid, cudaStream_t st) {
    switch (D) {
        case 32: return launch_d<32>(bf16, causal, tq, tk, tv, p, grid, st);
        case 64: return launch_d<64>(bf16, causal, tq, tk, tv, p, grid, st);
        case 128: return launch_d<128>(bf16, causal, tq, tk, tv, p, grid, st);
        case 256: return launch_d<256>(bf16, causal, tq, tk, tv, p, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

int fwd_tile_rows() { return 128; }

int fwd_box_inner_elems(int D) { return (2 * D >= 128) ? 64 : D; }

int fwd_kv_tile_rows(int D) { return (D == 256) ? 64 : 128; }

cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t st) {
    fa_selftest_wait_kernel<<<1, 32, 0, st>>>(limit_ns);
    return cudaGetLastError();
}

cudaError_t fwd_take_device_error(int *code, int *where) {
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_err_code, sizeof(int));
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(where, g_err_where, sizeof(int));
    if (e != cudaSuccess) return e;
    e = cudaMemcpyToSymbol(g_err_code, &zero, sizeof(int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_err_where, &zero, sizeof(int));
}

}  // namespace fa
