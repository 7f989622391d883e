// fa_fwd.cu -- the attention forward over contiguous K/V (dense and packed sequences, and the
// fused packed path): instantiations of the kernel in fa_fwd_kernel.cuh (dense persistent and
// packed), the bounded-wait self-test, and the host-side tile geometry shared with fa_api.cu.
#include <atomic>

#include "fa_fwd_kernel.cuh"

namespace fa {

// Counters of the dense item queue, {next item index, CTAs done} per slot (zero while no launch
// uses them: the last CTA of a launch zeroes its slot). Each launch takes the next slot, so
// launches in flight at the same time on other streams use other counters.
constexpr int kQueueSlots = 64;
static __device__ int g_item_queue[2 * kQueueSlots];
static std::atomic<unsigned> g_queue_seq{0};

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

template <int D, bool BF16>
static cudaError_t launch_c(bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, const FwdParams &p, dim3 grid, cudaStream_t st) {
    if (p.cu_seqlens)
        return causal ? launch_t<D, BF16, true, false, true>(tq, tk, tv, p, grid, st)
                      : launch_t<D, BF16, false, false, true>(tq, tk, tv, p, grid, st);
    if (causal)
        return p.num_groups > 1 ? launch_t<D, BF16, true, false, false, true>(tq, tk, tv, p, grid, st)
                                : launch_t<D, BF16, true, false, false>(tq, tk, tv, p, grid, st);
    return launch_t<D, BF16, false, false, false>(tq, tk, tv, p, grid, st);
}

template <int D>
static cudaError_t launch_d(bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                            const CUtensorMap &tv, const FwdParams &p, dim3 grid, cudaStream_t st) {
    return bf16 ? launch_c<D, true>(causal, tq, tk, tv, p, grid, st)
                : launch_c<D, false>(causal, tq, tk, tv, p, grid, st);
}

cudaError_t launch_fwd(int D, bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                       const CUtensorMap &tv, const FwdParams &p_in, dim3 grid, cudaStream_t st) {
    FwdParams p = p_in;
    p.queue = nullptr;
    // Dense inputs over more than one round of the persistent grid (D = 256: of its CTA pairs)
    // take their items from a queue.
    const int units = (D == 256) ? static_cast<int>(grid.x / 2) : static_cast<int>(grid.x);
    if (!p.cu_seqlens && p.num_items > units) {
        void *base = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&base, g_item_queue);  // on the current device
        if (e != cudaSuccess) return e;
        const unsigned slot = g_queue_seq.fetch_add(1u, std::memory_order_relaxed) % kQueueSlots;
        p.queue = static_cast<int *>(base) + 2 * slot;
    }
    switch (D) {
        case 32: return launch_d<32>(bf16, causal, tq, tk, tv, p, grid, st);
        case 64: return launch_d<64>(bf16, causal, tq, tk, tv, p, grid, st);
        case 128: return launch_d<128>(bf16, causal, tq, tk, tv, p, grid, st);
        case 256: return launch_d<256>(bf16, causal, tq, tk, tv, p, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

int fwd_tile_rows() { return 128; }

int fwd_tiles_per_cta(int D) { return (D == 256) ? 1 : 2; }

bool fwd_pair_mode(int D) { return D == 256; }

int fwd_box_inner_elems(int D) { return (2 * D >= 128) ? 64 : D; }

int fwd_kv_tile_rows(int D) { return 128; }
int fwd_v_box_rows(int D) { return (D == 256) ? 64 : 128; }
int fwd_gather_run_rows() { return 32; }
int fwd_paged_k_box_rows(int D, int page_size) { return page_size < fwd_kv_tile_rows(D) ? page_size : fwd_kv_tile_rows(D); }
int fwd_paged_v_box_rows(int D, int page_size) { return page_size < fwd_v_box_rows(D) ? page_size : fwd_v_box_rows(D); }

cudaError_t launch_selftest_wait(uint64_t limit_ns, cudaStream_t st) {
    fa_selftest_wait_kernel<<<1, 32, 0, st>>>(limit_ns);
    return cudaGetLastError();
}

cudaError_t fwd_error_addrs(int **code, int **where) { return device_error_addrs(code, where); }

}  // namespace fa
