// fa_fwd_paged.cu -- the attention forward with K/V read through a block table from page
// pools (fa_fwd_paged): the PAGED instantiations of the kernel in fa_fwd_kernel.cuh.
#include "fa_fwd_kernel.cuh"

namespace fa {

template <int D, bool BF16>
static cudaError_t launch_paged_c(bool causal, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                                  const FwdParams &p, dim3 grid, cudaStream_t st) {
    if (causal)
        return p.num_groups > 1 ? launch_t<D, BF16, true, true, false, true>(tq, tk, tv, p, grid, st)
                                : launch_t<D, BF16, true, true, false>(tq, tk, tv, p, grid, st);
    return launch_t<D, BF16, false, true, false>(tq, tk, tv, p, grid, st);
}

template <int D>
static cudaError_t launch_paged_d(bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                                  const CUtensorMap &tv, const FwdParams &p, dim3 grid, cudaStream_t st) {
    return bf16 ? launch_paged_c<D, true>(causal, tq, tk, tv, p, grid, st)
                : launch_paged_c<D, false>(causal, tq, tk, tv, p, grid, st);
}

cudaError_t launch_fwd_paged(int D, bool bf16, bool causal, const CUtensorMap &tq, const CUtensorMap &tk,
                             const CUtensorMap &tv, const FwdParams &p, dim3 grid, cudaStream_t st) {
    switch (D) {
        case 32: return launch_paged_d<32>(bf16, causal, tq, tk, tv, p, grid, st);
        case 64: return launch_paged_d<64>(bf16, causal, tq, tk, tv, p, grid, st);
        case 128: return launch_paged_d<128>(bf16, causal, tq, tk, tv, p, grid, st);
        case 256: return launch_paged_d<256>(bf16, causal, tq, tk, tv, p, grid, st);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t fwd_paged_error_addrs(int **code, int **where) { return device_error_addrs(code, where); }

}  // namespace fa
