// fa_seq.cuh -- which packed sequence a token belongs to: lookups in cu_seqlens shared by the
// forward and backward kernels (cu_seqlens[s] <= token < cu_seqlens[s + 1]).
#pragma once
#include <stdint.h>

namespace fa {

// Sequence that packed token `tok` belongs to: the s with cu[s] <= tok < cu[s+1]
// (binary search over the num_seqs + 1 offsets; empty sequences are skipped).
__device__ __forceinline__ int seq_of_token(const int32_t *cu, int num_seqs, int tok) {
    int lo = 0, hi = num_seqs;  // invariant: cu[lo] <= tok < cu[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(cu + mid) <= tok) lo = mid; else hi = mid;
    }
    return lo;
}

// seq_of_token for a token shared by the whole warp: 32 probes per dependent load.
__device__ __forceinline__ int warp_seq_of_token(const int32_t *cu, int num_seqs, int tok, int lane) {
    int lo = 0, hi = num_seqs;  // answer s in [lo, hi - 1]: the last s with cu[s] <= tok
    while (hi - lo > 32) {
        const int step = (hi - lo + 31) / 32;
        const int p = lo + lane * step;
        const bool le = p < hi && __ldg(cu + p) <= tok;
        const int c = __popc(__ballot_sync(0xffffffffu, le));  // probes <= tok form a prefix (c >= 1)
        const int new_lo = lo + (c - 1) * step;
        hi = min(hi, lo + c * step);
        lo = new_lo;
    }
    const int p = lo + lane;
    const bool le = p < hi && __ldg(cu + p) <= tok;
    return lo + __popc(__ballot_sync(0xffffffffu, le)) - 1;
}

// Sequence of each lane's token `tok` (tokens of one warp, >= cu[s0] where s0 is the sequence
// of the warp's first token): one 32-wide load of cu[s0 + 1 ..] and a 5-step search over the
// lanes; falls back to the plain search when the warp's tokens span more than 32 sequences.
__device__ __forceinline__ int lane_seq_of_token(const int32_t *cu, int num_seqs, int s0, int tok, int lane) {
    const int wi = s0 + 1 + lane;
    const int w = (wi <= num_seqs) ? __ldg(cu + wi) : 0x7fffffff;
    int lo = 0, hi = 32;  // count of window entries <= tok, in [lo, hi]
#pragma unroll
    for (int k = 0; k < 6; ++k) {
        const int mid = (lo + hi + 1) >> 1;
        const int v = __shfl_sync(0xffffffffu, w, (mid - 1) & 31);
        if (mid <= hi && lo < hi) {
            if (v <= tok) lo = mid; else hi = mid - 1;
        }
    }
    return (lo < 32) ? s0 + lo : seq_of_token(cu, num_seqs, tok);
}

// cu[0 .. num_seqs] held by a warp, entries lane and 32 + lane of every lane, when
// num_seqs < 64 (`ok`); then seq() and at() need no memory access. Every lane must take part
// in each call, with the same arguments for at().
struct CuWindow {
    int v0, v1;  // cu[lane], cu[32 + lane] (INT32 max past cu[num_seqs])
    int n;       // num_seqs
    bool ok;
    __device__ __forceinline__ CuWindow(const int32_t *cu, int num_seqs, int lane) : n(num_seqs) {
        ok = num_seqs < 64;
        v0 = (ok && lane <= num_seqs) ? __ldg(cu + lane) : 0x7fffffff;
        v1 = (ok && 32 + lane <= num_seqs) ? __ldg(cu + 32 + lane) : 0x7fffffff;
    }
    // the last s < num_seqs with cu[s] <= tok (the entries <= tok form a prefix)
    __device__ __forceinline__ int seq(int tok, int lane) const {
        const unsigned a = __ballot_sync(0xffffffffu, lane < n && v0 <= tok);
        const unsigned b = __ballot_sync(0xffffffffu, 32 + lane < n && v1 <= tok);
        return __popc(a) + __popc(b) - 1;
    }
    // cu[s] for 0 <= s <= num_seqs
    __device__ __forceinline__ int at(int s) const {
        const int x = __shfl_sync(0xffffffffu, v0, s & 31);
        const int y = __shfl_sync(0xffffffffu, v1, s & 31);
        return s < 32 ? x : y;
    }
};

}  // namespace fa
