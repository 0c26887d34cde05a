// Stable counting sort of token->expert assignments by expert, as a block
// function for a CTA of kPermuteThreads threads (used by the grouping kernel
// and by the decode path's preparation kernel).
//
//   pass 1: per-expert counts (shared-memory atomics; order-independent);
//   scan:   offsets[e] = exclusive prefix; padded offsets (each count rounded
//           up to `pad`) when asked for;
//   pass 2: the assignments are visited in ascending order, kPermuteThreads at
//           a time; inside a warp __match_any_sync groups lanes with the same
//           expert and a popcount of the lower lanes gives the stable rank;
//           per-warp counts are prefix-summed across the warps.  perm and inv
//           come out identical to a stable counting sort.
// Assignments whose expert id is outside [0, E) are left out of the groups
// (inv = -1) and raise kErrBadExpert in the device error word.  ids == nullptr
// means every assignment goes to expert 0 (the dense layer).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace jmoe {

constexpr int kPermuteThreads = 1024;
constexpr int kPermuteMaxE = 64;

__device__ __forceinline__ void block_permute(const int32_t* __restrict__ ids, int64_t A, int E,
                                              int pad, int32_t* __restrict__ offsets,
                                              int32_t* __restrict__ padded_offsets,
                                              int32_t* __restrict__ perm,
                                              int32_t* __restrict__ inv, unsigned* err) {
    constexpr int kWarps = kPermuteThreads / 32;
    __shared__ int s_count[kPermuteMaxE];
    __shared__ int s_cursor[kPermuteMaxE];
    __shared__ int s_warp_count[kWarps][kPermuteMaxE];
    __shared__ int s_warp_base[kWarps][kPermuteMaxE];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    auto expert = [&](int64_t a) { return ids ? ids[a] : 0; };

    if (tid < kPermuteMaxE) s_count[tid] = 0;
    __syncthreads();
    bool bad = false;
    for (int64_t a = tid; a < A; a += kPermuteThreads) {
        const int e = expert(a);
        if (e >= 0 && e < E)
            atomicAdd(&s_count[e], 1);
        else
            bad = true;
    }
    if (bad && err) flag_error(err, kErrBadExpert);
    __syncthreads();
    if (tid == 0) {
        int run = 0, prun = 0;
        for (int e = 0; e < E; ++e) {
            offsets[e] = run;
            if (padded_offsets) padded_offsets[e] = prun;
            s_cursor[e] = run;
            run += s_count[e];
            prun += (s_count[e] + pad - 1) / pad * pad;
        }
        offsets[E] = run;
        if (padded_offsets) padded_offsets[E] = prun;
    }
    for (int i = tid; i < kWarps * kPermuteMaxE; i += kPermuteThreads)
        (&s_warp_count[0][0])[i] = 0;
    __syncthreads();

    for (int64_t base = 0; base < A; base += kPermuteThreads) {
        const int64_t a = base + tid;
        int e = a < A ? expert(a) : -1;
        if (e < 0 || e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0 && rank == 0) s_warp_count[warp][e] = __popc(peers);
        __syncthreads();
        if (tid < E) {
            int run = 0;
            for (int w = 0; w < kWarps; ++w) {
                s_warp_base[w][tid] = run;
                run += s_warp_count[w][tid];
                s_warp_count[w][tid] = 0;
            }
            s_count[tid] = run;  // this chunk's total for expert tid
        }
        __syncthreads();
        if (e >= 0) {
            const int pos = s_cursor[e] + s_warp_base[warp][e] + rank;
            perm[pos] = (int32_t)a;
            if (inv) inv[a] = pos;
        } else if (a < A && inv) {
            inv[a] = -1;
        }
        __syncthreads();
        if (tid < E) s_cursor[tid] += s_count[tid];
        __syncthreads();
    }
}

}  // namespace jmoe
