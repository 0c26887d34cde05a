// Stable counting sort of token->expert assignments by expert, as a block
// function for a CTA of kPermuteThreads threads (used by the grouping kernel
// and by the decode path's preparation kernel); up to kPermuteWarpMaxA
// assignments one warp of it sorts (warp_permute), larger inputs go through:
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
constexpr int64_t kPermuteWarpMaxA = 1024;  // up to here one warp sorts (no block barriers)

// The same stable counting sort by one warp, 32 assignments at a time in
// ascending order: pass 1 counts (the lowest lane of each expert adds its
// group's size), a warp scan gives the offsets, pass 2 places every
// assignment at its expert's cursor plus its rank among the lower lanes of
// the same expert.  For the few assignments of a decode batch this replaces
// the block-wide passes and their barriers.
__device__ __forceinline__ void warp_permute(const int32_t* __restrict__ ids, int64_t A, int E,
                                             int pad, int32_t* __restrict__ offsets,
                                             int32_t* __restrict__ padded_offsets,
                                             int32_t* __restrict__ perm,
                                             int32_t* __restrict__ inv, unsigned* err,
                                             int* s_count, int* s_cursor) {
    const int lane = threadIdx.x & 31;
    auto expert = [&](int64_t a) {
        int e = a < A ? (ids ? ids[a] : 0) : -1;
        return e >= 0 && e < E ? e : -1;
    };
    s_count[lane] = 0;
    s_count[lane + 32] = 0;
    __syncwarp();
    bool bad = false;
    for (int64_t base = 0; base < A; base += 32) {
        const int64_t a = base + lane;
        const int e = expert(a);
        bad |= a < A && e < 0;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (peers & ((1u << lane) - 1u)) == 0) s_count[e] += __popc(peers);
        __syncwarp();
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0 && err) flag_error(err, kErrBadExpert);
    // exclusive scans of the counts (experts lane and lane + 32), plain and padded
    const int c0 = lane < E ? s_count[lane] : 0, c1 = lane + 32 < E ? s_count[lane + 32] : 0;
    const int p0 = (c0 + pad - 1) / pad * pad, p1 = (c1 + pad - 1) / pad * pad;
    int i0 = c0, i1 = c1, q0 = p0, q1 = p1;  // inclusive scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u0 = __shfl_up_sync(0xffffffffu, i0, o), u1 = __shfl_up_sync(0xffffffffu, i1, o);
        const int v0 = __shfl_up_sync(0xffffffffu, q0, o), v1 = __shfl_up_sync(0xffffffffu, q1, o);
        if (lane >= o) { i0 += u0; i1 += u1; q0 += v0; q1 += v1; }
    }
    const int tot0 = __shfl_sync(0xffffffffu, i0, 31), ptot0 = __shfl_sync(0xffffffffu, q0, 31);
    const int off0 = i0 - c0, off1 = tot0 + i1 - c1;
    const int poff0 = q0 - p0, poff1 = ptot0 + q1 - p1;
    if (lane < E) {
        offsets[lane] = off0;
        if (padded_offsets) padded_offsets[lane] = poff0;
    }
    if (lane + 32 < E) {
        offsets[lane + 32] = off1;
        if (padded_offsets) padded_offsets[lane + 32] = poff1;
    }
    if (lane == E - 1 || lane + 32 == E - 1) {
        offsets[E] = lane == E - 1 ? off0 + c0 : off1 + c1;
        if (padded_offsets) padded_offsets[E] = lane == E - 1 ? poff0 + p0 : poff1 + p1;
    }
    s_cursor[lane] = off0;
    s_cursor[lane + 32] = off1;
    __syncwarp();
    for (int64_t base = 0; base < A; base += 32) {
        const int64_t a = base + lane;
        const int e = expert(a);
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const unsigned lower = peers & ((1u << lane) - 1u);
        if (e >= 0) {
            const int pos = s_cursor[e] + __popc(lower);
            if (JMOE_CHECK(pos >= 0 && pos < A)) {
                perm[pos] = (int32_t)a;
                if (inv) inv[a] = pos;
            }
        } else if (a < A && inv) {
            inv[a] = -1;
        }
        __syncwarp();
        if (e >= 0 && lower == 0) s_cursor[e] += __popc(peers);
        __syncwarp();
    }
}

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
    if (A <= kPermuteWarpMaxA) {
        if (warp == 0)
            warp_permute(ids, A, E, pad, offsets, padded_offsets, perm, inv, err, s_count, s_cursor);
        return;
    }
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
            if (JMOE_CHECK(pos >= 0 && pos < A)) {
                perm[pos] = (int32_t)a;
                if (inv) inv[a] = pos;
            }
        } else if (a < A && inv) {
            inv[a] = -1;
        }
        __syncthreads();
        if (tid < E) s_cursor[tid] += s_count[tid];
        __syncthreads();
    }
}

}  // namespace jmoe
