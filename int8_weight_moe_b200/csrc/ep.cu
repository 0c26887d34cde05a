// Expert parallelism: the layer's experts split over G ranks (GPUs), each
// token's rows sent to the ranks that own its selected experts and the expert
// outputs sent back.
//
// "Jamba: A Hybrid Transformer-Mamba Language Model" (paper summary),
// sections "Training Infrastructure and Stabilization Techniques" (expert
// parallelism, with all-to-all communication routing tokens to the GPU that
// holds their selected experts) and "Mixture-of-Experts (MoE) in Jamba:
// Router, Top-K, and Load Balancing" (the MoE layers need all-to-all
// communication under expert parallelism).
//
// Rank g owns the E/G consecutive experts [g E/G, (g+1) E/G).  Grouping the
// assignments by expert (the stable counting sort of permute.cuh) therefore
// also groups them by owner rank, in rank order: the send buffer is the token
// rows in that order, and rank r's block is rows offsets[r E/G] ..
// offsets[(r+1) E/G].  These kernels build the send buffer and finish the
// combine; the exchange itself is an all-to-all between the two.
//   k_ep_pack:    x_send[i] = x[perm[i] / top_k], local_ids[i] = expert % (E/G)
//   k_ep_combine: out[t] = bf16( sum_j g_tj * y_back[inv[t top_k + j]] )
#include "common.cuh"
#include "kernels.h"

namespace jmoe {
namespace {

// One warp per send row, 16-byte moves; lane 0 writes the row's expert index
// within its owner rank.
__global__ void __launch_bounds__(256)
    k_ep_pack(const uint16_t* __restrict__ x, int64_t T, int64_t d, int top_k,
              const int32_t* __restrict__ ids, const int32_t* __restrict__ perm,
              const int32_t* __restrict__ offsets, int E, int E_local,
              uint16_t* __restrict__ x_send, int32_t* __restrict__ local_ids) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t rows = offsets[E];  // assignments with a valid expert id
    const int lane = threadIdx.x & 31;
    const int64_t nvec = d / 8;
    for (int64_t i = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); i < rows;
         i += (int64_t)gridDim.x * 8) {
        if (!JMOE_CHECK(i < T * top_k)) break;
        const int32_t a = perm[i];
        if (!JMOE_CHECK(a >= 0 && a < T * top_k)) continue;
        const int64_t t = a / top_k;
        const uint4* src = reinterpret_cast<const uint4*>(x + t * d);
        uint4* dst = reinterpret_cast<uint4*>(x_send + i * d);
        for (int64_t v = lane; v < nvec; v += 32) dst[v] = __ldg(src + v);
        if (lane == 0) local_ids[i] = ids[a] % E_local;
    }
}

// Block (chunk of 1024 channels, token): each thread sums 4 consecutive
// channels of the token's returned rows in assignment order, fp32, one
// rounding to bf16.  Assignments left out by the grouping (inv < 0) add
// nothing.
constexpr int kChunk = 1024;

__global__ void __launch_bounds__(256)
    k_ep_combine(const uint16_t* __restrict__ y_back, const int32_t* __restrict__ inv,
                 const float* __restrict__ gates, int64_t T, int64_t d, int top_k,
                 uint16_t* __restrict__ out) {
    pdl_wait();
    pdl_launch_dependents();
    const int64_t m = (int64_t)blockIdx.x * kChunk + threadIdx.x * 4;
    if (m >= d) return;
    for (int64_t t = blockIdx.y; t < T; t += gridDim.y) {
        float o[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < top_k; ++j) {
            const int64_t a = t * top_k + j;
            const int32_t slot = inv[a];
            if (slot < 0 || !JMOE_CHECK(slot < T * top_k)) continue;
            const float g = gates[a];
            const uint2 v = *reinterpret_cast<const uint2*>(y_back + (int64_t)slot * d + m);
            o[0] += g * bf16_bits_to_f32((uint16_t)(v.x & 0xffffu));
            o[1] += g * bf16_bits_to_f32((uint16_t)(v.x >> 16));
            o[2] += g * bf16_bits_to_f32((uint16_t)(v.y & 0xffffu));
            o[3] += g * bf16_bits_to_f32((uint16_t)(v.y >> 16));
        }
        uint2 r;
        r.x = pack_bf16x2(o[0], o[1]);
        r.y = pack_bf16x2(o[2], o[3]);
        *reinterpret_cast<uint2*>(out + t * d + m) = r;
    }
}

}  // namespace

cudaError_t launch_ep_dispatch(const void* x, int64_t T, int64_t d, const int32_t* ids, int top_k,
                               int E, int E_local, int32_t* offsets, int32_t* perm, int32_t* inv,
                               void* x_send, int32_t* local_ids, unsigned* err, int num_sms,
                               cudaStream_t stream) {
    const int64_t A = T * top_k;
    cudaError_t e = launch_permute(ids, A, E, 1, offsets, nullptr, perm, inv, err, stream);
    if (e != cudaSuccess) return e;
    int64_t blocks = (A + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return launch_pdl(k_ep_pack, dim3((unsigned)blocks), dim3(256), 0, stream,
                      static_cast<const uint16_t*>(x), T, d, top_k, ids,
                      static_cast<const int32_t*>(perm), static_cast<const int32_t*>(offsets), E,
                      E_local, static_cast<uint16_t*>(x_send), local_ids);
}

cudaError_t launch_ep_combine(const void* y_back, const int32_t* inv, const float* gates,
                              int64_t T, int64_t d, int top_k, void* out, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    return launch_pdl(k_ep_combine,
                      dim3((unsigned)((d + kChunk - 1) / kChunk), (unsigned)(T < 65535 ? T : 65535)),
                      dim3(256), 0, stream, static_cast<const uint16_t*>(y_back), inv, gates, T, d,
                      top_k, static_cast<uint16_t*>(out));
}

JMOE_DEFINE_CHECKS_READER(checks_take_ep)

}  // namespace jmoe
