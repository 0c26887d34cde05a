// Grouping of token->expert assignments by expert, and the row gather that
// feeds the tensor-core path.
//
// The fused MoE kernel of "Jamba-1.5: Hybrid Transformer-Mamba Models at
// Scale" (paper summary, section "Innovation 2") fuses expert routing with
// the expert computation; here routing is split into this bit-exact
// counting sort and the expert GEMMs that consume its output.
//
// k_permute: one CTA of 1024 threads running the stable counting sort of
// permute.cuh.
#include "common.cuh"
#include "kernels.h"
#include "permute.cuh"

namespace jmoe {
namespace {

constexpr int kMaxE = 64;

__global__ void __launch_bounds__(kPermuteThreads)
    k_permute(const int32_t* __restrict__ ids, int64_t A, int E, int pad, int32_t* __restrict__ offsets,
              int32_t* __restrict__ padded_offsets, int32_t* __restrict__ perm,
              int32_t* __restrict__ inv, unsigned* err) {
    block_permute(ids, A, E, pad, offsets, padded_offsets, perm, inv, err);
}

// x_perm[padded_offsets[e] + r] = x[perm[offsets[e] + r] / top_k] for
// r < count_e, zero rows up to the padded end.  One warp per row, 16-B moves.
__global__ void __launch_bounds__(256)
    k_gather_rows(const uint16_t* __restrict__ x, int64_t d, int top_k, int E,
                  const int32_t* __restrict__ offsets, const int32_t* __restrict__ padded_offsets,
                  const int32_t* __restrict__ perm, int64_t T, int64_t max_rows,
                  uint16_t* __restrict__ x_perm) {
    __shared__ int s_off[kMaxE + 1], s_poff[kMaxE + 1];
    if (threadIdx.x <= E) {
        s_off[threadIdx.x] = offsets[threadIdx.x];
        s_poff[threadIdx.x] = padded_offsets[threadIdx.x];
    }
    __syncthreads();
    const int64_t total = s_poff[E];
    const int lane = threadIdx.x & 31;
    const int64_t nvec = d / 8;
    for (int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); row < total && row < max_rows;
         row += (int64_t)gridDim.x * 8) {
        int e = 0;
        while (e + 1 < E && s_poff[e + 1] <= row) ++e;
        const int64_t r = row - s_poff[e];
        uint4* dst = reinterpret_cast<uint4*>(x_perm + row * d);
        if (r < s_off[e + 1] - s_off[e]) {
            const int64_t g = s_off[e] + r;
            if (!JMOE_CHECK(g < (int64_t)T * top_k)) continue;
            const int64_t t = perm[g] / top_k;
            if (!JMOE_CHECK(t >= 0 && t < T)) continue;
            const uint4* src = reinterpret_cast<const uint4*>(x + t * d);
            for (int64_t i = lane; i < nvec; i += 32) dst[i] = __ldg(src + i);
        } else {
            for (int64_t i = lane; i < nvec; i += 32) dst[i] = make_uint4(0, 0, 0, 0);
        }
    }
}

__global__ void k_fill_f32(float* __restrict__ p, float v, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        p[i] = v;
}

}  // namespace

cudaError_t launch_fill_f32(float* p, float v, int64_t n, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    k_fill_f32<<<(unsigned)blocks, 256, 0, stream>>>(p, v, n);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_permute(const int32_t* ids, int64_t A, int E, int pad, int32_t* offsets,
                           int32_t* padded_offsets, int32_t* perm, int32_t* inv, unsigned* err,
                           cudaStream_t stream) {
    k_permute<<<1, kPermuteThreads, 0, stream>>>(ids, A, E, pad, offsets, padded_offsets, perm, inv, err);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* x_bf16, int64_t T, int64_t d, int top_k, int E,
                               const int32_t* offsets, const int32_t* padded_offsets,
                               const int32_t* perm, int64_t max_rows, void* x_perm, int num_sms,
                               cudaStream_t stream) {
    if (max_rows == 0) return cudaSuccess;
    int64_t blocks = (max_rows + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 16;
    if (blocks > cap) blocks = cap;
    k_gather_rows<<<(unsigned)blocks, 256, 0, stream>>>((const uint16_t*)x_bf16, d, top_k, E,
                                                        offsets, padded_offsets, perm, T, max_rows,
                                                        (uint16_t*)x_perm);
    note_launch();
    return cudaGetLastError();
}

JMOE_DEFINE_CHECKS_READER(checks_take_permute)

}  // namespace jmoe
