// Final combine of the tensor-core path.  The down GEMM's epilogue writes
// every assignment's output row already multiplied by its gate (fp32); the
// layer output of a token is the sum of its slots' rows, rounded once to bf16
// ("Jamba: A Hybrid Transformer-Mamba Language Model", paper summary, section
// "Mixture-of-Experts (MoE) in Jamba: Router, Top-K, and Load Balancing":
// y = sum over the selected experts of g_i Expert_i(h)).
#include "common.cuh"
#include "kernels.h"

namespace jmoe {
namespace {

// out[t] = bf16( sum_j Y[t*top_k + j] ) over the token's valid assignments
// (j ascending).  A CTA takes whole tokens: the token's expert ids are read
// once, and the threads stride over its columns four at a time with every
// slot's row loaded before the first sum, so that each thread keeps several
// 16-byte loads in flight.
__global__ void __launch_bounds__(256)
    k_finalize(const float* __restrict__ Y, int64_t T, int64_t d, int top_k, int E,
               const int32_t* __restrict__ ids, uint16_t* __restrict__ out) {
    constexpr int kMaxK = 4;
    const int nvec = (int)(d / 4);
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        bool ok[kMaxK];
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            const int e = j < top_k ? __ldg(ids + t * top_k + j) : -1;
            ok[j] = e >= 0 && e < E;
        }
        const float* y0 = Y + t * top_k * d;
        uint16_t* o_row = out + t * d;
#pragma unroll 2
        for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
            float4 y[kMaxK];
#pragma unroll
            for (int j = 0; j < kMaxK; ++j)
                if (ok[j]) y[j] = __ldg(reinterpret_cast<const float4*>(y0 + j * d) + i);
            float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < kMaxK; ++j) {
                if (!ok[j]) continue;
                o[0] += y[j].x;
                o[1] += y[j].y;
                o[2] += y[j].z;
                o[3] += y[j].w;
            }
            uint2 r;
            r.x = pack_bf16x2(o[0], o[1]);
            r.y = pack_bf16x2(o[2], o[3]);
            *reinterpret_cast<uint2*>(o_row + 4 * (int64_t)i) = r;
        }
    }
}

}  // namespace

cudaError_t launch_finalize(const float* Y, int64_t T, int64_t d, int top_k, int E,
                            const int32_t* ids, void* out, int num_sms, cudaStream_t stream) {
    if (T <= 0) return cudaSuccess;
    const int64_t cap = (int64_t)num_sms * 8;  // 8 CTAs of 256 threads per SM
    k_finalize<<<(unsigned)(T < cap ? T : cap), 256, 0, stream>>>(Y, T, d, top_k, E, ids,
                                                                 static_cast<uint16_t*>(out));
    note_launch();
    return cudaGetLastError();
}

}  // namespace jmoe
