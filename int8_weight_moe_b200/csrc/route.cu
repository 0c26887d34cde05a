// Router: logits, softmax over the experts, top-k selection, renormalised
// gates.
//
// "Jamba: A Hybrid Transformer-Mamba Language Model" (paper summary), section
// "Mixture-of-Experts (MoE) in Jamba: Router, Top-K, and Load Balancing":
// g = softmax(W_r h) with W_r of shape [n, d]; the top K = 2 experts are
// selected and their probabilities renormalised over the selected set.
//
// One warp per token.  Lane j accumulates the fp64 partial sum
// p_j = sum over k = j, j+32, ... (ascending) of x_k * w_ek for every expert;
// the 32 partial sums are then combined by the halving tree
// p_j += p_{j+o}, o = 16, 8, 4, 2, 1 (a shuffle-down reduction), the bias is
// added in fp64 and the result rounded once to fp32.  The products are exact
// in fp64, so this fixed order makes the logits -- and the top-k ids chosen
// from them -- reproducible bit for bit.  Softmax and gates are fp32.
#include "common.cuh"
#include "kernels.h"

namespace jmoe {
namespace {

constexpr int kWarps = 8;
constexpr int kMaxE = 16;

__global__ void __launch_bounds__(kWarps * 32)
    k_route(const uint16_t* __restrict__ x, int64_t T, int64_t d, const float* __restrict__ wr,
            const float* __restrict__ bias, int E, int top_k, int32_t* __restrict__ ids,
            float* __restrict__ gates, float* __restrict__ logits) {
    const int lane = threadIdx.x & 31;
    const int64_t warp_global = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * kWarps;
    for (int64_t t = warp_global; t < T; t += nwarps) {
        const uint16_t* xr = x + t * d;
        double acc[kMaxE];
#pragma unroll
        for (int e = 0; e < kMaxE; ++e) acc[e] = 0.0;
        for (int64_t k = lane; k < d; k += 32) {
            const double xk = (double)bf16_bits_to_f32(__ldg(xr + k));
#pragma unroll
            for (int e = 0; e < kMaxE; ++e)
                if (e < E) acc[e] = fma(xk, (double)__ldg(wr + (int64_t)e * d + k), acc[e]);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
#pragma unroll
            for (int e = 0; e < kMaxE; ++e) acc[e] += __shfl_down_sync(0xffffffffu, acc[e], o);
        }
        if (lane == 0) {
            float l[kMaxE];
#pragma unroll
            for (int e = 0; e < kMaxE; ++e) {
                const double b = (bias && e < E) ? (double)bias[e] : 0.0;
                l[e] = e < E ? __double2float_rn(acc[e] + b) : -INFINITY;
            }
            if (logits)
                for (int e = 0; e < E; ++e) logits[t * E + e] = l[e];
            // top-k on the fp32 logits: strict '>' keeps the lower index on ties
            int e1 = 0;
            for (int e = 1; e < E; ++e)
                if (l[e] > l[e1]) e1 = e;
            int e2 = -1;
            if (top_k == 2) {
                for (int e = 0; e < E; ++e)
                    if (e != e1 && (e2 < 0 || l[e] > l[e2])) e2 = e;
            }
            // fp32 softmax over all E experts
            float p[kMaxE];
            const float m = l[e1];
            float z = 0.0f;
            for (int e = 0; e < E; ++e) {
                p[e] = expf(l[e] - m);
                z += p[e];
            }
            for (int e = 0; e < E; ++e) p[e] = p[e] / z;
            if (top_k == 1) {
                ids[t] = e1;
                gates[t] = 1.0f;
            } else {
                const float sel = p[e1] + p[e2];
                ids[2 * t] = e1;
                ids[2 * t + 1] = e2;
                gates[2 * t] = p[e1] / sel;
                gates[2 * t + 1] = p[e2] / sel;
            }
        }
    }
}

}  // namespace

cudaError_t launch_route(const void* x_bf16, int64_t T, int64_t d, const float* w_router,
                         const float* bias, int E, int top_k, int32_t* ids, float* gates,
                         float* logits, int num_sms, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    int64_t blocks = (T + kWarps - 1) / kWarps;
    const int64_t cap = (int64_t)num_sms * 16;
    if (blocks > cap) blocks = cap;
    k_route<<<(unsigned)blocks, kWarps * 32, 0, stream>>>((const uint16_t*)x_bf16, T, d, w_router,
                                                          bias, E, top_k, ids, gates, logits);
    return cudaGetLastError();
}

}  // namespace jmoe
