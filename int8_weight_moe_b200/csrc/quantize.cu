// Load-time ExpertsInt8 quantisation: BF16 weights -> INT8 + fp32 scale per
// output row.
//
// "Jamba-1.5: Hybrid Transformer-Mamba Models at Scale" (paper summary),
// section "ExpertsInt8 Quantization (Section 3.1)", step 1: the MoE and MLP
// weights are converted from BF16 to INT8 when the model loads, with no
// calibration data.  Scheme (symmetric, per output channel):
//   a = max_k |w_k|,  s = a / 127  (one correctly rounded fp32 division),
//   q_k = round_half_even(w_k / s) (one fp32 division per element), in
//   [-127, 127]; an all-zero row gets s = 0 and q = 0.
//
// One CTA per row; the row is read twice (absmax, then quantise), the second
// pass mostly from L2.  HBM-bound: 2 B read + 1 B written per weight.
#include "common.cuh"
#include "kernels.h"

namespace jmoe {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < kThreads / 32 ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    return red[0];
}

__device__ __forceinline__ int8_t quant1(float w, float s) {
    float v = rintf(__fdiv_rn(w, s));  // rint: round half to even
    v = fminf(fmaxf(v, -127.0f), 127.0f);
    return (int8_t)(int)v;
}

// cols % 8 == 0: every thread moves 8 bf16 (16 B) in and 8 int8 (8 B) out.
__global__ void __launch_bounds__(kThreads) k_quantize_rows(const uint16_t* __restrict__ w,
                                                            int64_t cols, int8_t* __restrict__ q,
                                                            float* __restrict__ scales) {
    __shared__ float red[kThreads / 32];
    const int64_t row = blockIdx.x;
    const uint16_t* wr = w + row * cols;
    int8_t* qr = q + row * cols;
    const int64_t nvec = cols / 8;

    float amax = 0.0f;
    for (int64_t i = threadIdx.x; i < nvec; i += kThreads) {
        uint4 v = *reinterpret_cast<const uint4*>(wr + i * 8);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            amax = fmaxf(amax, fabsf(__uint_as_float(u[j] << 16)));
            amax = fmaxf(amax, fabsf(__uint_as_float(u[j] & 0xffff0000u)));
        }
    }
    amax = block_max(amax, red);
    const float s = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
    if (threadIdx.x == 0) scales[row] = s;

    for (int64_t i = threadIdx.x; i < nvec; i += kThreads) {
        uint2 out = make_uint2(0u, 0u);
        if (s != 0.0f) {
            uint4 v = *reinterpret_cast<const uint4*>(wr + i * 8);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
            uint32_t b[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                b[2 * j] = (uint8_t)quant1(__uint_as_float(u[j] << 16), s);
                b[2 * j + 1] = (uint8_t)quant1(__uint_as_float(u[j] & 0xffff0000u), s);
            }
            out.x = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
            out.y = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
        }
        *reinterpret_cast<uint2*>(qr + i * 8) = out;
    }
}

}  // namespace

cudaError_t launch_quantize(const void* w_bf16, int64_t rows, int64_t cols, int8_t* q,
                            float* scales, cudaStream_t stream) {
    if (rows == 0) return cudaSuccess;
    k_quantize_rows<<<(unsigned)rows, kThreads, 0, stream>>>((const uint16_t*)w_bf16, cols, q,
                                                             scales);
    note_launch();
    return cudaGetLastError();
}

}  // namespace jmoe
