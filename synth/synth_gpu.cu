// Seeded synthetic inputs, device side.
//
// The same generator as synth_cpu.c (SplitMix64 counter stream, Irwin-Hall(12)
// normal approximation, one fp32 multiply by sigma, round-to-nearest-even to
// bfloat16); the two files must agree bit for bit.  It draws inputs only and
// holds none of the MoE method's arithmetic.  It lives in its own library so
// that large weight tensors (tens of GB at the biggest workloads) can be drawn
// directly in device memory instead of being copied from the host.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

constexpr uint64_t kGamma = 0x9e3779b97f4a7c15ULL;

__host__ __device__ __forceinline__ uint64_t mix(uint64_t z) {
    z ^= z >> 30;
    z *= 0xbf58476d1ce4e5b9ULL;
    z ^= z >> 27;
    z *= 0x94d049bb133111ebULL;
    z ^= z >> 31;
    return z;
}

__device__ __forceinline__ float value(uint64_t key, uint64_t i, float sigma) {
    int32_t s = 0;
#pragma unroll
    for (uint64_t j = 0; j < 3; ++j) {
        uint64_t w = mix(key + (3ULL * i + j + 1ULL) * kGamma);
        s += (int32_t)(w & 0xffffu) + (int32_t)((w >> 16) & 0xffffu) +
             (int32_t)((w >> 32) & 0xffffu) + (int32_t)(w >> 48);
    }
    float z = (float)(s - 393210) * (1.0f / 65536.0f);
    return __fmul_rn(z, sigma);  // one rounded multiply, never contracted
}

__device__ __forceinline__ uint16_t to_bf16_rne(float f) {
    uint32_t u = __float_as_uint(f);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

__global__ void k_normal_bf16(uint64_t key, float sigma, uint64_t start, int64_t n,
                              uint16_t* __restrict__ out) {
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride)
        out[k] = to_bf16_rne(value(key, start + (uint64_t)k, sigma));
}

__global__ void k_normal_f32(uint64_t key, float sigma, uint64_t start, int64_t n,
                             float* __restrict__ out) {
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += stride)
        out[k] = value(key, start + (uint64_t)k, sigma);
}

int grid_for(int64_t n) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t want = (n + 255) / 256;
    int64_t cap = (int64_t)sms * 8;
    return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

}  // namespace

extern "C" int synth_normal_bf16_gpu(uint64_t seed, uint64_t tensor, float sigma,
                                     uint64_t start, int64_t n, void* out,
                                     void* stream) {
    if (n <= 0) return 0;
    if (!out) return 1;
    uint64_t key = mix(seed + (tensor + 1ULL) * kGamma);
    k_normal_bf16<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(key, sigma, start, n,
                                                                  (uint16_t*)out);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

extern "C" int synth_normal_f32_gpu(uint64_t seed, uint64_t tensor, float sigma,
                                    uint64_t start, int64_t n, float* out, void* stream) {
    if (n <= 0) return 0;
    if (!out) return 1;
    uint64_t key = mix(seed + (tensor + 1ULL) * kGamma);
    k_normal_f32<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(key, sigma, start, n, out);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
