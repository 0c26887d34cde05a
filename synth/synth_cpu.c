/*
 * Seeded synthetic inputs, host side.
 *
 * This file holds no arithmetic of the MoE method: it only draws the
 * pseudo-random tensors (activations, router weights, BF16 expert weights)
 * that the CPU oracle and the CUDA path both consume.  The same definition is
 * implemented for the GPU in synth_gpu.cu; both must produce identical bits.
 *
 * Generator (counter based, so any element can be regenerated on its own):
 *   mix(z)       = SplitMix64 finaliser (Steele, Lea & Flood, "Fast
 *                  splittable pseudorandom number generators", OOPSLA 2014):
 *                  z ^= z>>30; z *= 0xbf58476d1ce4e5b9;
 *                  z ^= z>>27; z *= 0x94d049bb133111eb; z ^= z>>31
 *   gamma        = 0x9e3779b97f4a7c15 (the SplitMix64 increment)
 *   key(s, tau)  = mix(s + (tau + 1) * gamma)
 *   word(i, j)   = mix(key + (3*i + j + 1) * gamma),  j = 0, 1, 2
 *   S            = sum of the twelve 16-bit fields of word(i,0..2)
 *   z            = (S - 393210) * 2^-16   (exact in fp32: |S - 393210| < 2^19;
 *                  the Irwin-Hall(12) approximation of N(0,1): each field is
 *                  uniform on 0..65535 with mean 32767.5, so 393210 = 12 *
 *                  32767.5 is the mean of S and 2^-16 maps the spread of one
 *                  field to unit width, giving variance ~1 and |z| < 6)
 *   value        = fp32(z * sigma)        (one IEEE multiply, round to nearest)
 *   bf16 variant = round-to-nearest-even of the fp32 value to bfloat16.
 *
 * The element index i is the row-major linear index into the whole tensor,
 * so a slice [start, start+n) reproduces exactly the same values as the
 * corresponding part of the full tensor.
 */
#include <stdint.h>
#include <string.h>

#define SYNTH_GAMMA 0x9e3779b97f4a7c15ULL

static inline uint64_t synth_mix(uint64_t z) {
    z ^= z >> 30;
    z *= 0xbf58476d1ce4e5b9ULL;
    z ^= z >> 27;
    z *= 0x94d049bb133111ebULL;
    z ^= z >> 31;
    return z;
}

static inline uint64_t synth_key(uint64_t seed, uint64_t tensor) {
    return synth_mix(seed + (tensor + 1ULL) * SYNTH_GAMMA);
}

static inline float synth_value(uint64_t key, uint64_t i, float sigma) {
    int32_t s = 0;
    for (uint64_t j = 0; j < 3; ++j) {
        uint64_t w = synth_mix(key + (3ULL * i + j + 1ULL) * SYNTH_GAMMA);
        s += (int32_t)(w & 0xffffu) + (int32_t)((w >> 16) & 0xffffu) +
             (int32_t)((w >> 32) & 0xffffu) + (int32_t)(w >> 48);
    }
    float z = (float)(s - 393210) * (1.0f / 65536.0f);
    volatile float v = z * sigma; /* a single rounded multiply */
    return v;
}

static inline uint16_t synth_f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* Raw SplitMix64 stream, exposed only so the generator can be checked
 * against the published reference sequence: out[n] = mix(seed + (n+1)*gamma). */
void synth_splitmix64_stream(uint64_t seed, int64_t n, uint64_t* out) {
    for (int64_t k = 0; k < n; ++k) out[k] = synth_mix(seed + (uint64_t)(k + 1) * SYNTH_GAMMA);
}

void synth_normal_f32(uint64_t seed, uint64_t tensor, float sigma, uint64_t start,
                      int64_t n, float* out) {
    const uint64_t key = synth_key(seed, tensor);
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < n; ++k) out[k] = synth_value(key, start + (uint64_t)k, sigma);
}

void synth_normal_bf16(uint64_t seed, uint64_t tensor, float sigma, uint64_t start,
                       int64_t n, uint16_t* out) {
    const uint64_t key = synth_key(seed, tensor);
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < n; ++k)
        out[k] = synth_f32_to_bf16_rne(synth_value(key, start + (uint64_t)k, sigma));
}
