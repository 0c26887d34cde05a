// Decode path of the expert MLPs: few tokens per expert, so the work is a
// stream over the INT8 weights of the experts that some token selected
// (HBM-bound; weights of untouched experts are never read).
//
// ExpertsInt8 ("Jamba-1.5: Hybrid Transformer-Mamba Models at Scale", paper
// summary, section "ExpertsInt8 Quantization (Section 3.1)", steps 3-4): the
// INT8 weights cross HBM once and are turned back into BF16 on chip, the
// activations stay BF16.  Here each weight byte goes HBM -> registers, is
// converted exactly to bf16 (the scale is applied once per output channel
// after the dot product, an exact refactoring of sum_k x_k (q_k s)), and
// feeds an mma.sync m16n8k16 whose 8 columns are up to 8 tokens of the
// expert; accumulation is fp32.
//
// Fragment trick: the dot product does not care in which order k is summed,
// so the 16 k-columns of every MMA step are a permutation of the 64-wide
// k-block chosen such that thread (g = lane/4, c = lane%4) needs exactly
// bytes [16c, 16c+16) of weight rows g and g+8 for all four MMA steps of the
// block -- one 16-byte load per row -- and the matching 16 consecutive bf16
// of its token.  Step s uses physical k = 16c + 4s + {0,1} for the fragment
// columns 2c, 2c+1 and 16c + 4s + {2,3} for columns 2c+8, 2c+9.
//
// Kernels:
//   k_decode_gateup : h = silu(s_g * x.q_g) * (s_u * x.q_u) for every
//                     (expert, 16 channels) per warp, h stored bf16 in
//                     expert-grouped slot order;
//   k_decode_down   : raw partial sums of h.q_d over one K split;
//   k_decode_combine: out_t = bf16( sum_j g_tj * s_d[m] * sum_splits ).
#include "common.cuh"
#include "kernels.h"

namespace jmoe {
namespace {

constexpr int kWarpsPerBlock = 4;
constexpr int kChPerWarp = 16;
constexpr int kDepth = 3;  // weight steps in flight per warp (ring of registers)

// x (or h) fragment for one token row: 16 consecutive bf16 starting at p.
__device__ __forceinline__ void load_b(const uint16_t* p, uint32_t (&b)[8]) {
    if (p) {
        const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(p));
        const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(p + 8));
        b[0] = v0.x; b[1] = v0.y; b[2] = v0.z; b[3] = v0.w;
        b[4] = v1.x; b[5] = v1.y; b[6] = v1.z; b[7] = v1.w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) b[i] = 0u;
    }
}

// Four MMA steps of one 64-wide k-block: rows g (q0) and g+8 (q1).
__device__ __forceinline__ void mma_block(float (&acc)[4], const uint4& q0, const uint4& q1,
                                          const uint32_t (&b)[8]) {
    const uint32_t w0[4] = {q0.x, q0.y, q0.z, q0.w};
    const uint32_t w1[4] = {q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const uint32_t a[4] = {i8x2_to_bf16x2<0>(w0[s]), i8x2_to_bf16x2<0>(w1[s]),
                               i8x2_to_bf16x2<1>(w0[s]), i8x2_to_bf16x2<1>(w1[s])};
        mma_bf16_16816(acc, a, b[2 * s], b[2 * s + 1]);
    }
}

template <int NCH>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    k_decode_gateup(const uint16_t* __restrict__ x, int top_k, int64_t d, int64_t f,
                    const int8_t* __restrict__ wgu, const float* __restrict__ sgu,
                    const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm,
                    uint16_t* __restrict__ H) {
    const int e = blockIdx.y;
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const int64_t ch0 = ((int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5)) * kChPerWarp;
    if (ch0 >= f) return;
    const int base = offsets[e];
    const int cnt = offsets[e + 1] - base;
    if (cnt <= 0) return;

    const int8_t* wg0 = wgu + ((int64_t)e * 2 * f + ch0 + g) * d + 16 * c;
    const int8_t* wg1 = wg0 + 8 * d;
    const int8_t* wu0 = wg0 + f * d;
    const int8_t* wu1 = wu0 + 8 * d;
    const int64_t nsteps = d / 64;

    for (int pass = 0; pass * NCH * 8 < cnt; ++pass) {
        const int nch = min(NCH, (cnt - pass * NCH * 8 + 7) / 8);  // warp-uniform
        const uint16_t* xp[NCH];
#pragma unroll
        for (int n = 0; n < NCH; ++n) {
            const int slot = (pass * NCH + n) * 8 + g;
            xp[n] = slot < cnt ? x + (int64_t)(perm[base + slot] / top_k) * d + 16 * c : nullptr;
        }
        float ag[NCH][4], au[NCH][4];
#pragma unroll
        for (int n = 0; n < NCH; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) ag[n][i] = au[n][i] = 0.0f;

        uint4 ring[kDepth][4];
#pragma unroll
        for (int p = 0; p < kDepth - 1; ++p) {
            if (p < nsteps) {
                ring[p][0] = ldg_stream_v4(wg0 + p * 64);
                ring[p][1] = ldg_stream_v4(wg1 + p * 64);
                ring[p][2] = ldg_stream_v4(wu0 + p * 64);
                ring[p][3] = ldg_stream_v4(wu1 + p * 64);
            }
        }
        for (int64_t i0 = 0; i0 < nsteps; i0 += kDepth) {
#pragma unroll
            for (int j = 0; j < kDepth; ++j) {
                const int64_t i = i0 + j;
                if (i < nsteps) {
                    const int64_t ip = i + kDepth - 1;
                    if (ip < nsteps) {
                        const int slot = (j + kDepth - 1) % kDepth;
                        ring[slot][0] = ldg_stream_v4(wg0 + ip * 64);
                        ring[slot][1] = ldg_stream_v4(wg1 + ip * 64);
                        ring[slot][2] = ldg_stream_v4(wu0 + ip * 64);
                        ring[slot][3] = ldg_stream_v4(wu1 + ip * 64);
                    }
#pragma unroll
                    for (int n = 0; n < NCH; ++n) {
                        if (n < nch) {
                            uint32_t b[8];
                            load_b(xp[n] ? xp[n] + i * 64 : nullptr, b);
                            mma_block(ag[n], ring[j][0], ring[j][1], b);
                            mma_block(au[n], ring[j][2], ring[j][3], b);
                        }
                    }
                }
            }
        }
        // epilogue: rows = channels (g, g+8), cols = token slots (2c, 2c+1)
        const float sg0 = sgu[(int64_t)e * 2 * f + ch0 + g];
        const float sg1 = sgu[(int64_t)e * 2 * f + ch0 + g + 8];
        const float su0 = sgu[(int64_t)e * 2 * f + f + ch0 + g];
        const float su1 = sgu[(int64_t)e * 2 * f + f + ch0 + g + 8];
#pragma unroll
        for (int n = 0; n < NCH; ++n) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int slot = (pass * NCH + n) * 8 + 2 * c + (i & 1);
                const int row = g + (i >> 1) * 8;
                if (n < nch && slot < cnt) {
                    const float gs = (i >> 1) ? sg1 : sg0;
                    const float us = (i >> 1) ? su1 : su0;
                    const float h = silu_f32(gs * ag[n][i]) * (us * au[n][i]);
                    H[(int64_t)(base + slot) * f + ch0 + row] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(h));
                }
            }
        }
    }
}

// Raw partial sums P[z][slot][m] = sum over k in split z of h[slot][k] q_d[m][k].
template <int NCH>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    k_decode_down(const uint16_t* __restrict__ H, int64_t d, int64_t f, int64_t ksplit,
                  const int8_t* __restrict__ wd, const int32_t* __restrict__ offsets, int64_t A,
                  float* __restrict__ P) {
    const int e = blockIdx.y;
    const int z = blockIdx.z;
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const int64_t m0 = ((int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5)) * kChPerWarp;
    if (m0 >= d) return;
    const int base = offsets[e];
    const int cnt = offsets[e + 1] - base;
    if (cnt <= 0) return;
    const int64_t k_begin = (int64_t)z * ksplit;

    const int8_t* w0 = wd + ((int64_t)e * d + m0 + g) * f + k_begin + 16 * c;
    const int8_t* w1 = w0 + 8 * f;
    const int64_t nsteps = ksplit / 64;

    for (int pass = 0; pass * NCH * 8 < cnt; ++pass) {
        const int nch = min(NCH, (cnt - pass * NCH * 8 + 7) / 8);
        const uint16_t* hp[NCH];
#pragma unroll
        for (int n = 0; n < NCH; ++n) {
            const int slot = (pass * NCH + n) * 8 + g;
            hp[n] = slot < cnt ? H + (int64_t)(base + slot) * f + k_begin + 16 * c : nullptr;
        }
        float acc[NCH][4];
#pragma unroll
        for (int n = 0; n < NCH; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[n][i] = 0.0f;

        uint4 ring[kDepth][2];
#pragma unroll
        for (int p = 0; p < kDepth - 1; ++p) {
            if (p < nsteps) {
                ring[p][0] = ldg_stream_v4(w0 + p * 64);
                ring[p][1] = ldg_stream_v4(w1 + p * 64);
            }
        }
        for (int64_t i0 = 0; i0 < nsteps; i0 += kDepth) {
#pragma unroll
            for (int j = 0; j < kDepth; ++j) {
                const int64_t i = i0 + j;
                if (i < nsteps) {
                    const int64_t ip = i + kDepth - 1;
                    if (ip < nsteps) {
                        const int slot = (j + kDepth - 1) % kDepth;
                        ring[slot][0] = ldg_stream_v4(w0 + ip * 64);
                        ring[slot][1] = ldg_stream_v4(w1 + ip * 64);
                    }
#pragma unroll
                    for (int n = 0; n < NCH; ++n) {
                        if (n < nch) {
                            uint32_t b[8];
                            load_b(hp[n] ? hp[n] + i * 64 : nullptr, b);
                            mma_block(acc[n], ring[j][0], ring[j][1], b);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int n = 0; n < NCH; ++n) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int slot = (pass * NCH + n) * 8 + 2 * c + (i & 1);
                const int row = g + (i >> 1) * 8;
                if (n < nch && slot < cnt)
                    P[((int64_t)z * A + base + slot) * d + m0 + row] = acc[n][i];
            }
        }
    }
}

// out[t][m] = bf16( sum_j g_tj * (s_d[e_j][m] * sum_z P[z][inv[a]][m]) ), a = t*top_k + j.
__global__ void __launch_bounds__(256)
    k_decode_combine(const float* __restrict__ P, int nsplit, int64_t A, int64_t T, int64_t d,
                     int top_k, int E, const int32_t* __restrict__ ids,
                     const float* __restrict__ gates, const int32_t* __restrict__ inv,
                     const float* __restrict__ sd, uint16_t* __restrict__ out) {
    const int64_t nvec = d / 4;
    const int64_t total = T * nvec;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < total;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = v / nvec, m = (v % nvec) * 4;
        float o[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < top_k; ++j) {
            const int64_t a = t * top_k + j;
            const int e = ids[a];
            const int slot = inv[a];
            if (e < 0 || e >= E || slot < 0) continue;
            float y[4] = {0.f, 0.f, 0.f, 0.f};
            for (int z = 0; z < nsplit; ++z) {
                const float4 p = *reinterpret_cast<const float4*>(P + ((int64_t)z * A + slot) * d + m);
                y[0] += p.x; y[1] += p.y; y[2] += p.z; y[3] += p.w;
            }
            const float4 s = *reinterpret_cast<const float4*>(sd + (int64_t)e * d + m);
            const float gw = gates[a];
            o[0] += gw * (s.x * y[0]);
            o[1] += gw * (s.y * y[1]);
            o[2] += gw * (s.z * y[2]);
            o[3] += gw * (s.w * y[3]);
        }
        uint2 r;
        r.x = pack_bf16x2(o[0], o[1]);
        r.y = pack_bf16x2(o[2], o[3]);
        *reinterpret_cast<uint2*>(out + t * d + m) = r;
    }
}

template <int NCH>
cudaError_t launch_decode_nch(const DecodeArgs& a, cudaStream_t stream) {
    dim3 g1((unsigned)((a.f + kWarpsPerBlock * kChPerWarp - 1) / (kWarpsPerBlock * kChPerWarp)),
            (unsigned)a.E);
    if (a.mark) a.mark(2, false, stream);
    k_decode_gateup<NCH><<<g1, kWarpsPerBlock * 32, 0, stream>>>(
        (const uint16_t*)a.x, a.top_k, a.d, a.f, a.wgu, a.sgu, a.offsets, a.perm, (uint16_t*)a.H);
    if (a.mark) a.mark(2, true, stream);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    dim3 g2((unsigned)((a.d + kWarpsPerBlock * kChPerWarp - 1) / (kWarpsPerBlock * kChPerWarp)),
            (unsigned)a.E, (unsigned)a.nsplit);
    if (a.mark) a.mark(3, false, stream);
    k_decode_down<NCH><<<g2, kWarpsPerBlock * 32, 0, stream>>>(
        (const uint16_t*)a.H, a.d, a.f, a.f / a.nsplit, a.wd, a.offsets, a.A, a.P);
    if (a.mark) a.mark(3, true, stream);
    return cudaGetLastError();
}

}  // namespace

int decode_split_for(int64_t f) {
    // largest power of two <= 8 that keeps each K split a multiple of 64
    int s = 8;
    while (s > 1 && (f % (64 * s)) != 0) s >>= 1;
    return s;
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    if (a.T == 0) return cudaSuccess;
    cudaError_t err;
    if (a.max_per_expert <= 8)
        err = launch_decode_nch<1>(a, stream);
    else if (a.max_per_expert <= 16)
        err = launch_decode_nch<2>(a, stream);
    else
        err = launch_decode_nch<4>(a, stream);
    if (err != cudaSuccess) return err;
    const int64_t total = a.T * (a.d / 4);
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)a.num_sms * 8) blocks = (int64_t)a.num_sms * 8;
    if (a.mark) a.mark(4, false, stream);
    k_decode_combine<<<(unsigned)blocks, 256, 0, stream>>>(a.P, a.nsplit, a.A, a.T, a.d, a.top_k,
                                                           a.E, a.ids, a.gates, a.inv, a.sd,
                                                           (uint16_t*)a.out);
    if (a.mark) a.mark(4, true, stream);
    return cudaGetLastError();
}

}  // namespace jmoe
