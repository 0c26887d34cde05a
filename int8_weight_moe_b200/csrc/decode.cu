// Decode path of the expert MLPs: few tokens per expert, so the work is one
// stream over the INT8 weights of the experts that some token selected
// (HBM-bound; the weights of untouched experts are never read).
//
// ExpertsInt8 ("Jamba-1.5: Hybrid Transformer-Mamba Models at Scale", paper
// summary, section "ExpertsInt8 Quantization (Section 3.1)", steps 3-4): the
// INT8 weights cross HBM once and are turned back into BF16 on chip; the
// activations stay BF16.  Here every weight byte goes HBM -> registers, is
// converted exactly to bf16 (the scale is applied once per output channel
// after the dot product, an exact refactoring of sum_k x_k (q_k s)), and feeds
// an mma.sync m16n8k16 whose 8 columns are up to 8 tokens of the expert;
// accumulation is fp32.
//
// Fragment trick: the dot product does not care in which order k is summed,
// so the 16 k-columns of every MMA step are a permutation of the 64-wide
// k-block chosen such that thread (g = lane/4, c = lane%4) needs exactly
// bytes [16c, 16c+16) of weight rows g and g+8 for the block's four MMA
// steps -- one 16-byte load per row -- and the matching 16 consecutive bf16
// of its token.  Step s uses physical k = 16c + 4s + {0,1} for fragment
// columns 2c, 2c+1 and 16c + 4s + {2,3} for columns 2c+8, 2c+9.
//
// Work decomposition (persistent, one 16-warp CTA per SM): a work unit is
// (touched expert, 16 output channels, one pass of up to 8*NCH tokens).  The
// CTA's 16 warps split the unit's K range into equal contiguous pieces, so a
// unit is small (a 16-row weight slab) and the units divide evenly over the
// CTAs; each warp keeps a ring of kDepth weight steps in registers that runs
// ahead across unit boundaries, so HBM never waits for a reduction.  At the
// end of a unit the 16 partial accumulators are summed through shared memory
// in warp order (deterministic) and warp 0 writes the result:
//   k_gemv_gateup : h = silu(s_g * x.q_g) * (s_u * x.q_u) -> H (bf16, slot order)
//   k_gemv_down   : y = gate * (s_d * h.q_d)               -> Y (fp32, one row per
//                                                             token->expert assignment)
// and launch_finalize sums each token's rows of Y into the bf16 output.
#include "common.cuh"
#include "kernels.h"

namespace jmoe {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kDepth = 4;  // ring slots per warp: three 64-wide k steps in flight
constexpr int kMaxE = 16;

// Units of one launch, built by every CTA from the expert offsets.
struct Units {
    int start[kMaxE + 1];  // first unit of expert e
    int groups;            // 16-channel groups per expert
};

__device__ __forceinline__ void build_units(Units& u, const int32_t* offsets, int E, int groups,
                                            int tokens_per_pass) {
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            const int cnt = offsets[e + 1] - offsets[e];
            const int passes = cnt > 0 ? (cnt + tokens_per_pass - 1) / tokens_per_pass : 0;
            u.start[e] = run;
            run += passes * groups;
        }
        u.start[E] = run;
        u.groups = groups;
    }
}

struct Unit {
    int e, group, pass;
};

__device__ __forceinline__ Unit decode_unit(const Units& u, int E, int unit) {
    int e = 0;
    while (e + 1 < E && u.start[e + 1] <= unit) ++e;
    const int local = unit - u.start[e];
    Unit r;
    r.e = e;
    r.group = local % u.groups;
    r.pass = local / u.groups;
    return r;
}

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
__global__ void __launch_bounds__(kThreads, 1)
    k_gemv_gateup(const uint16_t* __restrict__ x, int top_k, int E, int64_t d, int64_t f,
                  const int8_t* __restrict__ wgu, const float* __restrict__ sgu,
                  const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm,
                  uint16_t* __restrict__ H) {
    __shared__ Units U;
    __shared__ int s_off[kMaxE + 1];
    // partial sums of the 16 warps, double-buffered by unit parity (dynamic:
    // 32 KB per token chunk)
    extern __shared__ float red_raw[];
    auto red = reinterpret_cast<float(*)[kWarps][32][NCH][8]>(red_raw);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, c = lane & 3;
    if (threadIdx.x <= E) s_off[threadIdx.x] = offsets[threadIdx.x];
    build_units(U, offsets, E, (int)(f / 16), 8 * NCH);
    __syncthreads();
    const int n_units = U.start[E];
    const int G = gridDim.x;
    const int n_mine = (int)blockIdx.x < n_units ? (n_units - 1 - (int)blockIdx.x) / G + 1 : 0;
    const int S = (int)(d / 64);
    const int nw = (S + kWarps - 1) / kWarps;
    const int s_lo = warp * nw;
    const int s_hi = min(S, s_lo + nw);
    const int64_t total = (int64_t)n_mine * nw;

    // ---- prefetch cursor (unit iteration pi, step pj) and its slab pointers
    int pi = 0, pj = 0;
    const int8_t* pw[4] = {nullptr, nullptr, nullptr, nullptr};
    auto set_prefetch_unit = [&](int it) {
        const Unit u = decode_unit(U, E, blockIdx.x + it * G);
        const int8_t* base = wgu + ((int64_t)u.e * 2 * f + u.group * 16 + g) * d + 16 * c +
                             (int64_t)s_lo * 64;
        pw[0] = base;
        pw[1] = base + 8 * d;
        pw[2] = base + f * d;
        pw[3] = base + f * d + 8 * d;
    };
    uint4 ring[kDepth][4];
    auto issue = [&](int slot) {
        // load step (pi, pj) into ring[slot]; the padding steps of short K pieces load nothing
        if (s_lo + pj < s_hi) {
#pragma unroll
            for (int m = 0; m < 4; ++m) ring[slot][m] = ldg_stream_v4(pw[m] + (int64_t)pj * 64);
        }
        if (++pj == nw) {
            pj = 0;
            if (++pi < n_mine) set_prefetch_unit(pi);
        }
    };
    if (n_mine > 0) set_prefetch_unit(0);
#pragma unroll
    for (int p = 0; p < kDepth - 1; ++p)
        if (p < total) issue(p);

    // ---- consumer state
    float ag[NCH][4], au[NCH][4];
#pragma unroll
    for (int n = 0; n < NCH; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) ag[n][i] = au[n][i] = 0.0f;
    Unit cu{};
    const uint16_t* xp[NCH];
    int cnt_pass = 0;
    int ci = 0, cj = 0;
    auto set_consumer_unit = [&](int it) {
        cu = decode_unit(U, E, blockIdx.x + it * G);
        const int base = s_off[cu.e];
        const int cnt = s_off[cu.e + 1] - base;
        const int t0 = cu.pass * 8 * NCH;
        cnt_pass = min(8 * NCH, cnt - t0);
#pragma unroll
        for (int n = 0; n < NCH; ++n) {
            const int slot = n * 8 + g;
            xp[n] = slot < cnt_pass
                        ? x + (int64_t)(perm[base + t0 + slot] / top_k) * d + 16 * c + s_lo * 64
                        : nullptr;
        }
    };
    if (n_mine > 0) set_consumer_unit(0);

    for (int64_t q0 = 0; q0 < total; q0 += kDepth) {
#pragma unroll
        for (int jj = 0; jj < kDepth; ++jj) {
            const int64_t q = q0 + jj;
            if (q < total) {
                if (q + kDepth - 1 < total) issue((jj + kDepth - 1) % kDepth);
                if (s_lo + cj < s_hi) {
#pragma unroll
                    for (int n = 0; n < NCH; ++n) {
                        if (n * 8 < cnt_pass) {
                            uint32_t b[8];
                            load_b(xp[n] ? xp[n] + cj * 64 : nullptr, b);
                            mma_block(ag[n], ring[jj][0], ring[jj][1], b);
                            mma_block(au[n], ring[jj][2], ring[jj][3], b);
                        }
                    }
                }
                if (++cj == nw) {
                    // end of unit: reduce the 16 warps' partials, warp 0 writes h
                    const int buf = ci & 1;
#pragma unroll
                    for (int n = 0; n < NCH; ++n)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            red[buf][warp][lane][n][i] = ag[n][i];
                            red[buf][warp][lane][n][4 + i] = au[n][i];
                            ag[n][i] = au[n][i] = 0.0f;
                        }
                    __syncthreads();
                    if (warp == 0) {
                        const int base = s_off[cu.e] + cu.pass * 8 * NCH;
                        const int64_t ch0 = (int64_t)cu.group * 16;
                        const float* sg = sgu + (int64_t)cu.e * 2 * f + ch0;
#pragma unroll
                        for (int n = 0; n < NCH; ++n) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                float vg = 0.f, vu = 0.f;
                                for (int w2 = 0; w2 < kWarps; ++w2) {
                                    vg += red[buf][w2][lane][n][i];
                                    vu += red[buf][w2][lane][n][4 + i];
                                }
                                const int slot = n * 8 + 2 * c + (i & 1);
                                const int row = g + (i >> 1) * 8;
                                if (slot < cnt_pass) {
                                    const float h = silu_f32(sg[row] * vg) * (sg[f + row] * vu);
                                    H[(int64_t)(base + slot) * f + ch0 + row] =
                                        __bfloat16_as_ushort(__float2bfloat16_rn(h));
                                }
                            }
                        }
                    }
                    cj = 0;
                    if (++ci < n_mine) set_consumer_unit(ci);
                }
            }
        }
    }
}

template <int NCH>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemv_down(const uint16_t* __restrict__ H, int E, int64_t d, int64_t f,
                const int8_t* __restrict__ wd, const float* __restrict__ sd,
                const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm,
                const float* __restrict__ gates, float* __restrict__ Y) {
    __shared__ Units U;
    __shared__ int s_off[kMaxE + 1];
    __shared__ float red[2][kWarps][32][NCH][4];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, c = lane & 3;
    if (threadIdx.x <= E) s_off[threadIdx.x] = offsets[threadIdx.x];
    build_units(U, offsets, E, (int)(d / 16), 8 * NCH);
    __syncthreads();
    const int n_units = U.start[E];
    const int G = gridDim.x;
    const int n_mine = (int)blockIdx.x < n_units ? (n_units - 1 - (int)blockIdx.x) / G + 1 : 0;
    const int S = (int)(f / 64);
    const int nw = (S + kWarps - 1) / kWarps;
    const int s_lo = warp * nw;
    const int s_hi = min(S, s_lo + nw);
    const int64_t total = (int64_t)n_mine * nw;

    int pi = 0, pj = 0;
    const int8_t* pw[2] = {nullptr, nullptr};
    auto set_prefetch_unit = [&](int it) {
        const Unit u = decode_unit(U, E, blockIdx.x + it * G);
        const int8_t* base =
            wd + ((int64_t)u.e * d + u.group * 16 + g) * f + 16 * c + (int64_t)s_lo * 64;
        pw[0] = base;
        pw[1] = base + 8 * f;
    };
    uint4 ring[kDepth][2];
    auto issue = [&](int slot) {
        if (s_lo + pj < s_hi) {
            ring[slot][0] = ldg_stream_v4(pw[0] + (int64_t)pj * 64);
            ring[slot][1] = ldg_stream_v4(pw[1] + (int64_t)pj * 64);
        }
        if (++pj == nw) {
            pj = 0;
            if (++pi < n_mine) set_prefetch_unit(pi);
        }
    };
    if (n_mine > 0) set_prefetch_unit(0);
#pragma unroll
    for (int p = 0; p < kDepth - 1; ++p)
        if (p < total) issue(p);

    float acc[NCH][4];
#pragma unroll
    for (int n = 0; n < NCH; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[n][i] = 0.0f;
    Unit cu{};
    const uint16_t* hp[NCH];
    int cnt_pass = 0;
    int ci = 0, cj = 0;
    auto set_consumer_unit = [&](int it) {
        cu = decode_unit(U, E, blockIdx.x + it * G);
        const int base = s_off[cu.e];
        const int cnt = s_off[cu.e + 1] - base;
        const int t0 = cu.pass * 8 * NCH;
        cnt_pass = min(8 * NCH, cnt - t0);
#pragma unroll
        for (int n = 0; n < NCH; ++n) {
            const int slot = n * 8 + g;
            hp[n] = slot < cnt_pass ? H + (int64_t)(base + t0 + slot) * f + 16 * c + s_lo * 64
                                    : nullptr;
        }
    };
    if (n_mine > 0) set_consumer_unit(0);

    for (int64_t q0 = 0; q0 < total; q0 += kDepth) {
#pragma unroll
        for (int jj = 0; jj < kDepth; ++jj) {
            const int64_t q = q0 + jj;
            if (q < total) {
                if (q + kDepth - 1 < total) issue((jj + kDepth - 1) % kDepth);
                if (s_lo + cj < s_hi) {
#pragma unroll
                    for (int n = 0; n < NCH; ++n) {
                        if (n * 8 < cnt_pass) {
                            uint32_t b[8];
                            load_b(hp[n] ? hp[n] + cj * 64 : nullptr, b);
                            mma_block(acc[n], ring[jj][0], ring[jj][1], b);
                        }
                    }
                }
                if (++cj == nw) {
                    const int buf = ci & 1;
#pragma unroll
                    for (int n = 0; n < NCH; ++n)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            red[buf][warp][lane][n][i] = acc[n][i];
                            acc[n][i] = 0.0f;
                        }
                    __syncthreads();
                    if (warp == 0) {
                        const int base = s_off[cu.e] + cu.pass * 8 * NCH;
                        const int64_t m0 = (int64_t)cu.group * 16;
                        const float* s = sd + (int64_t)cu.e * d + m0;
#pragma unroll
                        for (int n = 0; n < NCH; ++n) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                float v = 0.f;
                                for (int w2 = 0; w2 < kWarps; ++w2) v += red[buf][w2][lane][n][i];
                                const int slot = n * 8 + 2 * c + (i & 1);
                                const int row = g + (i >> 1) * 8;
                                if (slot < cnt_pass) {
                                    const int a = perm[base + slot];
                                    Y[(int64_t)a * d + m0 + row] = gates[a] * (s[row] * v);
                                }
                            }
                        }
                    }
                    cj = 0;
                    if (++ci < n_mine) set_consumer_unit(ci);
                }
            }
        }
    }
}

// out[t] = bf16( sum_j Y[t*top_k + j] ) over the token's valid assignments.
__global__ void __launch_bounds__(256)
    k_finalize(const float* __restrict__ Y, int64_t T, int64_t d, int top_k, int E,
               const int32_t* __restrict__ ids, uint16_t* __restrict__ out) {
    const int64_t nvec = d / 4;
    const int64_t total = T * nvec;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < total;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = v / nvec, m = (v % nvec) * 4;
        float o[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < top_k; ++j) {
            const int64_t a = t * top_k + j;
            const int e = ids[a];
            if (e < 0 || e >= E) continue;
            const float4 y = *reinterpret_cast<const float4*>(Y + a * d + m);
            o[0] += y.x;
            o[1] += y.y;
            o[2] += y.z;
            o[3] += y.w;
        }
        uint2 r;
        r.x = pack_bf16x2(o[0], o[1]);
        r.y = pack_bf16x2(o[2], o[3]);
        *reinterpret_cast<uint2*>(out + t * d + m) = r;
    }
}

template <int NCH>
cudaError_t launch_decode_nch(const DecodeArgs& a, cudaStream_t stream) {
    const int grid = a.num_sms;
    const int red_bytes = (int)(2 * kWarps * 32 * NCH * 8 * sizeof(float));
    cudaError_t err = cudaFuncSetAttribute(k_gemv_gateup<NCH>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, red_bytes);
    if (err != cudaSuccess) return err;
    if (a.mark) a.mark(2, false, stream);
    k_gemv_gateup<NCH><<<grid, kThreads, red_bytes, stream>>>((const uint16_t*)a.x, a.top_k, a.E, a.d,
                                                      a.f, a.wgu, a.sgu, a.offsets, a.perm,
                                                      (uint16_t*)a.H);
    if (a.mark) a.mark(2, true, stream);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    if (a.mark) a.mark(3, false, stream);
    k_gemv_down<NCH><<<grid, kThreads, 0, stream>>>((const uint16_t*)a.H, a.E, a.d, a.f, a.wd,
                                                    a.sd, a.offsets, a.perm, a.gates, a.Y);
    if (a.mark) a.mark(3, true, stream);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_finalize(const float* Y, int64_t T, int64_t d, int top_k, int E,
                            const int32_t* ids, void* out, int num_sms, cudaStream_t stream) {
    const int64_t total = T * (d / 4);
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    if (blocks < 1) blocks = 1;
    k_finalize<<<(unsigned)blocks, 256, 0, stream>>>(Y, T, d, top_k, E, ids,
                                                     static_cast<uint16_t*>(out));
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    if (a.T == 0) return cudaSuccess;
    cudaError_t err = a.max_per_expert <= 8 ? launch_decode_nch<1>(a, stream)
                                            : launch_decode_nch<2>(a, stream);
    if (err != cudaSuccess) return err;
    if (a.mark) a.mark(4, false, stream);
    err = launch_finalize(a.Y, a.T, a.d, a.top_k, a.E, a.ids, a.out, a.num_sms, stream);
    if (a.mark) a.mark(4, true, stream);
    return err;
}

}  // namespace jmoe
