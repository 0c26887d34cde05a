// Router: logits, softmax over the experts, top-k selection, renormalised
// gates.
//
// "Jamba: A Hybrid Transformer-Mamba Language Model" (paper summary), section
// "Mixture-of-Experts (MoE) in Jamba: Router, Top-K, and Load Balancing":
// g = softmax(W_r h) with W_r of shape [n, d]; the top K = 2 experts are
// selected and their probabilities renormalised over the selected set.
//
// Summation order (fixed, so the logits -- and the top-k ids chosen from them
// -- are reproducible bit for bit): for every (token, expert), lane j of a
// warp accumulates in fp64 the partial sum p_j = sum over k = j, j+32, ...
// (ascending) of x_k * w_ek; the 32 partial sums are combined by the halving
// tree p_j += p_{j+o}, o = 16, 8, 4, 2, 1 (a shuffle-down reduction); the bias
// is added in fp64 and the result rounded once to fp32.  The products are
// exact in fp64 (8-bit x 24-bit significands).
//
// Work split: for many tokens a CTA of 8 warps handles 16 tokens with the
// router rows and token rows staged in shared memory (k_route_tiles: each
// lane keeps 8 tokens x 4 experts of fp64 partial sums).
// For few tokens (decode) one warp per expert: a cluster of 4 CTAs per token
// (each warp's router row copied to shared memory in one round trip, logits
// gathered in the first CTA through distributed shared memory), or for rows
// too wide for that a 16-warp CTA per token streaming the rows in chunks.
// Softmax (fp32) and top-k run in one warp per token afterwards.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace jmoe {
namespace {

constexpr int kMaxE = 64;      // experts
constexpr int kMaxTopK = 4;
constexpr int kGroupE = 16;    // experts computed together (one warp each, or 4 per warp)

// Top-k on one token's fp32 logits (E <= 64), by one whole warp: k passes of
// a strict '>' argmax over the experts not yet chosen, scanning in index
// order (the lower index wins ties), fp32 softmax over all E experts, then
// the chosen probabilities -- renormalised over the selection (in selection
// order) when `renorm`, as they are otherwise.
//
// Lane i holds experts i and i + 32.  A scan in index order that starts at
// the first candidate f and moves on only to a strictly larger value ends at
// f when l[f] is NaN (nothing compares larger), and otherwise at the lowest
// index holding the largest non-NaN value; each pass takes exactly that,
// the second case by a shuffle reduction over (value, index).  The sum z of
// the exponentials runs in index order in every lane (shuffles), so the
// result is the same as one thread's loop.
__device__ __forceinline__ void warp_select_topk(const float* l, int64_t t, int E, int top_k,
                                                 int renorm, int32_t* ids, float* gates,
                                                 float* logits) {
    const int lane = threadIdx.x & 31;
    const bool has0 = lane < E, has1 = lane + 32 < E;
    const float v0 = has0 ? l[lane] : 0.0f, v1 = has1 ? l[lane + 32] : 0.0f;
    if (logits) {
        if (has0) logits[t * E + lane] = v0;
        if (has1) logits[t * E + lane + 32] = v1;
    }
    bool free0 = has0, free1 = has1;
    int chosen[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        if (j >= top_k) break;
        const unsigned b0 = __ballot_sync(0xffffffffu, free0), b1 = __ballot_sync(0xffffffffu, free1);
        const int f = b0 ? __ffs(b0) - 1 : 32 + __ffs(b1) - 1;  // first candidate
        const float lf = f < 32 ? __shfl_sync(0xffffffffu, v0, f) : __shfl_sync(0xffffffffu, v1, f - 32);
        int best;
        if (isnan(lf)) {
            best = f;
        } else {
            // this lane's best non-NaN candidate (its lower index first), then
            // the warp's: the larger value, the lower index on equal values
            float bv = 0.0f;
            int bi = -1;
            if (free0 && !isnan(v0)) { bv = v0; bi = lane; }
            if (free1 && !isnan(v1) && (bi < 0 || v1 > bv)) { bv = v1; bi = lane + 32; }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                const bool take = oi >= 0 && (bi < 0 || ov > bv || (ov == bv && oi < bi));
                if (take) { bv = ov; bi = oi; }
            }
            best = bi;
        }
        chosen[j] = best;
        if (best == lane) free0 = false;
        if (best == lane + 32) free1 = false;
    }
    const int c0 = chosen[0];
    const float m = c0 < 32 ? __shfl_sync(0xffffffffu, v0, c0) : __shfl_sync(0xffffffffu, v1, c0 - 32);
    const float p0 = has0 ? expf(v0 - m) : 0.0f, p1 = has1 ? expf(v1 - m) : 0.0f;
    float z = 0.0f;
    for (int e = 0; e < E && e < 32; ++e) z += __shfl_sync(0xffffffffu, p0, e);
    for (int e = 32; e < E; ++e) z += __shfl_sync(0xffffffffu, p1, e - 32);
    float q[kMaxTopK];
    float sel = 0.0f;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        if (j >= top_k) break;
        const int c = chosen[j];
        const float pc = c < 32 ? __shfl_sync(0xffffffffu, p0, c) : __shfl_sync(0xffffffffu, p1, c - 32);
        q[j] = pc / z;
        sel += q[j];
    }
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        if (j >= top_k) break;
        if (lane == j) {
            ids[t * top_k + j] = chosen[j];
            gates[t * top_k + j] = renorm ? q[j] / sel : q[j];
        }
    }
}

// RMSNorm of one bf16 row held by a warp's lanes in the canonical order:
// ss = sum of x_k^2 with lane j summing k = j (mod 32) ascending and the
// halving tree over the lanes (squares of bf16 values are exact in fp64),
// r = 1 / sqrt(ss / d + eps), each step one IEEE-rounded fp64 operation (no
// fused multiply-adds), so the result matches a plain fp64 evaluation.
__device__ __forceinline__ double rms_inv(double lane_sum, int64_t d, float eps) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) lane_sum += __shfl_down_sync(0xffffffffu, lane_sum, o);
    const double ss = __shfl_sync(0xffffffffu, lane_sum, 0);
    return __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, (double)d), (double)eps)));
}

// y_k = bf16((x_k * r) * gamma_k), rounded once from fp64.
__device__ __forceinline__ uint16_t rms_apply(uint16_t x, double r, uint16_t g) {
    const double v = __dmul_rn(__dmul_rn((double)bf16_bits_to_f32(x), r),
                               (double)bf16_bits_to_f32(g));
    return __bfloat16_as_ushort(__double2bfloat16(v));
}

// Few tokens, very wide rows: one CTA of 16 warps per token, warp w computing
// experts w, w + 16, ... (same per-lane order and halving tree).  The token
// row is staged in shared memory once; each warp streams its expert's router
// row through two 4 KB shared-memory buffers with 16-byte cp.async copies
// (all copies of a chunk in flight at once, the next chunk landing while this
// one is summed), and lane j then reads its own k = j (mod 32) entries,
// conflict-free.
constexpr int kChunk = 1024;  // router-row floats per chunk
constexpr int kChunkSmem = 2 * kChunk * 4;  // per warp: two chunks
constexpr size_t kWideMaxSmem = 200 * 1024;  // 128 KB of chunks + token rows up to d = 36864

__device__ __forceinline__ void route_chunk_copy(float* dst, const float* src, int n, int lane) {
    // n floats (a multiple of 64): n/4 copies of 16 bytes, spread over the lanes
    for (int i = lane; i < n / 4; i += 32) cp_async_16(dst + 4 * i, src + 4 * i, 16);
    cp_async_commit();
}

__global__ void __launch_bounds__(kGroupE * 32)
    k_route_wide(const uint16_t* __restrict__ x, int64_t d, const float* __restrict__ wr,
                 const float* __restrict__ bias, int E, int top_k, int renorm,
                 int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ logits) {
    extern __shared__ __align__(16) uint8_t route_smem[];
    float* s_w = reinterpret_cast<float*>(route_smem);  // [16 warps][2][kChunk]
    uint16_t* s_x = reinterpret_cast<uint16_t*>(route_smem + kGroupE * kChunkSmem);  // [d]
    __shared__ float s_logit[kMaxE];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t = blockIdx.x;
    const int nchunks = (int)((d + kChunk - 1) / kChunk);
    float* buf = s_w + warp * 2 * kChunk;
    const uint16_t* xr = x + t * d;
    for (int64_t k = threadIdx.x * 8; k < d; k += (int64_t)blockDim.x * 8)
        *reinterpret_cast<uint4*>(s_x + k) = __ldg(reinterpret_cast<const uint4*>(xr + k));
    __syncthreads();
    for (int e = warp; e < E; e += kGroupE) {
        const float* w = wr + (int64_t)e * d;
        route_chunk_copy(buf, w, (int)(d < kChunk ? d : (int64_t)kChunk), lane);
        double acc = 0.0;
        for (int c = 0; c < nchunks; ++c) {
            const int64_t base = (int64_t)c * kChunk;
            if (c + 1 < nchunks) {
                route_chunk_copy(buf + ((c + 1) & 1) * kChunk, w + base + kChunk,
                                 (int)(d - base - kChunk < kChunk ? d - base - kChunk : (int64_t)kChunk), lane);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncwarp();
            const float* cw = buf + (c & 1) * kChunk;
            const int n = (int)(d - base < kChunk ? d - base : (int64_t)kChunk);
#pragma unroll 8
            for (int k = lane; k < n; k += 32)
                acc = fma((double)bf16_bits_to_f32(s_x[base + k]), (double)cw[k], acc);
            __syncwarp();  // the buffer is refilled two chunks later
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_down_sync(0xffffffffu, acc, o);
        if (lane == 0) s_logit[e] = __double2float_rn(acc + (bias ? (double)bias[e] : 0.0));
    }
    __syncthreads();
    if (warp == 0) warp_select_topk(s_logit, t, E, top_k, renorm, ids, gates, logits);
}

// Few tokens, d_model up to about 11k: a cluster of 4 CTAs per token, 4
// warps per CTA, warp w of CTA r computing experts 4r + w, 4r + w + 16, ....
// Each warp pulls one whole router row into shared memory with 16-byte
// cp.async copies at once (one memory round trip per expert), sums in the
// canonical order, and writes its logit into the first CTA's shared memory
// (distributed shared memory); after the cluster barrier the first CTA
// selects the top-k.
constexpr int kRouteCluster = 4;
constexpr int kExpertsPerCta = kGroupE / kRouteCluster;
constexpr size_t kClusterMaxSmem = 200 * 1024;

// kNorm: the token row is RMS-normalised in shared memory first (every CTA
// of the cluster computes the same r; the first one writes the normalised
// row to y) and the logits are taken of the normalised row.
template <bool kNorm>
__global__ void __cluster_dims__(kRouteCluster, 1, 1) __launch_bounds__(kExpertsPerCta * 32)
    k_route_cluster(const uint16_t* __restrict__ x, int64_t d, const float* __restrict__ wr,
                    const float* __restrict__ bias, int E, int top_k, int renorm,
                    int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ logits,
                    const uint16_t* __restrict__ gamma, float eps, uint16_t* __restrict__ y) {
    namespace cg = cooperative_groups;
    extern __shared__ __align__(16) uint8_t route_smem[];
    float* s_w = reinterpret_cast<float*>(route_smem);  // [kExpertsPerCta][d]
    uint16_t* s_x = reinterpret_cast<uint16_t*>(route_smem + (size_t)kExpertsPerCta * d * 4);
    __shared__ float s_logit[kMaxE];  // filled in the cluster's first CTA
    cg::cluster_group cluster = cg::this_cluster();
    // first half of a cluster barrier: no CTA writes into another CTA's shared
    // memory before every CTA of the cluster has started (the wait is below)
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
    const unsigned rank = cluster.block_rank();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t = blockIdx.x / kRouteCluster;
    float* row = s_w + (size_t)warp * d;
    auto copy_row = [&](int e) {
        const float* w = wr + (int64_t)e * d;
        for (int64_t i = lane; i < d / 4; i += 32) cp_async_16(row + 4 * i, w + 4 * i, 16);
        cp_async_commit();
    };
    // The router rows are weights no kernel of the stream writes: their copy
    // starts before the wait for the previous kernel.
    const int e0 = (int)rank * kExpertsPerCta + warp;
    if (e0 < E) copy_row(e0);
    pdl_wait();  // the token rows come from, and ids/gates may still be read by, earlier kernels
    pdl_launch_dependents();
    const uint16_t* xr = x + t * d;
    for (int64_t k = threadIdx.x * 8; k < d; k += (int64_t)blockDim.x * 8)
        *reinterpret_cast<uint4*>(s_x + k) = __ldg(reinterpret_cast<const uint4*>(xr + k));
    __syncthreads();
    if (kNorm) {
        __shared__ double s_r;
        if (warp == 0) {
            double acc = 0.0;
            for (int64_t k = lane; k < d; k += 32) {
                const double v = (double)bf16_bits_to_f32(s_x[k]);
                acc = __dadd_rn(acc, __dmul_rn(v, v));
            }
            const double r = rms_inv(acc, d, eps);
            if (lane == 0) s_r = r;
        }
        __syncthreads();
        const double r = s_r;
        for (int64_t k = threadIdx.x; k < d; k += blockDim.x) {
            const uint16_t v = rms_apply(s_x[k], r, gamma[k]);
            s_x[k] = v;
            if (rank == 0) y[t * d + k] = v;
        }
        __syncthreads();
    }
    float* dst = cluster.map_shared_rank(s_logit, 0);
    auto logit_of_row = [&](int e) {
        cp_async_wait<0>();
        __syncwarp();
        double acc = 0.0;
#pragma unroll 8
        for (int64_t k = lane; k < d; k += 32)
            acc = fma((double)bf16_bits_to_f32(s_x[k]), (double)row[k], acc);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc += __shfl_down_sync(0xffffffffu, acc, o);
        return __double2float_rn(acc + (bias ? (double)bias[e] : 0.0));
    };
    float l0 = 0.0f;
    if (e0 < E) l0 = logit_of_row(e0);
    // second half of the start barrier, after the first row's sum: every CTA
    // of the cluster is running before the first remote write
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (e0 < E && lane == 0) dst[e0] = l0;
    for (int e = e0 + kGroupE; e < E; e += kGroupE) {
        __syncwarp();  // every lane is done with the row before it is refilled
        copy_row(e);
        const float l = logit_of_row(e);
        if (lane == 0) dst[e] = l;
    }
    cluster.sync();
    if (rank == 0 && warp == 0) warp_select_topk(s_logit, t, E, top_k, renorm, ids, gates, logits);
}

// One warp per token.
__global__ void __launch_bounds__(256)
    k_rmsnorm(const uint16_t* __restrict__ x, int64_t T, int64_t d, const uint16_t* __restrict__ gamma,
              float eps, uint16_t* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    for (int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); t < T;
         t += (int64_t)gridDim.x * 8) {
        const uint16_t* xr = x + t * d;
        double acc = 0.0;
        for (int64_t k = lane; k < d; k += 32) {
            const double v = (double)bf16_bits_to_f32(xr[k]);
            acc = __dadd_rn(acc, __dmul_rn(v, v));
        }
        const double r = rms_inv(acc, d, eps);
        for (int64_t k = lane; k < d; k += 32) y[t * d + k] = rms_apply(xr[k], r, gamma[k]);
    }
}

// Many tokens: a CTA of 8 warps computes the logits of 16 tokens, one group
// of 16 experts at a time.  The group's router rows and the tokens' rows go
// through shared memory in k-chunks of 512 (16-byte cp.async copies, the next
// chunk landing while this one is summed); warp w keeps the fp64 partial sums
// of tokens 8 (w / 4) .. +7 for experts w % 4, w % 4 + 4, w % 4 + 8, w % 4 + 12
// of the group.  Lane j accumulates k = j (mod 32) in ascending k across the
// chunks (the canonical order), so every router weight a lane reads serves 8
// tokens and every token value 4 experts, and a CTA reads each router row
// once per 16 tokens.
constexpr int kTileTok = 16, kTileWarps = 8, kTileChunk = 512;
constexpr int kTileTokPerWarp = 8, kTileExpPerWarp = 4;
constexpr int kTileWBytes = kGroupE * kTileChunk * 4;     // 32 KB of router rows
constexpr int kTileXBytes = kTileTok * kTileChunk * 2;    // 16 KB of token rows
constexpr size_t kTileSmem = 2 * (size_t)(kTileWBytes + kTileXBytes);
static_assert(kTileWarps * kTileTokPerWarp * kTileExpPerWarp == kTileTok * kGroupE,
              "the warps cover the 16 tokens x 16 experts of a group");

__global__ void __launch_bounds__(kTileWarps * 32, 2)
    k_route_tiles(const uint16_t* __restrict__ x, int64_t T, int64_t d, const float* __restrict__ wr,
                  const float* __restrict__ bias, int E, int top_k, int renorm,
                  int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ logits) {
    extern __shared__ __align__(16) uint8_t tile_smem[];
    __shared__ float s_logit[kTileTok][kMaxE];
    float* const sw0 = reinterpret_cast<float*>(tile_smem);
    uint16_t* const sx0 = reinterpret_cast<uint16_t*>(tile_smem + kTileWBytes);
    const size_t buf_bytes = kTileWBytes + kTileXBytes;
    auto sw = [&](int b) { return reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sw0) + b * buf_bytes); };
    auto sx = [&](int b) {
        return reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(sx0) + b * buf_bytes);
    };
    pdl_wait();  // the previous step may still read ids and gates
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int tg = warp / kTileExpPerWarp, eg = warp % kTileExpPerWarp;
    const int nchunks = (int)((d + kTileChunk - 1) / kTileChunk);
    for (int64_t t0 = (int64_t)blockIdx.x * kTileTok; t0 < T; t0 += (int64_t)gridDim.x * kTileTok) {
        for (int e0 = 0; e0 < E; e0 += kGroupE) {
            // copies of chunk c into buffer b: the group's router rows and the
            // tokens' rows (tokens past T repeat the last one; never written)
            auto stage = [&](int c, int b) {
                const int64_t base = (int64_t)c * kTileChunk;
                const int n = (int)(d - base < kTileChunk ? d - base : (int64_t)kTileChunk);
                const int wu = n / 4, xu = n / 8;  // 16-byte units per row
                float* w_dst = sw(b);
                uint16_t* x_dst = sx(b);
                for (int i = threadIdx.x; i < kGroupE * wu; i += blockDim.x) {
                    const int r = i / wu, u = i - r * wu;
                    if (e0 + r < E)
                        cp_async_16(w_dst + r * kTileChunk + 4 * u, wr + (int64_t)(e0 + r) * d + base + 4 * u, 16);
                }
                for (int i = threadIdx.x; i < kTileTok * xu; i += blockDim.x) {
                    const int r = i / xu, u = i - r * xu;
                    const int64_t tok = t0 + r < T ? t0 + r : T - 1;
                    cp_async_16(x_dst + r * kTileChunk + 8 * u, x + tok * d + base + 8 * u, 16);
                }
                cp_async_commit();
            };
            double acc[kTileTokPerWarp][kTileExpPerWarp];
#pragma unroll
            for (int t = 0; t < kTileTokPerWarp; ++t)
#pragma unroll
                for (int i = 0; i < kTileExpPerWarp; ++i) acc[t][i] = 0.0;
            stage(0, 0);
            for (int c = 0; c < nchunks; ++c) {
                if (c + 1 < nchunks) {
                    stage(c + 1, (c + 1) & 1);
                    cp_async_wait<1>();
                } else {
                    cp_async_wait<0>();
                }
                __syncthreads();
                const float* W = sw(c & 1);
                const uint16_t* X = sx(c & 1) + tg * kTileTokPerWarp * kTileChunk;
                const int n = (int)(d - (int64_t)c * kTileChunk < kTileChunk ? d - (int64_t)c * kTileChunk
                                                                            : (int64_t)kTileChunk);
#pragma unroll 2
                for (int k = lane; k < n; k += 32) {
                    double xv[kTileTokPerWarp];
#pragma unroll
                    for (int t = 0; t < kTileTokPerWarp; ++t)
                        xv[t] = (double)bf16_bits_to_f32(X[t * kTileChunk + k]);
#pragma unroll
                    for (int i = 0; i < kTileExpPerWarp; ++i) {
                        const int e = eg + kTileExpPerWarp * i;
                        if (e0 + e < E) {
                            const double w = (double)W[e * kTileChunk + k];
#pragma unroll
                            for (int t = 0; t < kTileTokPerWarp; ++t) acc[t][i] = fma(xv[t], w, acc[t][i]);
                        }
                    }
                }
                __syncthreads();  // buffer c & 1 is refilled for chunk c + 2
            }
#pragma unroll
            for (int t = 0; t < kTileTokPerWarp; ++t)
#pragma unroll
                for (int i = 0; i < kTileExpPerWarp; ++i) {
                    double v = acc[t][i];
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
                    const int e = e0 + eg + kTileExpPerWarp * i;
                    if (lane == 0 && e < E)
                        s_logit[tg * kTileTokPerWarp + t][e] =
                            __double2float_rn(v + (bias ? (double)bias[e] : 0.0));
                }
        }
        __syncthreads();
        for (int r = warp; r < kTileTok; r += kTileWarps)
            if (t0 + r < T) warp_select_topk(s_logit[r], t0 + r, E, top_k, renorm, ids, gates, logits);
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_route(const void* x_bf16, int64_t T, int64_t d, const float* w_router,
                         const float* bias, int E, int top_k, int renorm, int32_t* ids,
                         float* gates, float* logits, int num_sms, cudaStream_t stream) {
    return launch_norm_route(x_bf16, T, d, nullptr, 0.0f, nullptr, w_router, bias, E, top_k,
                             renorm, ids, gates, logits, num_sms, stream);
}

cudaError_t launch_rmsnorm(const void* x_bf16, int64_t T, int64_t d, const void* gamma_bf16,
                           float eps, void* y_bf16, int num_sms, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    int64_t blocks = (T + 7) / 8;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    k_rmsnorm<<<(unsigned)blocks, 256, 0, stream>>>(static_cast<const uint16_t*>(x_bf16), T, d,
                                                   static_cast<const uint16_t*>(gamma_bf16), eps,
                                                   static_cast<uint16_t*>(y_bf16));
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_norm_route(const void* x_bf16, int64_t T, int64_t d, const void* gamma_bf16,
                              float eps, void* y_bf16, const float* w_router, const float* bias,
                              int E, int top_k, int renorm, int32_t* ids, float* gates,
                              float* logits, int num_sms, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    const bool norm = gamma_bf16 != nullptr;
    // Few tokens: a cluster of 4 CTAs per token, the RMSNorm (if any) fused in
    // front of the logits (or, for very wide rows, a 16-warp CTA streaming the
    // router rows in chunks); many tokens: 16 tokens per 8-warp CTA with the
    // rows staged in shared memory (k_route_tiles).  Outside the fused kernel the
    // RMSNorm runs first, into y, and the router reads y.
    const size_t csmem = (size_t)kExpertsPerCta * d * sizeof(float) + (size_t)d * sizeof(uint16_t);
    const size_t smem = (size_t)kGroupE * kChunkSmem + (size_t)d * sizeof(uint16_t);
    if (T < (int64_t)num_sms * 8 && csmem <= kClusterMaxSmem && T * kRouteCluster < (1LL << 31)) {
        const auto kernel = norm ? k_route_cluster<true> : k_route_cluster<false>;
        const cudaError_t e = cudaFuncSetAttribute(
            kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kClusterMaxSmem);
        if (e != cudaSuccess) return e;
        return launch_pdl(kernel, dim3((unsigned)(T * kRouteCluster)), dim3(kExpertsPerCta * 32),
                          csmem, stream, (const uint16_t*)x_bf16, d, w_router, bias, E, top_k,
                          renorm, ids, gates, logits, (const uint16_t*)gamma_bf16, eps,
                          (uint16_t*)y_bf16);
    }
    const void* xr = x_bf16;
    if (norm) {
        const cudaError_t e = launch_rmsnorm(x_bf16, T, d, gamma_bf16, eps, y_bf16, num_sms, stream);
        if (e != cudaSuccess) return e;
        xr = y_bf16;
    }
    if (T < (int64_t)num_sms * 8 && smem <= kWideMaxSmem) {
        const cudaError_t e = cudaFuncSetAttribute(
            k_route_wide, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWideMaxSmem);
        if (e != cudaSuccess) return e;
        k_route_wide<<<(unsigned)T, kGroupE * 32, smem, stream>>>(
            (const uint16_t*)xr, d, w_router, bias, E, top_k, renorm, ids, gates, logits);
        note_launch();
    } else {
        int64_t blocks = (T + kTileTok - 1) / kTileTok;
        const int64_t cap = (int64_t)num_sms * 2;  // one wave: two CTAs per SM
        if (blocks > cap) blocks = cap;
        const cudaError_t e = cudaFuncSetAttribute(
            k_route_tiles, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTileSmem);
        if (e != cudaSuccess) return e;
        return launch_pdl(k_route_tiles, dim3((unsigned)blocks), dim3(kTileWarps * 32), kTileSmem,
                          stream, (const uint16_t*)xr, T, d, w_router, bias, E, top_k, renorm, ids,
                          gates, logits);
    }
    return cudaGetLastError();
}

}  // namespace jmoe
