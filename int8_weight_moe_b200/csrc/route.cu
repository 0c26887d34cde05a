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
// Work split: for many tokens a CTA of 8 warps handles 32 tokens with the
// router rows and token rows staged in shared memory (k_route_tiles: each
// lane keeps 8 tokens x 8 experts of fp64 partial sums).
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

// Many tokens: a CTA of 8 warps computes the logits of 32 tokens, one group
// of 16 experts at a time, the router rows and token rows streamed through
// shared memory in k-chunks of 256 (16-byte cp.async copies, four chunks in
// flight).  Warp w keeps the fp64 partial sums of tokens 8 (w / 2) .. +7 for
// the experts w % 2, w % 2 + 2, ..., w % 2 + 14 of the group; lane j
// accumulates k = j (mod 32) in ascending k across the chunks (the canonical
// order), so every router weight a lane reads serves 8 tokens and every token
// value 8 experts.
//
// No conversion instruction runs in the inner loop (an fp32 -> fp64
// conversion issues at a small fraction of the fp64 FMA rate).  Each product
// x * w is formed as (x * 2^-896) * (w * 2^896), which is the same real
// number, so every fused multiply-add -- and every rounding of the canonical
// order -- is unchanged:
// - x * 2^-896 is the bf16 bit pattern moved into the fp64 fields: the 8-bit
//   exponent field read with the fp64 bias (1023 instead of 127) is exactly
//   that scaling, for zeros and subnormals too; only an all-ones exponent
//   (inf, NaN) maps wrongly, so a chunk holding one takes the exact
//   conversion for it (a CTA-wide flag found while the chunk is staged);
// - w * 2^896 is exact for every fp32 value (2^127 * 2^896 = 2^1023 still
//   fits) and is written to shared memory in fp64 once per CTA and chunk,
//   by integer field arithmetic for normal numbers and by the conversion
//   instruction otherwise.
constexpr int kRtTok = 32, kRtK = 256, kRtStages = 4;
constexpr int kRtTokPerWarp = 8, kRtExpPerWarp = 8;
constexpr int kRtEStride = kGroupE / kRtExpPerWarp;  // warps per token group; expert stride
constexpr int kRtWarps = kRtTok / kRtTokPerWarp * kRtEStride;
constexpr int kRtSums = kRtTokPerWarp * kRtExpPerWarp / 32;  // sums a lane holds after the tree
constexpr int kRtPrep = kGroupE * kRtK / 4 / (kRtWarps * 32);  // 16-byte pieces per thread and half
constexpr int kRtWRawBytes = kGroupE * kRtK * 4;          // 16 KB: fp32 router rows
constexpr int kRtXBytes = kRtTok * kRtK * 2;              // 16 KB: bf16 token rows
constexpr int kRtStageBytes = kRtWRawBytes + kRtXBytes;
constexpr int kRtW64Bytes = kGroupE * kRtK * 8;           // 32 KB: scaled fp64 router rows
constexpr int kRtLogitBytes = kRtTok * kMaxE * 4;         // 8 KB
constexpr size_t kTileSmem = (size_t)kRtStages * kRtStageBytes + 2 * (size_t)kRtW64Bytes +
                             2 * (size_t)kRtLogitBytes;
static_assert(kRtWarps * kRtTokPerWarp * kRtExpPerWarp == kRtTok * kGroupE,
              "the warps cover the 32 tokens x 16 experts of a group");
static_assert(kRtK % 64 == 0, "chunks hold whole 64-wide pieces of a row");
static_assert(kRtTok * kRtK / 8 == kGroupE * kRtK / 4, "token and router rows split alike");

// x * 2^-896 from the bf16 bits sign-extended to 32 bits (s << 13 puts the
// exponent field at bits 20..27, the mantissa at 13..19 and copies of the
// sign at 28..31; the mask keeps bit 31 of those).
__device__ __forceinline__ double rt_x_scaled(int s) {
    return __hiloint2double((int)(((uint32_t)s << 13) & 0x8fffe000u), 0);
}

// w * 2^896 in fp64 (the exponent field grows by 1792 = 896 + 1023 - 127).
__device__ __forceinline__ double rt_w_scaled(uint32_t b) {
    if ((b & 0x7f800000u) - 0x00800000u < 0x7f000000u) {  // normal
        const uint32_t hi = ((uint32_t)((int32_t)b >> 3) & 0x8fffffffu) + 0x70000000u;
        return __hiloint2double((int)hi, (int)(b << 29));
    }
    return (double)__uint_as_float(b) * 0x1p896;
}

// One chunk of the warp's kRtTokPerWarp tokens x kRtExpPerWarp experts: n
// (a multiple of 32) values of each row, X the warp's first token row, Wd its
// first scaled router row (the warp's experts are kRtEStride rows apart); ne
// of its experts exist (all of them when kFull).  The operands of the next k
// are loaded while this one's fused multiply-adds issue.
template <bool kExact, bool kFull>
__device__ __forceinline__ void rt_chunk(const int16_t* __restrict__ X, const double* __restrict__ Wd,
                                         int n, int ne, double (&acc)[kRtTokPerWarp][kRtExpPerWarp]) {
    const int lane = threadIdx.x & 31;
    int xs[kRtTokPerWarp];
    double wv[kRtExpPerWarp];
#pragma unroll
    for (int t = 0; t < kRtTokPerWarp; ++t) xs[t] = X[t * kRtK + lane];
#pragma unroll
    for (int i = 0; i < kRtExpPerWarp; ++i)
        wv[i] = kFull || i < ne ? Wd[kRtEStride * i * kRtK + lane] : 0.0;
#pragma unroll 1
    for (int k = lane; k < n; k += 32) {
        double xv[kRtTokPerWarp], wc[kRtExpPerWarp];
#pragma unroll
        for (int t = 0; t < kRtTokPerWarp; ++t) {
            xv[t] = rt_x_scaled(xs[t]);
            if (kExact && (xs[t] & 0x7f80) == 0x7f80)
                xv[t] = (double)bf16_bits_to_f32((uint16_t)xs[t]);  // inf or NaN: unscaled is exact
        }
#pragma unroll
        for (int i = 0; i < kRtExpPerWarp; ++i) wc[i] = wv[i];
        const int kn = k + 32;
        if (kn < n) {
#pragma unroll
            for (int t = 0; t < kRtTokPerWarp; ++t) xs[t] = X[t * kRtK + kn];
#pragma unroll
            for (int i = 0; i < kRtExpPerWarp; ++i)
                if (kFull || i < ne) wv[i] = Wd[kRtEStride * i * kRtK + kn];
        }
#pragma unroll
        for (int i = 0; i < kRtExpPerWarp; ++i)
            if (kFull || i < ne)
#pragma unroll
                for (int t = 0; t < kRtTokPerWarp; ++t) acc[t][i] = fma(xv[t], wc[i], acc[t][i]);
    }
}

// The halving tree p_j += p_{j+o} (o = 16 ... 1) of all the warp's sums at
// once: at each step a lane keeps half of its sums and hands the other half
// to lane ^ o, which adds them to its own (addition is commutative, so each
// pair is summed exactly as in the one-sum-at-a-time tree).  Afterwards lane
// L holds the sums q = kRtSums * L + m, m < kRtSums (q = token * experts per
// warp + expert slot), in v[m].
__device__ __forceinline__ void rt_tree(double (&v)[kRtTokPerWarp * kRtExpPerWarp]) {
    const int lane = threadIdx.x & 31;
    constexpr int kAll = kRtTokPerWarp * kRtExpPerWarp;
#pragma unroll
    for (int o = 16, half = kAll / 2; o >= 1; o >>= 1, half >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int m = 0; m < half; ++m) {
            const double keep = upper ? v[m + half] : v[m];
            const double send = upper ? v[m] : v[m + half];
            v[m] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
}

__global__ void __launch_bounds__(kRtWarps * 32, 1)
    k_route_tiles(const uint16_t* __restrict__ x, int64_t T, int64_t d, const float* __restrict__ wr,
                  const float* __restrict__ bias, int E, int top_k, int renorm,
                  int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ logits) {
    extern __shared__ __align__(16) uint8_t tile_smem[];
    auto w_raw = [&](int s) { return reinterpret_cast<float*>(tile_smem + s * kRtStageBytes); };
    auto x_raw = [&](int s) {
        return reinterpret_cast<int16_t*>(tile_smem + s * kRtStageBytes + kRtWRawBytes);
    };
    auto w64 = [&](int b) {
        return reinterpret_cast<double*>(tile_smem + kRtStages * kRtStageBytes + b * kRtW64Bytes);
    };
    auto s_logit = [&](int b) {
        return reinterpret_cast<float*>(tile_smem + kRtStages * kRtStageBytes + 2 * kRtW64Bytes +
                                        b * kRtLogitBytes);
    };
    pdl_wait();  // the previous step may still read ids and gates
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tg = warp / kRtEStride, eq = warp % kRtEStride;
    const int nch = (int)((d + kRtK - 1) / kRtK);
    const int ngroups = (E + kGroupE - 1) / kGroupE;
    const int64_t ntiles = (T + kRtTok - 1) / kRtTok;
    const int64_t my_tiles = ntiles > blockIdx.x ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int64_t U = my_tiles * ngroups * nch;  // (tile, group, chunk) units of this CTA
    // a unit's place, advanced one unit at a time (no divisions)
    struct Unit {
        int tile_i, g, c;
        __device__ void next(int nch_, int ngroups_) {
            if (++c == nch_) {
                c = 0;
                if (++g == ngroups_) { g = 0; ++tile_i; }
            }
        }
    };
    auto t0_of = [&](const Unit& r) { return ((int64_t)blockIdx.x + (int64_t)r.tile_i * gridDim.x) * kRtTok; };
    auto n_of = [&](const Unit& r) {
        const int64_t base = (int64_t)r.c * kRtK;
        return (int)(d - base < kRtK ? d - base : (int64_t)kRtK);
    };
    auto rows_of = [&](const Unit& r) { return E - r.g * kGroupE < kGroupE ? E - r.g * kGroupE : kGroupE; };
    // copies of unit u (at r) into stage u % kRtStages (tokens past T repeat
    // the last one; their logits are never written); one commit group per
    // unit, empty past the end, so the group count stays uniform
    auto stage = [&](int64_t u, const Unit& r) {
        if (u < U) {
            const int s = (int)(u % kRtStages);
            const int64_t base = (int64_t)r.c * kRtK, t0 = t0_of(r);
            const int n = n_of(r), rows = rows_of(r), e0 = r.g * kGroupE;
            float* wd = w_raw(s);
            int16_t* xd = x_raw(s);
            for (int i = tid; i < kGroupE * (kRtK / 4); i += kRtWarps * 32) {
                const int row = i / (kRtK / 4), p = i % (kRtK / 4);
                if (row < rows && 4 * p < n)
                    cp_async_16(wd + row * kRtK + 4 * p, wr + (int64_t)(e0 + row) * d + base + 4 * p, 16);
            }
            for (int i = tid; i < kRtTok * (kRtK / 8); i += kRtWarps * 32) {
                const int row = i / (kRtK / 8), p = i % (kRtK / 8);
                const int64_t tok = t0 + row < T ? t0 + row : T - 1;
                if (8 * p < n) cp_async_16(xd + row * kRtK + 8 * p, x + tok * d + base + 8 * p, 16);
            }
        }
        cp_async_commit();
    };
    // piece j (0 .. 2 kRtPrep - 1) of the preparation of unit u (at r): the
    // first kRtPrep scale the thread's share of the router rows into
    // w64[u & 1], the others look for an all-ones exponent in its share of the
    // token rows (returned as nonzero bits)
    auto prep = [&](int64_t u, const Unit& r, int j) -> uint32_t {
        const int s = (int)(u % kRtStages);
        const int n = n_of(r);
        if (j < kRtPrep) {
            const int f = tid + j * kRtWarps * 32;  // float4 index in [16][kRtK / 4]
            const int row = f / (kRtK / 4), k = 4 * (f % (kRtK / 4));
            if (row < rows_of(r) && k < n) {
                const uint4 b = *reinterpret_cast<const uint4*>(w_raw(s) + row * kRtK + k);
                double* dst = w64(u & 1) + row * kRtK + k;
                *reinterpret_cast<double2*>(dst) = make_double2(rt_w_scaled(b.x), rt_w_scaled(b.y));
                *reinterpret_cast<double2*>(dst + 2) = make_double2(rt_w_scaled(b.z), rt_w_scaled(b.w));
            }
            return 0u;
        }
        const int f = tid + (j - kRtPrep) * kRtWarps * 32;  // uint4 index in [32][kRtK / 8]
        const int row = f / (kRtK / 8), k = 8 * (f % (kRtK / 8));
        if (k >= n) return 0u;
        const uint4 b = *reinterpret_cast<const uint4*>(x_raw(s) + row * kRtK + k);
        uint32_t bad = ((b.x & 0x7f807f80u) + 0x00800080u) | ((b.y & 0x7f807f80u) + 0x00800080u) |
                       ((b.z & 0x7f807f80u) + 0x00800080u) | ((b.w & 0x7f807f80u) + 0x00800080u);
        return bad & 0x80008000u;
    };

    double acc[kRtTokPerWarp][kRtExpPerWarp];
    Unit st{0, 0, 0};  // the next unit to stage
    for (int s = 0; s < kRtStages; ++s) {
        stage(s, st);
        st.next(nch, ngroups);
    }
    cp_async_wait<kRtStages - 2>();  // units 0 and 1 have landed
    __syncthreads();
    int exact = 0;
    Unit r{0, 0, 0};
    if (U > 0) {
        uint32_t bad = 0;
        for (int j = 0; j < 2 * kRtPrep; ++j) bad |= prep(0, r, j);
        exact = __syncthreads_or(bad != 0);
    }
    for (int64_t u = 0; u < U; ++u) {
        // here: w64[u & 1] holds unit u's scaled router rows, `exact` says
        // whether its token rows hold an inf or NaN, and unit u + 1 has landed
        if (r.c == 0) {
#pragma unroll
            for (int t = 0; t < kRtTokPerWarp; ++t)
#pragma unroll
                for (int i = 0; i < kRtExpPerWarp; ++i) acc[t][i] = 0.0;
        }
        const int first = r.g * kGroupE + eq;  // the warp's first expert in this group
        const int avail = first < E ? (E - first + kRtEStride - 1) / kRtEStride : 0;
        const int ne = avail < kRtExpPerWarp ? avail : kRtExpPerWarp;
        const int n = n_of(r);
        const int16_t* X = x_raw((int)(u % kRtStages)) + tg * kRtTokPerWarp * kRtK;
        const double* Wd = w64(u & 1) + eq * kRtK;
        if (ne == kRtExpPerWarp) {
            if (exact) rt_chunk<true, true>(X, Wd, n, ne, acc);
            else rt_chunk<false, true>(X, Wd, n, ne, acc);
        } else {
            if (exact) rt_chunk<true, false>(X, Wd, n, ne, acc);
            else rt_chunk<false, false>(X, Wd, n, ne, acc);
        }
        Unit rn = r;
        rn.next(nch, ngroups);
        uint32_t bad = 0;
        if (u + 1 < U)
            for (int j = 0; j < 2 * kRtPrep; ++j) bad |= prep(u + 1, rn, j);
        const bool last_chunk = r.c == nch - 1;
        if (last_chunk) {
            double v[kRtTokPerWarp * kRtExpPerWarp];
#pragma unroll
            for (int t = 0; t < kRtTokPerWarp; ++t)
#pragma unroll
                for (int i = 0; i < kRtExpPerWarp; ++i) v[t * kRtExpPerWarp + i] = acc[t][i];
            rt_tree(v);
            float* sl = s_logit(r.tile_i & 1);
#pragma unroll
            for (int m = 0; m < kRtSums; ++m) {
                const int q = kRtSums * lane + m;
                const int t = q / kRtExpPerWarp, i = q % kRtExpPerWarp;
                const int e = first + kRtEStride * i;
                if (e < E)
                    sl[(tg * kRtTokPerWarp + t) * kMaxE + e] =
                        __double2float_rn(v[m] + (bias ? (double)bias[e] : 0.0));
            }
        }
        cp_async_wait<1>();  // unit u + 2 has landed
        exact = __syncthreads_or(bad != 0);
        stage(u + kRtStages, st);  // into the stage unit u used
        st.next(nch, ngroups);
        if (last_chunk && r.g == ngroups - 1) {
            const float* sl = s_logit(r.tile_i & 1);
            const int64_t t0 = t0_of(r);
            for (int row = warp; row < kRtTok; row += kRtWarps)
                if (t0 + row < T)
                    warp_select_topk(sl + row * kMaxE, t0 + row, E, top_k, renorm, ids, gates, logits);
        }
        r = rn;
    }
    cp_async_wait<0>();
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

// Whether the tiled kernel beats the per-token clusters for T tokens of width
// d.  Measured on the B200 (router alone, 16 experts): a wave of clusters (as
// many four-CTA clusters as fit at once, shared memory deciding how many CTAs
// share an SM) takes about 5.8 + 0.4 d/1024 us, a round of 32-token tiles (one
// per SM) about 4 + 0.0151 d us.  d_model 4096: clusters 0.039 ms at 512
// tokens and 0.069 ms at 1024, tiles 0.070 ms from 1184 to 4736 tokens;
// d_model 8192: clusters 0.071 ms at 256 tokens, 0.131 at 512, 0.250 at 1024,
// tiles 0.125 ms.  More experts scale both alike.
static bool route_tiles_cheaper(int64_t T, int64_t d, size_t cluster_smem, int num_sms) {
    constexpr int64_t kSmemPerSm = 227 * 1024;
    int64_t per_sm = kSmemPerSm / (int64_t)(cluster_smem + 1024);
    if (per_sm < 1) per_sm = 1;
    const int64_t at_once = (int64_t)num_sms * per_sm;
    const int64_t waves = (T * kRouteCluster + at_once - 1) / at_once;
    const int64_t rounds = (T + (int64_t)kRtTok * num_sms - 1) / ((int64_t)kRtTok * num_sms);
    const double cluster_us = (double)waves * (5.8 + 0.4 * (double)d / 1024.0);
    const double tiles_us = (double)rounds * (4.0 + 0.0151 * (double)d);
    return tiles_us < cluster_us;
}

cudaError_t launch_norm_route(const void* x_bf16, int64_t T, int64_t d, const void* gamma_bf16,
                              float eps, void* y_bf16, const float* w_router, const float* bias,
                              int E, int top_k, int renorm, int32_t* ids, float* gates,
                              float* logits, int num_sms, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    const bool norm = gamma_bf16 != nullptr;
    // Few tokens: a cluster of 4 CTAs per token, the RMSNorm (if any) fused in
    // front of the logits, while that is cheaper than the tiles (or, for rows too
    // wide for the clusters, a 16-warp CTA per token streaming the router rows in
    // chunks); otherwise 32 tokens per 8-warp CTA with the rows staged in shared
    // memory (k_route_tiles).  Outside the fused kernel the RMSNorm runs first,
    // into y, and the router reads y.
    const size_t csmem = (size_t)kExpertsPerCta * d * sizeof(float) + (size_t)d * sizeof(uint16_t);
    const size_t smem = (size_t)kGroupE * kChunkSmem + (size_t)d * sizeof(uint16_t);
    const bool few = T < (int64_t)num_sms * 8;
    const bool cluster_fits = csmem <= kClusterMaxSmem && T * kRouteCluster < (1LL << 31);
    if (few && cluster_fits && !route_tiles_cheaper(T, d, csmem, num_sms)) {
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
    if (few && !cluster_fits && smem <= kWideMaxSmem) {
        const cudaError_t e = cudaFuncSetAttribute(
            k_route_wide, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kWideMaxSmem);
        if (e != cudaSuccess) return e;
        k_route_wide<<<(unsigned)T, kGroupE * 32, smem, stream>>>(
            (const uint16_t*)xr, d, w_router, bias, E, top_k, renorm, ids, gates, logits);
        note_launch();
    } else {
        int64_t blocks = (T + kRtTok - 1) / kRtTok;
        const int64_t cap = (int64_t)num_sms;  // one CTA per SM (208 KB of shared memory)
        if (blocks > cap) blocks = cap;
        const cudaError_t e = cudaFuncSetAttribute(
            k_route_tiles, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTileSmem);
        if (e != cudaSuccess) return e;
        return launch_pdl(k_route_tiles, dim3((unsigned)blocks), dim3(kRtWarps * 32), kTileSmem,
                          stream, (const uint16_t*)xr, T, d, w_router, bias, E, top_k, renorm, ids,
                          gates, logits);
    }
    return cudaGetLastError();
}

}  // namespace jmoe
