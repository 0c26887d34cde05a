// Decode path of the expert MLPs: few tokens per expert, so the work is one
// stream over the INT8 weights of the experts that some token selected
// (HBM-bound; the weights of untouched experts are never read).
//
// ExpertsInt8 ("Jamba-1.5: Hybrid Transformer-Mamba Models at Scale", paper
// summary, section "ExpertsInt8 Quantization (Section 3.1)", steps 3-4): the
// INT8 weights cross HBM once and are turned back into BF16 on chip; the
// activations stay BF16.  Here the weight bytes go HBM -> shared memory by
// bulk asynchronous copies (1 byte per weight), are converted exactly to bf16
// in registers (the scale is applied once per output channel after the dot
// product, an exact refactoring of sum_k x_k (q_k s)), and feed mma.sync
// m16n8k16 tiles whose 8 columns are up to 8 tokens of the expert; fp32
// accumulation.
//
// One CTA per SM, persistent: 1 producer warp + 16 consumer warps.
//  - A work unit is (touched expert, 16 output channels, one pass of up to
//    8*NCH tokens): a slab of R weight rows (gate/up: 16 gate + the matching
//    16 up rows; down: 16 rows) over the whole contraction length K.  Units
//    are dealt to the CTAs round-robin; they are small, so the CTAs finish
//    together.
//  - The producer streams each slab in stages of R rows x KC bytes (32 KB),
//    one cp.async.bulk per row (lane r copies row r), into a ring of 4-5
//    stages: about 130-160 KB of weights in flight per SM, independent of
//    what the consumers are doing.
//  - Consumer warp w takes k-blocks [w*KB_W, (w+1)*KB_W) of every stage (64 B
//    each) and accumulates its partial dot products over the whole unit.  Rows
//    sit at a pitch of KC + 64 bytes, which spreads the 16-byte fragment reads
//    of a warp over all banks.
//  - At the end of a unit the 16 partials go to shared memory (double
//    buffered by unit parity), an mbarrier collects the 16 warps, and all 512
//    consumer threads sum them in warp order (deterministic) and write:
//      gate/up : h = silu(s_g * x.q_g) * (s_u * x.q_u) -> H (bf16, slot order)
//      down    : y = gate * (s_d * h.q_d)               -> Y (fp32, one row per
//                                                          token->expert assignment)
//    launch_finalize then sums each token's rows of Y into the bf16 output.
// Fragment trick: the dot product does not care in which order k is summed,
// so the 16 k-columns of an MMA step are a permutation of the 64-wide k-block
// chosen such that thread (g = lane/4, c = lane%4) reads exactly bytes
// [16c, 16c+16) of rows g and g+8 for the block's four MMA steps, and the
// matching 16 consecutive bf16 of its token.  Step s uses physical
// k = 16c + 4s + {0,1} for fragment columns 2c, 2c+1 and 16c + 4s + {2,3} for
// columns 2c+8, 2c+9.
// Every wait is bounded (a stuck wait raises the abort flag, sets the device
// error word and lets all warps leave).
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace jmoe {
namespace {

using namespace sm100;

constexpr int kConsumers = 16;
constexpr int kProducer = kConsumers;  // warp index of the producer
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kPad = 64;
constexpr int kMaxE = 16;
constexpr int kMaxStages = 5;

enum { kGateUp = 0, kDown = 1 };

template <int MODE, int NCH>
struct Cfg {
    static constexpr int R = MODE == kGateUp ? 32 : 16;       // slab rows
    static constexpr int KC = MODE == kGateUp ? 1024 : 2048;  // stage bytes per row
    static constexpr int KBW = KC / 64 / kConsumers;          // 64-B k-blocks per warp per stage
    static constexpr int kPitch = KC + kPad;
    static constexpr int kStage = R * kPitch;
    static constexpr int kStages = NCH == 1 ? 5 : 4;
    static constexpr int NMAT = MODE == kGateUp ? 2 : 1;  // weight matrices per slab
    static constexpr int kAcc = NMAT * 4;                 // fp32 per token chunk per thread
    static constexpr int kRedFloats = 2 * kConsumers * NCH * kAcc * 32;
    static constexpr int kSmem = kStages * kStage + kRedFloats * 4;
};

struct Units {
    int start[kMaxE + 1];  // first unit of expert e
    int groups;            // 16-channel groups per expert
};

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

struct GemvParams {
    int E, top_k;
    int64_t d, f;
    const int8_t* w;        // gate/up [E][2f][d] or down [E][d][f]
    const float* scale;     // [E][2f] or [E][d]
    const int32_t* offsets; // [E+1]
    const int32_t* perm;    // [A]
    const float* gates;     // [A]        (down)
    const uint16_t* b_src;  // x [T][d] (gate/up) or H [A][f] (down)
    uint16_t* H;            // out of gate/up: bf16 [A][f]
    float* Y;               // out of down: fp32 [A][d]
    unsigned* err;
};

template <int MODE, int NCH>
__global__ void __launch_bounds__(kThreads, 1) k_gemv(const GemvParams p) {
    using C = Cfg<MODE, NCH>;
    extern __shared__ __align__(128) uint8_t smem[];
    float* red = reinterpret_cast<float*>(smem + C::kStages * C::kStage);
    __shared__ uint64_t full[kMaxStages], empty[kMaxStages], red_full[2];
    __shared__ Units U;
    __shared__ int s_off[kMaxE + 1];
    __shared__ int s_abort;

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int E = p.E;
    const int64_t K = MODE == kGateUp ? p.d : p.f;
    const int64_t rows_out = MODE == kGateUp ? p.f : p.d;  // output channels per expert
    const int nst = (int)((K + C::KC - 1) / C::KC);       // stages per unit

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumers);
        }
        mbar_init(&red_full[0], kConsumers);
        mbar_init(&red_full[1], kConsumers);
        s_abort = 0;
        int run = 0;
        for (int e = 0; e < E; ++e) {
            const int cnt = p.offsets[e + 1] - p.offsets[e];
            U.start[e] = run;
            run += cnt > 0 ? (cnt + 8 * NCH - 1) / (8 * NCH) * (int)(rows_out / 16) : 0;
        }
        U.start[E] = run;
        U.groups = (int)(rows_out / 16);
        fence_mbar_init();
    }
    if (threadIdx.x <= E) s_off[threadIdx.x] = p.offsets[threadIdx.x];
    __syncthreads();
    volatile int* abort = &s_abort;
    const int n_units = U.start[E];
    const int G = gridDim.x;
    const int n_mine = (int)blockIdx.x < n_units ? (n_units - 1 - (int)blockIdx.x) / G + 1 : 0;

    if (warp == kProducer) {
        uint32_t g = 0;
        bool ok = true;
        for (int it = 0; it < n_mine && ok; ++it) {
            const Unit u = decode_unit(U, E, blockIdx.x + it * G);
            const int8_t* src = nullptr;
            if (lane < C::R) {
                int64_t row;
                if (MODE == kGateUp)
                    row = (int64_t)u.e * 2 * p.f + (lane < 16 ? 0 : p.f) + u.group * 16 + (lane & 15);
                else
                    row = (int64_t)u.e * p.d + u.group * 16 + lane;
                src = p.w + row * K;
            }
            for (int st = 0; st < nst; ++st, ++g) {
                const int s = g % C::kStages;
                const uint32_t ph = (g / C::kStages) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, abort)) {
                    ok = false;
                    break;
                }
                const int64_t k0 = (int64_t)st * C::KC;
                const uint32_t bytes = (uint32_t)min((int64_t)C::KC, K - k0);
                if (lane == 0) mbar_arrive_expect_tx(&full[s], C::R * bytes);
                __syncwarp();
                if (lane < C::R) bulk_load(smem + s * C::kStage + lane * C::kPitch, src + k0, bytes,
                                           &full[s]);
            }
        }
        // do not leave while a copy may still be landing in shared memory
        for (uint32_t h = (g > (uint32_t)C::kStages ? g - C::kStages : 0); h < g; ++h) {
            const long long t0 = clock64();
            while (!mbar_try_wait(&full[h % C::kStages], (h / C::kStages) & 1))
                if (clock64() - t0 > kWaitCycles) break;
        }
    } else {
        const int g8 = lane >> 2, c = lane & 3;
        float acc[NCH][C::NMAT][4];
#pragma unroll
        for (int n = 0; n < NCH; ++n)
#pragma unroll
            for (int m = 0; m < C::NMAT; ++m)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[n][m][i] = 0.0f;
        uint32_t g = 0;
        bool ok = true;
        for (int it = 0; it < n_mine && ok; ++it) {
            const Unit u = decode_unit(U, E, blockIdx.x + it * G);
            const int base = s_off[u.e] + u.pass * 8 * NCH;
            const int cnt_pass = min(8 * NCH, s_off[u.e + 1] - base);
            const uint16_t* bp[NCH];
#pragma unroll
            for (int n = 0; n < NCH; ++n) {
                const int slot = n * 8 + g8;
                if (slot < cnt_pass) {
                    const int64_t row =
                        MODE == kGateUp ? (int64_t)(p.perm[base + slot] / p.top_k) : base + slot;
                    bp[n] = p.b_src + row * K + 16 * c;
                } else {
                    bp[n] = nullptr;
                }
            }
            for (int st = 0; st < nst; ++st, ++g) {
                const int s = g % C::kStages;
                const uint32_t ph = (g / C::kStages) & 1;
                if (!mbar_wait(&full[s], ph, abort)) {
                    ok = false;
                    break;
                }
                const int64_t k0 = (int64_t)st * C::KC;
                const int valid = (int)min((int64_t)C::KC, K - k0);
                const uint8_t* stage = smem + s * C::kStage;
#pragma unroll
                for (int kb = 0; kb < C::KBW; ++kb) {
                    const int kbyte = (warp * C::KBW + kb) * 64;
                    if (kbyte < valid) {
                        const uint8_t* r0 = stage + g8 * C::kPitch + kbyte + 16 * c;
                        const uint4 q0 = *reinterpret_cast<const uint4*>(r0);
                        const uint4 q1 = *reinterpret_cast<const uint4*>(r0 + 8 * C::kPitch);
                        uint4 q2, q3;
                        if (MODE == kGateUp) {
                            q2 = *reinterpret_cast<const uint4*>(r0 + 16 * C::kPitch);
                            q3 = *reinterpret_cast<const uint4*>(r0 + 24 * C::kPitch);
                        }
#pragma unroll
                        for (int n = 0; n < NCH; ++n) {
                            if (n * 8 < cnt_pass) {
                                uint32_t b[8];
                                load_b(bp[n] ? bp[n] + k0 + kbyte : nullptr, b);
                                mma_block(acc[n][0], q0, q1, b);
                                if (MODE == kGateUp) mma_block(acc[n][C::NMAT - 1], q2, q3, b);
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            if (!ok) break;
            // ---- end of unit: partials -> shared, then 512 threads finish
            const int buf = it & 1;
            float* rb = red + buf * (kConsumers * NCH * C::kAcc * 32);
#pragma unroll
            for (int n = 0; n < NCH; ++n)
#pragma unroll
                for (int m = 0; m < C::NMAT; ++m)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        rb[((warp * NCH + n) * C::kAcc + 4 * m + i) * 32 + lane] = acc[n][m][i];
                        acc[n][m][i] = 0.0f;
                    }
            __syncwarp();
            if (lane == 0) mbar_arrive(&red_full[buf]);
            if (!mbar_wait(&red_full[buf], (it >> 1) & 1, abort)) break;
            const int pos = threadIdx.x;  // 0..511: (n, i, lane') with lane' fastest
            if (pos < NCH * 4 * 32) {
                const int ln = pos & 31, i = (pos >> 5) & 3, n = pos >> 7;
                float v0 = 0.f, v1 = 0.f;
                for (int w2 = 0; w2 < kConsumers; ++w2) {
                    v0 += rb[((w2 * NCH + n) * C::kAcc + i) * 32 + ln];
                    if (MODE == kGateUp) v1 += rb[((w2 * NCH + n) * C::kAcc + 4 + i) * 32 + ln];
                }
                const int slot = n * 8 + 2 * (ln & 3) + (i & 1);
                const int row = (ln >> 2) + (i >> 1) * 8;
                const int64_t ch = (int64_t)u.group * 16 + row;
                if (slot < cnt_pass) {
                    if (MODE == kGateUp) {
                        const float* sg = p.scale + (int64_t)u.e * 2 * p.f;
                        const float h = silu_f32(sg[ch] * v0) * (sg[p.f + ch] * v1);
                        p.H[(int64_t)(base + slot) * p.f + ch] =
                            __bfloat16_as_ushort(__float2bfloat16_rn(h));
                    } else {
                        const int a = p.perm[base + slot];
                        p.Y[(int64_t)a * p.d + ch] =
                            p.gates[a] * (p.scale[(int64_t)u.e * p.d + ch] * v0);
                    }
                }
            }
        }
    }
    if (s_abort && threadIdx.x == kProducer * 32) flag_error(p.err, kErrTimeout);
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

template <int MODE, int NCH>
cudaError_t launch_gemv(const GemvParams& p, int grid, cudaStream_t stream) {
    using C = Cfg<MODE, NCH>;
    cudaError_t err = cudaFuncSetAttribute(k_gemv<MODE, NCH>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (err != cudaSuccess) return err;
    k_gemv<MODE, NCH><<<grid, kThreads, C::kSmem, stream>>>(p);
    return cudaGetLastError();
}

template <int NCH>
cudaError_t launch_decode_nch(const DecodeArgs& a, cudaStream_t stream) {
    GemvParams p{};
    p.E = a.E;
    p.top_k = a.top_k;
    p.d = a.d;
    p.f = a.f;
    p.offsets = a.offsets;
    p.perm = a.perm;
    p.gates = a.gates;
    p.err = a.err;
    p.w = a.wgu;
    p.scale = a.sgu;
    p.b_src = static_cast<const uint16_t*>(a.x);
    p.H = static_cast<uint16_t*>(a.H);
    if (a.mark) a.mark(2, false, stream);
    cudaError_t err = launch_gemv<kGateUp, NCH>(p, a.num_sms, stream);
    if (a.mark) a.mark(2, true, stream);
    if (err != cudaSuccess) return err;
    p.w = a.wd;
    p.scale = a.sd;
    p.b_src = static_cast<const uint16_t*>(a.H);
    p.H = nullptr;
    p.Y = a.Y;
    if (a.mark) a.mark(3, false, stream);
    err = launch_gemv<kDown, NCH>(p, a.num_sms, stream);
    if (a.mark) a.mark(3, true, stream);
    return err;
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
