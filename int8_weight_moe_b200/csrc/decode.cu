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
// an mma.sync m16n8k16 whose 8 columns are up to 8 tokens of the expert; fp32
// accumulation.
//
// Fragment trick: the dot product does not care in which order k is summed,
// so the 16 k-columns of an MMA step are a permutation of the 64-wide k-block
// chosen such that thread (g = lane/4, c = lane%4) reads exactly bytes
// [16c, 16c+16) of rows g and g+8 for the block's four MMA steps -- one
// 16-byte load per row -- and the matching 16 consecutive bf16 of its token.
// Step s uses physical k = 16c + 4s + {0,1} for fragment columns 2c, 2c+1 and
// 16c + 4s + {2,3} for columns 2c+8, 2c+9.
//
// Work decomposition: every warp is an independent streaming worker.  A work
// item is (touched expert, 16 output channels, one pass of up to 8*NCH
// tokens, one K piece of S): a slab of 16 rows (gate/up: 16 gate + the same
// 16 up rows) x K/S bytes.  Items are small (16-32 KB) and dealt round-robin
// to all warps of the GPU, so the warps finish together; each warp keeps a
// ring of kDepth 64-byte steps of weights -- and of the matching activation
// fragments -- in shared memory, filled by cp.async three steps ahead of use
// and across item boundaries (the bytes in flight live in shared memory, not
// in registers), so there are no bubbles and no barriers at all.  An item
// stores its raw fp32 partial sums; the small follow-up kernels add the S
// pieces in a fixed order (deterministic) and apply scales, SwiGLU, gates:
//   k_gemv<gate/up> -> P_gu[S][slot][2f] -> k_swiglu -> H (bf16, slot order)
//   k_gemv<down>    -> P_d [S][slot][d]  -> k_combine -> out (bf16)
#include "common.cuh"
#include "kernels.h"

namespace jmoe {
namespace {

constexpr int kWarpsPerBlock = 4;
constexpr int kDepth = 4;  // ring slots per warp: three 64-byte steps in flight
constexpr int kMaxE = 16;

enum { kGateUp = 0, kDown = 1 };

struct GemvParams {
    int E, top_k, S;           // experts, experts per token, K pieces
    int64_t d, f;
    const int8_t* w;           // gate/up [E][2f][d] or down [E][d][f]
    const int32_t* offsets;    // [E+1]
    const int32_t* perm;       // [A]
    const uint16_t* b_src;     // x [T][d] (gate/up) or H [A][f] (down)
    float* P;                  // partial sums [S][A][cols]
    int64_t A;
};

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

// Four MMA steps of one 64-wide k-block: rows g (q0) and g+8 (q1).  Even and
// odd steps accumulate into separate tiles (two independent MMA chains).
__device__ __forceinline__ void mma_block(float (&acc)[2][4], const uint4& q0, const uint4& q1,
                                          const uint32_t (&b)[8]) {
    const uint32_t w0[4] = {q0.x, q0.y, q0.z, q0.w};
    const uint32_t w1[4] = {q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        const uint32_t a[4] = {i8x2_to_bf16x2<0>(w0[s]), i8x2_to_bf16x2<0>(w1[s]),
                               i8x2_to_bf16x2<1>(w0[s]), i8x2_to_bf16x2<1>(w1[s])};
        mma_bf16_16816(acc[s & 1], a, b[2 * s], b[2 * s + 1]);
    }
}

struct Item {
    int e, group, pass, z;
};

// Shared-memory bytes of one ring slot: per lane, 2*NMAT weight and NCH*2
// activation 16-byte pieces.
template <int MODE, int NCH>
constexpr int slot_bytes() {
    return (2 * (MODE == kGateUp ? 2 : 1) + 2 * NCH) * 32 * 16;
}

template <int MODE, int NCH>
constexpr int gemv_smem() {
    return kWarpsPerBlock * kDepth * slot_bytes<MODE, NCH>();
}

template <int MODE, int NCH>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    k_gemv(const GemvParams p) {
    constexpr int NMAT = MODE == kGateUp ? 2 : 1;
    constexpr int kPieces = 2 * NMAT + 2 * NCH;  // 16-byte pieces per lane per step
    extern __shared__ __align__(16) uint4 ring_smem[];
    __shared__ int s_start[kMaxE + 1];  // first item of expert e
    __shared__ int s_off[kMaxE + 1];
    const int lane = threadIdx.x & 31, g8 = lane >> 2, c = lane & 3;
    // this lane's pieces of slot q: ring[(q * kPieces + piece) * 32]
    uint4* ring = ring_smem + (threadIdx.x >> 5) * kDepth * kPieces * 32 + lane;
    const int E = p.E, S = p.S;
    const int64_t K = MODE == kGateUp ? p.d : p.f;
    const int64_t rows_out = MODE == kGateUp ? p.f : p.d;
    const int groups = (int)(rows_out / 16);
    if (threadIdx.x <= E) s_off[threadIdx.x] = p.offsets[threadIdx.x];
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            const int cnt = s_off[e + 1] - s_off[e];
            s_start[e] = run;
            run += cnt > 0 ? (cnt + 8 * NCH - 1) / (8 * NCH) * groups * S : 0;
        }
        s_start[E] = run;
    }
    __syncthreads();
    const int n_items = s_start[E];
    const int W = gridDim.x * kWarpsPerBlock;
    const int wid = blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    const int n_mine = wid < n_items ? (n_items - 1 - wid) / W + 1 : 0;
    const int nw = (int)(K / S / 64);  // 64-byte steps per item
    const int64_t total = (int64_t)n_mine * nw;
    if (total == 0) return;

    auto item_of = [&](int it) {
        const int idx = wid + it * W;
        int e = 0;
        while (e + 1 < E && s_start[e + 1] <= idx) ++e;
        const int local = idx - s_start[e];
        Item r;
        r.e = e;
        r.z = local % S;
        r.group = (local / S) % groups;
        r.pass = local / S / groups;
        return r;
    };

    // ---- prefetch cursor (item iteration pi, step pj): weight rows and the
    // activation (x or h) rows of the item's tokens, both loaded kDepth-1
    // steps ahead of use
    int pi = 0, pj = 0;
    const int8_t* pw[2 * NMAT];
    const uint16_t* pb[NCH];
    auto set_prefetch_item = [&](int it) {
        const Item u = item_of(it);
        const int64_t kz = (int64_t)u.z * nw * 64;
        if (MODE == kGateUp) {
            const int8_t* base = p.w + ((int64_t)u.e * 2 * p.f + u.group * 16 + g8) * K + 16 * c + kz;
            pw[0] = base;
            pw[1] = base + 8 * K;
            pw[NMAT] = base + p.f * K;
            pw[NMAT + 1] = base + p.f * K + 8 * K;
        } else {
            const int8_t* base = p.w + ((int64_t)u.e * p.d + u.group * 16 + g8) * K + 16 * c + kz;
            pw[0] = base;
            pw[1] = base + 8 * K;
        }
        const int b0 = s_off[u.e] + u.pass * 8 * NCH;
        const int cp = min(8 * NCH, s_off[u.e + 1] - b0);
#pragma unroll
        for (int n = 0; n < NCH; ++n) {
            const int slot = n * 8 + g8;
            if (slot < cp) {
                const int64_t row = MODE == kGateUp ? (int64_t)(p.perm[b0 + slot] / p.top_k)
                                                    : (int64_t)(b0 + slot);
                pb[n] = p.b_src + row * K + 16 * c + kz;
            } else {
                pb[n] = nullptr;
            }
        }
    };
    // each thread copies (cp.async) exactly the pieces it will later read, so
    // the shared ring needs no synchronisation beyond the thread's own waits
    auto issue = [&](int slot) {
        uint4* dst = ring + slot * kPieces * 32;
#pragma unroll
        for (int m = 0; m < 2 * NMAT; ++m) {
            cp_async_16(dst + m * 32, pw[m], 16);
            pw[m] += 64;
        }
#pragma unroll
        for (int n = 0; n < NCH; ++n) {
            const uint16_t* src = pb[n] ? pb[n] : p.b_src;
            const uint32_t bytes = pb[n] ? 16u : 0u;
            cp_async_16(dst + (2 * NMAT + 2 * n) * 32, src, bytes);
            cp_async_16(dst + (2 * NMAT + 2 * n + 1) * 32, src + 8, bytes);
            if (pb[n]) pb[n] += 64;
        }
        if (++pj == nw) {
            pj = 0;
            if (++pi < n_mine) set_prefetch_item(pi);
        }
    };
    set_prefetch_item(0);
#pragma unroll
    for (int q = 0; q < kDepth - 1; ++q) {
        if (q < total) issue(q);
        cp_async_commit();
    }

    // ---- consumer state
    float acc[NCH][NMAT][2][4];
#pragma unroll
    for (int n = 0; n < NCH; ++n)
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[n][m][0][i] = acc[n][m][1][i] = 0.0f;
    Item cu{};
    int base = 0, cnt_pass = 0;
    int ci = 0, cj = 0;
    auto set_consumer_item = [&](int it) {
        cu = item_of(it);
        base = s_off[cu.e] + cu.pass * 8 * NCH;
        cnt_pass = min(8 * NCH, s_off[cu.e + 1] - base);
    };
    set_consumer_item(0);

    int cslot = 0, pslot = kDepth - 1;  // consumed slot, next slot to fill
    for (int64_t q = 0; q < total; ++q) {
        {
            if (q + kDepth - 1 < total) issue(pslot);
            pslot = pslot == kDepth - 1 ? 0 : pslot + 1;
            cp_async_commit();  // one group per step, empty ones included
            cp_async_wait<kDepth - 1>();  // step q has landed
            const uint4* src = ring + cslot * kPieces * 32;
            cslot = cslot == kDepth - 1 ? 0 : cslot + 1;
            uint4 wq[2 * NMAT];
#pragma unroll
            for (int m = 0; m < 2 * NMAT; ++m) wq[m] = src[m * 32];
#pragma unroll
            for (int n = 0; n < NCH; ++n) {
                if (n * 8 < cnt_pass) {
                    const uint4 b0 = src[(2 * NMAT + 2 * n) * 32];
                    const uint4 b1 = src[(2 * NMAT + 2 * n + 1) * 32];
                    const uint32_t b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                    mma_block(acc[n][0], wq[0], wq[1], b);
                    if (MODE == kGateUp) mma_block(acc[n][NMAT - 1], wq[2], wq[3], b);
                }
            }
                if (++cj == nw) {
                    // end of item: raw partial sums -> P[z][slot][col]
                    const int64_t cols = MODE == kGateUp ? 2 * p.f : p.d;
                    float* P = p.P + (int64_t)cu.z * p.A * cols;
#pragma unroll
                    for (int n = 0; n < NCH; ++n)
#pragma unroll
                        for (int m = 0; m < NMAT; ++m)
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int slot = n * 8 + 2 * c + (i & 1);
                                const int64_t col = (int64_t)m * p.f + cu.group * 16 + g8 + (i >> 1) * 8;
                                if (slot < cnt_pass)
                                    P[(int64_t)(base + slot) * cols + col] = acc[n][m][0][i] + acc[n][m][1][i];
                                acc[n][m][0][i] = acc[n][m][1][i] = 0.0f;
                            }
                    cj = 0;
                    if (++ci < n_mine) set_consumer_item(ci);
                }
        }
    }
    cp_async_wait<0>();
}

// Expert of a grouped slot (offsets[e] <= slot < offsets[e+1]).
__device__ __forceinline__ int expert_of_slot(const int* off, int E, int slot) {
    int e = 0;
    while (e + 1 < E && off[e + 1] <= slot) ++e;
    return e;
}

// H[slot][n] = bf16( silu(s_g * sum_z Pg) * (s_u * sum_z Pu) ), pieces in order.
__global__ void __launch_bounds__(256)
    k_swiglu(const float* __restrict__ P, int S, int64_t A, int64_t f, int E,
             const int32_t* __restrict__ offsets, const float* __restrict__ sgu,
             uint16_t* __restrict__ H) {
    __shared__ int s_off[kMaxE + 1];
    if (threadIdx.x <= E) s_off[threadIdx.x] = offsets[threadIdx.x];
    __syncthreads();
    const int64_t total = (int64_t)s_off[E] * f;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < total;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int slot = (int)(v / f);
        const int64_t n = v % f;
        const int e = expert_of_slot(s_off, E, slot);
        float vg = 0.f, vu = 0.f;
        for (int z = 0; z < S; ++z) {
            const float* row = P + ((int64_t)z * A + slot) * 2 * f;
            vg += row[n];
            vu += row[f + n];
        }
        const float* s = sgu + (int64_t)e * 2 * f;
        H[(int64_t)slot * f + n] =
            __bfloat16_as_ushort(__float2bfloat16_rn(silu_f32(s[n] * vg) * (s[f + n] * vu)));
    }
}

// out[t][m] = bf16( sum_j g_tj * (s_d[e_j][m] * sum_z P[z][inv[a]][m]) ), a = t*top_k + j.
__global__ void __launch_bounds__(256)
    k_combine(const float* __restrict__ P, int S, int64_t A, int64_t T, int64_t d, int top_k,
              int E, const int32_t* __restrict__ ids, const float* __restrict__ gates,
              const int32_t* __restrict__ inv, const float* __restrict__ sd,
              uint16_t* __restrict__ out) {
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
            for (int z = 0; z < S; ++z) {
                const float4 q = *reinterpret_cast<const float4*>(P + ((int64_t)z * A + slot) * d + m);
                y[0] += q.x; y[1] += q.y; y[2] += q.z; y[3] += q.w;
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

int grid_for(int64_t work, int num_sms, int per_sm) {
    int64_t blocks = (work + 255) / 256;
    const int64_t cap = (int64_t)num_sms * per_sm;
    if (blocks > cap) blocks = cap;
    return (int)(blocks < 1 ? 1 : blocks);
}

// One full wave: the resident CTAs per SM at the kernel's register use.
template <int MODE, int NCH>
int gemv_grid(int num_sms) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gemv<MODE, NCH>,
                                                      kWarpsPerBlock * 32,
                                                      gemv_smem<MODE, NCH>()) != cudaSuccess ||
        per_sm < 1)
        per_sm = 2;
    return num_sms * per_sm;
}

template <int MODE, int NCH>
cudaError_t set_gemv_smem() {
    return cudaFuncSetAttribute(k_gemv<MODE, NCH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                gemv_smem<MODE, NCH>());
}

template <int NCH>
cudaError_t launch_decode_nch(const DecodeArgs& a, cudaStream_t stream) {
    cudaError_t err = set_gemv_smem<kGateUp, NCH>();
    if (err == cudaSuccess) err = set_gemv_smem<kDown, NCH>();
    if (err != cudaSuccess) return err;
    const int grid = gemv_grid<kGateUp, NCH>(a.num_sms);
    GemvParams p{};
    p.E = a.E;
    p.top_k = a.top_k;
    p.d = a.d;
    p.f = a.f;
    p.A = a.A;
    p.offsets = a.offsets;
    p.perm = a.perm;
    p.w = a.wgu;
    p.S = a.split_gu;
    p.b_src = static_cast<const uint16_t*>(a.x);
    p.P = a.P_gu;
    if (a.mark) a.mark(2, false, stream);
    k_gemv<kGateUp, NCH><<<grid, kWarpsPerBlock * 32, gemv_smem<kGateUp, NCH>(), stream>>>(p);
    err = cudaGetLastError();
    if (err == cudaSuccess)
        k_swiglu<<<grid_for(a.A * a.f, a.num_sms, 8), 256, 0, stream>>>(
            a.P_gu, a.split_gu, a.A, a.f, a.E, a.offsets, a.sgu, static_cast<uint16_t*>(a.H));
    if (a.mark) a.mark(2, true, stream);
    if (err != cudaSuccess) return err;
    p.w = a.wd;
    p.S = a.split_d;
    p.b_src = static_cast<const uint16_t*>(a.H);
    p.P = a.P_d;
    if (a.mark) a.mark(3, false, stream);
    k_gemv<kDown, NCH><<<gemv_grid<kDown, NCH>(a.num_sms), kWarpsPerBlock * 32,
                         gemv_smem<kDown, NCH>(), stream>>>(p);
    if (a.mark) a.mark(3, true, stream);
    return cudaGetLastError();
}

}  // namespace

int decode_split(int64_t K, int64_t want, int64_t cap) {
    const int64_t steps = K / 64;
    if (cap < 1) cap = 1;
    int64_t best_below = 1;
    for (int64_t s = 1; s <= steps && s <= cap; ++s) {
        if (steps % s != 0 || steps / s < 8) continue;
        if (s >= want) return (int)s;
        best_below = s;
    }
    return (int)best_below;
}

cudaError_t launch_finalize(const float* Y, int64_t T, int64_t d, int top_k, int E,
                            const int32_t* ids, void* out, int num_sms, cudaStream_t stream) {
    k_finalize<<<grid_for(T * (d / 4), num_sms, 8), 256, 0, stream>>>(
        Y, T, d, top_k, E, ids, static_cast<uint16_t*>(out));
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    if (a.T == 0) return cudaSuccess;
    cudaError_t err = a.max_per_expert <= 8 ? launch_decode_nch<1>(a, stream)
                                            : launch_decode_nch<2>(a, stream);
    if (err != cudaSuccess) return err;
    if (a.mark) a.mark(4, false, stream);
    k_combine<<<grid_for(a.T * (a.d / 4), a.num_sms, 8), 256, 0, stream>>>(
        a.P_d, a.split_d, a.A, a.T, a.d, a.top_k, a.E, a.ids, a.gates, a.inv, a.sd,
        static_cast<uint16_t*>(a.out));
    if (a.mark) a.mark(4, true, stream);
    return cudaGetLastError();
}

}  // namespace jmoe
