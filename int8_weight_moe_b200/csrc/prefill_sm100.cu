// Tensor-core path of the expert MLPs (many tokens per expert): a persistent
// grouped GEMM on the 5th-generation tensor cores (tcgen05, accumulators in
// TMEM), with the ExpertsInt8 dequantisation inside the kernel.
//
// "Jamba-1.5: Hybrid Transformer-Mamba Models at Scale" (paper summary),
// section "ExpertsInt8 Quantization (Section 3.1)", step 3: the INT8 weights
// are turned back into BF16 inside the fused MoE kernel as they move from HBM
// to on-chip memory, by a scaling and a cast.  Here: TMA brings each INT8
// weight tile HBM -> shared memory (1 byte per weight), converter warps turn
// it exactly into BF16 in the 128-byte-swizzled K-major layout the tensor core
// reads, and the per-output-channel scale is applied once in the epilogue
// (sum_k x_k (q_k s) = s sum_k x_k q_k).  Activations stay BF16 (step 4);
// accumulation is fp32 in TMEM.
//
// One CTA per SM, 16 warps:
//   warp 0      TMA producer of the activation tile A [256 rows x 64 k] bf16
//               (two 128-row boxes; the second is skipped when the expert ends)
//   warp 1      TMEM allocator and MMA issuer of the first 128-row half
//   warp 2      TMA producer of the INT8 weight tile [128 rows x 64 k]
//   warps 3-10  converters INT8 -> BF16 (shared -> shared, swizzled)
//   warps 11-14 epilogue: TMEM -> registers -> scale / SwiGLU / gate -> HBM
//   warp 15     MMA issuer of the second 128-row half
// Two issuing threads, one per half (each with its own accumulator, so the
// order of every accumulation stays fixed): a thread that waits on an
// mbarrier stops issuing until the MMAs it already queued have been
// dispatched, and the tensor pipe would idle through every such wait if one
// thread issued everything; with two, the other thread's MMAs fill it.
// Rings: A + converted B share 3 stages (48 KB each); the INT8 tiles, which
// come from HBM, have 8 stages (8 KB each) to cover its latency.  Each weight tile, once converted, feeds two M = 128
// MMAs (256 token rows), which halves the conversion work per multiply-add
// compared with one 128-row MMA.  Two accumulators of 2 x 128 x 128 fp32
// (512 TMEM columns) let the epilogue of one tile overlap the main loop of
// the next.
//
// Tiles: 256 expert-grouped rows (each expert's rows are padded to a
// multiple of 128, so a tile never mixes experts; its second half may be
// absent) x 128 MMA columns.  Gate/up mode: the 128 columns are 64 gate
// channels and the same 64 up channels, so the SwiGLU pairs sit in one
// thread.  Down mode: 128 output channels; the epilogue multiplies by the
// routing gate and writes one fp32 row per token->expert assignment.  Tiles
// are visited expert by expert in groups of 16 m-tiles (see decode_tile).
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "prefill.h"
#include "sm100.cuh"

namespace jmoe {
namespace {

using namespace sm100;

constexpr int BH = 128;       // rows of one MMA (a "half" of the tile)
constexpr int BM = 2 * BH;    // token rows per tile: two MMAs share one weight tile
constexpr int BN = 128, BK = 64;
constexpr int kStagesAB = 3, kStages8 = 8;
constexpr int kGroupM = 16;  // m-tiles per raster group (activation rows kept in L2)
constexpr int kHalfBytes = BH * BK * 2;  // 16 KB
constexpr int kABytes = 2 * kHalfBytes;  // 32 KB
constexpr int kBbfBytes = BN * BK * 2;   // 16 KB
constexpr int kB8Bytes = BN * BK;        // 8 KB
constexpr int kABStage = kABytes + kBbfBytes;
constexpr int kSmemAB = kStagesAB * kABStage;
constexpr int kSmem8 = kStages8 * kB8Bytes;
constexpr uint32_t kTmemCols = 512;   // 2 buffers x 2 halves x 128 fp32 columns
constexpr uint32_t kIdesc = idesc_bf16_f32(BH, BN);

constexpr int kWarpProdA = 0, kWarpMMA = 1, kWarpProdB = 2;
constexpr int kConvWarp0 = 3, kConvWarps = 8;
constexpr int kEpiWarp0 = kConvWarp0 + kConvWarps, kEpiWarps = 4;
constexpr int kWarpMMA2 = kEpiWarp0 + kEpiWarps;
constexpr int kThreads = (kWarpMMA2 + 1) * 32;
constexpr int kIssuers = 2;  // MMA-issuing threads (one per 128-row half)
constexpr int kMaxE = 64;

enum Mode { kGateUp = 0, kDown = 1 };

struct GemmParams {
    int E;
    int K;                // contraction length (d_model or d_ff)
    int n_valid;          // valid output channels (d_ff or d_model)
    int n_tiles;          // N tiles per expert
    int w_rows;           // weight rows per expert (2 d_ff or d_model)
    int up_offset;        // d_ff (gate/up mode)
    const int32_t* poff;  // [E+1] padded row offsets
    const int32_t* off;   // [E+1] assignment offsets
    const int32_t* perm;  // [A]
    const float* scale;   // [E][w_rows]
    const float* gates;   // [A]
    uint16_t* H;          // gate/up output, bf16 [rows_padded][d_ff]
    float* Y;             // down output, fp32 [A][d_model]
    unsigned* err;
};

struct Shared {
    uint64_t ab_full[kStagesAB], ab_empty[kStagesAB];
    uint64_t b8_full[kStages8], b8_empty[kStages8];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int poff[kMaxE + 1];
    int off[kMaxE + 1];
    int tile_start[kMaxE + 1];
};

constexpr int kSmemBytes = kSmemAB + kSmem8 + (int)sizeof(Shared) + 1024;

struct Tile {
    int e, row0, n, halves;  // halves: 1 or 2 valid 128-row halves
};

// Tile order inside an expert: groups of kGroupM m-tiles; within a group all
// n-tiles, m fastest.  The CTAs of a wave then share a few weight tiles and
// at most kGroupM x 256 activation rows, which stay in L2.
__device__ __forceinline__ Tile decode_tile(const Shared& s, int E, int n_tiles, int tile) {
    int e = 0;
    while (e + 1 < E && s.tile_start[e + 1] <= tile) ++e;
    const int local = tile - s.tile_start[e];
    const int nh = (s.poff[e + 1] - s.poff[e]) / BH;  // 128-row halves of this expert
    const int mt = (nh + 1) / 2;
    const int mg = local / (kGroupM * n_tiles);
    const int gm = min(kGroupM, mt - mg * kGroupM);  // m-tiles in this group
    const int rem = local - mg * kGroupM * n_tiles;
    Tile t;
    t.e = e;
    t.n = rem / gm;
    const int m = mg * kGroupM + rem % gm;
    t.row0 = s.poff[e] + m * BM;
    t.halves = min(2, nh - 2 * m);
    return t;
}

// Bounded wait that ignores the abort flag (used only while draining).
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitCycles) return;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Shared& S = *reinterpret_cast<Shared*>(smem + kSmemAB + kSmem8);
    auto tileA = [&](int s) { return smem + s * kABStage; };
    auto tileBbf = [&](int s) { return smem + s * kABStage + kABytes; };
    auto tileB8 = [&](int s) { return smem + kSmemAB + s * kB8Bytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int KB = p.K / BK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStagesAB; ++i) {
            // the A producer's expect-tx arrival (plus the TMA bytes) and the
            // converter warps' arrivals
            mbar_init(&S.ab_full[i], 1 + kConvWarps);
            mbar_init(&S.ab_empty[i], kIssuers);
        }
        for (int i = 0; i < kStages8; ++i) {
            mbar_init(&S.b8_full[i], 1);
            mbar_init(&S.b8_empty[i], kConvWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.acc_full[i], kIssuers);
            mbar_init(&S.acc_empty[i], kEpiWarps);
        }
        mbar_init(&S.drain, kIssuers);
        S.abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x <= E) {
        S.poff[threadIdx.x] = p.poff[threadIdx.x];
        S.off[threadIdx.x] = p.off[threadIdx.x];
    }
    if (warp == kWarpProdA && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            S.tile_start[e] = run;
            run += ((S.poff[e + 1] - S.poff[e]) / BH + 1) / 2 * p.n_tiles;
        }
        S.tile_start[E] = run;
    }
    if (warp == kWarpMMA) {
        tmem_alloc(&S.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const int total = S.tile_start[E];
    volatile int* abort = &S.abort;

    if (warp == kWarpProdA) {
        if (lane == 0) {
            uint32_t g = 0;
            for (int tile = blockIdx.x; tile < total && !*abort; tile += gridDim.x) {
                const Tile t = decode_tile(S, E, p.n_tiles, tile);
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int s = g % kStagesAB;
                    const uint32_t ph = (g / kStagesAB) & 1;
                    if (!mbar_wait(&S.ab_empty[s], ph ^ 1, abort)) break;
                    mbar_arrive_expect_tx(&S.ab_full[s], t.halves * kHalfBytes);
                    tma_load_2d(tileA(s), &tmA, &S.ab_full[s], kb * BK, t.row0);
                    if (t.halves == 2)
                        tma_load_2d(tileA(s) + kHalfBytes, &tmA, &S.ab_full[s], kb * BK,
                                    t.row0 + BH);
                }
            }
            // make sure no copy is still landing in shared memory when the CTA exits
            for (uint32_t h = (g > (uint32_t)kStagesAB ? g - kStagesAB : 0); h < g; ++h)
                wait_drain(&S.ab_full[h % kStagesAB], (h / kStagesAB) & 1);
        }
    } else if (warp == kWarpProdB) {
        if (lane == 0) {
            uint32_t g = 0;
            for (int tile = blockIdx.x; tile < total && !*abort; tile += gridDim.x) {
                const Tile t = decode_tile(S, E, p.n_tiles, tile);
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int s = g % kStages8;
                    const uint32_t ph = (g / kStages8) & 1;
                    if (!mbar_wait(&S.b8_empty[s], ph ^ 1, abort)) break;
                    mbar_arrive_expect_tx(&S.b8_full[s], kB8Bytes);
                    if (MODE == kGateUp) {
                        const int y = t.e * p.w_rows + t.n * (BN / 2);
                        tma_load_2d(tileB8(s), &tmB, &S.b8_full[s], kb * BK, y);
                        tma_load_2d(tileB8(s) + kB8Bytes / 2, &tmB, &S.b8_full[s], kb * BK,
                                    y + p.up_offset);
                    } else {
                        tma_load_2d(tileB8(s), &tmB, &S.b8_full[s], kb * BK,
                                    t.e * p.w_rows + t.n * BN);
                    }
                }
            }
            for (uint32_t h = (g > (uint32_t)kStages8 ? g - kStages8 : 0); h < g; ++h)
                wait_drain(&S.b8_full[h % kStages8], (h / kStages8) & 1);
        }
    } else if (warp == kWarpMMA || warp == kWarpMMA2) {
        if (lane == 0) {
            const int h = warp == kWarpMMA ? 0 : 1;  // the 128-row half this thread issues
            uint32_t g = 0;
            int it = 0;
            for (int tile = blockIdx.x; tile < total && !*abort; tile += gridDim.x, ++it) {
                const bool active = h < decode_tile(S, E, p.n_tiles, tile).halves;
                const int buf = it & 1;
                if (!mbar_wait(&S.acc_empty[buf], ((it >> 1) & 1) ^ 1, abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + buf * 2 * BN + h * BN;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int s = g % kStagesAB;
                    const uint32_t ph = (g / kStagesAB) & 1;
                    if (!mbar_wait(&S.ab_full[s], ph, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (active) {
                        const uint32_t a0 = smem_u32(tileA(s)) + h * kHalfBytes;
                        const uint32_t b0 = smem_u32(tileBbf(s));
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            mma_bf16_ss(d_tmem, desc_sw128(a0 + kk * 32), desc_sw128(b0 + kk * 32),
                                        kIdesc, (kb | kk) != 0);
                    }
                    mma_commit(&S.ab_empty[s]);
                }
                if (!ok) break;
                mma_commit(&S.acc_full[buf]);
            }
            mma_commit(&S.drain);
            wait_drain(&S.drain, 0);
        }
    } else if (warp >= kConvWarp0 && warp < kConvWarp0 + kConvWarps) {
        // Thread ct converts the 16-byte int8 chunks q = ct and ct + 256 of the
        // tile (row q / 4, bytes 16 (q % 4) .. +16): both loads are issued
        // before any conversion, and each chunk becomes two 16-byte bf16 units
        // 2 (q % 4) and 2 (q % 4) + 1 of the row's 128-byte swizzled line.
        const int ct = threadIdx.x - kConvWarp0 * 32;  // 0..255
        uint32_t g = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok && !*abort; tile += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb, ++g) {
                const int s = g % kStagesAB;
                const uint32_t ph = (g / kStagesAB) & 1;
                const int s8 = g % kStages8;
                const uint32_t ph8 = (g / kStages8) & 1;
                if (!mbar_wait(&S.b8_full[s8], ph8, abort) ||
                    !mbar_wait(&S.ab_empty[s], ph ^ 1, abort)) {
                    ok = false;
                    break;
                }
                const uint8_t* src = tileB8(s8);
                uint8_t* dst = tileBbf(s);
                uint4 v[2];
#pragma unroll
                for (int j = 0; j < 2; ++j)
                    v[j] = *reinterpret_cast<const uint4*>(src + (ct + 256 * j) * 16);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int q = ct + 256 * j, row = q >> 2, u0 = 2 * (q & 3);
                    uint8_t* line = dst + (row >> 3) * 1024 + (row & 7) * 128;
                    const uint4 o0 = make_uint4(i8x2_to_bf16x2<0>(v[j].x), i8x2_to_bf16x2<1>(v[j].x),
                                                i8x2_to_bf16x2<0>(v[j].y), i8x2_to_bf16x2<1>(v[j].y));
                    const uint4 o1 = make_uint4(i8x2_to_bf16x2<0>(v[j].z), i8x2_to_bf16x2<1>(v[j].z),
                                                i8x2_to_bf16x2<0>(v[j].w), i8x2_to_bf16x2<1>(v[j].w));
                    *reinterpret_cast<uint4*>(line + ((u0 ^ (row & 7)) << 4)) = o0;
                    *reinterpret_cast<uint4*>(line + (((u0 + 1) ^ (row & 7)) << 4)) = o1;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&S.ab_full[s]);
                    mbar_arrive(&S.b8_empty[s8]);
                }
            }
        }
    } else {
        // epilogue warps: TMEM lane quadrant = warp % 4, both halves of the tile
        const int quad = warp & 3;
        int it = 0;
        for (int tile = blockIdx.x; tile < total && !*abort; tile += gridDim.x, ++it) {
            const Tile t = decode_tile(S, E, p.n_tiles, tile);
            const int buf = it & 1;
            if (!mbar_wait(&S.acc_full[buf], (it >> 1) & 1, abort)) break;
            tc_fence_after();
            __syncwarp();
            for (int h = 0; h < t.halves; ++h) {
                const uint32_t taddr =
                    tmem + buf * 2 * BN + h * BN + ((uint32_t)(quad * 32) << 16);
                const int row = t.row0 + h * BH + quad * 32 + lane;
                if (MODE == kGateUp) {
                    const int n0 = t.n * (BN / 2);
                    const float* sg = p.scale + (size_t)t.e * p.w_rows + n0;
                    const float* su = sg + p.up_offset;
#pragma unroll 1
                    for (int c = 0; c < BN / 2 / 32; ++c) {
                        uint32_t gv[32], uv[32];
                        tmem_ld_32x32b_x32(taddr + c * 32, gv);
                        tmem_ld_32x32b_x32(taddr + BN / 2 + c * 32, uv);
                        tmem_ld_wait();
                        const int ch = n0 + c * 32;
                        if (ch < p.n_valid) {
                            uint32_t packed[16];
#pragma unroll
                            for (int j = 0; j < 32; j += 4) {
                                const float4 g4 = __ldg(reinterpret_cast<const float4*>(sg + c * 32 + j));
                                const float4 u4 = __ldg(reinterpret_cast<const float4*>(su + c * 32 + j));
                                const float g0 = g4.x * __uint_as_float(gv[j]);
                                const float g1 = g4.y * __uint_as_float(gv[j + 1]);
                                const float g2 = g4.z * __uint_as_float(gv[j + 2]);
                                const float g3 = g4.w * __uint_as_float(gv[j + 3]);
                                const float u0 = u4.x * __uint_as_float(uv[j]);
                                const float u1 = u4.y * __uint_as_float(uv[j + 1]);
                                const float u2 = u4.z * __uint_as_float(uv[j + 2]);
                                const float u3 = u4.w * __uint_as_float(uv[j + 3]);
                                packed[j / 2] = pack_bf16x2(silu_f32(g0) * u0, silu_f32(g1) * u1);
                                packed[j / 2 + 1] = pack_bf16x2(silu_f32(g2) * u2, silu_f32(g3) * u3);
                            }
                            uint4* dst = reinterpret_cast<uint4*>(p.H + (size_t)row * p.n_valid + ch);
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1],
                                                    packed[4 * q + 2], packed[4 * q + 3]);
                        }
                    }
                } else {
                    const int m0 = t.n * BN;
                    const int r = row - S.poff[t.e];
                    const bool valid = r < S.off[t.e + 1] - S.off[t.e];
                    const int a = valid ? p.perm[S.off[t.e] + r] : 0;
                    const float gate = valid ? p.gates[a] : 0.0f;
                    const float* sd = p.scale + (size_t)t.e * p.w_rows;
#pragma unroll 1
                    for (int c = 0; c < BN / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(taddr + c * 32, v);
                        tmem_ld_wait();
                        const int m = m0 + c * 32;
                        if (valid && m < p.n_valid) {
                            float4* dst = reinterpret_cast<float4*>(p.Y + (size_t)a * p.n_valid + m);
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float4 s4 = __ldg(reinterpret_cast<const float4*>(sd + m) + q);
                                float4 o;
                                o.x = gate * (s4.x * __uint_as_float(v[4 * q]));
                                o.y = gate * (s4.y * __uint_as_float(v[4 * q + 1]));
                                o.z = gate * (s4.z * __uint_as_float(v[4 * q + 2]));
                                o.w = gate * (s4.w * __uint_as_float(v[4 * q + 3]));
                                dst[q] = o;
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.acc_empty[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && S.abort) flag_error(p.err, kErrTimeout);
    if (warp == kWarpMMA) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ----------------------------------------------------------------------------- host side

template <int MODE>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p,
                        int num_sms, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    k_grouped_gemm<MODE><<<num_sms, kThreads, kSmemBytes, stream>>>(a, b, p);
    note_launch();
    return cudaGetLastError();
}

}  // namespace

bool prefill_available() { return tensormap_available(); }

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
    if (a.T == 0) return cudaSuccess;
    if (a.d > INT32_MAX / 2 || a.f > INT32_MAX / 2 || a.rows_padded > INT32_MAX)
        return cudaErrorInvalidValue;
    cudaError_t err;
    // 1. gather the routed activation rows, grouped by expert, padded per expert
    if (a.mark) a.mark(1, false, stream);
    err = launch_gather_rows(a.x, a.d, a.top_k, a.E, a.offsets, a.padded_offsets, a.perm,
                             a.rows_padded, a.xperm, a.num_sms, stream);
    if (a.mark) a.mark(1, true, stream);
    if (err != cudaSuccess) return err;

    CUtensorMap mA1, mB1, mA2, mB2;
    const bool ok =
        encode_2d(&mA1, a.xperm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.rows_padded, a.d, BH, BK,
                 CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_2d(&mB1, a.wgu, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.E * 2 * a.f, a.d,
                 BN / 2, BK, CU_TENSOR_MAP_SWIZZLE_NONE) &&
        encode_2d(&mA2, a.H, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.rows_padded, a.f, BH, BK,
                 CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_2d(&mB2, a.wd, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.E * a.d, a.f, BN, BK,
                 CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;

    // 2. gate/up GEMM + SwiGLU -> H (bf16, grouped rows)
    GemmParams g1{};
    g1.E = a.E;
    g1.K = (int)a.d;
    g1.n_valid = (int)a.f;
    g1.n_tiles = (int)((a.f + BN / 2 - 1) / (BN / 2));
    g1.w_rows = (int)(2 * a.f);
    g1.up_offset = (int)a.f;
    g1.poff = a.padded_offsets;
    g1.off = a.offsets;
    g1.perm = a.perm;
    g1.scale = a.sgu;
    g1.gates = a.gates;
    g1.H = static_cast<uint16_t*>(a.H);
    g1.err = a.err;
    if (a.mark) a.mark(2, false, stream);
    err = launch_gemm<kGateUp>(mA1, mB1, g1, a.num_sms, stream);
    if (a.mark) a.mark(2, true, stream);
    if (err != cudaSuccess) return err;

    // 3. down GEMM, scale and routing gate -> Y (fp32, one row per assignment)
    GemmParams g2 = g1;
    g2.K = (int)a.f;
    g2.n_valid = (int)a.d;
    g2.n_tiles = (int)((a.d + BN - 1) / BN);
    g2.w_rows = (int)a.d;
    g2.up_offset = 0;
    g2.scale = a.sd;
    g2.H = nullptr;
    g2.Y = a.Yg;
    if (a.mark) a.mark(3, false, stream);
    err = launch_gemm<kDown>(mA2, mB2, g2, a.num_sms, stream);
    if (a.mark) a.mark(3, true, stream);
    if (err != cudaSuccess) return err;

    // 4. out[t] = bf16(sum over the token's assignments)
    if (a.mark) a.mark(4, false, stream);
    err = launch_finalize(a.Yg, a.T, a.d, a.top_k, a.E, a.ids, a.out, a.num_sms, stream);
    if (a.mark) a.mark(4, true, stream);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace jmoe
