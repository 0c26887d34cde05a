// Tensor-core path of the expert MLPs (many tokens per expert): a persistent
// grouped GEMM on the 5th-generation tensor cores (tcgen05, accumulators in
// TMEM), with the ExpertsInt8 dequantisation inside the kernel.
//
// "Jamba-1.5: Hybrid Transformer-Mamba Models at Scale" (paper summary),
// section "ExpertsInt8 Quantization (Section 3.1)", step 3: the INT8 weights
// are turned back into BF16 inside the fused MoE kernel as they move from HBM
// to on-chip memory, by a scaling and a cast.  Here: TMA brings each INT8
// weight tile HBM -> shared memory (1 byte per weight), converter warps turn
// it exactly into BF16 and store it straight into tensor memory, where the
// tensor core reads it as the A operand; the per-output-channel scale is
// applied once in the epilogue (sum_k x_k (q_k s) = s sum_k x_k q_k).
// Activations stay BF16 (step 4) and are the B operand, from shared memory;
// accumulation is fp32 in TMEM.
//
// The product is computed transposed, D[channel][token] = W[channel][k] *
// X[token][k]: M = 128 weight rows (output channels), N = up to 192 token
// rows, K in steps of 64.  Keeping the converted weights in tensor memory
// takes them off the shared-memory path entirely (no bf16 tile written and
// read back there), which was what bounded the multiply rate.
//
// One CTA per SM, 16 warps:
//   warp 0      TMA producer of the activation tile X [192 rows x 64 k] bf16
//               (three 64-row boxes; trailing boxes skipped when the expert ends)
//   warp 1      TMEM allocator and MMA issuer of tokens 0..95 of the tile
//   warp 2      TMA producer of the INT8 weight tile [128 rows x 64 k]
//   warps 3-10  converters INT8 -> BF16 (shared -> tensor memory): two groups
//               of four (one warp per TMEM lane quadrant) that take the
//               k-steps in turn, so each group has two MMA periods for one
//               conversion and its wait for the tensor-memory stores
//   warps 11-14 epilogue: TMEM -> registers -> scale / SwiGLU / gate -> HBM
//   warp 15     MMA issuer of tokens 96..191
// Two issuing threads, each with its own accumulator (so the order of every
// accumulation stays fixed): a thread that waits on an mbarrier stops issuing
// until the MMAs it already queued have been dispatched, and the tensor pipe
// would idle through every such wait if one thread issued everything.
// Tensor memory (512 columns): two accumulators of 192 fp32 columns (the
// epilogue of one tile overlaps the main loop of the next) and four stages of
// 32 columns for the converted weights (64 bf16 per row).  Shared memory: four
// activation stages (24 KB) paired with the four weight stages, and eight
// INT8 stages (8 KB) to cover the latency of HBM.
//
// Tiles: 192 expert-grouped token rows (each expert's rows are padded to a
// multiple of 128, so a tile never mixes experts and holds 64, 128 or 192 of
// them) x 128 weight rows.  Gate/up mode: the 128 rows are 64 gate channels
// and the same 64 up channels, arranged so that each TMEM lane quadrant holds
// 16 gate rows and their 16 up rows (lanes 0-15 and 16-31): the SwiGLU pairs
// meet with one warp shuffle.  Down mode: 128 output channels; the epilogue
// multiplies by the routing gate and writes one fp32 row per token->expert
// assignment.  Tiles are visited expert by expert in groups of 16 m-tiles.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "prefill.h"
#include "sm100.cuh"

namespace jmoe {
namespace {

using namespace sm100;

constexpr int BT = 192;       // token rows per tile (MMA N, split over two issuers)
constexpr int BTH = BT / 2;   // token rows per issuer
constexpr int BC = 128;       // weight rows (output channels) per tile: MMA M
constexpr int BK = 64;
constexpr int kXBox = 64;     // token rows per activation TMA box
constexpr int kStages = 4, kStages8 = 8;
constexpr int kGroupM = 16;   // m-tiles per raster group (activation rows kept in L2)
constexpr int kXBytes = BT * BK * 2;     // 24 KB
constexpr int kXBoxBytes = kXBox * BK * 2;
constexpr int kB8Bytes = BC * BK;        // 8 KB
constexpr int kSmemX = kStages * kXBytes;
constexpr int kSmem8 = kStages8 * kB8Bytes;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 2 * BT;    // two accumulators
constexpr uint32_t kACols = BK / 2;      // one converted k-tile: 64 bf16 per lane
static_assert(kAccCols + kStages * kACols <= kTmemCols, "tensor memory budget");

constexpr int kWarpProdX = 0, kWarpMMA = 1, kWarpProdW = 2;
constexpr int kConvWarp0 = 3, kConvWarps = 8;
constexpr int kConvGroups = 2, kConvPerStep = kConvWarps / kConvGroups;
constexpr int kEpiWarp0 = kConvWarp0 + kConvWarps, kEpiWarps = 4;
constexpr int kWarpMMA2 = kEpiWarp0 + kEpiWarps;
constexpr int kThreads = (kWarpMMA2 + 1) * 32;
constexpr int kIssuers = 2;
constexpr int kMaxE = 64;

enum Mode { kGateUp = 0, kDown = 1 };

struct GemmParams {
    int E;
    int K;                // contraction length (d_model or d_ff)
    int n_valid;          // valid output channels (d_ff or d_model)
    int n_tiles;          // channel tiles per expert
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
    uint64_t full[kStages], empty[kStages];
    uint64_t b8_full[kStages8], b8_empty[kStages8];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int poff[kMaxE + 1];
    int off[kMaxE + 1];
    int tile_start[kMaxE + 1];
};

constexpr int kSmemBytes = kSmemX + kSmem8 + (int)sizeof(Shared) + 1024;

struct Tile {
    int e, row0, n, rows;  // rows: valid token rows of the tile (64, 128 or 192)
};

// Tile order inside an expert: groups of kGroupM m-tiles; within a group all
// channel tiles, m fastest.  The CTAs of a wave then share a few weight tiles
// and at most kGroupM x 192 activation rows, which stay in L2.
__device__ __forceinline__ Tile decode_tile(const Shared& s, int E, int n_tiles, int tile) {
    int e = 0;
    while (e + 1 < E && s.tile_start[e + 1] <= tile) ++e;
    const int local = tile - s.tile_start[e];
    const int rows_e = s.poff[e + 1] - s.poff[e];
    const int mt = (rows_e + BT - 1) / BT;
    const int mg = local / (kGroupM * n_tiles);
    const int gm = min(kGroupM, mt - mg * kGroupM);  // m-tiles in this group
    const int rem = local - mg * kGroupM * n_tiles;
    Tile t;
    t.e = e;
    t.n = rem / gm;
    const int m = mg * kGroupM + rem % gm;
    t.row0 = s.poff[e] + m * BT;
    t.rows = min(BT, rows_e - m * BT);
    return t;
}

// Token rows of issuer h in a tile with `rows` valid rows (0: nothing to do).
__device__ __forceinline__ int issuer_rows(int rows, int h) {
    return max(0, min(BTH, rows - h * BTH));
}

// Bounded wait that ignores the abort flag (used only while draining).
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitCycles) return;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                   const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Shared& S = *reinterpret_cast<Shared*>(smem + kSmemX + kSmem8);
    auto tileX = [&](int s) { return smem + s * kXBytes; };
    auto tileW8 = [&](int s) { return smem + kSmemX + s * kB8Bytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E;
    const int KB = p.K / BK;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            // the X producer's expect-tx arrival (plus the TMA bytes) and the
            // converter warps' arrivals (weights stored in tensor memory)
            mbar_init(&S.full[i], 1 + kConvPerStep);
            mbar_init(&S.empty[i], kIssuers);
        }
        for (int i = 0; i < kStages8; ++i) {
            mbar_init(&S.b8_full[i], 1);
            mbar_init(&S.b8_empty[i], kConvPerStep);
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
    if (warp == kWarpProdX && lane == 0) {
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            S.tile_start[e] = run;
            run += (S.poff[e + 1] - S.poff[e] + BT - 1) / BT * p.n_tiles;
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

    if (warp == kWarpProdX) {
        if (lane == 0) {
            uint32_t g = 0;
            for (int tile = blockIdx.x; tile < total && !*abort; tile += gridDim.x) {
                const Tile t = decode_tile(S, E, p.n_tiles, tile);
                const int boxes = t.rows / kXBox;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int s = g % kStages;
                    const uint32_t ph = (g / kStages) & 1;
                    if (!mbar_wait(&S.empty[s], ph ^ 1, abort)) break;
                    mbar_arrive_expect_tx(&S.full[s], boxes * kXBoxBytes);
                    for (int b = 0; b < boxes; ++b)
                        tma_load_2d(tileX(s) + b * kXBoxBytes, &tmX, &S.full[s], kb * BK,
                                    t.row0 + b * kXBox);
                }
            }
            // make sure no copy is still landing in shared memory when the CTA exits
            for (uint32_t h = (g > (uint32_t)kStages ? g - kStages : 0); h < g; ++h)
                wait_drain(&S.full[h % kStages], (h / kStages) & 1);
        }
    } else if (warp == kWarpProdW) {
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
                        // rows 0-63: gate channels, rows 64-127: the same up channels
                        const int y = t.e * p.w_rows + t.n * (BC / 2);
                        tma_load_2d(tileW8(s), &tmW, &S.b8_full[s], kb * BK, y);
                        tma_load_2d(tileW8(s) + kB8Bytes / 2, &tmW, &S.b8_full[s], kb * BK,
                                    y + p.up_offset);
                    } else {
                        tma_load_2d(tileW8(s), &tmW, &S.b8_full[s], kb * BK,
                                    t.e * p.w_rows + t.n * BC);
                    }
                }
            }
            for (uint32_t h = (g > (uint32_t)kStages8 ? g - kStages8 : 0); h < g; ++h)
                wait_drain(&S.b8_full[h % kStages8], (h / kStages8) & 1);
        }
    } else if (warp == kWarpMMA || warp == kWarpMMA2) {
        if (lane == 0) {
            const int h = warp == kWarpMMA ? 0 : 1;  // token rows [96 h, 96 h + 96) of the tile
            uint32_t g = 0;
            int it = 0;
            for (int tile = blockIdx.x; tile < total && !*abort; tile += gridDim.x, ++it) {
                const int nh = issuer_rows(decode_tile(S, E, p.n_tiles, tile).rows, h);
                const uint32_t idesc = idesc_bf16_f32(BC, nh > 0 ? nh : 16);
                const int buf = it & 1;
                if (!mbar_wait(&S.acc_empty[buf], ((it >> 1) & 1) ^ 1, abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + buf * BT + h * BTH;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int s = g % kStages;
                    const uint32_t ph = (g / kStages) & 1;
                    if (!mbar_wait(&S.full[s], ph, abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (nh > 0) {
                        const uint32_t a_tmem = tmem + kAccCols + s * kACols;
                        const uint32_t b0 = smem_u32(tileX(s)) + h * BTH * BK * 2;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            mma_bf16_ts(d_tmem, a_tmem + kk * 8, desc_sw128(b0 + kk * 32), idesc,
                                        (kb | kk) != 0);
                    }
                    mma_commit(&S.empty[s]);
                }
                if (!ok) break;
                mma_commit(&S.acc_full[buf]);
            }
            mma_commit(&S.drain);
            wait_drain(&S.drain, 0);
        }
    } else if (warp >= kConvWarp0 && warp < kConvWarp0 + kConvWarps) {
        // Thread = TMEM lane L = 32 quad + lane = one weight row of the tile;
        // group grp converts the k-steps g with g % 2 == grp.  The INT8 tile
        // arrives 64-byte swizzled (16-byte chunk c of row r at r*64 +
        // 16 (c ^ ((r >> 1) & 3))), so a warp's 16-byte reads of 32 rows are
        // free of bank conflicts.
        const int cw = warp - kConvWarp0;
        const int quad = warp & 3, grp = cw / kConvPerStep;
        int r;  // shared-memory row of this lane's weight row
        if (MODE == kGateUp)
            r = lane < 16 ? 16 * quad + lane : BC / 2 + 16 * quad + (lane - 16);
        else
            r = 32 * quad + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        uint32_t g = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok && !*abort; tile += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb, ++g) {
                if ((int)(g % kConvGroups) != grp) continue;
                const int s = g % kStages;
                const uint32_t ph = (g / kStages) & 1;
                const int s8 = g % kStages8;
                const uint32_t ph8 = (g / kStages8) & 1;
                if (!mbar_wait(&S.b8_full[s8], ph8, abort) ||
                    !mbar_wait(&S.empty[s], ph ^ 1, abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t* row = tileW8(s8) + r * BK;
                uint4 v[4];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    v[c] = *reinterpret_cast<const uint4*>(row + ((c ^ ((r >> 1) & 3)) << 4));
                uint32_t o[32];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    o[8 * c + 0] = i8x2_to_bf16x2<0>(v[c].x);
                    o[8 * c + 1] = i8x2_to_bf16x2<1>(v[c].x);
                    o[8 * c + 2] = i8x2_to_bf16x2<0>(v[c].y);
                    o[8 * c + 3] = i8x2_to_bf16x2<1>(v[c].y);
                    o[8 * c + 4] = i8x2_to_bf16x2<0>(v[c].z);
                    o[8 * c + 5] = i8x2_to_bf16x2<1>(v[c].z);
                    o[8 * c + 6] = i8x2_to_bf16x2<0>(v[c].w);
                    o[8 * c + 7] = i8x2_to_bf16x2<1>(v[c].w);
                }
                tmem_st_32x32b_x32(tmem + lane_addr + kAccCols + s * kACols, o);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&S.full[s]);
                    mbar_arrive(&S.b8_empty[s8]);
                }
            }
        }
    } else {
        // epilogue warps: TMEM lane quadrant = warp % 4; lane = weight row of
        // the tile, columns = token rows
        const int quad = warp & 3;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        int it = 0;
        for (int tile = blockIdx.x; tile < total && !*abort; tile += gridDim.x, ++it) {
            const Tile t = decode_tile(S, E, p.n_tiles, tile);
            const int buf = it & 1;
            if (!mbar_wait(&S.acc_full[buf], (it >> 1) & 1, abort)) break;
            tc_fence_after();
            __syncwarp();
            if (MODE == kGateUp) {
                // lanes 0-15: gate channel ch, lanes 16-31: up channel ch; after
                // one exchange the gate lane finishes tokens 0-15 of each
                // 32-token chunk and the up lane tokens 16-31
                const bool up = lane >= 16;
                const int ch = t.n * (BC / 2) + 16 * quad + (lane & 15);
                const float* sc = p.scale + (size_t)t.e * p.w_rows;
                const float sg = __ldg(sc + ch), su = __ldg(sc + p.up_offset + ch);
                for (int h = 0; h < kIssuers; ++h) {
                    const int nh = issuer_rows(t.rows, h);
#pragma unroll 1
                    for (int c = 0; c < nh / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(tmem + lane_addr + buf * BT + h * BTH + c * 32, v);
                        tmem_ld_wait();
                        const int tok0 = t.row0 + h * BTH + c * 32 + (up ? 16 : 0);
                        uint16_t* dst = p.H + (size_t)tok0 * p.n_valid + ch;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const uint32_t mine = up ? v[16 + j] : v[j];
                            const uint32_t other =
                                __shfl_xor_sync(0xffffffffu, up ? v[j] : v[16 + j], 16);
                            const float gv = sg * __uint_as_float(up ? other : mine);
                            const float uv = su * __uint_as_float(up ? mine : other);
                            dst[(size_t)j * p.n_valid] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(silu_f32(gv) * uv));
                        }
                    }
                }
            } else {
                const int m = t.n * BC + 32 * quad + lane;
                const bool m_ok = m < p.n_valid;
                const float sd = m_ok ? __ldg(p.scale + (size_t)t.e * p.w_rows + m) : 0.0f;
                const int cnt = S.off[t.e + 1] - S.off[t.e];
                const int r0 = t.row0 - S.poff[t.e];  // expert-local row of column 0
                for (int h = 0; h < kIssuers; ++h) {
                    const int nh = issuer_rows(t.rows, h);
#pragma unroll 1
                    for (int c = 0; c < nh / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(tmem + lane_addr + buf * BT + h * BTH + c * 32, v);
                        // lane j looks up the assignment and gate of token column j
                        const int rl = r0 + h * BTH + c * 32 + lane;
                        const bool tok_ok = rl < cnt;
                        const int a_l = tok_ok ? p.perm[S.off[t.e] + rl] : 0;
                        const float g_l = tok_ok ? p.gates[a_l] : 0.0f;
                        tmem_ld_wait();
                        const unsigned valid = __ballot_sync(0xffffffffu, tok_ok);
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int a = __shfl_sync(0xffffffffu, a_l, j);
                            const float gate = __shfl_sync(0xffffffffu, g_l, j);
                            if (((valid >> j) & 1u) && m_ok)
                                p.Y[(size_t)a * p.n_valid + m] = gate * (sd * __uint_as_float(v[j]));
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
cudaError_t launch_gemm(const CUtensorMap& x, const CUtensorMap& w, const GemmParams& p,
                        int num_sms, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    k_grouped_gemm<MODE><<<num_sms, kThreads, kSmemBytes, stream>>>(x, w, p);
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

    CUtensorMap mX1, mW1, mX2, mW2;
    const bool ok =
        encode_2d(&mX1, a.xperm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.rows_padded, a.d, kXBox,
                  BK, CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_2d(&mW1, a.wgu, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.E * 2 * a.f, a.d,
                  BC / 2, BK, CU_TENSOR_MAP_SWIZZLE_64B) &&
        encode_2d(&mX2, a.H, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.rows_padded, a.f, kXBox, BK,
                  CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_2d(&mW2, a.wd, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.E * a.d, a.f, BC, BK,
                  CU_TENSOR_MAP_SWIZZLE_64B);
    if (!ok) return cudaErrorInvalidValue;

    // 2. gate/up GEMM + SwiGLU -> H (bf16, grouped rows)
    GemmParams g1{};
    g1.E = a.E;
    g1.K = (int)a.d;
    g1.n_valid = (int)a.f;
    g1.n_tiles = (int)((a.f + BC / 2 - 1) / (BC / 2));
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
    err = launch_gemm<kGateUp>(mX1, mW1, g1, a.num_sms, stream);
    if (a.mark) a.mark(2, true, stream);
    if (err != cudaSuccess) return err;

    // 3. down GEMM, scale and routing gate -> Y (fp32, one row per assignment)
    GemmParams g2 = g1;
    g2.K = (int)a.f;
    g2.n_valid = (int)a.d;
    g2.n_tiles = (int)((a.d + BC - 1) / BC);
    g2.w_rows = (int)a.d;
    g2.up_offset = 0;
    g2.scale = a.sd;
    g2.H = nullptr;
    g2.Y = a.Yg;
    if (a.mark) a.mark(3, false, stream);
    err = launch_gemm<kDown>(mX2, mW2, g2, a.num_sms, stream);
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
