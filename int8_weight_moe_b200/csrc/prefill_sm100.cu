// Tensor-core path of the expert MLPs (many tokens per expert): a persistent
// grouped GEMM on the 5th-generation tensor cores (tcgen05, accumulators in
// TMEM), run by CTA pairs, with the ExpertsInt8 dequantisation inside the
// kernel.
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
// A cluster of two CTAs (a pair, on two SMs) computes one tile of 512 token
// rows x 256 output columns with CTA-pair MMAs (tcgen05.mma.cta_group::2,
// M = 256, N = 256, K = 16).  The tile's rows are four quarters of 128: CTA
// r holds quarters r and 2 + r of A and converts 128 of the 256 weight rows
// (B).  Issuer h (two threads of the even CTA) multiplies quarters 2h (even
// CTA) and 2h + 1 (odd CTA) by the whole B into accumulator h; the tensor
// cores of both SMs read both CTAs' operands, and each CTA's TMEM receives
// its rows x 256 columns.  While one issuer waits for its next stage the
// MMAs the other queued keep the tensor pipe busy.  Every converted weight
// tile feeds both issuers: each weight is converted once per 512 token rows,
// and per 64-wide k-step a CTA's shared memory carries 32 KB of A (TMA),
// 8 KB of INT8 (TMA), the converters' 8 KB read + 16 KB write and 64 KB of
// MMA operand reads for 256 x 256 x 64 multiply-adds.
//
// Warps of each CTA (16):
//   warp 0      TMA producer of the CTA's two A quarters [128 x 64 k] bf16
//               (a quarter past the expert's rows is not loaded)
//   warp 1      TMEM allocator (both CTAs); issuer 0 (even CTA only)
//   warp 2      TMA producer of the CTA's INT8 weight rows [128 x 64 k]
//   warps 3-10  converters INT8 -> BF16 (shared -> shared, swizzled), in two
//               groups of 4 that take alternate k-steps; group h also drains
//               the second half of accumulator h while the ring is full
//   warps 11-14 epilogue: TMEM -> registers -> scale / SwiGLU / gate -> HBM,
//               the first half of every accumulator
//   warp 15     issuer 1 (even CTA only)
//
// Gate/up tiles: the even CTA converts 128 gate channels, the odd CTA the
// same 128 up channels, so TMEM columns r and 128 + r of a row hold the gate
// and up sums of one channel (the SwiGLU pair sits in one thread).  Down
// tiles: 256 output channels, 128 per CTA.  Expert rows are padded to 128.
// An issuer whose two quarters lie past the expert's rows issues no MMAs
// for the tile (it still takes part in every stage's hand-over); a quarter
// of the odd CTA past the expert's rows leaves that CTA's A stale and
// nothing is stored for it (the MMA rows are independent).
//
// Synchronisation (mbarriers; every wait is bounded and a wait that runs out
// raises the abort flags of both CTAs, after which every role drains its own
// copies and the pair frees its TMEM):
//   a_full[s]   (each CTA)  its A copies of stage s landed
//   empty_a[s]  (each CTA)  both issuers' MMAs reading A stage s are done
//                           (commit multicast)
//   b8_full/b8_empty (each CTA)  INT8 ring between its TMA and its converters
//   full[s]     (even CTA)  the converter warps of both CTAs wrote stage s's
//                           BF16 weights after seeing their CTA's A land
//   empty_b[s]  (each CTA)  both issuers' MMAs reading BF16 stage s are done
//   acc_full[h] (each CTA)  accumulator h is final (issuer h's commit multicast)
//   acc_empty[h] (even CTA) the epilogue warps and converter group h of both
//                           CTAs read it
// The two accumulators of 256 fp32 columns take all 512 TMEM columns.  A
// drain (about 5 us for a whole accumulator with four warps, the SwiGLU's
// exponentials and divisions the largest part) is split: the epilogue warps
// take the first half of accumulator 0 and then of 1, converter group h the
// second half of accumulator h; the converters are idle then anyway, since
// the ring stays full until the issuers restart, and the issuers restart
// only after the drain.  Tiles are visited expert by
// expert in groups of 16 m-tiles (see decode_tile).  No TMA load is
// multicast; every copy reads global memory into its own CTA.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "prefill.h"
#include "sm100.cuh"

namespace jmoe {
namespace {

using namespace sm100;

constexpr int BH = 128;       // token rows of one quarter of the pair tile (one CTA, one issuer)
constexpr int BM = 4 * BH;    // token rows of a pair tile: each CTA holds 2 quarters
constexpr int BN = 256;       // MMA N: output columns of a pair tile
constexpr int BNC = BN / 2;   // weight rows each CTA converts
constexpr int BK = 64;
// Ring depths (4 x 32 KB of A, 4 x 16 KB of BF16 weights, 4 x 8 KB of INT8
// weights: 224 KB).  A k-step's MMAs take about 1024 cycles.  Even depths:
// stage s of the BF16 and INT8 rings always goes to converter group s & 1.
#ifndef JMOE_GEMM_STAGES_A
#define JMOE_GEMM_STAGES_A 4
#endif
#ifndef JMOE_GEMM_STAGES_B
#define JMOE_GEMM_STAGES_B 4
#endif
#ifndef JMOE_GEMM_STAGES_8
#define JMOE_GEMM_STAGES_8 4
#endif
constexpr int kStagesA = JMOE_GEMM_STAGES_A, kStagesB = JMOE_GEMM_STAGES_B;
constexpr int kStages8 = JMOE_GEMM_STAGES_8;
#ifndef JMOE_GEMM_GROUP_M
#define JMOE_GEMM_GROUP_M 16
#endif
constexpr int kGroupM = JMOE_GEMM_GROUP_M;  // pair m-tiles per raster group (rows kept in L2)
constexpr int kABytes = BH * BK * 2;     // 16 KB
constexpr int kBbfBytes = BNC * BK * 2;  // 16 KB
constexpr int kB8Bytes = BNC * BK;       // 8 KB
constexpr int kAStage = 2 * kABytes;     // the CTA's two quarters
constexpr int kSmemA = kStagesA * kAStage;
constexpr int kSmemB = kStagesB * kBbfBytes;
constexpr int kSmem8 = kStages8 * kB8Bytes;
constexpr uint32_t kTmemCols = 512;   // 2 accumulators x 256 fp32 columns
constexpr int kIssuers = 2;           // issuer h: quarters 2h, 2h+1 (M = 256), N = 256
constexpr uint32_t kIdesc = idesc_bf16_f32(2 * BH, BN);
constexpr uint16_t kPairMask = 0x3;   // both CTAs of the cluster

constexpr int kWarpProdA = 0, kWarpMMA = 1, kWarpProdB = 2;
constexpr int kConvWarp0 = 3, kConvGroupWarps = 4, kConvWarps = 2 * kConvGroupWarps;
constexpr int kConvThreads = kConvGroupWarps * 32;  // threads of one converter group
constexpr int kEpiWarp0 = kConvWarp0 + kConvWarps, kEpiWarps = 4;
constexpr int kWarpMMA2 = kEpiWarp0 + kEpiWarps;  // second issuer (kIssuers == 2)
constexpr int kThreads = (kEpiWarp0 + kEpiWarps + kIssuers - 1) * 32;
constexpr int kChunks = kB8Bytes / 16 / kConvThreads;  // 16-byte INT8 chunks per thread per k-step
constexpr int kMaxE = 64;

static_assert(kStagesB % 2 == 0 && kStages8 % 2 == 0, "converter groups alternate k-steps");
// The converters run kStagesB k-steps into the next tile before they help
// drain the previous one; each of those steps waits for its A copy, which the
// A producer can issue only while the A ring has a free stage -- and stages of
// the next tile are freed by MMAs that need the drain.  A shallower A ring
// waits in a cycle (seen as every bounded wait running out).
static_assert(kStagesA >= kStagesB, "the A ring must hold the steps converted before the drain");
static_assert(kChunks * 16 * kConvThreads == kB8Bytes, "converter work split");

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
    long long wait_cycles;  // bound of every mbarrier wait (SM cycles)
    int fault_tile;         // < 0: none; else the weight producers stop before this tile
    int rows_padded;        // rows of H (bounds checks)
    int A;                  // assignments: rows of Y, entries of perm and gates (bounds checks)
};

struct Shared {
    uint64_t full[kStagesB], empty_b[kStagesB];
    uint64_t a_full[kStagesA], empty_a[kStagesA];
    uint64_t b8_full[kStages8], b8_empty[kStages8];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int poff[kMaxE + 1];
    int off[kMaxE + 1];
    int tile_start[kMaxE + 1];
};

constexpr int kSmemBytes = kSmemA + kSmemB + kSmem8 + (int)sizeof(Shared) + 1024;
static_assert(kSmemBytes <= 232448, "more shared memory than a CTA can have");

struct Tile {
    int e, row0, n, quarters;  // quarters: 1..4 valid 128-row quarters
};

// Tile order inside an expert: groups of kGroupM m-tiles; within a group all
// n-tiles, m fastest.  The pairs of a wave then share a few weight tiles and
// at most kGroupM x 512 activation rows, which stay in L2.
__device__ __forceinline__ Tile decode_tile(const Shared& s, int E, int n_tiles, int tile) {
    int e = 0;
    while (e + 1 < E && s.tile_start[e + 1] <= tile) ++e;
    const int local = tile - s.tile_start[e];
    const int nh = (s.poff[e + 1] - s.poff[e]) / BH;  // 128-row quarters of this expert
    const int mt = (nh + 3) / 4;
    const int mg = local / (kGroupM * n_tiles);
    const int gm = min(kGroupM, mt - mg * kGroupM);  // m-tiles in this group
    const int rem = local - mg * kGroupM * n_tiles;
    Tile t;
    t.e = e;
    t.n = rem / gm;
    const int m = mg * kGroupM + rem % gm;
    t.row0 = s.poff[e] + m * BM;
    t.quarters = min(4, nh - 4 * m);
    return t;
}

// Bounded wait that ignores the abort flags (used only while draining).
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, long long limit) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > limit) return;
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    k_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Shared& S = *reinterpret_cast<Shared*>(smem + kSmemA + kSmemB + kSmem8);
    auto tileA = [&](int s) { return smem + s * kAStage; };
    auto tileBbf = [&](int s) { return smem + kSmemA + s * kBbfBytes; };
    auto tileB8 = [&](int s) { return smem + kSmemA + kSmemB + s * kB8Bytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs; 1: its partner
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int E = p.E;
    const int KB = p.K / BK;
    const long long limit = p.wait_cycles;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStagesB; ++i) {
            mbar_init(&S.full[i], 2 * kConvGroupWarps);  // one converter group of each CTA
            mbar_init(&S.empty_b[i], kIssuers);           // the issuers' MMA commits
        }
        for (int i = 0; i < kStagesA; ++i) {
            mbar_init(&S.a_full[i], 1);                   // the A producer (+ TMA bytes)
            mbar_init(&S.empty_a[i], kIssuers);           // the issuers' MMA commits
        }
        for (int i = 0; i < kStages8; ++i) {
            mbar_init(&S.b8_full[i], 1);
            mbar_init(&S.b8_empty[i], kConvGroupWarps);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&S.acc_full[i], 1);  // issuer i's commit
            mbar_init(&S.acc_empty[i], 2 * (kEpiWarps + kConvGroupWarps));  // both CTAs' drainers
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
            run += ((S.poff[e + 1] - S.poff[e]) / BH + 3) / 4 * p.n_tiles;
        }
        S.tile_start[E] = run;
    }
    if (warp == kWarpMMA) {
        tmem_alloc_pair(&S.tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    // both CTAs' barriers initialised and TMEM allocated before any role
    // touches the partner
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;
    const int total = S.tile_start[E];
    volatile int* abort = &S.abort;
    const uint32_t peer_abort = mapa_shared(smem_u32(&S.abort), rank ^ 1u);
    auto wait = [&](uint64_t* bar, uint32_t parity) {
        return mbar_wait_pair(bar, parity, abort, peer_abort, limit);
    };

    // Drains chunks [c_lo, c_hi) (32 columns each; gate/up: 32 channels, whose
    // gate and up columns sit 128 apart) of accumulator h of tile t into H or
    // Y, from this warp's TMEM lane quadrant: wait for the accumulator, read,
    // scale (SwiGLU / gate), store, and arrive on acc_empty[h] of the even CTA.
    // The epilogue warps drain the first half of every accumulator, converter
    // group h the second half of accumulator h.
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(&S.acc_empty[0]), 0);
    auto drain = [&](const Tile& t, int h, int& uses_h, int c_lo, int c_hi) {
        const int quad = warp & 3;
        if (!__all_sync(0xffffffffu, wait(&S.acc_full[h], uses_h & 1))) return false;
        ++uses_h;
        tc_fence_after();
        const int q = 2 * h + (int)rank;
        if (q < t.quarters) {
            const uint32_t taddr = tmem + h * BN + ((uint32_t)(quad * 32) << 16);
            const int row = t.row0 + q * BH + quad * 32 + lane;
            if (MODE == kGateUp) {
                const int n0 = t.n * BNC;
                const float* sg = p.scale + (size_t)t.e * p.w_rows + n0;
                const float* su = sg + p.up_offset;
#pragma unroll 1
                for (int c = c_lo; c < c_hi; ++c) {
                    const int ch = n0 + c * 32;
                    if (ch >= p.n_valid) break;  // n_valid is a multiple of 64
                    // gate channel n0 + r: column r (the even CTA's B row r);
                    // its up channel: column 128 + r (the odd CTA's row r)
                    uint32_t gv[32], uv[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, gv);
                    tmem_ld_32x32b_x32(taddr + BNC + c * 32, uv);
                    tmem_ld_wait();
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
                    if (JMOE_CHECK(row >= 0 && row < p.rows_padded))
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq)
                            dst[qq] = make_uint4(packed[4 * qq], packed[4 * qq + 1],
                                                 packed[4 * qq + 2], packed[4 * qq + 3]);
                }
            } else {
                const int m0 = t.n * BN;
                const int r = row - S.poff[t.e];
                const int gi = S.off[t.e] + r;  // grouped index of the row
                bool valid = r < S.off[t.e + 1] - S.off[t.e];
                valid = valid && JMOE_CHECK(gi >= 0 && gi < p.A);
                const int a = valid ? p.perm[gi] : 0;
                valid = valid && JMOE_CHECK(a >= 0 && a < p.A);
                const float gate = valid ? p.gates[a] : 0.0f;
                const float* sd = p.scale + (size_t)t.e * p.w_rows;
#pragma unroll 1
                for (int c = c_lo; c < c_hi; ++c) {
                    const int m = m0 + c * 32;  // column c: the even CTA's rows, then the odd's
                    if (m >= p.n_valid) break;  // n_valid is a multiple of 64
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, v);
                    tmem_ld_wait();
                    if (valid) {
                        float4* dst = reinterpret_cast<float4*>(p.Y + (size_t)a * p.n_valid + m);
#pragma unroll
                        for (int qq = 0; qq < 8; ++qq) {
                            const float4 s4 = __ldg(reinterpret_cast<const float4*>(sd + m) + qq);
                            float4 o;
                            o.x = gate * (s4.x * __uint_as_float(v[4 * qq]));
                            o.y = gate * (s4.y * __uint_as_float(v[4 * qq + 1]));
                            o.z = gate * (s4.z * __uint_as_float(v[4 * qq + 2]));
                            o.w = gate * (s4.w * __uint_as_float(v[4 * qq + 3]));
                            dst[qq] = o;
                        }
                    }
                }
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty_leader + h * (uint32_t)sizeof(uint64_t));
        return true;
    };
    constexpr int kAccChunks = (MODE == kGateUp ? BNC : BN) / 32;  // chunks of an accumulator

    if (warp == kWarpProdA) {
        if (lane == 0) {
            uint32_t g = 0;
            for (int tile = pair; tile < total && !*abort; tile += npairs) {
                const Tile t = decode_tile(S, E, p.n_tiles, tile);
                // this CTA's quarters of the tile: 2h + rank for h = 0, 1
                const int nq = ((int)rank < t.quarters) + (2 + (int)rank < t.quarters);
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int s = g % kStagesA;
                    const uint32_t ph = (g / kStagesA) & 1;
                    if (!wait(&S.empty_a[s], ph ^ 1)) break;
                    if (nq > 0) {
                        mbar_arrive_expect_tx(&S.a_full[s], nq * kABytes);
                        for (int h = 0; h < nq; ++h)
                            tma_load_2d(tileA(s) + h * kABytes, &tmA, &S.a_full[s], kb * BK,
                                        t.row0 + (2 * h + (int)rank) * BH);
                    } else {
                        mbar_arrive(&S.a_full[s]);
                    }
                }
            }
            // leave only when no copy is still landing in shared memory
            for (uint32_t h = (g > (uint32_t)kStagesA ? g - kStagesA : 0); h < g; ++h)
                wait_drain(&S.a_full[h % kStagesA], (h / kStagesA) & 1, limit);
        }
    } else if (warp == kWarpProdB) {
        if (lane == 0) {
            uint32_t g = 0;
            for (int tile = pair; tile < total && !*abort; tile += npairs) {
                if (tile == p.fault_tile) break;  // test hook: this tile's weights never come
                const Tile t = decode_tile(S, E, p.n_tiles, tile);
                // gate/up: the even CTA's gate rows, the odd CTA's up rows of the same
                // channels; down: the CTA's half of the 256 output channels
                const int y = MODE == kGateUp ? t.e * p.w_rows + (int)rank * p.up_offset + t.n * BNC
                                              : t.e * p.w_rows + t.n * BN + (int)rank * BNC;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int s = g % kStages8;
                    const uint32_t ph = (g / kStages8) & 1;
                    if (!wait(&S.b8_empty[s], ph ^ 1)) break;
                    mbar_arrive_expect_tx(&S.b8_full[s], kB8Bytes);
                    tma_load_2d(tileB8(s), &tmB, &S.b8_full[s], kb * BK, y);
                }
            }
            for (uint32_t h = (g > (uint32_t)kStages8 ? g - kStages8 : 0); h < g; ++h)
                wait_drain(&S.b8_full[h % kStages8], (h / kStages8) & 1, limit);
        }
    } else if (warp == kWarpMMA || warp == kWarpMMA2) {
        if (rank == 0 && lane == 0) {
            // issuer h: M slice h (quarter 2h from this CTA, 2h + 1 from the
            // partner) into accumulator h; an issuer whose slice lies past the
            // expert's rows still waits and commits every stage, without MMAs
            const int h = warp == kWarpMMA ? 0 : 1;
            uint32_t g = 0;
            int uses = 0;
            for (int tile = pair; tile < total && !*abort; tile += npairs) {
                const bool active = 2 * h < decode_tile(S, E, p.n_tiles, tile).quarters;
                if (active) {
                    if (!mbar_wait_pair(&S.acc_empty[h], (uses & 1) ^ 1, abort, peer_abort, limit))
                        break;
                    tc_fence_after();
                }
                const uint32_t d_tmem = tmem + h * BN;
                bool ok = true;
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int sa = g % kStagesA;
                    const int s = g % kStagesB;
                    const uint32_t ph = (g / kStagesB) & 1;
                    if (!mbar_wait_pair(&S.full[s], ph, abort, peer_abort, limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(tileA(sa)) + h * kABytes;
                    const uint32_t b0 = smem_u32(tileBbf(s));
                    if (active) {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            mma_bf16_ss_pair(d_tmem, desc_sw128(a0 + kk * 32), desc_sw128(b0 + kk * 32),
                                             kIdesc, (kb | kk) != 0);
                    }
                    mma_commit_pair_mc(&S.empty_a[sa], kPairMask);
                    mma_commit_pair_mc(&S.empty_b[s], kPairMask);
                }
                if (!ok) break;
                if (active) {
                    mma_commit_pair_mc(&S.acc_full[h], kPairMask);
                    ++uses;
                }
            }
            // every MMA done (both CTAs' TMEM written, both CTAs' shared memory read)
            mma_commit_pair(&S.drain);
            wait_drain(&S.drain, 0, limit);
        }
    } else if (warp >= kConvWarp0 && warp < kConvWarp0 + kConvWarps) {
        // Group G converts the k-steps g with g % 2 == G.  Thread ct converts the
        // 16-byte INT8 chunks q = ct + 128 j (row q / 4, bytes 16 (q % 4) ..
        // +16) of the CTA's 128 x 64 tile: all loads first, then each chunk
        // becomes the two 16-byte bf16 units 2 (q % 4) and 2 (q % 4) + 1 of the
        // row's 128-byte swizzled line.
        const int G = (warp - kConvWarp0) / kConvGroupWarps;
        const int ct = threadIdx.x - (kConvWarp0 + G * kConvGroupWarps) * 32;  // 0..127
        const uint32_t full_leader = mapa_shared(smem_u32(&S.full[0]), 0);
        uint32_t g = 0;
        bool ok = true;
        // The group also drains the second half of accumulator G of the
        // previous tile, at the point where it would otherwise wait for this
        // tile's MMAs to free a stage -- which needs issuer G to restart, which
        // needs the drain: k-step kStagesB of the next tile, or the end of the
        // next tile's k-steps when it has fewer, or after the last tile.
        int help_uses = 0, pending = -1;
        auto help = [&](int tile) {
            const Tile t = decode_tile(S, E, p.n_tiles, tile);
            if (2 * G >= t.quarters) return true;  // issuer G had no rows in this tile
            return drain(t, G, help_uses, kAccChunks / 2, kAccChunks);
        };
        for (int tile = pair; tile < total && ok && !*abort; tile += npairs) {
            for (int kb = 0; kb < KB; ++kb, ++g) {
                if (pending >= 0 && kb == kStagesB) {
                    ok = help(pending);
                    pending = -1;
                    if (!ok) break;
                }
                if ((int)(g & 1) != G) continue;
                const int s = g % kStagesB;
                const uint32_t ph = (g / kStagesB) & 1;
                const int sa = g % kStagesA;
                const uint32_t pha = (g / kStagesA) & 1;
                const int s8 = g % kStages8;
                const uint32_t ph8 = (g / kStages8) & 1;
                // every lane waits; the vote keeps the warp together if one lane
                // gave up just as the phase completed for another
                if (!__all_sync(0xffffffffu, wait(&S.b8_full[s8], ph8) && wait(&S.empty_b[s], ph ^ 1))) {
                    ok = false;
                    break;
                }
                const uint8_t* src = tileB8(s8);
                uint8_t* dst = tileBbf(s);
                uint4 v[kChunks];
#pragma unroll
                for (int j = 0; j < kChunks; ++j)
                    v[j] = *reinterpret_cast<const uint4*>(src + (ct + kConvThreads * j) * 16);
#pragma unroll
                for (int j = 0; j < kChunks; ++j) {
                    const int q = ct + kConvThreads * j, row = q >> 2, u0 = 2 * (q & 3);
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
                int good = 1;
                if (lane == 0) {
                    mbar_arrive(&S.b8_empty[s8]);
                    // the stage is complete in this CTA once its A rows landed too
                    if (wait(&S.a_full[sa], pha))
                        mbar_arrive_cluster(full_leader + s * (uint32_t)sizeof(uint64_t));
                    else
                        good = 0;
                }
                if (!__shfl_sync(0xffffffffu, good, 0)) {
                    ok = false;
                    break;
                }
            }
            if (ok && pending >= 0) ok = help(pending);
            pending = tile;
        }
        if (ok && pending >= 0 && !*abort) help(pending);  // the last tile
    } else {
        // epilogue warps (TMEM lane quadrant = warp % 4): per tile, the first
        // half of accumulator h (this CTA's quarter 2h + rank: 128 rows x 256
        // columns), accumulator 0 first
        int uses[2] = {0, 0};
        bool ok = true;
        for (int tile = pair; tile < total && ok && !*abort; tile += npairs) {
            const Tile t = decode_tile(S, E, p.n_tiles, tile);
            for (int h = 0; h < 2 && ok; ++h) {
                if (2 * h >= t.quarters) break;  // issuer h had no rows in this tile
                ok = drain(t, h, uses[h], 0, kAccChunks / 2);
            }
        }
    }

    // Neither CTA frees its TMEM or leaves before every MMA (which reads both
    // CTAs' shared memory and writes both CTAs' TMEM) and every arrival on the
    // partner's barriers is done: the issuer waited for its drain commit above,
    // and the cluster barrier orders everything before it.
    tc_fence_before();
    __syncwarp();
    cluster_sync();
    if (threadIdx.x == 0 && S.abort) flag_error(p.err, kErrTimeout);
    if (warp == kWarpMMA) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// ----------------------------------------------------------------------------- host side

// CTA pairs resident at once (one CTA per SM), at most `want`.  The kernel's
// cluster shape is fixed at compile time, so the query leaves it unspecified.
template <int MODE>
int resident_pairs(int num_sms, int want) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * want);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, k_grouped_gemm<MODE>, &cfg) != cudaSuccess ||
        clusters < 1)
        clusters = num_sms / 2;
    return clusters < want ? clusters : want;
}

template <int MODE>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const GemmParams& p,
                        int num_sms, int tiles, cudaStream_t stream) {
    if (tiles <= 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(k_grouped_gemm<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    const int pairs = resident_pairs<MODE>(num_sms, tiles);
    k_grouped_gemm<MODE><<<2 * pairs, kThreads, kSmemBytes, stream>>>(a, b, p);
    note_launch();
    return cudaGetLastError();
}

// Pair tiles of one GEMM: per expert, ceil(128-row quarters / 4) m-tiles times
// n_tiles (the kernel derives the same count from the padded offsets; the
// host only needs an upper bound to size the grid).
int64_t tile_bound(const PrefillArgs& a, int n_tiles) {
    const int64_t quarters = a.rows_padded / BH;
    return (quarters / 4 + a.E) * n_tiles;
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
    err = launch_gather_rows(a.x, a.T, a.d, a.top_k, a.E, a.offsets, a.padded_offsets, a.perm,
                             a.rows_padded, a.xperm, a.num_sms, stream);
    if (a.mark) a.mark(1, true, stream);
    if (err != cudaSuccess) return err;

    CUtensorMap mA1, mB1, mA2, mB2;
    const bool ok =
        encode_2d(&mA1, a.xperm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.rows_padded, a.d, BH, BK,
                 CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_2d(&mB1, a.wgu, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.E * 2 * a.f, a.d,
                 BNC, BK, CU_TENSOR_MAP_SWIZZLE_NONE) &&
        encode_2d(&mA2, a.H, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.rows_padded, a.f, BH, BK,
                 CU_TENSOR_MAP_SWIZZLE_128B) &&
        encode_2d(&mB2, a.wd, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)a.E * a.d, a.f, BNC, BK,
                 CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;

    // 2. gate/up GEMM + SwiGLU -> H (bf16, grouped rows)
    GemmParams g1{};
    g1.E = a.E;
    g1.K = (int)a.d;
    g1.n_valid = (int)a.f;
    g1.n_tiles = (int)((a.f + BNC - 1) / BNC);
    g1.w_rows = (int)(2 * a.f);
    g1.up_offset = (int)a.f;
    g1.poff = a.padded_offsets;
    g1.off = a.offsets;
    g1.perm = a.perm;
    g1.scale = a.sgu;
    g1.gates = a.gates;
    g1.H = static_cast<uint16_t*>(a.H);
    g1.err = a.err;
    g1.wait_cycles = a.wait_cycles > 0 ? a.wait_cycles : kWaitCycles;
    g1.fault_tile = a.fault_tile;
    g1.rows_padded = (int)a.rows_padded;
    g1.A = (int)a.A;
    if (a.mark) a.mark(2, false, stream);
    err = launch_gemm<kGateUp>(mA1, mB1, g1, a.num_sms, (int)tile_bound(a, g1.n_tiles), stream);
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
    g2.fault_tile = -1;
    if (a.mark) a.mark(3, false, stream);
    err = launch_gemm<kDown>(mA2, mB2, g2, a.num_sms, (int)tile_bound(a, g2.n_tiles), stream);
    if (a.mark) a.mark(3, true, stream);
    if (err != cudaSuccess) return err;

    // 4. out[t] = bf16(sum over the token's assignments)
    if (a.mark) a.mark(4, false, stream);
    err = launch_finalize(a.Yg, a.T, a.d, a.top_k, a.E, a.ids, a.out, a.num_sms, stream);
    if (a.mark) a.mark(4, true, stream);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

JMOE_DEFINE_CHECKS_READER(checks_take_prefill)

}  // namespace jmoe
