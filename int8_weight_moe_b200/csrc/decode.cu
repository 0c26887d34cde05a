// Decode path of the expert MLPs: few tokens per expert, so the work is one
// stream over the INT8 weights of the experts that some token selected
// (HBM-bound; the weights of untouched experts are never read).
//
// ExpertsInt8 ("Jamba-1.5: Hybrid Transformer-Mamba Models at Scale", paper
// summary, section "ExpertsInt8 Quantization (Section 3.1)", steps 3-4): the
// INT8 weights cross HBM once and are turned back into 16-bit floating point
// on chip; the activations keep their BF16 values.  Every weight byte goes
// HBM -> shared (TMA) -> registers and is converted exactly (|q| <= 127) into
// fp16 -- the same number BF16 would hold, at half the ALU cost of an
// int8 -> bf16 conversion.  The activation operand (token rows for gate/up,
// BF16-rounded hidden rows for down) is staged as fp16 after a power-of-two
// shift per row that brings the row maximum into [2^14, 2^15): a bf16 value
// has 8 significant bits, so the staged values are exact and every product
// equals the bf16 one; the shifts are undone exactly after the dot products.
// The per-output-channel scale is applied once after the dot product (an
// exact refactoring of sum_k x_k (q_k s)).  mma.sync m16n8k16 (f16 in, fp32
// accumulate), up to 8 tokens of the expert as the columns.

// Fragment trick: the dot product does not care in which order k is summed,
// so the 16 k-columns of an MMA step are a permutation of the 64-wide k-block
// chosen such that thread (g = lane/4, c = lane%4) reads exactly bytes
// [16c, 16c+16) of rows g and g+8 for the block's four MMA steps -- one
// 16-byte load per row -- and the matching 16 consecutive bf16 of its token.
// Step s uses physical k = 16c + 4s + {0,1} for fragment columns 2c, 2c+1 and
// 16c + 4s + {2,3} for columns 2c+8, 2c+9.
//
// Work decomposition: every warp is an independent streaming worker.  A work
// item is (touched expert, one unit of output channels, one pass of up to 8
// tokens, one K piece of S): two 16-row matrices x K/S bytes (gate/up: 16
// gate rows and the same 16 up rows; down: the two halves of 32 output
// rows).  Items (32-112 KB at Mini sizes) are dealt round-robin to all warps
// of the GPU, the K pieces and passes of a unit to neighbouring warps, so the
// warps finish together and the rows being read at any moment are few and
// shared by several warps (DRAM rows stay open for more of their bytes).
// Each warp keeps a ring of 4 KB slots in its own shared memory, filled by
// TMA two slots ahead of use and across item boundaries, with the matching
// activation fragments loaded one slot ahead (their lines prefetched into L1
// two slots ahead); there are no barriers.  An
// item stores its raw fp32 partial sums; the small follow-up kernels add the
// S pieces in a fixed order (deterministic) and apply scales, SwiGLU, gates.
// (Finishing units inside the streaming warps instead -- a counter per unit,
// the last piece's warp adding them -- measured much slower: every fence,
// atomic and dependent read at an item's end stalls that warp's short ring.)
//   k_dprep -> grouping by expert (one CTA) + x16 (fp16, per-token shift)
//   k_gemv<gate/up> -> P_gu[S][slot][2f] -> k_swiglu -> Hb (bf16) + row maxima
//                                         -> k_h16 -> H (fp16, per-slot shift)
//   k_gemv<down>    -> P_d [S][slot][d]  -> k_combine -> out (bf16)
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "permute.cuh"
#include "sm100.cuh"

namespace jmoe {
namespace {

constexpr int kWarpsPerBlock = 4;
constexpr int kMaxE = 64;

enum { kGateUp = 0, kDown = 1 };

// x (or h) fragment for one token row: 16 consecutive fp16 starting at p.
__device__ __forceinline__ void load_b(const uint16_t* p, uint32_t (&b)[8]) {
    const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(p));
    const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(p + 8));
    b[0] = v0.x; b[1] = v0.y; b[2] = v0.z; b[3] = v0.w;
    b[4] = v1.x; b[5] = v1.y; b[6] = v1.z; b[7] = v1.w;
}

// Bring the 128-byte line at p into L1 without waiting for it.
__device__ __forceinline__ void prefetch_l1(const void* p) {
    asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// Four MMA steps of one 64-wide k-block: rows g (q0) and g+8 (q1).  Even and
// odd steps accumulate into separate tiles (two independent MMA chains).  The
// weights are converted to fp16 (the activation operand is fp16 too).
__device__ __forceinline__ void mma_block(float (&acc)[2][4], const uint4& q0, const uint4& q1,
                                          const uint32_t (&b)[8]) {
    const uint32_t w0[4] = {q0.x, q0.y, q0.z, q0.w};
    const uint32_t w1[4] = {q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        uint32_t l0, h0, l1, h1;
        i8x4_to_f16x2x2(w0[s], l0, h0);
        i8x4_to_f16x2x2(w1[s], l1, h1);
        const uint32_t a[4] = {l0, l1, h0, h1};
        mma_f16_16816(acc[s & 1], a, b[2 * s], b[2 * s + 1]);
    }
}

struct Item {
    int e, group, pass, z;
};

// The first of the last `slots` slot fills a warp issued (the ones whose
// copies may still be in flight when the warp leaves).
__device__ __forceinline__ int64_t q_drain_begin(int64_t total, int slots) {
    return total > slots ? total - slots : 0;
}

constexpr int kSlots = 3;  // ring slots per warp: two 4 KB slots in flight

// Every item reads two 16-row weight matrices that share the activation
// fragments: gate/up, the 16 gate rows and the same 16 up rows of a unit of 16
// channels; down, the two 16-row halves of a unit of 32 output channels.  A
// ring slot holds 2 k-blocks (one 128-byte line per row) of both: 4 KB, filled
// by a single TMA box (gate/up: a 4-D view that puts the up rows f rows below
// the gate rows; down: 32 adjacent rows).
template <int MODE>
constexpr int nb_of() {
    return 2;
}

// Output channels of one unit.
template <int MODE>
constexpr int unit_rows() {
    return MODE == kGateUp ? 16 : 32;
}

// Shared memory of one warp: kSlots x [matrix][16 rows][128 B], stored with
// the TMA 128-byte swizzle (16-byte chunk j of row r at chunk j ^ (r & 7)), so
// that the fragment reads of a warp -- 8 rows x the same 4 chunks -- hit all
// banks once.  The swizzle needs 1024-byte aligned slots; the extra 1 KB of
// the allocation pays for aligning the ring.
template <int MODE>
constexpr int slot_bytes() {
    return 2 * nb_of<MODE>() * 16 * 64;
}

template <int MODE>
constexpr int gemv_smem() {
    return kWarpsPerBlock * kSlots * slot_bytes<MODE>() + 1024;
}

template <int MODE, int NCH>
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    k_gemv(const __grid_constant__ CUtensorMap tmW, const GemvParams p) {
    constexpr int NMAT = 2;
    constexpr int kNB = nb_of<MODE>();
    constexpr int kSlotBytes = slot_bytes<MODE>();
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ uint64_t full[kWarpsPerBlock][kSlots];
    __shared__ int s_start[kMaxE + 1];  // first item of expert e
    __shared__ int s_off[kMaxE + 1];
    __shared__ int s_np[kMaxE];         // passes of expert e
    __shared__ int s_abort;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g8 = lane >> 2, c = lane & 3;
    uint8_t* const ring_base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* ring = ring_base + warp * kSlots * kSlotBytes;
    const int E = p.E, S = p.S;
    const int64_t K = MODE == kGateUp ? p.d : p.f;
    const int64_t rows_out = MODE == kGateUp ? p.f : p.d;
    const int groups = (int)(rows_out / unit_rows<MODE>());
    if (lane == 0) {
        for (int i = 0; i < kSlots; ++i) sm100::mbar_init(&full[warp][i], 1);
        sm100::tma_prefetch_desc(&tmW);
    }
    if (threadIdx.x == 0) {
        s_abort = 0;
        sm100::fence_mbar_init();
    }
    // The gate/up GEMV reads the grouping tables of the kernel it follows, so
    // it waits first.  The down GEMV follows k_h16, which lets it start only
    // after its own wait, i.e. once k_swiglu and everything before it (the
    // grouping tables included) are complete: it plans its items and starts
    // its first weight copies, and waits only before it reads hidden rows.
    if (MODE == kGateUp) {
        pdl_wait();
        pdl_launch_dependents();
    }
    if (threadIdx.x <= E) s_off[threadIdx.x] = p.offsets[threadIdx.x];
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            const int np = (s_off[e + 1] - s_off[e] + 8 * NCH - 1) / (8 * NCH);
            s_np[e] = np;
            s_start[e] = run;
            run += np * groups * S;
        }
        s_start[E] = run;
    }
    __syncthreads();
    volatile int* abort = &s_abort;
    const int n_items = s_start[E];
    const int W = gridDim.x * kWarpsPerBlock;
    const int wid = blockIdx.x * kWarpsPerBlock + warp;
    const int n_mine = wid < n_items ? (n_items - 1 - wid) / W + 1 : 0;
    const int kb_item = (int)(K / 64 / S);            // k-blocks per item
    const int nsl = (kb_item + kNB - 1) / kNB;        // ring slots per item
    const int64_t total = (int64_t)n_mine * nsl;
    if (total == 0) return;

    // The warp's it-th item.  Items come in increasing order, so each cursor
    // (producer, consumer) keeps its expert `e` and only moves it forward; the
    // search stops below E because every index is below s_start[E].  The
    // passes of one (unit, piece) are neighbours, so the warps that read the
    // same weights run side by side and all but one hit in L2.
    auto item_at = [&](int it, int& e) {
        const int idx = wid + it * W;
        while (s_start[e + 1] <= idx) ++e;
        const int local = idx - s_start[e];
        const int np = s_np[e];
        int rest = local;
        Item r;
        r.e = e;
        r.pass = 0;
        if (np > 1) {
            r.pass = local % np;
            rest = local / np;
        }
        r.z = rest % S;
        r.group = rest / S;
        return r;
    };

    // ---- producer cursor (lane 0 issues the TMA boxes of slot-sized pieces)
    int pe = 0, pi = 0, pj = 0;
    int pexp = 0, prow = 0, pk = 0;  // expert, first weight row of the item, first k byte of the piece
    int64_t issued = 0;    // slot fills issued so far (fill h uses slot h % kSlots)
    int64_t skipped = -1;  // the fill the test hook left out (its barrier never completes)
    auto set_prefetch_item = [&](int it) {
        const Item u = item_at(it, pe);
        pexp = u.e;
        prow = MODE == kGateUp ? u.group * 16 : u.e * (int)p.d + u.group * unit_rows<MODE>();
        pk = u.z * kb_item * 64;
    };
    auto issue = [&](int slot) {
        const bool skip = p.fault && wid == 0 && issued == 0;
        if (skip) skipped = issued;
        if (lane == 0 && !skip) {
            (void)JMOE_CHECK(pk + pj * kNB * 64 < K && pexp < E &&
                             prow + (MODE == kGateUp ? 16 : 32) <= (MODE == kGateUp ? p.f : (int64_t)E * p.d));
            uint8_t* dst = ring + slot * kSlotBytes;
            sm100::mbar_arrive_expect_tx(&full[warp][slot], kSlotBytes);
            if (MODE == kGateUp)  // [expert][gate|up][row][k]: 16 rows of both halves
                sm100::tma_load_4d(dst, &tmW, &full[warp][slot], pk + pj * kNB * 64, prow, 0, pexp);
            else                  // [row][k]: the unit's 32 rows
                sm100::tma_load_2d(dst, &tmW, &full[warp][slot], pk + pj * kNB * 64, prow);
        }
        ++issued;
        if (++pj == nsl) {
            pj = 0;
            if (++pi < n_mine) set_prefetch_item(pi);
        }
    };
    set_prefetch_item(0);
#pragma unroll
    for (int q = 0; q < kSlots - 1; ++q)
        if (q < total) issue(q);
    if (MODE == kDown) {
        pdl_wait();
        pdl_launch_dependents();
    }

    // ---- consumer state: activation fragments are loaded one slot ahead,
    // into the one of two register buffers the current slot does not use
    float acc[NCH][NMAT][2][4];
#pragma unroll
    for (int n = 0; n < NCH; ++n)
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[n][m][0][i] = acc[n][m][1][i] = 0.0f;
    struct Cur {
        Item u;
        int base, cnt_pass;
        const uint16_t* b[NCH];
    };
    int ce = 0;
    auto make_cur = [&](int it) {
        Cur r;
        r.u = item_at(it, ce);
        r.base = s_off[r.u.e] + r.u.pass * 8 * NCH;
        r.cnt_pass = min(8 * NCH, s_off[r.u.e + 1] - r.base);
        const int64_t kz = (int64_t)r.u.z * kb_item * 64;
#pragma unroll
        for (int n = 0; n < NCH; ++n) {
            // A column without a token reads the pass's first row instead: the
            // MMA keeps columns apart and that output column is never stored.
            const int slot = n * 8 + g8 < r.cnt_pass ? n * 8 + g8 : 0;
            const int gi = r.base + slot;  // grouped index of the column's assignment
            int64_t row = 0;
            if (JMOE_CHECK(gi >= 0 && gi < p.A)) {
                row = MODE == kGateUp ? (int64_t)(p.perm[gi] / p.top_k) : (int64_t)gi;
                if (!JMOE_CHECK(row >= 0 && row < (MODE == kGateUp ? p.T : p.A))) row = 0;
            }
            const int64_t k0 = JMOE_CHECK(kz + (int64_t)kb_item * 64 <= K) ? kz : 0;
            r.b[n] = p.b_src + row * K + 16 * c + k0;
        }
        return r;
    };
    using Frag = uint32_t[kNB][NCH][8];
    auto load_slot_b = [&](const Cur& r, int j, Frag& dst) {
#pragma unroll
        for (int b = 0; b < kNB; ++b) {
            // a k-block past the item's end (odd count) is read but not used
            const int kb = min(j * kNB + b, kb_item - 1);
#pragma unroll
            for (int n = 0; n < NCH; ++n) load_b(r.b[n] + kb * 64, dst[b][n]);
        }
    };
    Frag fa, fb;
    Cur cur = make_cur(0), nxt{};
    load_slot_b(cur, 0, fa);
    int ci = 0, cj = 0, cslot = 0;
    uint32_t cphase = 0;
    bool ok = true;
    // Slot q: refill the slot consumed by q-1, fetch the fragments of q+1 into
    // `fnext`, wait for q's weights and multiply them with `fcur`.
    auto step = [&](int64_t q, const Frag& fcur, Frag& fnext) {
        if (q + kSlots - 1 < total) {
            __syncwarp();
            if (lane == 0) sm100::fence_proxy_async_smem();
            issue((int)((q + kSlots - 1) % kSlots));
        }
        if (cj + 1 < nsl) {
            load_slot_b(cur, cj + 1, fnext);
        } else if (ci + 1 < n_mine) {
            nxt = make_cur(ci + 1);
            load_slot_b(nxt, 0, fnext);
        }
        // Warm L1 with the activation lines of slot q+2 (one per row and
        // k-block; a prefetch holds no register).  While the weight stream
        // keeps DRAM busy an L2 hit takes longer than one slot, so without
        // this the loads above wait whenever several token rows share a pass.
        if (cj + 2 < nsl && c == 0) {
#pragma unroll
            for (int b = 0; b < kNB; ++b)
#pragma unroll
                for (int n = 0; n < NCH; ++n)
                    prefetch_l1(cur.b[n] + min((cj + 2) * kNB + b, kb_item - 1) * 64);
        }
        // every lane waits; the vote keeps the warp on one path
        if (!__all_sync(0xffffffffu,
                        sm100::mbar_wait(&full[warp][cslot], cphase, abort, p.wait_cycles))) {
            ok = false;
            return;
        }
        // rows g8 and g8 + 8 of matrix m: byte m * 2048 + row * 128 + the
        // swizzled position of chunk 4b + c (row & 7 == g8 for both rows)
        const uint8_t* src = ring + cslot * kSlotBytes + g8 * 128;
#pragma unroll
        for (int b = 0; b < kNB; ++b) {
            if (cj * kNB + b < kb_item) {
                uint4 wq[2 * NMAT];
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    const int off = m * 2048 + (((4 * b + c) ^ g8) << 4);
                    wq[2 * m] = *reinterpret_cast<const uint4*>(src + off);
                    wq[2 * m + 1] = *reinterpret_cast<const uint4*>(src + off + 8 * 128);
                }
#pragma unroll
                for (int n = 0; n < NCH; ++n) {
                    if (n * 8 < cur.cnt_pass) {
                        mma_block(acc[n][0], wq[0], wq[1], fcur[b][n]);
                        mma_block(acc[n][1], wq[2], wq[3], fcur[b][n]);
                    }
                }
            }
        }
        if (++cslot == kSlots) {
            cslot = 0;
            cphase ^= 1u;
        }
        if (++cj == nsl) {
            // end of item: raw partial sums -> P[z][slot][col]
            const int64_t cols = MODE == kGateUp ? 2 * p.f : p.d;
            float* P = p.P + (int64_t)cur.u.z * p.A * cols;
#pragma unroll
            for (int n = 0; n < NCH; ++n)
#pragma unroll
                for (int m = 0; m < NMAT; ++m)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int slot = n * 8 + 2 * c + (i & 1);
                        const int64_t col =
                            MODE == kGateUp
                                ? (int64_t)m * p.f + cur.u.group * 16 + g8 + (i >> 1) * 8
                                : (int64_t)cur.u.group * 32 + m * 16 + g8 + (i >> 1) * 8;
                        if (slot < cur.cnt_pass &&
                            JMOE_CHECK(cur.base + slot < p.A && col < cols && cur.u.z < S))
                            P[(int64_t)(cur.base + slot) * cols + col] = acc[n][m][0][i] + acc[n][m][1][i];
                        acc[n][m][0][i] = acc[n][m][1][i] = 0.0f;
                    }
            cj = 0;
            if (++ci < n_mine) cur = nxt;
        }
    };
    for (int64_t q = 0; q < total; q += 2) {
        step(q, fa, fb);
        if (!ok || q + 1 >= total) break;
        step(q + 1, fb, fa);
        if (!ok) break;
    }
    // leave only when no copy is still landing in this warp's ring: the last
    // kSlots fills issued (all of them on the normal path, where issued equals
    // total; fewer when a wait ran out), each the newest fill of its slot
    if (lane == 0) {
        for (int64_t h = q_drain_begin(issued, kSlots); h < issued; ++h) {
            if (h == skipped) continue;
            const long long t0 = clock64();
            while (!sm100::mbar_try_wait(&full[warp][h % kSlots], (uint32_t)((h / kSlots) & 1)))
                if (clock64() - t0 > p.wait_cycles) break;
        }
        if (!ok && p.err) flag_error(p.err, kErrTimeout);
    }
}

// Power-of-two shift that puts the largest |value| of a row (biased fp32 /
// bf16 exponent field emax) into [2^14, 2^15), inside fp16's normal range.
__device__ __forceinline__ int row_shift(int emax) {
    if (emax == 0) return 0;
    return max(emax - 127 - 14, -100);
}

__device__ __forceinline__ int block_max_int(int v, int* red) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    int m = 0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = max(m, red[i]);
    __syncthreads();
    return m;
}

// Block T: the stable grouping of the assignments by expert (offsets, perm,
// inv; invalid expert ids are left out and flagged).  Blocks t < T:
// x16[t] = fp16(x[t] * 2^-xexp[t]).  A bf16 value has 8 significant bits, so
// the scaled value is exactly representable in fp16 unless it falls below
// fp16's normal range (2^-14, i.e. 2^28 times smaller than the row maximum).
__global__ void __launch_bounds__(kPermuteThreads)
    k_dprep(const uint16_t* __restrict__ x, int64_t T, int64_t d, uint16_t* __restrict__ x16,
            int32_t* __restrict__ xexp, int32_t* __restrict__ hmax, const int32_t* __restrict__ ids,
            int E, int top_k, int32_t* __restrict__ offsets, int32_t* __restrict__ perm,
            int32_t* __restrict__ inv, unsigned* err) {
    pdl_wait();
    pdl_launch_dependents();
    if (blockIdx.x == T) {
        block_permute(ids, T * top_k, E, 1, offsets, nullptr, perm, inv, err);
        return;
    }
    __shared__ int red[kPermuteThreads / 32];
    const int64_t t = blockIdx.x;
    if (threadIdx.x < top_k) hmax[t * top_k + threadIdx.x] = 0;  // for k_swiglu's maxima
    const uint16_t* xr = x + t * d;
    int m = 0;
    for (int64_t k = threadIdx.x * 8; k < d; k += (int64_t)blockDim.x * 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(xr + k);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) m = max(m, (int)max((u[i] >> 7) & 0xffu, (u[i] >> 23) & 0xffu));
    }
    const int sh = row_shift(block_max_int(m, red));
    if (threadIdx.x == 0) xexp[t] = sh;
    const float scale = ldexpf(1.0f, -sh);
    for (int64_t k = threadIdx.x * 8; k < d; k += (int64_t)blockDim.x * 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(xr + k);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __half2 h = __floats2half2_rn(__uint_as_float(u[i] << 16) * scale,
                                                __uint_as_float(u[i] & 0xffff0000u) * scale);
            o[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(x16 + t * d + k) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// h = bf16( silu(s_g * u_g) * (s_u * u_u) ), u = 2^xexp[token] * sum_z P
// (pieces in order; the power-of-two factor undoes the fp16 staging of x
// exactly).  h goes to Hb (bf16) and the largest exponent field of each slot
// to hmax[slot] (zeroed by k_dprep).  Block (chunk, slot): the slot's expert
// and shift are looked up once, each thread takes 4 consecutive channels
// (16-byte loads of every piece), and one atomic per block publishes the
// block's maximum.
constexpr int kSwigluChunk = 1024;  // channels per block (256 threads x 4)

__global__ void __launch_bounds__(256)
    k_swiglu(const float* __restrict__ P, int S, int64_t A, int64_t f, int E, int top_k,
             const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm,
             const int32_t* __restrict__ xexp, const float* __restrict__ sgu,
             uint16_t* __restrict__ Hb, int32_t* __restrict__ hmax) {
    __shared__ int s_e;
    __shared__ float s_sx;
    __shared__ int red[8];
    const int64_t n = (int64_t)blockIdx.x * kSwigluChunk + threadIdx.x * 4;
    // The slot's expert, its token's shift and the channel scales depend only
    // on the grouping kernel's tables, complete before the gate/up GEMV (the
    // kernel this one follows) started: the first slot's lookups run before
    // the wait, which only the partial sums P need.
    float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
    auto lookup = [&](int slot) {
        if (threadIdx.x == 0) {
            int e = 0;
            while (e + 1 < E && offsets[e + 1] <= slot) ++e;
            s_e = e;
            const int a = JMOE_CHECK(slot < A) ? perm[slot] : 0;
            s_sx = ldexpf(1.0f, xexp[JMOE_CHECK(a >= 0 && a < A) ? a / top_k : 0]);
        }
        __syncthreads();
        if (n < f) {
            const float* sg = sgu + (int64_t)s_e * 2 * f;
            s0 = __ldg(reinterpret_cast<const float4*>(sg + n));
            s1 = __ldg(reinterpret_cast<const float4*>(sg + f + n));
        }
    };
    const int used = offsets[E];  // dropped assignments leave trailing slots unused
    int slot = blockIdx.y;
    if (slot < used) lookup(slot);
    pdl_wait();
    pdl_launch_dependents();
    for (; slot < used; slot += gridDim.y) {
        int ex = 0;
        if (n < f && JMOE_CHECK(slot < A)) {
            const float sx = s_sx;
            float vg[4] = {0.f, 0.f, 0.f, 0.f}, vu[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int z = 0; z < S; ++z) {
                const float* row = P + ((int64_t)z * A + slot) * 2 * f;
                const float4 g = __ldg(reinterpret_cast<const float4*>(row + n));
                const float4 u = __ldg(reinterpret_cast<const float4*>(row + f + n));
                vg[0] += g.x; vg[1] += g.y; vg[2] += g.z; vg[3] += g.w;
                vu[0] += u.x; vu[1] += u.y; vu[2] += u.z; vu[3] += u.w;
            }
            const float sgv[4] = {s0.x, s0.y, s0.z, s0.w}, suv[4] = {s1.x, s1.y, s1.z, s1.w};
            uint16_t hb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                hb[i] = __bfloat16_as_ushort(__float2bfloat16_rn(
                    silu_f32(sgv[i] * (vg[i] * sx)) * (suv[i] * (vu[i] * sx))));
                ex = max(ex, (int)((hb[i] >> 7) & 0xff));
            }
            *reinterpret_cast<uint2*>(Hb + (int64_t)slot * f + n) =
                make_uint2(hb[0] | ((uint32_t)hb[1] << 16), hb[2] | ((uint32_t)hb[3] << 16));
        }
        const int m = block_max_int(ex, red);  // ends with a barrier: s_e, s_sx reusable
        if (threadIdx.x == 0 && m > 0) atomicMax(&hmax[slot], m);
        if (slot + (int)gridDim.y < used) lookup(slot + (int)gridDim.y);
    }
}

// H16[slot][n] = fp16( Hb[slot][n] * 2^-hexp ), hexp = row_shift(hmax[slot]):
// the bf16 values are kept exactly (8 significant bits, row maximum brought
// into [2^14, 2^15)).
__global__ void __launch_bounds__(256)
    k_h16(const uint16_t* __restrict__ Hb, int64_t f, int64_t A, const int32_t* __restrict__ offsets,
          int E, const int32_t* __restrict__ hmax, uint16_t* __restrict__ H16) {
    pdl_wait();
    // only after the wait: the down GEMV relies on it (it reads the grouping
    // tables before its own wait)
    pdl_launch_dependents();
    const int64_t total = (int64_t)offsets[E] * f / 2;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < total;
         v += (int64_t)gridDim.x * blockDim.x) {
        const int slot = (int)((2 * v) / f);
        if (!JMOE_CHECK(slot < A)) break;
        const float scale = ldexpf(1.0f, -row_shift(hmax[slot]));
        const uint32_t u = reinterpret_cast<const uint32_t*>(Hb)[v];
        const __half2 h = __floats2half2_rn(__uint_as_float(u << 16) * scale,
                                            __uint_as_float(u & 0xffff0000u) * scale);
        reinterpret_cast<uint32_t*>(H16)[v] = *reinterpret_cast<const uint32_t*>(&h);
    }
}

// out[t][m] = bf16( sum_j g_tj * (s_d[e_j][m] * (2^hexp * sum_z P[z][inv[a]][m])) ),
// a = t*top_k + j, hexp = row_shift(hmax[inv[a]]).  Block (chunk, token): the
// token's slots, experts, gates and shifts are looked up once; each thread
// takes 4 consecutive channels (16-byte loads).
constexpr int kCombineChunk = 1024;  // channels per block (256 threads x 4)
constexpr int kMaxTopK = 4;

__global__ void __launch_bounds__(256)
    k_combine(const float* __restrict__ P, int S, int64_t A, int64_t T, int64_t d, int top_k,
              int E, const int32_t* __restrict__ ids, const float* __restrict__ gates,
              const int32_t* __restrict__ inv, const int32_t* __restrict__ hmax,
              const float* __restrict__ sd, uint16_t* __restrict__ out) {
    __shared__ int s_slot[kMaxTopK], s_e[kMaxTopK];
    __shared__ float s_gw[kMaxTopK], s_hs[kMaxTopK];
    const int64_t m = (int64_t)blockIdx.x * kCombineChunk + threadIdx.x * 4;
    // The token's slots, experts, gates, hidden-row shifts and the scales are
    // all final before the down GEMV (the kernel this one follows) starts: the
    // first token's lookups run before the wait, which only the partial sums P
    // need.
    float4 sv[kMaxTopK];
    auto lookup = [&](int64_t t) {
        if (threadIdx.x < top_k) {
            const int64_t a = t * top_k + threadIdx.x;
            const int e = ids[a];
            const int slot = inv[a];
            const bool ok = e >= 0 && e < E && slot >= 0 && JMOE_CHECK(slot < A);
            s_slot[threadIdx.x] = ok ? slot : -1;
            s_e[threadIdx.x] = ok ? e : 0;
            s_gw[threadIdx.x] = gates[a];
            s_hs[threadIdx.x] = ok ? ldexpf(1.0f, row_shift(hmax[slot])) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j)
            if (j < top_k && m < d && s_slot[j] >= 0)
                sv[j] = __ldg(reinterpret_cast<const float4*>(sd + (int64_t)s_e[j] * d + m));
    };
    int64_t t = blockIdx.y;
    if (t < T) lookup(t);
    pdl_wait();
    pdl_launch_dependents();
    for (; t < T; t += gridDim.y) {
        if (m < d) {
            float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                const int slot = j < top_k ? s_slot[j] : -1;
                if (slot < 0) continue;
                float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                for (int z = 0; z < S; ++z) {
                    const float4 q = __ldg(
                        reinterpret_cast<const float4*>(P + ((int64_t)z * A + slot) * d + m));
                    y[0] += q.x; y[1] += q.y; y[2] += q.z; y[3] += q.w;
                }
                const float hs = s_hs[j];
                const float gw = s_gw[j];
                o[0] += gw * (sv[j].x * (y[0] * hs));
                o[1] += gw * (sv[j].y * (y[1] * hs));
                o[2] += gw * (sv[j].z * (y[2] * hs));
                o[3] += gw * (sv[j].w * (y[3] * hs));
            }
            uint2 r;
            r.x = pack_bf16x2(o[0], o[1]);
            r.y = pack_bf16x2(o[2], o[3]);
            *reinterpret_cast<uint2*>(out + t * d + m) = r;
        }
        if (t + (int64_t)gridDim.y < T) {
            __syncthreads();  // the next token's lookups overwrite the shared values
            lookup(t + gridDim.y);
        }
    }
}

int grid_for(int64_t work, int num_sms, int per_sm) {
    int64_t blocks = (work + 255) / 256;
    const int64_t cap = (int64_t)num_sms * per_sm;
    if (blocks > cap) blocks = cap;
    return (int)(blocks < 1 ? 1 : blocks);
}

// One full wave: the resident CTAs per SM at the kernel's register and
// shared-memory use.
template <int MODE, int NCH>
int gemv_grid(int num_sms) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gemv<MODE, NCH>,
                                                      kWarpsPerBlock * 32,
                                                      gemv_smem<MODE>()) != cudaSuccess ||
        per_sm < 1)
        per_sm = 2;
    return num_sms * per_sm;
}

template <int MODE, int NCH>
cudaError_t launch_gemv(const GemvParams& p, int num_sms, cudaStream_t stream) {
    // int8 weights, one 4 KB box per ring slot, 128-byte swizzle.  gate/up
    // [E][2f][d] seen as 4-D [E][2][f][d]: box 128 bytes x 16 rows x both
    // halves; down [E*d][f]: box 128 bytes x 32 rows.
    CUtensorMap map;
    bool ok;
    if (MODE == kGateUp) {
        const uint64_t K = (uint64_t)p.d, f = (uint64_t)p.f;
        const uint64_t dims[4] = {K, f, 2, (uint64_t)p.E};
        const uint64_t strides[3] = {K, f * K, 2 * f * K};
        const uint32_t box[4] = {128, 16, 2, 1};
        ok = encode_4d_u8(&map, p.w, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
    } else {
        ok = encode_2d(&map, p.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)p.E * p.d,
                       (uint64_t)p.f, 32, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    if (!ok) return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(k_gemv<MODE, NCH>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           gemv_smem<MODE>());
    if (err != cudaSuccess) return err;
    return launch_pdl(k_gemv<MODE, NCH>, dim3(gemv_grid<MODE, NCH>(num_sms)),
                      dim3(kWarpsPerBlock * 32), gemv_smem<MODE>(), stream, map, p);
}

template <int NCH>
cudaError_t launch_decode_nch(const DecodeArgs& a, cudaStream_t stream) {
    GemvParams p{};
    p.E = a.E;
    p.top_k = a.top_k;
    p.d = a.d;
    p.f = a.f;
    p.A = a.A;
    p.T = a.T;
    p.offsets = a.offsets;
    p.perm = a.perm;
    p.err = a.err;
    p.wait_cycles = a.wait_cycles > 0 ? a.wait_cycles : sm100::kWaitCycles;
    p.fault = a.fault;
    p.w = a.wgu;
    p.S = a.split_gu;
    p.b_src = static_cast<const uint16_t*>(a.x16);
    p.P = a.P_gu;
    if (a.mark) a.mark(0, false, stream);
    const cudaError_t prep = launch_pdl(
        k_dprep, dim3((unsigned)(a.T + 1)), dim3(kPermuteThreads), 0, stream,
        static_cast<const uint16_t*>(a.x), a.T, a.d, static_cast<uint16_t*>(a.x16), a.xexp,
        a.hmax, a.ids, a.E, a.top_k, a.offsets, a.perm, a.inv, a.err);
    if (a.mark) a.mark(0, true, stream);
    if (prep != cudaSuccess) return prep;
    if (a.mark) a.mark(2, false, stream);
    cudaError_t err = launch_gemv<kGateUp, NCH>(p, a.num_sms, stream);
    if (a.mark) a.mark(2, true, stream);
    if (a.mark) a.mark(5, false, stream);
    if (err == cudaSuccess) {
        err = launch_pdl(k_swiglu,
                         dim3((unsigned)((a.f + kSwigluChunk - 1) / kSwigluChunk),
                              (unsigned)(a.A < 65535 ? a.A : 65535)),
                         dim3(256), 0, stream, static_cast<const float*>(a.P_gu), a.split_gu,
                         a.A, a.f, a.E, a.top_k, a.offsets, a.perm, a.xexp, a.sgu,
                         static_cast<uint16_t*>(a.Hb), a.hmax);
        if (err == cudaSuccess)
            err = launch_pdl(k_h16, dim3(grid_for(a.A * a.f / 2, a.num_sms, 8)), dim3(256), 0,
                             stream, static_cast<const uint16_t*>(a.Hb), a.f, a.A, a.offsets, a.E,
                             a.hmax, static_cast<uint16_t*>(a.H));
    }
    if (a.mark) a.mark(5, true, stream);
    if (err != cudaSuccess) return err;
    p.w = a.wd;
    p.fault = 0;
    p.S = a.split_d;
    p.b_src = static_cast<const uint16_t*>(a.H);
    p.P = a.P_d;
    if (a.mark) a.mark(3, false, stream);
    err = launch_gemv<kDown, NCH>(p, a.num_sms, stream);
    if (a.mark) a.mark(3, true, stream);
    return err;
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

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
    if (a.T == 0) return cudaSuccess;
    // One 8-token tile per pass: a 16-token tile needs 167 registers per
    // thread (3 CTAs per SM instead of 4), which costs more than the extra
    // passes of experts with more than 8 tokens, whose weights come from L2.
    cudaError_t err = launch_decode_nch<1>(a, stream);
    if (err != cudaSuccess) return err;
    if (a.mark) a.mark(4, false, stream);
    err = launch_pdl(k_combine,
                     dim3((unsigned)((a.d + kCombineChunk - 1) / kCombineChunk),
                          (unsigned)(a.T < 65535 ? a.T : 65535)),
                     dim3(256), 0, stream, static_cast<const float*>(a.P_d), a.split_d, a.A, a.T,
                     a.d, a.top_k, a.E, a.ids, a.gates, static_cast<const int32_t*>(a.inv),
                     static_cast<const int32_t*>(a.hmax), a.sd, static_cast<uint16_t*>(a.out));
    if (a.mark) a.mark(4, true, stream);
    return err;
}

JMOE_DEFINE_CHECKS_READER(checks_take_decode)

namespace {
// The bounds-check build's self-test: one check that fails (n > 0), no access.
__global__ void k_check_probe(int n) { (void)JMOE_CHECK(n <= 0); }
}  // namespace

bool checks_built() { return JMOE_CHECKS != 0; }

cudaError_t launch_check_probe(cudaStream_t stream) {
    k_check_probe<<<1, 1, 0, stream>>>(1);
    note_launch();
    return cudaGetLastError();
}

}  // namespace jmoe
