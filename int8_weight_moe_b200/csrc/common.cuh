// Device helpers shared by the jmoe kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "kernels.h"

namespace jmoe {

__device__ __forceinline__ void flag_error(unsigned* err, unsigned bit) {
    if (err) atomicOr(err, bit);
}

// Device bounds checks, compiled only into the JMOE_CHECKS=1 build
// (libjmoe_checks.so): JMOE_CHECK(cond) is true when cond holds; when it does
// not, it raises kErrBounds in this translation unit's check word and is
// false, and the caller skips the access.  A check never traps.  In the
// normal build it is the constant true and costs nothing.  Every source file
// with checks defines its reader of the word (JMOE_DEFINE_CHECKS_READER);
// jmoe_last_error reads and clears them all.
#ifndef JMOE_CHECKS
#define JMOE_CHECKS 0
#endif
#if JMOE_CHECKS
namespace {
__device__ unsigned s_check_word;  // one per translation unit
}  // namespace
#define JMOE_CHECK(cond) \
    ((cond) ? true : (atomicOr(&::jmoe::s_check_word, ::jmoe::kErrBounds), false))
#define JMOE_DEFINE_CHECKS_READER(name)                                                      \
    unsigned name() {                                                                        \
        unsigned v = 0;                                                                      \
        if (cudaMemcpyFromSymbol(&v, s_check_word, sizeof(v)) != cudaSuccess) return kErrBounds; \
        if (v) {                                                                             \
            const unsigned z = 0;                                                            \
            cudaMemcpyToSymbol(s_check_word, &z, sizeof(z));                                 \
        }                                                                                    \
        return v;                                                                            \
    }
#else
#define JMOE_CHECK(cond) true
#define JMOE_DEFINE_CHECKS_READER(name) \
    unsigned name() { return 0; }
#endif

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __uint_as_float(((uint32_t)b) << 16);
}

// Two int8 values (bytes 0,1 or 2,3 of `w`) to a packed bf16x2, exactly.
//
// For a byte b (two's complement), let m = b & 0x7f and s = b & 0x80.  The
// bf16 pattern 0x4300 | m is the number 128 + m (exponent 2^7, mantissa m),
// and 0x4300 | s is 128 (s = 0) or 256 (s = 0x80).  Their difference is
// m - 128*[s != 0] = b, which is exactly representable (|b| <= 128 needs 8
// significant bits), so one round-to-nearest bf16x2 subtraction is exact.
// Cost: one byte permute, two logic ops and one bf16x2 subtract per pair.
template <int kHigh>
__device__ __forceinline__ uint32_t i8x2_to_bf16x2(uint32_t w) {
    // byte layout of t: [b_lo, 0x43, b_hi, 0x43] -> halves 0x43bb
    const uint32_t t = __byte_perm(w, 0x43u, kHigh ? 0x4342u : 0x4140u);
    const uint32_t v = t & 0xff7fff7fu;                // 0x43 | m  -> 128 + m
    const uint32_t c = (t & 0x00800080u) | 0x43004300u;  // 128 or 256
    __nv_bfloat162 r = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&v),
                               *reinterpret_cast<const __nv_bfloat162*>(&c));
    return *reinterpret_cast<uint32_t*>(&r);
}

// Four int8 values (one 32-bit word) to two packed f16x2 words, exactly.
//
// u = b + 128 (flip the sign bit) is an unsigned byte; the f16 pattern
// 0x6400 | u is 1024 + u (exponent 2^10, ten mantissa bits hold 0..1023), and
// subtracting 1152 = 1024 + 128 (0x6480) gives b exactly.  One logic op per
// word, then one byte permute and one f16x2 subtract per pair.
__device__ __forceinline__ void i8x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t u = w ^ 0x80808080u;
    const uint32_t tlo = __byte_perm(u, 0x64646464u, 0x4140u);  // [u0, 0x64, u1, 0x64]
    const uint32_t thi = __byte_perm(u, 0x64646464u, 0x4342u);  // [u2, 0x64, u3, 0x64]
    const uint32_t k = 0x64806480u;
    __half2 rl = __hsub2(*reinterpret_cast<const __half2*>(&tlo), *reinterpret_cast<const __half2*>(&k));
    __half2 rh = __hsub2(*reinterpret_cast<const __half2*>(&thi), *reinterpret_cast<const __half2*>(&k));
    lo = *reinterpret_cast<uint32_t*>(&rl);
    hi = *reinterpret_cast<uint32_t*>(&rh);
}

// D = A * B + D for one m16n8k16 tile, f16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4],
                                              uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16-byte asynchronous global -> shared copy (bypasses L1).  src_bytes = 0
// writes 16 zero bytes instead of reading.
__device__ __forceinline__ void cp_async_16(void* dst_smem, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem))),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// Wait until at most N of this thread's committed copy groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// silu(z) = z / (1 + e^-z), with the fast exponential and the fast division
// (a reciprocal and a multiply, within 2 ulp of the quotient in fp32): the
// result is rounded to bf16 (8 significant bits) before anyone reads it.
// For z < -88, e^-z overflows to inf and the quotient is 0.
__device__ __forceinline__ float silu_f32(float z) {
    return __fdividef(z, 1.0f + __expf(-z));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&r);
}

// Programmatic dependent launch.  pdl_wait: block until the preceding kernel
// on the stream (launched before this one with the programmatic-serialisation
// attribute set on this launch) has completed and its writes are visible; a
// no-op when this kernel was launched without that attribute.
// pdl_launch_dependents: let the next such kernel start launching once every
// CTA of this grid has executed it (or exited), so its launch overlaps this
// kernel's tail; it grants no access to this kernel's results.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous kernel on the stream is still finishing; every kernel
// launched this way calls pdl_wait() before it reads anything the previous
// kernels wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    note_launch();
    return e;
}

struct GemvParams {
    int E, top_k, S;           // experts, experts per token, K pieces
    int64_t d, f;
    const int8_t* w;           // gate/up [E][2f][d] or down [E][d][f]
    const int32_t* offsets;    // [E+1]
    const int32_t* perm;       // [A]
    const uint16_t* b_src;     // x [T][d] (gate/up) or H [A][f] (down)
    float* P;                  // partial sums [S][A][cols]
    int64_t A;                 // assignment slots (rows of P and H)
    int64_t T;                 // tokens (rows of the gate/up activation operand)
    unsigned* err;
    long long wait_cycles;     // bound of every mbarrier wait (SM cycles)
    int fault;                 // test hook: warp 0 of block 0 never issues its first copy
};

}  // namespace jmoe
