// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace jmoe {

// Counts one kernel launch (process-wide, all devices); every launch site in
// the library calls it right after the launch.
void note_launch();

// Whether the driver's tensor-map encoder could be looked up.
bool tensormap_available();

// TMA tensor map of a row-major 2-D tensor [rows][cols] with boxes of
// box_rows x box_cols elements (false if the driver entry point is missing or
// the encoder rejects the arguments).
bool encode_2d(CUtensorMap* map, const void* base, CUtensorMapDataType type, int elem_bytes,
               uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
               CUtensorMapSwizzle swizzle);

// TMA tensor map of a 4-D byte tensor: dims innermost first, byte strides of
// dims 1..3, box extents innermost first (false as for encode_2d).
bool encode_4d_u8(CUtensorMap* map, const void* base, const uint64_t (&dims)[4],
                  const uint64_t (&strides)[3], const uint32_t (&box)[4],
                  CUtensorMapSwizzle swizzle);

// Bits of the sticky device error word (see jmoe_last_error).
enum : unsigned {
    kErrTimeout = 1u,    // a bounded wait ran out
    kErrBadExpert = 2u,  // an expert id outside [0, E)
    kErrBounds = 4u,     // a device bounds check failed (JMOE_CHECKS build only)
};

// Readers of the per-file device check words of the JMOE_CHECKS build (read
// and clear; 0 in the normal build).  Call with the device current, after a
// synchronisation.
unsigned checks_take_decode();
unsigned checks_take_prefill();
unsigned checks_take_permute();
unsigned checks_take_ep();
// Whether this is the JMOE_CHECKS build, and a kernel whose one check fails
// while touching no memory (the jmoe_test_check hook; a no-op in the normal
// build, which has no checks).
bool checks_built();
cudaError_t launch_check_probe(cudaStream_t stream);

// Largest bound a caller may give the kernels' mbarrier waits (SM cycles,
// about 4 s at 2 GHz).
constexpr long long kMaxWaitCycles = 8000000000LL;

// Rows of the tensor-core path's M tile; expert groups are padded to it.
constexpr int kPrefillTileM = 128;

cudaError_t launch_quantize(const void* w_bf16, int64_t rows, int64_t cols, int8_t* q,
                            float* scales, cudaStream_t stream);

// renorm != 0: the chosen softmax probabilities renormalised over the
// selection; 0: the plain softmax probabilities.
cudaError_t launch_route(const void* x_bf16, int64_t T, int64_t d, const float* w_router,
                         const float* bias, int E, int top_k, int renorm, int32_t* ids,
                         float* gates, float* logits, int num_sms, cudaStream_t stream);
// RMSNorm y = bf16((x * r) * gamma), r = 1/sqrt(mean(x^2) + eps) (fp64, fixed order).
cudaError_t launch_rmsnorm(const void* x_bf16, int64_t T, int64_t d, const void* gamma_bf16,
                           float eps, void* y_bf16, int num_sms, cudaStream_t stream);
// Router on the RMS-normalised rows (written to y_bf16); gamma_bf16 == nullptr
// routes x itself (as launch_route).
cudaError_t launch_norm_route(const void* x_bf16, int64_t T, int64_t d, const void* gamma_bf16,
                              float eps, void* y_bf16, const float* w_router, const float* bias,
                              int E, int top_k, int renorm, int32_t* ids, float* gates,
                              float* logits, int num_sms, cudaStream_t stream);

cudaError_t launch_permute(const int32_t* ids, int64_t A, int E, int pad, int32_t* offsets,
                           int32_t* padded_offsets, int32_t* perm, int32_t* inv, unsigned* err,
                           cudaStream_t stream);

cudaError_t launch_gather_rows(const void* x_bf16, int64_t T, int64_t d, int top_k, int E,
                               const int32_t* offsets, const int32_t* padded_offsets,
                               const int32_t* perm, int64_t max_rows, void* x_perm, int num_sms,
                               cudaStream_t stream);

// Optional stage-timing callback (see jmoe_profile_events).
using StageMark = void (*)(int stage, bool after, cudaStream_t stream);

struct DecodeArgs {
    const void* x;        // bf16 [T][d]
    int64_t T, A, d, f;
    int E, top_k;
    const int8_t* wgu;    // int8 [E][2f][d]
    const float* sgu;     // [E][2f]
    const int8_t* wd;     // int8 [E][d][f]
    const float* sd;      // [E][d]
    const int32_t* ids;   // [T][top_k]
    const float* gates;   // [T][top_k]
    int32_t* offsets;     // [E+1] (workspace, written by the path)
    int32_t* perm;        // [A]   (workspace)
    int32_t* inv;         // [A]   (workspace)
    void* x16;            // fp16 [T][d]: x * 2^-xexp[t] (workspace)
    int32_t* xexp;        // [T] power-of-two shift of each token row (workspace)
    void* Hb;             // bf16 [A][f]: hidden activations, expert-grouped slot order
    void* H;              // fp16 [A][f]: Hb * 2^-shift(hmax[slot]) (workspace)
    int32_t* hmax;        // [A] largest exponent field of each hidden row (workspace)
    float* P_gu;          // fp32 [split_gu][A][2f] partial sums (workspace)
    float* P_d;           // fp32 [split_d][A][d] partial sums (workspace; may alias P_gu)
    int split_gu, split_d;   // K pieces of the two GEMVs
    void* out;            // bf16 [T][d]
    int num_sms;
    StageMark mark;
    unsigned* err;        // device error word
    long long wait_cycles;  // bound of the kernels' mbarrier waits (0: the default)
    int fault;            // test hook: the gate/up GEMV's first warp skips its first copy
};

// K pieces for a decode GEMV: the smallest divisor s of K/64 with s >= want
// (and K/s >= 512 B, s <= cap); if there is none, the largest allowed one.
int decode_split(int64_t K, int64_t want, int64_t cap);
cudaError_t launch_finalize(const float* Y, int64_t T, int64_t d, int top_k, int E,
                            const int32_t* ids, void* out, int num_sms, cudaStream_t stream);
cudaError_t launch_fill_f32(float* p, float v, int64_t n, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);

// Expert parallelism (ep.cu): grouping + send buffer, and the final combine.
cudaError_t launch_ep_dispatch(const void* x, int64_t T, int64_t d, const int32_t* ids, int top_k,
                               int E, int E_local, int32_t* offsets, int32_t* perm, int32_t* inv,
                               void* x_send, int32_t* local_ids, unsigned* err, int num_sms,
                               cudaStream_t stream);
cudaError_t launch_ep_combine(const void* y_back, const int32_t* inv, const float* gates,
                              int64_t T, int64_t d, int top_k, void* out, cudaStream_t stream);

}  // namespace jmoe
