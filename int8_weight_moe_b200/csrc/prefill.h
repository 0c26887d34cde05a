// Internal interface of the tensor-core (tcgen05 / TMEM) expert path.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"

namespace jmoe {

struct PrefillArgs {
    const void* x;                 // bf16 [T][d]
    int64_t T, A, d, f;
    int E, top_k;
    const int8_t* wgu;             // int8 [E][2f][d]
    const float* sgu;              // [E][2f]
    const int8_t* wd;              // int8 [E][d][f]
    const float* sd;               // [E][d]
    const int32_t* ids;            // [T][top_k]
    const float* gates;            // [T][top_k]
    const int32_t* offsets;        // [E+1]
    const int32_t* padded_offsets; // [E+1], multiples of kPrefillTileM
    const int32_t* perm;           // [A]
    const int32_t* inv;            // [A]
    void* xperm;                   // bf16 [rows_padded][d]  (workspace)
    void* H;                       // bf16 [rows_padded][f]  (workspace)
    float* Yg;                     // fp32 [A][d]            (workspace)
    int64_t rows_padded;
    void* out;                     // bf16 [T][d]
    int num_sms;
    unsigned* err;
    StageMark mark;
    bool dense;                    // one expert, every token routed to it with gate 1
    long long wait_cycles;         // bound of the kernels' mbarrier waits (0: the default)
    int fault_tile;                // test hook (< 0: off): the gate/up GEMM's weight
                                   // producers stop before this tile
};

bool prefill_available();
cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t stream);

}  // namespace jmoe
