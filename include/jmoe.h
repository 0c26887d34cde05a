/*
 * jmoe -- the ExpertsInt8 mixture-of-experts layer on NVIDIA B200 (sm_100a).
 *
 * C ABI of libjmoe.so.  Plain pointers and sizes only; no CUDA or PyTorch
 * types appear in the signatures.  A `stream` argument is a cudaStream_t
 * passed as `void*` (NULL = the legacy default stream).
 *
 * The method (sources cited by page title and section):
 *  - "Jamba-1.5: Hybrid Transformer-Mamba Models at Scale" (paper summary,
 *    arXiv 2408.12570), section "ExpertsInt8 Quantization (Section 3.1)":
 *    step 1, MoE and MLP weights are quantised BF16 -> INT8 once at load time
 *    without calibration; step 2, they are stored as INT8; step 3, they are
 *    dequantised back to BF16 inside the fused MoE kernel as they move from
 *    HBM to on-chip memory; step 4, activations stay BF16.
 *  - same page, section "The Jamba Hybrid Block Structure": the MoE layer
 *    output MoE(x) = sum over the top-2 experts of g_i(x) * Expert_i(x),
 *    16 experts.  (The library takes 1..64 experts and top-k 1..4.)
 *  - "Jamba: A Hybrid Transformer-Mamba Language Model" (paper summary,
 *    arXiv 2403.19887), section "Mixture-of-Experts (MoE) in Jamba: Router,
 *    Top-K, and Load Balancing": g = softmax(W_r h), top-K selection, and
 *    y = sum over the selected set of g_i * Expert_i(h) with g renormalised
 *    over the selected set; its layer list: experts are MLPs with SwiGLU.
 *
 * Conventions shared by every call:
 *  - Ownership: the caller owns every buffer.  The library never allocates,
 *    frees or synchronises on these calls (jmoe_last_error excepted); all
 *    work is enqueued on `stream` in order and may be captured in a CUDA graph.
 *  - Layouts are row-major.  A weight row is one output channel and its
 *    elements run along the input dimension (the contraction dimension is
 *    contiguous).  bf16 buffers hold IEEE bfloat16 bit patterns.
 *  - Pointers named *device* must be device-accessible CUDA allocations and
 *    16-byte aligned; d_model and d_ff must be multiples of 64.
 *  - Argument and shape errors return a status before anything is launched.
 *    A failed launch returns JMOE_ECUDA.  Conditions only the device can see
 *    (an expert id out of range, a bounded wait that ran out) set a sticky
 *    device error word that jmoe_last_error() reports; kernels never trap.
 *  - Non-finite inputs are outside the contract and are not checked.
 */
#ifndef JMOE_H
#define JMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    JMOE_OK = 0,
    JMOE_EINVAL = 1,       /* a null pointer, a negative size, an out-of-range count */
    JMOE_EALIGN = 2,       /* a pointer is not 16-byte aligned */
    JMOE_EUNSUPPORTED = 3, /* a shape or option this library does not implement */
    JMOE_EWORKSPACE = 4,   /* workspace smaller than the size query returned */
    JMOE_ECUDA = 5,        /* a CUDA runtime call or launch failed */
    JMOE_ETIMEOUT = 6,     /* (device word) a bounded wait inside a kernel ran out */
    JMOE_EDEVICE = 7,      /* (device word) a kernel saw an invalid expert id */
    JMOE_EBOUNDS = 8       /* (device word) a device bounds check failed; only the
                              JMOE_CHECKS=1 build (libjmoe_checks.so) has them */
} jmoe_status;

/* Which expert-GEMM kernels jmoe_forward / jmoe_mlp_forward use. */
typedef enum {
    JMOE_PATH_AUTO = 0,    /* decode kernels below max(128, k E) assignments, k = 26 per
                              expert at d_model <= 4096, 21 at >= 8192 (linear in between),
                              else tensor-core kernels */
    JMOE_PATH_DECODE = 1,  /* bandwidth-bound GEMV-like kernels (any size; slow when large) */
    JMOE_PATH_PREFILL = 2  /* tcgen05 / TMEM grouped GEMM kernels */
} jmoe_path;

/* The quantised expert weights of one MoE layer (all device pointers).
 *   w_gu : int8  [E][2*d_ff][d_model]  rows 0..d_ff-1 of each expert are the
 *          gate projection, rows d_ff..2*d_ff-1 the up projection
 *   s_gu : fp32  [E][2*d_ff]           one scale per row of w_gu
 *   w_d  : int8  [E][d_model][d_ff]    down projection
 *   s_d  : fp32  [E][d_model]          one scale per row of w_d
 * A row's dequantised weights are q * s (ExpertsInt8 step 3). */
typedef struct {
    int32_t E;       /* number of experts, 1..64 */
    int32_t top_k;   /* experts per token, 1..4, <= E */
    int64_t d_model; /* hidden size, multiple of 64 */
    int64_t d_ff;    /* expert intermediate size, multiple of 64 */
    const int8_t* w_gu;
    const float* s_gu;
    const int8_t* w_d;
    const float* s_d;
    int32_t path;    /* a jmoe_path value */
} jmoe_moe_desc;

/* ExpertsInt8 step 1 (load-time, calibration-free quantisation).
 * w_bf16 : device, bf16 [rows][cols], row = output channel
 * q      : device, int8 [rows][cols]   (written)
 * scales : device, fp32 [rows]         (written)
 * Per row: a = max |w|; s = a / 127 (one correctly rounded fp32 division);
 * q = round-half-even(w / s) (one fp32 division per element) clamped to
 * [-127, 127]; an all-zero row gets s = 0, q = 0.  cols must be a multiple
 * of 8 (16-byte rows of bf16); rows >= 0 (0 is a no-op). */
jmoe_status jmoe_quantize(const void* w_bf16, int64_t rows, int64_t cols, int8_t* q,
                          float* scales, void* stream);

/* Router (Jamba summary, "Router mechanism" and "Top-K selection").
 * x_bf16   : device, bf16 [T][d]
 * w_router : device, fp32 [E][d]
 * bias     : device, fp32 [E] added to the logits, or NULL (the pages' router
 *            has no bias; it exists to build skewed-routing workloads)
 * topk_ids : device, int32 [T][top_k] (written) largest logit first, ties to
 *            the lower expert index
 * topk_w   : device, fp32 [T][top_k]  (written) softmax probabilities of the
 *            selected experts renormalised to sum to 1 (1.0 when top_k = 1)
 * logits   : device, fp32 [T][E] (written) or NULL
 * Logits are fp64 dot products summed in a fixed order (lane j of 32 sums
 * the elements k = j mod 32 in ascending k, then a halving tree over the 32
 * lanes), plus the bias, rounded once to fp32; selection uses these fp32
 * logits, so ids are reproducible bit for bit.  E in 1..64, top_k in 1..4
 * (<= E), d a multiple of 64, T >= 0. */
jmoe_status jmoe_route(const void* x_bf16, int64_t T, int64_t d, const float* w_router,
                       const float* bias, int32_t E, int32_t top_k, int32_t* topk_ids,
                       float* topk_w, float* logits, void* stream);

/* jmoe_route with a choice of gates.  The two pages differ here: the Jamba
 * summary ("Top-K selection") renormalises the selected probabilities over
 * the selected set, the Jamba-1.5 summary ("The Jamba Hybrid Block
 * Structure") calls the gates softmax-normalised.  flags = 0 gives the
 * renormalised gates of jmoe_route; JMOE_ROUTE_SOFTMAX_GATES gives the plain
 * softmax probability (over all E experts) of each selected expert.  Other
 * bits are JMOE_EINVAL.  Everything else is as jmoe_route. */
#define JMOE_ROUTE_SOFTMAX_GATES 1u
jmoe_status jmoe_route_ex(const void* x_bf16, int64_t T, int64_t d, const float* w_router,
                          const float* bias, int32_t E, int32_t top_k, uint32_t flags,
                          int32_t* topk_ids, float* topk_w, float* logits, void* stream);

/* RMSNorm ("Jamba: A Hybrid Transformer-Mamba Language Model", paper
 * summary: section "The major components and their responsibilities" places
 * an RMSNorm at the input of the block's modules; section "Training
 * Infrastructure and Stabilization Techniques" defines RMSNorm(x) =
 * x / sqrt(mean(x^2) + eps) * gamma).  Every rounding is fixed, so the
 * routing that follows is reproducible bit for bit:
 *   ss = sum of x_k^2 in fp64 in the router's order (lane j of 32 sums
 *        k = j mod 32 ascending, then a halving tree over the lanes);
 *   r  = 1 / sqrt(ss / d + eps), IEEE-rounded fp64 steps;
 *   y_k = bf16((x_k * r) * gamma_k), fp64 products rounded once to bf16.
 * x_bf16 : device, bf16 [T][d];  gamma_bf16 : device, bf16 [d]
 * y_bf16 : device, bf16 [T][d] (written; must not overlap x)
 * eps >= 0 and finite; d a multiple of 64; all pointers 16-byte aligned. */
jmoe_status jmoe_rmsnorm(const void* x_bf16, int64_t T, int64_t d, const void* gamma_bf16,
                         float eps, void* y_bf16, void* stream);

/* RMSNorm, then the router on the normalised rows: the pre-MoE prologue of a
 * Jamba MoE layer.  y_bf16 receives the normalised rows (the expert input);
 * the routing outputs are those of jmoe_route_ex on y.  For few tokens the
 * normalisation is fused into the router kernel; otherwise jmoe_rmsnorm
 * runs first.  Arguments as jmoe_rmsnorm and jmoe_route_ex. */
jmoe_status jmoe_rmsnorm_route(const void* x_bf16, int64_t T, int64_t d, const void* gamma_bf16,
                               float eps, void* y_bf16, const float* w_router, const float* bias,
                               int32_t E, int32_t top_k, uint32_t flags, int32_t* topk_ids,
                               float* topk_w, float* logits, void* stream);

/* Grouping of the T*top_k token->expert assignments by expert (the dispatch
 * step the fused MoE kernel performs; Jamba-1.5 summary, "Innovation 2").
 * Assignment a = t*top_k + j.  offsets: device int32 [E+1] (written),
 * exclusive prefix of the per-expert counts (offsets[E] = T*top_k); perm:
 * device int32 [T*top_k] (written), the assignments of expert 0 in
 * ascending a, then expert 1, ...; inv: device int32 [T*top_k] (written),
 * inv[perm[i]] = i.  Deterministic and bit-exact.  An id outside [0, E)
 * sets JMOE_EDEVICE in the device error word and the assignment is dropped.
 * A single thread block does the work (T*top_k up to 2^24).  E in 1..64,
 * top_k in 1..4. */
jmoe_status jmoe_permute(const int32_t* topk_ids, int64_t T, int32_t top_k, int32_t E,
                         int32_t* offsets, int32_t* perm, int32_t* inv, void* stream);

/* Workspace bytes jmoe_forward needs for T tokens with this descriptor. */
jmoe_status jmoe_forward_workspace_size(const jmoe_moe_desc* desc, int64_t T, size_t* bytes);

/* The MoE layer forward (ExpertsInt8 steps 3-4 with the MoE equation).
 * x_bf16   : device, bf16 [T][d_model]
 * topk_ids : device, int32 [T][top_k] (from jmoe_route or the caller)
 * topk_w   : device, fp32 [T][top_k]
 * out_bf16 : device, bf16 [T][d_model] (written)
 * workspace: device, >= jmoe_forward_workspace_size bytes, 256-byte aligned
 * out_t = sum_j topk_w[t][j] * Expert_{topk_ids[t][j]}(x_t), where
 * Expert_e(x) = W_d (silu(W_g x) * (W_u x)) with W = q * s.  The hidden
 * activation between the two projections is stored as bf16 and every dot
 * product accumulates in fp32.  T >= 0 (0 is a no-op). */
jmoe_status jmoe_forward(const jmoe_moe_desc* desc, const void* x_bf16, int64_t T,
                         const int32_t* topk_ids, const float* topk_w, void* out_bf16,
                         void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes jmoe_mlp_forward needs. */
jmoe_status jmoe_mlp_workspace_size(int64_t T, int64_t d_model, int64_t d_ff, int32_t path,
                                    size_t* bytes);

/* The dense SwiGLU MLP with INT8 weights (ExpertsInt8 quantises "MoE and
 * MLP weights"): out_t = Expert(x_t) with one expert (E = 1, gate 1).
 * w_gu int8 [2*d_ff][d_model], s_gu fp32 [2*d_ff], w_d int8 [d_model][d_ff],
 * s_d fp32 [d_model]; other arguments as jmoe_forward. */
jmoe_status jmoe_mlp_forward(const void* x_bf16, int64_t T, int64_t d_model, int64_t d_ff,
                             const int8_t* w_gu, const float* s_gu, const int8_t* w_d,
                             const float* s_d, void* out_bf16, void* workspace,
                             size_t ws_bytes, int32_t path, void* stream);

/* Allocation-free variant of jmoe_forward.
 * This call has no counterpart in the method's sources; it exists for callers
 * that cannot obtain device memory at call time -- for example a plugin inside
 * a serving engine whose memory planner has already handed every byte of HBM
 * to its own pool, or a latency-critical path that must not pay the implicit
 * device-wide synchronisation cudaMalloc/cudaFree can cause.  Such a caller
 * still passes its inputs and its output buffer, but no workspace.
 *
 * It runs the decode (GEMV-like) kernels of jmoe_forward, whatever desc->path
 * says, with their scratch (grouping tables, the hidden activations and the
 * split-K partial sums) placed in one fixed array of JMOE_NOALLOC_SCRATCH_BYTES
 * bytes that is part of the library image: every GPU on which the library is
 * used holds that array until the process exits.  The call allocates nothing
 * and calls no allocating routine.
 *  - Size limit: if the scratch jmoe_forward_workspace_size would report for
 *    the decode kernels exceeds JMOE_NOALLOC_SCRATCH_BYTES, the call returns
 *    JMOE_EWORKSPACE before launching anything.  Roughly: the hidden
 *    activations take T*top_k * d_ff * 4 bytes (bf16 and fp16 copies) and
 *    the split-K partial sums of the two projections, which share one
 *    buffer, up to 16 MB (for example, 32 tokens at d_model 8192, d_ff 24576
 *    and top-2 fit; 64 tokens at those sizes do not).
 *  - The first call on a device looks up the array's device address for that
 *    device (with that device current) and caches it; make that first call
 *    before capturing any stream work on the device.  After a device reset
 *    (cudaDeviceReset) the device has a new context, and the next call looks
 *    the address up again: the cached one is tied to the context it came from.
 *  - All calls share the one array and it keeps whatever the last call left
 *    there.  Nothing in it has to start at zero for these kernels, so nothing
 *    is cleared.  Two calls whose work overlaps on the GPU (different
 *    streams, or different host threads without ordering) race on the array
 *    and give wrong results: order them on one stream or synchronise.
 * Arguments, layouts, validation and results are those of jmoe_forward. */
#define JMOE_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
jmoe_status jmoe_forward_noalloc(const jmoe_moe_desc* desc, const void* x_bf16, int64_t T,
                                 const int32_t* topk_ids, const float* topk_w, void* out_bf16,
                                 void* stream);

/* Expert parallelism ("Jamba: A Hybrid Transformer-Mamba Language Model",
 * paper summary, section "Training Infrastructure and Stabilization
 * Techniques": expert parallelism with all-to-all communication that routes
 * tokens to the GPU holding their selected experts; section
 * "Mixture-of-Experts (MoE) in Jamba: Router, Top-K, and Load Balancing":
 * MoE layers need all-to-all communication under expert parallelism).
 * The E experts are split over G ranks: rank g owns the E/G consecutive
 * experts g*E/G .. (g+1)*E/G - 1.  One layer forward on rank g is
 *   jmoe_ep_dispatch  -> all-to-all of the send rows (and their local expert
 *   ids) -> jmoe_forward on the received rows with the owned experts' weights
 *   (desc.E = E/G, top_k = 1, gates 1) -> all-to-all back -> jmoe_ep_combine.
 * The library does not communicate; the exchange is the caller's (the Python
 * binding uses torch.distributed's all_to_all_single).
 *
 * jmoe_ep_dispatch groups the T*top_k assignments by expert (as jmoe_permute,
 * which orders them by owner rank too) and builds the send buffer:
 *   offsets   : device int32 [E+1] (written), as jmoe_permute; the rows for
 *               rank r are offsets[r*E/G] .. offsets[(r+1)*E/G] - 1
 *   perm, inv : device int32 [T*top_k] (written), as jmoe_permute
 *   x_send    : device bf16 [T*top_k][d] (written up to row offsets[E] - 1):
 *               x_send[i] = x[perm[i] / top_k]
 *   local_ids : device int32 [T*top_k] (written): expert of perm[i] minus the
 *               owner's first expert
 * x_bf16 bf16 [T][d], topk_ids int32 [T][top_k].  E in 1..64, G >= 1 with
 * E % G == 0, top_k in 1..4, d a multiple of 64.  Ids outside [0, E) are
 * dropped (JMOE_EDEVICE in the device error word). */
jmoe_status jmoe_ep_dispatch(const void* x_bf16, int64_t T, int64_t d, const int32_t* topk_ids,
                             int32_t top_k, int32_t E, int32_t G, int32_t* offsets,
                             int32_t* perm, int32_t* inv, void* x_send, int32_t* local_ids,
                             void* stream);

/* The combine after the return exchange: y_back bf16 [T*top_k][d] holds the
 * expert output of send row i in row i; out_bf16 [T][d] (written):
 *   out[t] = bf16( sum_j topk_w[t][j] * y_back[inv[t*top_k + j]] )
 * summed in fp32 in assignment order (rows with inv < 0 add nothing).
 * inv int32 [T*top_k] from jmoe_ep_dispatch, topk_w fp32 [T][top_k]. */
jmoe_status jmoe_ep_combine(const void* y_back, const int32_t* inv, const float* topk_w,
                            int64_t T, int64_t d, int32_t top_k, void* out_bf16, void* stream);

/* Stage timing hook (diagnostics).  Registers `n` CUDA events (cudaEvent_t
 * handles passed as void*) that the following jmoe_forward / jmoe_mlp_forward
 * calls record on their stream around their kernels: events[2*i] before and
 * events[2*i+1] after stage i, where the stages are 0 = grouping by expert
 * (on the decode path together with the fp16 token rows), 1 = row gather
 * (tensor-core path), 2 = gate/up GEMM (on the tensor-core path with SwiGLU
 * in its epilogue), 3 = down GEMM, 4 = combine, 5 = SwiGLU and the fp16
 * hidden rows (decode path).
 * Stages that do not run record nothing, and neither do stages whose two
 * entries are NULL (so a caller can time one stage without the cost of the
 * other records); one NULL entry of a pair is JMOE_EINVAL.  n = 0 or
 * events = NULL switches recording off.  The registration is process-wide and
 * not thread-safe; the caller keeps the events alive.  n must be 0 or 12. */
jmoe_status jmoe_profile_events(void* const* events, int32_t n);

/* Launch counter (diagnostics; the pages have no counterpart).  Stores in
 * *count the number of kernels this library has launched in this process
 * since it was loaded, over all devices and host threads; a caller takes the
 * difference around a region to count the launches inside it.  Never
 * synchronises.  Returns JMOE_EINVAL when count is NULL. */
jmoe_status jmoe_launch_count(uint64_t* count);

/* Test hook (diagnostics; the pages have no counterpart): exercises the
 * bounded waits without any GPU fault.  Arms a stall for the next
 * jmoe_forward / jmoe_mlp_forward call in the process (one call only, then it
 * disarms itself):
 *   JMOE_STALL_TENSOR_GEMM: the tensor-core path's gate/up GEMM; its weight
 *     producers stop before their first tile, so the converter warps wait for
 *     copies that never come;
 *   JMOE_STALL_DECODE_GEMV: the decode path's gate/up GEMV; the first warp
 *     never issues its first weight copy, so its consumer waits for nothing.
 * During that call every mbarrier wait of the stalled kernel gives up after
 * wait_cycles SM cycles (1000 .. 8e9; the default bound is about 2 s), the
 * kernel drains the copies it did issue, frees its TMEM and sets
 * JMOE_ETIMEOUT in the device error word; the call's output is undefined.
 * The context stays usable and the next call runs normally.  target 0
 * disarms; other values are JMOE_EINVAL. */
#define JMOE_STALL_TENSOR_GEMM 1
#define JMOE_STALL_DECODE_GEMV 2
jmoe_status jmoe_test_stall(int32_t target, int64_t wait_cycles);

/* Reads and clears the device error word of the current device.  Unlike the
 * other calls it synchronises the device.  Returns JMOE_OK when no kernel
 * has flagged anything since the last call. */
jmoe_status jmoe_last_error(void);

/* Test hook of the bounds-check build (libjmoe_checks.so, compiled with
 * JMOE_CHECKS=1): launches on `stream` a kernel whose single bounds check
 * fails without touching memory, so that the next jmoe_last_error returns
 * JMOE_EBOUNDS.  The normal build has no checks and returns JMOE_EUNSUPPORTED
 * without launching anything.  The pages define no such operation: it tests
 * the library's own fault reporting. */
jmoe_status jmoe_test_check(void* stream);

/* A static, human-readable name for a status. */
const char* jmoe_status_string(jmoe_status status);

/* The CUDA runtime's description of the error behind the calling thread's
 * most recent JMOE_ECUDA ("no CUDA error" if there was none).  Static
 * storage; it stays until a later JMOE_ECUDA on the same thread. */
const char* jmoe_cuda_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* JMOE_H */
