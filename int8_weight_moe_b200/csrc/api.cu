// C ABI of libjmoe.so (declared in include/jmoe.h): argument validation,
// workspace layout and kernel dispatch.  Nothing here allocates, frees or
// synchronises, except jmoe_last_error.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "../../include/jmoe.h"
#include "kernels.h"
#include "prefill.h"

namespace {

__device__ unsigned g_jmoe_err_word;

constexpr int kMaxDevices = 64;
constexpr int kStages = 6;
cudaEvent_t g_stage_events[2 * kStages];
std::atomic<bool> g_profile_on{false};
std::atomic<int> g_num_sms[kMaxDevices];
std::atomic<uint64_t> g_launches{0};

// Test hook (jmoe_test_stall): armed for the next expert forward only.
std::mutex g_stall_mu;
int g_stall_target = 0;
long long g_stall_wait_cycles = 0;

// Takes the armed stall, if any, for this forward (and disarms it).
void take_stall(int& target, long long& wait_cycles) {
    std::lock_guard<std::mutex> lock(g_stall_mu);
    target = g_stall_target;
    wait_cycles = g_stall_wait_cycles;
    g_stall_target = 0;
    g_stall_wait_cycles = 0;
}

// The automatic path: the decode (GEMV-like) kernels while there are fewer
// than max(128, k E) token->expert assignments, the tcgen05 grouped GEMM from
// there on.  The decode kernels re-read an expert's weights (mostly from L2)
// for every pass of 8 of its tokens; the grouped GEMM streams them once but
// pads each expert's rows to 128, so its time is flat at small A.  k falls
// with the width: 26 per expert at d_model 4096 or less, 21 at 8192 or more,
// linear in between.  Measured on the B200 (16 experts, top-2, the forward
// alone): d_model 4096, d_ff 14336: decode 1.167 / 1.313 / 1.724 ms at 320 /
// 384 / 512 assignments against 1.392 / 1.400 / 1.404 ms; d_model 8192, d_ff
// 24576: decode 4.352 / 4.955 ms at 320 / 384 against 4.635 / 4.537 ms.  With
// one expert (the dense MLP) the bound stays 128.
constexpr int64_t kDecodeMinAssignments = 128;

int64_t decode_tokens_per_expert(int64_t d) {
    if (d <= 4096) return 26;
    if (d >= 8192) return 21;
    return 26 - 5 * (d - 4096) / 4096;
}

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

// Unique id of the calling thread's current CUDA context (0 if the driver
// cannot tell).  Device addresses of the library's __device__ arrays belong to
// one context: after cudaDeviceReset the device gets a new primary context,
// and addresses looked up in the old one are stale.
unsigned long long current_context_id() {
    using GetCurrentFn = CUresult (*)(CUcontext*);
    using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of a __device__ symbol in the current context, looked up
// with cudaGetSymbolAddress the first time a device (or, after a device
// reset, its new context) needs it, then cached per device.
struct SymbolCache {
    std::mutex mu;
    unsigned long long ctx[kMaxDevices] = {};
    void* addr[kMaxDevices] = {};
};

void* symbol_address(SymbolCache& c, const void* symbol) {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(c.mu);
    if (c.addr[dev] && c.ctx[dev] == ctx) return c.addr[dev];
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, symbol) != cudaSuccess || !addr) return nullptr;
    c.addr[dev] = addr;
    // the lookup has made the device's context current if nothing had yet
    c.ctx[dev] = current_context_id();
    return addr;
}

SymbolCache g_err_cache;

unsigned* err_word() {
    return static_cast<unsigned*>(symbol_address(g_err_cache, &g_jmoe_err_word));
}

int num_sms() {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return 148;
    int n = g_num_sms[dev].load();
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        g_num_sms[dev].store(n);
    }
    return n;
}

void stage_mark(int stage, bool after, cudaStream_t s) {
    if (g_profile_on.load(std::memory_order_relaxed)) {
        cudaEvent_t ev = g_stage_events[2 * stage + (after ? 1 : 0)];
        if (ev) cudaEventRecord(ev, s);
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The CUDA error behind the calling thread's most recent JMOE_ECUDA.
thread_local cudaError_t t_last_cuda = cudaSuccess;

jmoe_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return JMOE_OK;
    t_last_cuda = e;
    return JMOE_ECUDA;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace carve-up shared by the size query and the forward calls.
struct Workspace {
    size_t offsets, padded_offsets, perm, inv;  // routing tables
    size_t H, Hb, P, x16, xexp, hmax;           // decode path
    int split_gu, split_d;
    size_t xperm, Hp, Yg;                       // tensor-core path
    size_t total;
    int64_t rows_padded;  // upper bound of the padded expert-grouped rows
};

Workspace plan(int64_t T, int64_t A, int E, int64_t d, int64_t f, bool prefill) {
    Workspace w{};
    size_t at = 0;
    auto take = [&](size_t bytes) {
        size_t off = at;
        at = round_up(at + bytes, 256);
        return off;
    };
    w.offsets = take(sizeof(int32_t) * (size_t)(E + 1));
    w.padded_offsets = take(sizeof(int32_t) * (size_t)(E + 1));
    w.perm = take(sizeof(int32_t) * (size_t)A);
    w.inv = take(sizeof(int32_t) * (size_t)A);
    if (!prefill) {
        // K pieces: about 16 work items per warp on a 148-SM GPU for gate/up
        // and 2 for down (measured best: larger down items halve the per-item
        // overhead and the partial sums the combine reads), with the partial
        // sums capped at 16 MB for gate/up and 8 MB for down.  The two GEMVs
        // share one partial-sum buffer: the gate/up sums are used up (SwiGLU)
        // before the down GEMV writes its own.
        const int64_t target_gu = 148LL * 16 * 16, target_d = 148LL * 16 * 2;
        const int64_t touched = A < E ? A : E;
        const int64_t units_gu = touched * (f / 16), units_d = touched * (d / 32);
        const int64_t row_gu = A * 2 * f * (int64_t)sizeof(float);
        const int64_t row_d = A * d * (int64_t)sizeof(float);
        w.split_gu = jmoe::decode_split(d, units_gu > 0 ? (target_gu + units_gu - 1) / units_gu : 1,
                                        row_gu > 0 ? (16LL << 20) / row_gu : 1);
        w.split_d = jmoe::decode_split(f, units_d > 0 ? (target_d + units_d - 1) / units_d : 1,
                                       row_d > 0 ? (8LL << 20) / row_d : 1);
        const size_t pgu = (size_t)w.split_gu * (size_t)row_gu;
        const size_t pd = (size_t)w.split_d * (size_t)row_d;
        w.H = take(sizeof(uint16_t) * (size_t)A * (size_t)f);
        w.Hb = take(sizeof(uint16_t) * (size_t)A * (size_t)f);
        w.x16 = take(sizeof(uint16_t) * (size_t)T * (size_t)d);
        w.xexp = take(sizeof(int32_t) * (size_t)T);
        w.hmax = take(sizeof(int32_t) * (size_t)A);
        w.P = take(pgu > pd ? pgu : pd);
    } else {
        const int64_t tm = jmoe::kPrefillTileM;
        w.rows_padded = (A + (int64_t)E * (tm - 1) + tm - 1) / tm * tm;
        w.xperm = take(sizeof(uint16_t) * (size_t)w.rows_padded * (size_t)d);
        w.Hp = take(sizeof(uint16_t) * (size_t)w.rows_padded * (size_t)f);
        w.Yg = take(sizeof(float) * (size_t)A * (size_t)d);
    }
    w.total = at;
    return w;
}

bool use_prefill(int32_t path, int64_t A, int E, int64_t d) {
    if (path == JMOE_PATH_DECODE) return false;
    if (path == JMOE_PATH_PREFILL) return true;
    const int64_t per_expert = decode_tokens_per_expert(d) * E;
    const int64_t bound = per_expert > kDecodeMinAssignments ? per_expert : kDecodeMinAssignments;
    return A >= bound && jmoe::prefill_available();
}

jmoe_status check_norm(const void* x_bf16, int64_t T, int64_t d, const void* gamma_bf16,
                       float eps, const void* y_bf16) {
    if (T < 0 || d <= 0) return JMOE_EINVAL;
    if (!(eps >= 0.0f) || eps > 3.0e38f) return JMOE_EINVAL;  // negative, NaN or inf
    if (d % 64) return JMOE_EUNSUPPORTED;
    if (T == 0) return JMOE_OK;
    if (!x_bf16 || !gamma_bf16 || !y_bf16) return JMOE_EINVAL;
    if (!aligned16(x_bf16) || !aligned16(gamma_bf16) || !aligned16(y_bf16)) return JMOE_EALIGN;
    const char* xa = static_cast<const char*>(x_bf16);
    const char* ya = static_cast<const char*>(y_bf16);
    const size_t bytes = (size_t)T * (size_t)d * 2;
    if (xa < ya + bytes && ya < xa + bytes) return JMOE_EINVAL;  // overlap
    return JMOE_OK;
}

jmoe_status check_desc(const jmoe_moe_desc* desc) {
    if (!desc) return JMOE_EINVAL;
    if (desc->E < 1 || desc->E > 64) return JMOE_EUNSUPPORTED;
    if (desc->top_k < 1 || desc->top_k > 4 || desc->top_k > desc->E) return JMOE_EUNSUPPORTED;
    if (desc->d_model <= 0 || desc->d_ff <= 0) return JMOE_EINVAL;
    if (desc->d_model % 64 || desc->d_ff % 64) return JMOE_EUNSUPPORTED;
    if (desc->path < JMOE_PATH_AUTO || desc->path > JMOE_PATH_PREFILL) return JMOE_EINVAL;
    if (!desc->w_gu || !desc->s_gu || !desc->w_d || !desc->s_d) return JMOE_EINVAL;
    if (!aligned16(desc->w_gu) || !aligned16(desc->s_gu) || !aligned16(desc->w_d) ||
        !aligned16(desc->s_d))
        return JMOE_EALIGN;
    return JMOE_OK;
}

// The expert MLPs over routed rows, shared by the MoE and dense entries.
jmoe_status run_experts(const jmoe_moe_desc* desc, const void* x, int64_t T,
                        const int32_t* ids, const float* gates, void* out, void* ws,
                        size_t ws_bytes, bool dense, cudaStream_t stream) {
    const int E = desc->E, k = desc->top_k;
    const int64_t A = T * k, d = desc->d_model, f = desc->d_ff;
    const bool prefill = use_prefill(desc->path, A, desc->E, desc->d_model);
    if (prefill && !jmoe::prefill_available()) return JMOE_EUNSUPPORTED;
    const Workspace w = plan(T, A, E, d, f, prefill);
    if (!ws || ws_bytes < w.total) return JMOE_EWORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return JMOE_EALIGN;
    char* base = static_cast<char*>(ws);
    auto at = [&](size_t off) { return static_cast<void*>(base + off); };
    int32_t* offsets = static_cast<int32_t*>(at(w.offsets));
    int32_t* poff = static_cast<int32_t*>(at(w.padded_offsets));
    int32_t* perm = static_cast<int32_t*>(at(w.perm));
    int32_t* inv = static_cast<int32_t*>(at(w.inv));
    unsigned* err = err_word();
    const int sms = num_sms();
    int stall = 0;
    long long wait_cycles = 0;
    take_stall(stall, wait_cycles);

    if (!prefill) {
        // grouping happens inside the decode path's first kernel
        jmoe::DecodeArgs a{};
        a.x = x; a.T = T; a.A = A; a.d = d; a.f = f; a.E = E; a.top_k = k;
        a.wgu = desc->w_gu; a.sgu = desc->s_gu; a.wd = desc->w_d; a.sd = desc->s_d;
        a.ids = ids; a.gates = gates; a.offsets = offsets; a.perm = perm; a.inv = inv;
        a.H = at(w.H); a.Hb = at(w.Hb);
        a.P_gu = static_cast<float*>(at(w.P)); a.P_d = a.P_gu;
        a.split_gu = w.split_gu; a.split_d = w.split_d;
        a.x16 = at(w.x16); a.xexp = static_cast<int32_t*>(at(w.xexp));
        a.hmax = static_cast<int32_t*>(at(w.hmax));
        a.out = out; a.num_sms = sms;
        a.mark = stage_mark;
        a.err = err;
        a.wait_cycles = wait_cycles;
        a.fault = stall == JMOE_STALL_DECODE_GEMV ? 1 : 0;
        return from_cuda(jmoe::launch_decode(a, stream));
    }
    stage_mark(0, false, stream);
    cudaError_t e = jmoe::launch_permute(ids, A, E, jmoe::kPrefillTileM, offsets, poff, perm, inv,
                                         err, stream);
    stage_mark(0, true, stream);
    if (e != cudaSuccess) return JMOE_ECUDA;
    jmoe::PrefillArgs p{};
    p.x = x; p.T = T; p.A = A; p.d = d; p.f = f; p.E = E; p.top_k = k;
    p.wgu = desc->w_gu; p.sgu = desc->s_gu; p.wd = desc->w_d; p.sd = desc->s_d;
    p.ids = ids; p.gates = gates; p.offsets = offsets; p.padded_offsets = poff; p.perm = perm;
    p.inv = inv; p.xperm = at(w.xperm); p.H = at(w.Hp); p.Yg = static_cast<float*>(at(w.Yg));
    p.rows_padded = w.rows_padded; p.out = out; p.num_sms = sms; p.err = err;
    p.mark = stage_mark; p.dense = dense;
    p.wait_cycles = wait_cycles;
    p.fault_tile = stall == JMOE_STALL_TENSOR_GEMM ? 0 : -1;
    return from_cuda(jmoe::launch_prefill(p, stream));
}

// Scratch of jmoe_forward_noalloc: a fixed array in the library image, one
// per device.  In host code its name is only a stand-in for the symbol; the
// device address is looked up per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[JMOE_NOALLOC_SCRATCH_BYTES];
SymbolCache g_noalloc_cache;

// The array's device address on the current device (looked up once per
// device and context, with that device current), or nullptr if the lookup
// failed.
void* noalloc_scratch() { return symbol_address(g_noalloc_cache, &g_noalloc_scratch); }

}  // namespace

void jmoe::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

extern "C" {

jmoe_status jmoe_launch_count(uint64_t* count) {
    if (!count) return JMOE_EINVAL;
    *count = g_launches.load(std::memory_order_relaxed);
    return JMOE_OK;
}

const char* jmoe_status_string(jmoe_status s) {
    switch (s) {
        case JMOE_OK: return "JMOE_OK";
        case JMOE_EINVAL: return "JMOE_EINVAL: invalid argument";
        case JMOE_EALIGN: return "JMOE_EALIGN: pointer not aligned";
        case JMOE_EUNSUPPORTED: return "JMOE_EUNSUPPORTED: unsupported shape or option";
        case JMOE_EWORKSPACE: return "JMOE_EWORKSPACE: workspace too small";
        case JMOE_ECUDA: return "JMOE_ECUDA: CUDA call or launch failed";
        case JMOE_ETIMEOUT: return "JMOE_ETIMEOUT: a bounded device wait ran out";
        case JMOE_EDEVICE: return "JMOE_EDEVICE: invalid expert id seen on the device";
        case JMOE_EBOUNDS: return "JMOE_EBOUNDS: a device bounds check failed";
    }
    return "unknown jmoe_status";
}

jmoe_status jmoe_test_check(void* stream) {
    if (!jmoe::checks_built()) return JMOE_EUNSUPPORTED;
    return from_cuda(jmoe::launch_check_probe((cudaStream_t)stream));
}

const char* jmoe_cuda_error_string(void) {
    return t_last_cuda == cudaSuccess ? "no CUDA error" : cudaGetErrorString(t_last_cuda);
}

jmoe_status jmoe_quantize(const void* w_bf16, int64_t rows, int64_t cols, int8_t* q,
                          float* scales, void* stream) {
    if (rows < 0 || cols <= 0) return JMOE_EINVAL;
    if (cols % 8) return JMOE_EUNSUPPORTED;
    if (rows == 0) return JMOE_OK;
    if (rows > 0x7fffffffLL) return JMOE_EUNSUPPORTED;
    if (!w_bf16 || !q || !scales) return JMOE_EINVAL;
    if (!aligned16(w_bf16) || !aligned16(q) || !aligned16(scales)) return JMOE_EALIGN;
    return from_cuda(jmoe::launch_quantize(w_bf16, rows, cols, q, scales, (cudaStream_t)stream));
}

jmoe_status jmoe_route(const void* x_bf16, int64_t T, int64_t d, const float* w_router,
                       const float* bias, int32_t E, int32_t top_k, int32_t* topk_ids,
                       float* topk_w, float* logits, void* stream) {
    return jmoe_route_ex(x_bf16, T, d, w_router, bias, E, top_k, 0u, topk_ids, topk_w, logits,
                         stream);
}

jmoe_status jmoe_route_ex(const void* x_bf16, int64_t T, int64_t d, const float* w_router,
                          const float* bias, int32_t E, int32_t top_k, uint32_t flags,
                          int32_t* topk_ids, float* topk_w, float* logits, void* stream) {
    if (T < 0 || d <= 0) return JMOE_EINVAL;
    if (flags & ~JMOE_ROUTE_SOFTMAX_GATES) return JMOE_EINVAL;
    if (E < 1 || E > 64 || top_k < 1 || top_k > 4 || top_k > E) return JMOE_EUNSUPPORTED;
    if (d % 64) return JMOE_EUNSUPPORTED;
    if (T == 0) return JMOE_OK;
    if (!x_bf16 || !w_router || !topk_ids || !topk_w) return JMOE_EINVAL;
    if (!aligned16(x_bf16) || !aligned16(w_router) || !aligned16(topk_ids) || !aligned16(topk_w) ||
        (bias && !aligned16(bias)) || (logits && !aligned16(logits)))
        return JMOE_EALIGN;
    const int renorm = (flags & JMOE_ROUTE_SOFTMAX_GATES) ? 0 : 1;
    return from_cuda(jmoe::launch_route(x_bf16, T, d, w_router, bias, E, top_k, renorm, topk_ids, topk_w,
                                        logits, num_sms(), (cudaStream_t)stream));
}

jmoe_status jmoe_rmsnorm(const void* x_bf16, int64_t T, int64_t d, const void* gamma_bf16,
                         float eps, void* y_bf16, void* stream) {
    const jmoe_status st = check_norm(x_bf16, T, d, gamma_bf16, eps, y_bf16);
    if (st != JMOE_OK || T == 0) return st;
    return from_cuda(jmoe::launch_rmsnorm(x_bf16, T, d, gamma_bf16, eps, y_bf16, num_sms(),
                                          (cudaStream_t)stream));
}

jmoe_status jmoe_rmsnorm_route(const void* x_bf16, int64_t T, int64_t d, const void* gamma_bf16,
                               float eps, void* y_bf16, const float* w_router, const float* bias,
                               int32_t E, int32_t top_k, uint32_t flags, int32_t* topk_ids,
                               float* topk_w, float* logits, void* stream) {
    jmoe_status st = check_norm(x_bf16, T, d, gamma_bf16, eps, y_bf16);
    if (st != JMOE_OK) return st;
    if (flags & ~JMOE_ROUTE_SOFTMAX_GATES) return JMOE_EINVAL;
    if (E < 1 || E > 64 || top_k < 1 || top_k > 4 || top_k > E) return JMOE_EUNSUPPORTED;
    if (T == 0) return JMOE_OK;
    if (!w_router || !topk_ids || !topk_w) return JMOE_EINVAL;
    if (!aligned16(w_router) || !aligned16(topk_ids) || !aligned16(topk_w) ||
        (bias && !aligned16(bias)) || (logits && !aligned16(logits)))
        return JMOE_EALIGN;
    const int renorm = (flags & JMOE_ROUTE_SOFTMAX_GATES) ? 0 : 1;
    return from_cuda(jmoe::launch_norm_route(x_bf16, T, d, gamma_bf16, eps, y_bf16, w_router, bias,
                                             E, top_k, renorm, topk_ids, topk_w, logits, num_sms(),
                                             (cudaStream_t)stream));
}

jmoe_status jmoe_permute(const int32_t* topk_ids, int64_t T, int32_t top_k, int32_t E,
                         int32_t* offsets, int32_t* perm, int32_t* inv, void* stream) {
    if (T < 0) return JMOE_EINVAL;
    if (E < 1 || E > 64 || top_k < 1 || top_k > 4) return JMOE_EUNSUPPORTED;
    if (T * top_k > (1LL << 24)) return JMOE_EUNSUPPORTED;
    if (!offsets) return JMOE_EINVAL;
    if (T > 0 && (!topk_ids || !perm || !inv)) return JMOE_EINVAL;
    if (!aligned16(offsets) || (T > 0 && (!aligned16(topk_ids) || !aligned16(perm) ||
                                          !aligned16(inv))))
        return JMOE_EALIGN;
    return from_cuda(jmoe::launch_permute(topk_ids, T * top_k, E, jmoe::kPrefillTileM, offsets,
                                          nullptr, perm, inv, err_word(), (cudaStream_t)stream));
}

jmoe_status jmoe_forward_workspace_size(const jmoe_moe_desc* desc, int64_t T, size_t* bytes) {
    if (!bytes || !desc) return JMOE_EINVAL;
    if (T < 0) return JMOE_EINVAL;
    if (desc->E < 1 || desc->E > 64 || desc->top_k < 1 || desc->top_k > 4 ||
        desc->top_k > desc->E)
        return JMOE_EUNSUPPORTED;
    if (desc->d_model <= 0 || desc->d_ff <= 0) return JMOE_EINVAL;
    if (desc->d_model % 64 || desc->d_ff % 64) return JMOE_EUNSUPPORTED;
    if (desc->path < JMOE_PATH_AUTO || desc->path > JMOE_PATH_PREFILL) return JMOE_EINVAL;
    const int64_t A = T * desc->top_k;
    *bytes = plan(T, A, desc->E, desc->d_model, desc->d_ff,
                  use_prefill(desc->path, A, desc->E, desc->d_model)).total;
    return JMOE_OK;
}

jmoe_status jmoe_forward(const jmoe_moe_desc* desc, const void* x_bf16, int64_t T,
                         const int32_t* topk_ids, const float* topk_w, void* out_bf16,
                         void* workspace, size_t ws_bytes, void* stream) {
    jmoe_status st = check_desc(desc);
    if (st != JMOE_OK) return st;
    if (T < 0) return JMOE_EINVAL;
    if (T == 0) return JMOE_OK;
    if (T * desc->top_k > (1LL << 24)) return JMOE_EUNSUPPORTED;
    if (!x_bf16 || !topk_ids || !topk_w || !out_bf16) return JMOE_EINVAL;
    if (!aligned16(x_bf16) || !aligned16(topk_ids) || !aligned16(topk_w) || !aligned16(out_bf16))
        return JMOE_EALIGN;
    return run_experts(desc, x_bf16, T, topk_ids, topk_w, out_bf16, workspace, ws_bytes, false,
                       (cudaStream_t)stream);
}

jmoe_status jmoe_mlp_workspace_size(int64_t T, int64_t d_model, int64_t d_ff, int32_t path,
                                    size_t* bytes) {
    if (!bytes) return JMOE_EINVAL;
    jmoe_moe_desc desc{};
    desc.E = 1;
    desc.top_k = 1;
    desc.d_model = d_model;
    desc.d_ff = d_ff;
    desc.path = path;
    size_t inner = 0;
    const jmoe_status st = jmoe_forward_workspace_size(&desc, T, &inner);
    if (st != JMOE_OK) return st;
    // ids and gates tables of the single-expert routing, then the MoE workspace
    *bytes = 2 * round_up(sizeof(float) * (size_t)(T > 0 ? T : 0), 256) + inner;
    return JMOE_OK;
}

jmoe_status jmoe_mlp_forward(const void* x_bf16, int64_t T, int64_t d_model, int64_t d_ff,
                             const int8_t* w_gu, const float* s_gu, const int8_t* w_d,
                             const float* s_d, void* out_bf16, void* workspace, size_t ws_bytes,
                             int32_t path, void* stream) {
    jmoe_moe_desc desc{};
    desc.E = 1;
    desc.top_k = 1;
    desc.d_model = d_model;
    desc.d_ff = d_ff;
    desc.w_gu = w_gu;
    desc.s_gu = s_gu;
    desc.w_d = w_d;
    desc.s_d = s_d;
    desc.path = path;
    jmoe_status st = check_desc(&desc);
    if (st != JMOE_OK) return st;
    if (T < 0) return JMOE_EINVAL;
    if (T == 0) return JMOE_OK;
    if (T > (1LL << 24)) return JMOE_EUNSUPPORTED;
    if (!x_bf16 || !out_bf16) return JMOE_EINVAL;
    if (!aligned16(x_bf16) || !aligned16(out_bf16)) return JMOE_EALIGN;
    size_t need = 0;
    st = jmoe_mlp_workspace_size(T, d_model, d_ff, path, &need);
    if (st != JMOE_OK) return st;
    if (!workspace || ws_bytes < need) return JMOE_EWORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return JMOE_EALIGN;
    // The dense layer is the MoE machinery with one expert, every token
    // routed to it with gate 1: ids (all 0) and gates (all 1) live at the
    // front of the workspace, filled on the stream.
    char* base = static_cast<char*>(workspace);
    const size_t tbl = round_up(sizeof(float) * (size_t)T, 256);
    int32_t* ids = reinterpret_cast<int32_t*>(base);
    float* gates = reinterpret_cast<float*>(base + tbl);
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemsetAsync(ids, 0, sizeof(int32_t) * (size_t)T, s) != cudaSuccess) return JMOE_ECUDA;
    if (jmoe::launch_fill_f32(gates, 1.0f, T, s) != cudaSuccess) return JMOE_ECUDA;
    return run_experts(&desc, x_bf16, T, ids, gates, out_bf16, base + 2 * tbl, ws_bytes - 2 * tbl,
                       true, s);
}

jmoe_status jmoe_forward_noalloc(const jmoe_moe_desc* desc, const void* x_bf16, int64_t T,
                                 const int32_t* topk_ids, const float* topk_w, void* out_bf16,
                                 void* stream) {
    jmoe_status st = check_desc(desc);
    if (st != JMOE_OK) return st;
    if (T < 0) return JMOE_EINVAL;
    if (T == 0) return JMOE_OK;
    if (T * desc->top_k > (1LL << 24)) return JMOE_EUNSUPPORTED;
    if (!x_bf16 || !topk_ids || !topk_w || !out_bf16) return JMOE_EINVAL;
    if (!aligned16(x_bf16) || !aligned16(topk_ids) || !aligned16(topk_w) || !aligned16(out_bf16))
        return JMOE_EALIGN;
    jmoe_moe_desc dec = *desc;
    dec.path = JMOE_PATH_DECODE;
    const size_t need =
        plan(T, T * dec.top_k, dec.E, dec.d_model, dec.d_ff, /*prefill=*/false).total;
    if (need > JMOE_NOALLOC_SCRATCH_BYTES) return JMOE_EWORKSPACE;
    void* scratch = noalloc_scratch();
    if (!scratch) return JMOE_ECUDA;
    return run_experts(&dec, x_bf16, T, topk_ids, topk_w, out_bf16, scratch,
                       JMOE_NOALLOC_SCRATCH_BYTES, false, (cudaStream_t)stream);
}

jmoe_status jmoe_ep_dispatch(const void* x_bf16, int64_t T, int64_t d, const int32_t* topk_ids,
                             int32_t top_k, int32_t E, int32_t G, int32_t* offsets, int32_t* perm,
                             int32_t* inv, void* x_send, int32_t* local_ids, void* stream) {
    if (T < 0 || d <= 0) return JMOE_EINVAL;
    if (E < 1 || E > 64 || top_k < 1 || top_k > 4 || top_k > E) return JMOE_EUNSUPPORTED;
    if (G < 1 || E % G != 0) return JMOE_EUNSUPPORTED;
    if (d % 64) return JMOE_EUNSUPPORTED;
    if (T * top_k > (1LL << 24)) return JMOE_EUNSUPPORTED;
    if (!offsets) return JMOE_EINVAL;
    if (T > 0 && (!x_bf16 || !topk_ids || !perm || !inv || !x_send || !local_ids))
        return JMOE_EINVAL;
    if (!aligned16(offsets) || (T > 0 && (!aligned16(x_bf16) || !aligned16(topk_ids) ||
                                          !aligned16(perm) || !aligned16(inv) ||
                                          !aligned16(x_send) || !aligned16(local_ids))))
        return JMOE_EALIGN;
    return from_cuda(jmoe::launch_ep_dispatch(x_bf16, T, d, topk_ids, top_k, E, E / G, offsets,
                                              perm, inv, x_send, local_ids, err_word(), num_sms(),
                                              (cudaStream_t)stream));
}

jmoe_status jmoe_ep_combine(const void* y_back, const int32_t* inv, const float* topk_w, int64_t T,
                            int64_t d, int32_t top_k, void* out_bf16, void* stream) {
    if (T < 0 || d <= 0) return JMOE_EINVAL;
    if (top_k < 1 || top_k > 4) return JMOE_EUNSUPPORTED;
    if (d % 64) return JMOE_EUNSUPPORTED;
    if (T == 0) return JMOE_OK;
    if (!y_back || !inv || !topk_w || !out_bf16) return JMOE_EINVAL;
    if (!aligned16(y_back) || !aligned16(inv) || !aligned16(topk_w) || !aligned16(out_bf16))
        return JMOE_EALIGN;
    return from_cuda(jmoe::launch_ep_combine(y_back, inv, topk_w, T, d, top_k, out_bf16,
                                             (cudaStream_t)stream));
}

jmoe_status jmoe_profile_events(void* const* events, int32_t n) {
    if (n == 0 || events == nullptr) {
        g_profile_on.store(false);
        return JMOE_OK;
    }
    if (n != 2 * kStages) return JMOE_EINVAL;
    for (int i = 0; i < n; i += 2)
        if ((events[i] == nullptr) != (events[i + 1] == nullptr)) return JMOE_EINVAL;
    for (int i = 0; i < n; ++i) g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
    g_profile_on.store(true);
    return JMOE_OK;
}

jmoe_status jmoe_test_stall(int32_t target, int64_t wait_cycles) {
    if (target < 0 || target > JMOE_STALL_DECODE_GEMV) return JMOE_EINVAL;
    if (target != 0 && (wait_cycles < 1000 || wait_cycles > jmoe::kMaxWaitCycles))
        return JMOE_EINVAL;
    std::lock_guard<std::mutex> lock(g_stall_mu);
    g_stall_target = target;
    g_stall_wait_cycles = target ? (long long)wait_cycles : 0;
    return JMOE_OK;
}

jmoe_status jmoe_last_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return JMOE_ECUDA;
    unsigned* p = err_word();
    if (!p) return JMOE_ECUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return JMOE_ECUDA;
    if (v != 0 && cudaMemset(p, 0, sizeof(unsigned)) != cudaSuccess) return JMOE_ECUDA;
    v |= jmoe::checks_take_decode() | jmoe::checks_take_prefill() | jmoe::checks_take_permute() |
         jmoe::checks_take_ep();
    if (v & jmoe::kErrBounds) return JMOE_EBOUNDS;
    if (v & jmoe::kErrBadExpert) return JMOE_EDEVICE;
    if (v & jmoe::kErrTimeout) return JMOE_ETIMEOUT;
    return JMOE_OK;
}

}  // extern "C"
