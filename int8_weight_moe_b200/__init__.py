"""Python binding of libjmoe.so, the ExpertsInt8 MoE layer for B200 (sm_100a).

Argument marshalling only: every function below validates tensor dtypes and
devices, takes raw pointers and the current CUDA stream from PyTorch, and calls
the C entry point of the same name (declared in ``include/jmoe.h``).  Every step
of the layer runs in the library's CUDA kernels; there is no CPU or PyTorch
fallback -- if ``libjmoe.so`` is missing or a call fails, an exception says so.

Allocation of outputs and workspaces happens here, through PyTorch's caching
allocator (the C library itself never allocates).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libjmoe.so")
# The bounds-check build (same ABI, device checks compiled in); tests load it
# by setting LIB_PATH to this path before the first call.
CHECKS_LIB_PATH = os.path.join(HERE, "libjmoe_checks.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "jmoe.h")

JMOE_OK, JMOE_EINVAL, JMOE_EALIGN, JMOE_EUNSUPPORTED = 0, 1, 2, 3
JMOE_EWORKSPACE, JMOE_ECUDA, JMOE_ETIMEOUT, JMOE_EDEVICE = 4, 5, 6, 7
JMOE_EBOUNDS = 8
JMOE_PATH_AUTO, JMOE_PATH_DECODE, JMOE_PATH_PREFILL = 0, 1, 2

# Every C entry point the header declares.
EXPORTED = ("jmoe_quantize", "jmoe_route", "jmoe_route_ex", "jmoe_rmsnorm", "jmoe_rmsnorm_route",
            "jmoe_permute", "jmoe_forward_workspace_size",
            "jmoe_forward", "jmoe_forward_noalloc", "jmoe_mlp_workspace_size", "jmoe_mlp_forward",
            "jmoe_ep_dispatch", "jmoe_ep_combine",
            "jmoe_profile_events", "jmoe_launch_count", "jmoe_test_stall", "jmoe_last_error",
            "jmoe_test_check", "jmoe_status_string", "jmoe_cuda_error_string")
NOALLOC_SCRATCH_BYTES = 32 << 20  # JMOE_NOALLOC_SCRATCH_BYTES
JMOE_ROUTE_SOFTMAX_GATES = 1
JMOE_STALL_TENSOR_GEMM, JMOE_STALL_DECODE_GEMV = 1, 2
STAGES = ("permute", "gather", "gate_up", "down", "combine", "act")


class JmoeError(RuntimeError):
    """A jmoe call returned a status other than JMOE_OK."""

    def __init__(self, fn: str, status: int):
        self.status = status
        msg = f"{fn} failed: {status_string(status)}"
        if status == JMOE_ECUDA:
            msg += f" ({load().jmoe_cuda_error_string().decode()})"
        super().__init__(msg)


class MoeDesc(ctypes.Structure):
    """Mirror of ``jmoe_moe_desc``."""

    _fields_ = [("E", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("d_model", ctypes.c_int64), ("d_ff", ctypes.c_int64),
                ("w_gu", ctypes.c_void_p), ("s_gu", ctypes.c_void_p),
                ("w_d", ctypes.c_void_p), ("s_d", ctypes.c_void_p),
                ("path", ctypes.c_int32)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libjmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); run "
                          "`python -m int8_weight_moe_b200.build` or __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    st = ctypes.c_int
    lib.jmoe_quantize.argtypes = [vp, i64, i64, vp, vp, vp]
    lib.jmoe_route.argtypes = [vp, i64, i64, vp, vp, i32, i32, vp, vp, vp, vp]
    lib.jmoe_route_ex.argtypes = [vp, i64, i64, vp, vp, i32, i32, ctypes.c_uint32, vp, vp, vp,
                                  vp]
    lib.jmoe_rmsnorm.argtypes = [vp, i64, i64, vp, ctypes.c_float, vp, vp]
    lib.jmoe_rmsnorm_route.argtypes = [vp, i64, i64, vp, ctypes.c_float, vp, vp, vp, i32, i32,
                                       ctypes.c_uint32, vp, vp, vp, vp]
    lib.jmoe_permute.argtypes = [vp, i64, i32, i32, vp, vp, vp, vp]
    lib.jmoe_forward_workspace_size.argtypes = [ctypes.POINTER(MoeDesc), i64, ctypes.POINTER(sz)]
    lib.jmoe_forward.argtypes = [ctypes.POINTER(MoeDesc), vp, i64, vp, vp, vp, vp, sz, vp]
    lib.jmoe_forward_noalloc.argtypes = [ctypes.POINTER(MoeDesc), vp, i64, vp, vp, vp, vp]
    lib.jmoe_mlp_workspace_size.argtypes = [i64, i64, i64, i32, ctypes.POINTER(sz)]
    lib.jmoe_mlp_forward.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, vp, sz, i32, vp]
    lib.jmoe_ep_dispatch.argtypes = [vp, i64, i64, vp, i32, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.jmoe_ep_combine.argtypes = [vp, vp, vp, i64, i64, i32, vp, vp]
    lib.jmoe_profile_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), i32]
    lib.jmoe_launch_count.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
    lib.jmoe_test_stall.argtypes = [i32, i64]
    lib.jmoe_test_check.argtypes = [vp]
    lib.jmoe_last_error.argtypes = []
    for name in EXPORTED[:-2]:
        getattr(lib, name).restype = st
    lib.jmoe_status_string.argtypes = [st]
    lib.jmoe_status_string.restype = ctypes.c_char_p
    lib.jmoe_cuda_error_string.argtypes = []
    lib.jmoe_cuda_error_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().jmoe_status_string(status).decode()


def _check(fn: str, status: int) -> None:
    if status != JMOE_OK:
        raise JmoeError(fn, status)


def _stream(t) -> int:
    import torch

    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t, dtype, name):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


# ----------------------------------------------------------------------------- entry points


def jmoe_quantize(w, q=None, scales=None):
    """bf16 [rows, cols] -> (int8 [rows, cols], fp32 [rows]); see jmoe.h."""
    import torch

    _need(w, torch.bfloat16, "w")
    if q is None:
        q = torch.empty(w.shape, dtype=torch.int8, device=w.device)
    if scales is None:
        scales = torch.empty(w.shape[:-1], dtype=torch.float32, device=w.device)
    rows = w.numel() // w.shape[-1]
    cols = w.shape[-1]
    _check("jmoe_quantize", load().jmoe_quantize(_ptr(w), rows, cols, _ptr(q), _ptr(scales),
                                                 _stream(w)))
    return q, scales


def jmoe_route(x, w_router, top_k: int = 2, bias=None, topk_ids=None, topk_w=None,
               logits=None, want_logits: bool = False, softmax_gates: bool = False):
    """Router logits -> (topk_ids int32 [T, k], topk_w fp32 [T, k][, logits]).

    Gates are the selected softmax probabilities renormalised over the
    selection, or with softmax_gates=True the plain softmax probabilities
    (jmoe_route_ex with JMOE_ROUTE_SOFTMAX_GATES)."""
    import torch

    _need(x, torch.bfloat16, "x")
    _need(w_router, torch.float32, "w_router")
    T, d = x.shape
    E = w_router.shape[0]
    if bias is not None:
        _need(bias, torch.float32, "bias")
    if topk_ids is None:
        topk_ids = torch.empty((T, top_k), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((T, top_k), dtype=torch.float32, device=x.device)
    if want_logits and logits is None:
        logits = torch.empty((T, E), dtype=torch.float32, device=x.device)
    flags = JMOE_ROUTE_SOFTMAX_GATES if softmax_gates else 0
    _check("jmoe_route_ex", load().jmoe_route_ex(_ptr(x), T, d, _ptr(w_router), _ptr(bias), E,
                                                 top_k, flags, _ptr(topk_ids), _ptr(topk_w),
                                                 _ptr(logits), _stream(x)))
    return (topk_ids, topk_w, logits) if want_logits else (topk_ids, topk_w)


def jmoe_rmsnorm(x, gamma, eps: float, out=None):
    """RMSNorm of bf16 rows: bf16((x * r) * gamma), r = 1/sqrt(mean(x^2) + eps)."""
    import torch

    _need(x, torch.bfloat16, "x")
    _need(gamma, torch.bfloat16, "gamma")
    T, d = x.shape
    if out is None:
        out = torch.empty_like(x)
    _check("jmoe_rmsnorm", load().jmoe_rmsnorm(_ptr(x), T, d, _ptr(gamma), float(eps), _ptr(out),
                                               _stream(x)))
    return out


def jmoe_rmsnorm_route(x, gamma, eps: float, w_router, top_k: int = 2, bias=None, x_norm=None,
                       topk_ids=None, topk_w=None, logits=None, want_logits: bool = False,
                       softmax_gates: bool = False):
    """The pre-MoE prologue: RMSNorm, then the router on the normalised rows.
    Returns (x_norm, topk_ids, topk_w[, logits])."""
    import torch

    _need(x, torch.bfloat16, "x")
    _need(gamma, torch.bfloat16, "gamma")
    _need(w_router, torch.float32, "w_router")
    T, d = x.shape
    E = w_router.shape[0]
    if bias is not None:
        _need(bias, torch.float32, "bias")
    if x_norm is None:
        x_norm = torch.empty_like(x)
    if topk_ids is None:
        topk_ids = torch.empty((T, top_k), dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty((T, top_k), dtype=torch.float32, device=x.device)
    if want_logits and logits is None:
        logits = torch.empty((T, E), dtype=torch.float32, device=x.device)
    flags = JMOE_ROUTE_SOFTMAX_GATES if softmax_gates else 0
    _check("jmoe_rmsnorm_route", load().jmoe_rmsnorm_route(
        _ptr(x), T, d, _ptr(gamma), float(eps), _ptr(x_norm), _ptr(w_router), _ptr(bias), E, top_k,
        flags, _ptr(topk_ids), _ptr(topk_w), _ptr(logits), _stream(x)))
    out = (x_norm, topk_ids, topk_w)
    return out + (logits,) if want_logits else out


def jmoe_permute(topk_ids, E: int):
    """Stable grouping of the assignments by expert -> (offsets, perm, inv)."""
    import torch

    _need(topk_ids, torch.int32, "topk_ids")
    T, k = topk_ids.shape
    offsets = torch.empty(E + 1, dtype=torch.int32, device=topk_ids.device)
    perm = torch.empty(T * k, dtype=torch.int32, device=topk_ids.device)
    inv = torch.empty(T * k, dtype=torch.int32, device=topk_ids.device)
    _check("jmoe_permute", load().jmoe_permute(_ptr(topk_ids), T, k, E, _ptr(offsets), _ptr(perm),
                                               _ptr(inv), _stream(topk_ids)))
    return offsets, perm, inv


def make_desc(w_gu, s_gu, w_d, s_d, top_k: int = 2, path: int = JMOE_PATH_AUTO) -> MoeDesc:
    """Descriptor of one MoE layer's quantised weights (tensors must stay alive)."""
    import torch

    _need(w_gu, torch.int8, "w_gu")
    _need(s_gu, torch.float32, "s_gu")
    _need(w_d, torch.int8, "w_d")
    _need(s_d, torch.float32, "s_d")
    E, two_f, d = w_gu.shape
    if tuple(w_d.shape) != (E, d, two_f // 2):
        raise ValueError(f"w_d shape {tuple(w_d.shape)} does not match w_gu {tuple(w_gu.shape)}")
    return MoeDesc(E, top_k, d, two_f // 2, w_gu.data_ptr(), s_gu.data_ptr(), w_d.data_ptr(),
                   s_d.data_ptr(), path)


def jmoe_forward_workspace_size(desc: MoeDesc, T: int) -> int:
    n = ctypes.c_size_t(0)
    _check("jmoe_forward_workspace_size",
           load().jmoe_forward_workspace_size(ctypes.byref(desc), T, ctypes.byref(n)))
    return n.value


def uses_prefill_path(desc: MoeDesc, T: int) -> bool:
    """Whether jmoe_forward's automatic path choice is the tensor-core path
    for T tokens (read off the workspace sizes the library reports)."""
    auto = MoeDesc.from_buffer_copy(desc)
    auto.path = JMOE_PATH_AUTO
    dec = MoeDesc.from_buffer_copy(desc)
    dec.path = JMOE_PATH_DECODE
    return jmoe_forward_workspace_size(auto, T) != jmoe_forward_workspace_size(dec, T)


def jmoe_forward(desc: MoeDesc, x, topk_ids, topk_w, out=None, workspace=None):
    """MoE layer output bf16 [T, d] (see jmoe.h)."""
    import torch

    _need(x, torch.bfloat16, "x")
    _need(topk_ids, torch.int32, "topk_ids")
    _need(topk_w, torch.float32, "topk_w")
    T = x.shape[0]
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = torch.empty(max(jmoe_forward_workspace_size(desc, T), 1), dtype=torch.uint8,
                                device=x.device)
    _check("jmoe_forward", load().jmoe_forward(ctypes.byref(desc), _ptr(x), T, _ptr(topk_ids),
                                               _ptr(topk_w), _ptr(out), _ptr(workspace),
                                               workspace.numel(), _stream(x)))
    return out


def jmoe_forward_noalloc(desc: MoeDesc, x, topk_ids, topk_w, out=None):
    """jmoe_forward without a workspace: for callers that cannot allocate device
    memory when they call the layer; the scratch is a fixed array inside the
    library (see jmoe.h for its size limit and sharing rules)."""
    import torch

    _need(x, torch.bfloat16, "x")
    _need(topk_ids, torch.int32, "topk_ids")
    _need(topk_w, torch.float32, "topk_w")
    if out is None:
        out = torch.empty_like(x)
    _check("jmoe_forward_noalloc",
           load().jmoe_forward_noalloc(ctypes.byref(desc), _ptr(x), x.shape[0], _ptr(topk_ids),
                                       _ptr(topk_w), _ptr(out), _stream(x)))
    return out


def jmoe_mlp_workspace_size(T: int, d_model: int, d_ff: int, path: int = JMOE_PATH_AUTO) -> int:
    n = ctypes.c_size_t(0)
    _check("jmoe_mlp_workspace_size",
           load().jmoe_mlp_workspace_size(T, d_model, d_ff, path, ctypes.byref(n)))
    return n.value


def jmoe_mlp_forward(x, w_gu, s_gu, w_d, s_d, out=None, workspace=None, path=JMOE_PATH_AUTO):
    """Dense SwiGLU MLP with INT8 weights: bf16 [T, d] -> bf16 [T, d]."""
    import torch

    _need(x, torch.bfloat16, "x")
    _need(w_gu, torch.int8, "w_gu")
    _need(s_gu, torch.float32, "s_gu")
    _need(w_d, torch.int8, "w_d")
    _need(s_d, torch.float32, "s_d")
    T, d = x.shape
    f = w_d.shape[-1]
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = torch.empty(max(jmoe_mlp_workspace_size(T, d, f, path), 1), dtype=torch.uint8,
                                device=x.device)
    _check("jmoe_mlp_forward", load().jmoe_mlp_forward(_ptr(x), T, d, f, _ptr(w_gu), _ptr(s_gu),
                                                       _ptr(w_d), _ptr(s_d), _ptr(out),
                                                       _ptr(workspace), workspace.numel(), path,
                                                       _stream(x)))
    return out


def jmoe_ep_dispatch(x, topk_ids, E: int, G: int):
    """Expert-parallel send buffer (see jmoe.h) -> (offsets, perm, inv, x_send, local_ids)."""
    import torch

    _need(x, torch.bfloat16, "x")
    _need(topk_ids, torch.int32, "topk_ids")
    T, d = x.shape
    k = topk_ids.shape[1]
    dev = x.device
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    inv = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    x_send = torch.empty((max(T * k, 1), d), dtype=torch.bfloat16, device=dev)
    local_ids = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)
    _check("jmoe_ep_dispatch", load().jmoe_ep_dispatch(
        _ptr(x), T, d, _ptr(topk_ids), k, E, G, _ptr(offsets), _ptr(perm), _ptr(inv),
        _ptr(x_send), _ptr(local_ids), _stream(x)))
    return offsets, perm[:T * k], inv[:T * k], x_send[:T * k], local_ids[:T * k]


def jmoe_ep_combine(y_back, inv, topk_w, out=None):
    """out[t] = bf16(sum_j topk_w[t, j] * y_back[inv[t * k + j]]) (see jmoe.h)."""
    import torch

    _need(y_back, torch.bfloat16, "y_back")
    _need(inv, torch.int32, "inv")
    _need(topk_w, torch.float32, "topk_w")
    T, k = topk_w.shape
    d = y_back.shape[1]
    if out is None:
        out = torch.empty((T, d), dtype=torch.bfloat16, device=y_back.device)
    _check("jmoe_ep_combine", load().jmoe_ep_combine(_ptr(y_back), _ptr(inv), _ptr(topk_w), T, d,
                                                     k, _ptr(out), _stream(y_back)))
    return out


def jmoe_profile_events(events) -> None:
    """Register torch.cuda.Event objects (2 per stage, see jmoe.h; None skips a
    stage) or None to stop."""
    if not events:
        _check("jmoe_profile_events", load().jmoe_profile_events(None, 0))
        return
    arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event if ev is not None else None
                                            for ev in events])
    _check("jmoe_profile_events", load().jmoe_profile_events(arr, len(events)))


def jmoe_launch_count() -> int:
    """Kernels launched by the library so far in this process (all devices)."""
    n = ctypes.c_uint64(0)
    _check("jmoe_launch_count", load().jmoe_launch_count(ctypes.byref(n)))
    return int(n.value)


def jmoe_test_stall(target: int, wait_cycles: int = 0) -> None:
    """Arm the bounded-wait test hook for the next forward call (see jmoe.h)."""
    _check("jmoe_test_stall", load().jmoe_test_stall(target, wait_cycles))


def jmoe_last_error() -> int:
    """Read and clear the device error word (synchronises the device)."""
    return load().jmoe_last_error()


def jmoe_test_check(stream=None) -> int:
    """Bounds-check build only: make one device check fail (no memory access),
    so that the next jmoe_last_error() is JMOE_EBOUNDS.  Returns the status
    (JMOE_EUNSUPPORTED from the normal build)."""
    import torch

    s = torch.cuda.current_stream().cuda_stream if stream is None else stream
    return load().jmoe_test_check(s)


def jmoe_cuda_error_string() -> str:
    """The CUDA error text behind this thread's most recent JMOE_ECUDA."""
    return load().jmoe_cuda_error_string().decode()


def jmoe_status_string(status: int) -> str:
    return status_string(status)


class MoeLayerGraph:
    """A whole MoE layer -- RMSNorm + router (or router alone) + experts --
    captured once in a CUDA graph for a fixed token count and replayed.

    The graph reads the static input buffer ``x`` and writes ``out``; copy a
    batch into ``x`` (or pass it to ``run``) before each replay.  Every buffer
    the kernels touch (routing tables, workspace, normalised rows) is owned by
    this object, so replays allocate nothing."""

    def __init__(self, desc: MoeDesc, w_router, T: int, gamma=None, eps: float = 1e-6,
                 bias=None, softmax_gates: bool = False, device=None):
        import torch

        device = device or w_router.device
        d = desc.d_model
        self.desc, self.w_router, self.gamma, self.eps = desc, w_router, gamma, eps
        self.bias, self.softmax_gates = bias, softmax_gates
        self.x = torch.zeros((T, d), dtype=torch.bfloat16, device=device)
        self.x_norm = torch.empty_like(self.x) if gamma is not None else None
        self.ids = torch.empty((T, desc.top_k), dtype=torch.int32, device=device)
        self.gates = torch.empty((T, desc.top_k), dtype=torch.float32, device=device)
        self.out = torch.empty_like(self.x)
        self.ws = torch.empty(max(jmoe_forward_workspace_size(desc, T), 1), dtype=torch.uint8,
                              device=device)
        stream = torch.cuda.Stream(device=device)
        stream.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(stream):
            self._body()  # warm-up outside the capture (per-device first-use setup)
        torch.cuda.current_stream(device).wait_stream(stream)
        torch.cuda.synchronize(device)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=stream):
            self._body()

    def _body(self):
        if self.gamma is not None:
            jmoe_rmsnorm_route(self.x, self.gamma, self.eps, self.w_router, self.desc.top_k,
                               self.bias, x_norm=self.x_norm, topk_ids=self.ids,
                               topk_w=self.gates, softmax_gates=self.softmax_gates)
            xin = self.x_norm
        else:
            jmoe_route(self.x, self.w_router, self.desc.top_k, self.bias, topk_ids=self.ids,
                       topk_w=self.gates, softmax_gates=self.softmax_gates)
            xin = self.x
        jmoe_forward(self.desc, xin, self.ids, self.gates, out=self.out, workspace=self.ws)

    def run(self, x=None):
        """Replay on the current stream (after copying ``x`` in, if given); returns ``out``."""
        if x is not None:
            self.x.copy_(x)
        self.graph.replay()
        return self.out


def moe_layer(x, w_router, desc: MoeDesc, bias=None, workspace=None):
    """Route then run the layer: the whole MoE forward of one batch of tokens."""
    ids, gates = jmoe_route(x, w_router, desc.top_k, bias)
    return jmoe_forward(desc, x, ids, gates, workspace=workspace)
