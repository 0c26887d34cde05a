"""CPU oracle for the ExpertsInt8 MoE layer -- TEST INFRASTRUCTURE ONLY.

A thin numpy/ctypes wrapper around ``oracle.c`` (plain C, fp64).  Only the
tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package; the product path never does, and this package imports
nothing from the CUDA library.  Inputs come from :mod:`synth` (bf16 values are
passed as uint16 bit patterns).

Every function here restates a step of the pages (see ``oracle.c`` for the
citations and the readings taken where the pages are silent).  Parity status:
all functions are pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` against exact rational arithmetic, brute force,
closed forms, textbook special cases and invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")


def compile_oracle(source: str, out_so: str, verbose: bool = False) -> None:
    """Compile an oracle source with gcc (fp64, OpenMP, no FMA contraction, no fast-math)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
           "-fno-fast-math", "-o", out_so, source, "-lm"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)


def build(verbose: bool = False) -> None:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it."""
    compile_oracle(SOURCE, _SO, verbose)


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


class Oracle:
    """The oracle's entry points, bound to one compiled copy of ``oracle.c``.

    The default instance (module-level functions) loads ``liboracle.so``; the
    mutation tests bind deliberately broken copies to check that the pins
    reject them.
    """

    def __init__(self, so_path: str = _SO):
        if so_path == _SO and (not os.path.exists(_SO) or
                               os.path.getmtime(_SO) < os.path.getmtime(SOURCE)):
            build()  # missing, or older than its source (a stale signature would crash)
        lib = ctypes.CDLL(so_path)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.oracle_quantize.argtypes = [vp, i64, i64, vp, vp]
        lib.oracle_quantize.restype = None
        lib.oracle_router_logits.argtypes = [vp, i64, i64, vp, i32, vp, vp]
        lib.oracle_router_logits.restype = None
        lib.oracle_topk_gates.argtypes = [vp, i64, i32, i32, vp, vp]
        lib.oracle_topk_gates.restype = ctypes.c_int
        lib.oracle_topk_gates_mode.argtypes = [vp, i64, i32, i32, i32, vp, vp]
        lib.oracle_topk_gates_mode.restype = ctypes.c_int
        lib.oracle_rmsnorm.argtypes = [vp, i64, i64, vp, ctypes.c_float, vp]
        lib.oracle_rmsnorm.restype = None
        lib.oracle_permute.argtypes = [vp, i64, i32, i32, vp, vp, vp]
        lib.oracle_permute.restype = None
        lib.oracle_moe_forward.argtypes = [vp, i64, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp,
                                           vp]
        lib.oracle_moe_forward.restype = ctypes.c_int
        lib.oracle_mlp_forward.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp]
        lib.oracle_mlp_forward.restype = None
        self.lib = lib

    def quantize(self, w_bits: np.ndarray):
        """Per-row symmetric INT8 quantisation of a bf16 matrix [rows, cols].

        Returns ``(q int8 [rows, cols], scales fp32 [rows])``.
        """
        w = _c(w_bits, np.uint16)
        rows, cols = w.shape
        q = np.empty((rows, cols), dtype=np.int8)
        s = np.empty(rows, dtype=np.float32)
        self.lib.oracle_quantize(w.ctypes.data, rows, cols, q.ctypes.data, s.ctypes.data)
        return q, s

    def router_logits(self, x_bits: np.ndarray, w_router: np.ndarray,
                      bias: Optional[np.ndarray] = None) -> np.ndarray:
        """fp32 router logits [T, E] summed in the canonical fp64 order."""
        x = _c(x_bits, np.uint16)
        wr = _c(w_router, np.float32)
        T, d = x.shape
        E = wr.shape[0]
        assert wr.shape[1] == d
        b = None if bias is None else _c(bias, np.float32)
        out = np.empty((T, E), dtype=np.float32)
        self.lib.oracle_router_logits(x.ctypes.data, T, d, wr.ctypes.data, E,
                                      None if b is None else b.ctypes.data, out.ctypes.data)
        return out

    def topk_gates(self, logits: np.ndarray, top_k: int, renorm: bool = True):
        """Top-k expert ids (ties to the lower index) and fp64 gates: the
        selected softmax probabilities renormalised over the selection, or
        (renorm=False) the plain softmax probabilities."""
        l = _c(logits, np.float32)
        T, E = l.shape
        ids = np.empty((T, top_k), dtype=np.int32)
        g = np.empty((T, top_k), dtype=np.float64)
        rc = self.lib.oracle_topk_gates_mode(l.ctypes.data, T, E, top_k, 1 if renorm else 0,
                                             ids.ctypes.data, g.ctypes.data)
        if rc != 0:
            raise ValueError("oracle_topk_gates: unsupported E/top_k")
        return ids, g

    def rmsnorm(self, x_bits: np.ndarray, gamma_bits: np.ndarray, eps: float) -> np.ndarray:
        """RMSNorm of bf16 rows: bf16 bits of (x * r) * gamma, r = 1/sqrt(mean(x^2) + eps)."""
        x = _c(x_bits, np.uint16)
        gm = _c(gamma_bits, np.uint16)
        T, d = x.shape
        assert gm.shape == (d,)
        out = np.empty((T, d), dtype=np.uint16)
        self.lib.oracle_rmsnorm(x.ctypes.data, T, d, gm.ctypes.data, float(eps), out.ctypes.data)
        return out

    def route(self, x_bits, w_router, top_k: int, bias=None, renorm: bool = True):
        """Router logits, top-k ids and gates for every token."""
        logits = self.router_logits(x_bits, w_router, bias)
        ids, g = self.topk_gates(logits, top_k, renorm)
        return logits, ids, g

    def permute(self, ids: np.ndarray, E: int):
        """Stable grouping by expert: ``(offsets [E+1], perm [A], inv [A])``."""
        i = _c(ids, np.int32)
        T, k = i.shape
        offsets = np.empty(E + 1, dtype=np.int32)
        perm = np.empty(T * k, dtype=np.int32)
        inv = np.empty(T * k, dtype=np.int32)
        self.lib.oracle_permute(i.ctypes.data, T, k, E, offsets.ctypes.data, perm.ctypes.data,
                                inv.ctypes.data)
        return offsets, perm, inv

    def moe_forward(self, x_bits: np.ndarray, ids: np.ndarray, gates: np.ndarray,
                    q_gu: Sequence[Optional[np.ndarray]], s_gu: Sequence[Optional[np.ndarray]],
                    q_d: Sequence[Optional[np.ndarray]], s_d: Sequence[Optional[np.ndarray]]
                    ) -> np.ndarray:
        """fp64 MoE output [T, d] = sum_j gates[t,j] * Expert_{ids[t,j]}(x_t).

        ``q_gu[e]`` is expert e's int8 gate/up matrix [2*d_ff, d] (gate rows
        first), ``s_gu[e]`` its scales [2*d_ff]; ``q_d[e]`` [d, d_ff], ``s_d[e]``
        [d].  Entries of experts that no token selects may be None.
        """
        x = _c(x_bits, np.uint16)
        T, d = x.shape
        i = _c(ids, np.int32)
        k = i.shape[1]
        g = _c(gates, np.float64)
        E = len(q_gu)
        keep = []

        def table(arrs, dtype):
            ptrs = (ctypes.c_void_p * E)()
            for e, a in enumerate(arrs):
                if a is None:
                    ptrs[e] = None
                else:
                    c = _c(a, dtype)
                    keep.append(c)
                    ptrs[e] = c.ctypes.data
            return ptrs

        f = None
        for a in q_d:
            if a is not None:
                f = a.shape[1]
                break
        if f is None:
            raise ValueError("no expert weights given")
        t_qgu, t_sgu = table(q_gu, np.int8), table(s_gu, np.float32)
        t_qd, t_sd = table(q_d, np.int8), table(s_d, np.float32)
        out = np.empty((T, d), dtype=np.float64)
        rc = self.lib.oracle_moe_forward(x.ctypes.data, T, d, f, E, k, i.ctypes.data,
                                         g.ctypes.data, t_qgu, t_sgu, t_qd, t_sd,
                                         out.ctypes.data)
        if rc != 0:
            raise ValueError("oracle_moe_forward: a selected expert has no weights")
        return out

    def mlp_forward(self, x_bits, q_gu, s_gu, q_d, s_d) -> np.ndarray:
        """fp64 dense SwiGLU MLP output [T, d] with INT8 weights (the E=1 entry)."""
        x = _c(x_bits, np.uint16)
        T, d = x.shape
        qgu, sgu = _c(q_gu, np.int8), _c(s_gu, np.float32)
        qd, sd = _c(q_d, np.int8), _c(s_d, np.float32)
        f = qd.shape[1]
        out = np.empty((T, d), dtype=np.float64)
        self.lib.oracle_mlp_forward(x.ctypes.data, T, d, f, qgu.ctypes.data, sgu.ctypes.data,
                                    qd.ctypes.data, sd.ctypes.data, out.ctypes.data)
        return out


_default: Optional[Oracle] = None


def default() -> Oracle:
    """The oracle bound to ``liboracle.so`` (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def quantize(w_bits):
    return default().quantize(w_bits)


def router_logits(x_bits, w_router, bias=None):
    return default().router_logits(x_bits, w_router, bias)


def topk_gates(logits, top_k, renorm=True):
    return default().topk_gates(logits, top_k, renorm)


def rmsnorm(x_bits, gamma_bits, eps):
    return default().rmsnorm(x_bits, gamma_bits, eps)


def route(x_bits, w_router, top_k, bias=None, renorm=True):
    return default().route(x_bits, w_router, top_k, bias, renorm)


def permute(ids, E):
    return default().permute(ids, E)


def moe_forward(x_bits, ids, gates, q_gu, s_gu, q_d, s_d):
    return default().moe_forward(x_bits, ids, gates, q_gu, s_gu, q_d, s_d)


def mlp_forward(x_bits, q_gu, s_gu, q_d, s_d):
    return default().mlp_forward(x_bits, q_gu, s_gu, q_d, s_d)


def tolerance_report(got: np.ndarray, ref: np.ndarray) -> dict:
    """The parity metrics: max|d| / max|ref| and sum|d| / sum|ref|."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = np.abs(got - ref)
    mref = float(np.max(np.abs(ref))) if ref.size else 0.0
    sref = float(np.sum(np.abs(ref))) if ref.size else 0.0
    return {
        "max_abs_diff": float(diff.max()) if diff.size else 0.0,
        "max_ref": mref,
        "max_rel": float(diff.max() / mref) if mref > 0 else float(diff.max() if diff.size else 0),
        "mean_rel": float(diff.sum() / sref) if sref > 0 else float(diff.sum()),
    }
