"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This module draws tensors only; it contains none of the MoE method's
arithmetic.  The generator is defined in ``synth_cpu.c`` (host, used for the
oracle's inputs) and ``synth_gpu.cu`` (device, used to fill large weight
tensors in HBM); both produce identical bits for the same (seed, tensor id,
sigma, element index).

Tensor ids used by the workloads (:mod:`synth.workloads`):

=========  =====================================================
``X``      activations ``x`` [T, d_model], bf16, sigma = 1
``WR``     router weights ``W_r`` [E, d_model], fp32, sigma = 0.02
``WGU``    expert gate/up weights [E, 2*d_ff, d_model], bf16, sigma = 0.02
``WD``     expert down weights [E, d_model, d_ff], bf16, sigma = 0.02
=========  =====================================================
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

X, WR, WGU, WD = 1, 2, 3, 4

_HERE = os.path.dirname(os.path.abspath(__file__))
_CPU_SO = os.path.join(_HERE, "libsynth_cpu.so")
_GPU_SO = os.path.join(_HERE, "libsynth_gpu.so")
_cpu = None
_gpu = None


def build(verbose: bool = False) -> None:
    """Compile the host generator (gcc) and the device generator (nvcc, sm_100a)."""
    cmds = [
        ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
         "-o", _CPU_SO, os.path.join(_HERE, "synth_cpu.c")],
        ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3",
         "-Xcompiler", "-fPIC", "-shared", "-fmad=false", "-o", _GPU_SO,
         os.path.join(_HERE, "synth_gpu.cu")],
    ]
    for c in cmds:
        if verbose:
            print(" ".join(c))
        subprocess.run(c, check=True)


def _load_cpu():
    global _cpu
    if _cpu is None:
        if not os.path.exists(_CPU_SO):
            build()
        lib = ctypes.CDLL(_CPU_SO)
        u64, i64, f32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_float
        lib.synth_normal_f32.argtypes = [u64, u64, f32, u64, i64, ctypes.c_void_p]
        lib.synth_normal_bf16.argtypes = [u64, u64, f32, u64, i64, ctypes.c_void_p]
        lib.synth_splitmix64_stream.argtypes = [u64, i64, ctypes.c_void_p]
        for f in (lib.synth_normal_f32, lib.synth_normal_bf16, lib.synth_splitmix64_stream):
            f.restype = None
        _cpu = lib
    return _cpu


def _load_gpu():
    global _gpu
    if _gpu is None:
        if not os.path.exists(_GPU_SO):
            raise RuntimeError(f"device generator not built: {_GPU_SO} missing (run synth.build())")
        lib = ctypes.CDLL(_GPU_SO)
        u64, i64, f32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
        lib.synth_normal_bf16_gpu.argtypes = [u64, u64, f32, u64, i64, vp, vp]
        lib.synth_normal_f32_gpu.argtypes = [u64, u64, f32, u64, i64, vp, vp]
        lib.synth_normal_bf16_gpu.restype = ctypes.c_int
        lib.synth_normal_f32_gpu.restype = ctypes.c_int
        _gpu = lib
    return _gpu


def splitmix64_stream(seed: int, n: int) -> np.ndarray:
    """The raw SplitMix64 stream out[k] = mix(seed + (k+1)*gamma)."""
    out = np.empty(n, dtype=np.uint64)
    _load_cpu().synth_splitmix64_stream(seed, n, out.ctypes.data)
    return out


def normal_f32(seed: int, tensor: int, sigma: float, shape, start: int = 0) -> np.ndarray:
    """fp32 samples for elements [start, start+prod(shape)) of tensor ``tensor``."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    _load_cpu().synth_normal_f32(seed, tensor, sigma, start, n, out.ctypes.data)
    return out.reshape(shape)


def normal_bf16_bits(seed: int, tensor: int, sigma: float, shape, start: int = 0) -> np.ndarray:
    """bf16 samples (as uint16 bit patterns) for elements [start, start+prod(shape))."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    _load_cpu().synth_normal_bf16(seed, tensor, sigma, start, n, out.ctypes.data)
    return out.reshape(shape)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 values (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def normal_bf16_gpu(seed: int, tensor: int, sigma: float, shape, start: int = 0, device="cuda"):
    """A torch.bfloat16 CUDA tensor holding the same values as :func:`normal_bf16_bits`."""
    import torch

    out = torch.empty(tuple(shape), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(out.device).cuda_stream
    rc = _load_gpu().synth_normal_bf16_gpu(seed, tensor, sigma, start, out.numel(),
                                           out.data_ptr(), stream)
    if rc != 0:
        raise RuntimeError(f"synth_normal_bf16_gpu failed ({rc})")
    return out


def normal_f32_gpu(seed: int, tensor: int, sigma: float, shape, start: int = 0, device="cuda"):
    """A torch.float32 CUDA tensor holding the same values as :func:`normal_f32`."""
    import torch

    out = torch.empty(tuple(shape), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(out.device).cuda_stream
    rc = _load_gpu().synth_normal_f32_gpu(seed, tensor, sigma, start, out.numel(),
                                          out.data_ptr(), stream)
    if rc != 0:
        raise RuntimeError(f"synth_normal_f32_gpu failed ({rc})")
    return out
