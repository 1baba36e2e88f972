"""Seeded synthetic inputs for the MoRE router (bf16 Gaussian tensors).

This package only draws numbers: SplitMix64 as a counter-based stream, Box–Muller
normals, rounding to bf16 (the recipe is written out in ``synthetic.c``).  It holds
none of the routing arithmetic, so the CUDA path and the fp64 oracle can both be
fed bit-identical inputs from it.

Tensor ids of the router inputs: X = 0, R1 = 1, R2 = 2.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synthetic.c")
_LIB = os.path.join(_HERE, "libsynthetic.so")

TENSOR_X, TENSOR_R1, TENSOR_R2 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile ``libsynthetic.so`` next to its source (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.synth_normal_bf16.restype = ctypes.c_int
        lib.synth_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_int64, ctypes.c_double, ctypes.c_int, ctypes.c_void_p,
                                          ctypes.c_int]
        lib.synth_normal_at.restype = ctypes.c_double
        lib.synth_normal_at.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_stream_key.restype = ctypes.c_uint64
        lib.synth_stream_key.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_f32_to_bf16.restype = ctypes.c_uint16
        lib.synth_f32_to_bf16.argtypes = [ctypes.c_float]
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def normal_bf16(seed: int, tensor_id: int, rows: int, cols: int, sigma: float = 1.0,
                unit_rms_rows: bool = False, row_begin: int = 0, n_rows: int | None = None,
                out: np.ndarray | None = None, threads: int | None = None) -> np.ndarray:
    """Rows ``[row_begin, row_begin + n_rows)`` of the seeded ``rows x cols`` tensor.

    Returns the raw bf16 bit patterns as a ``uint16`` array of shape ``(n_rows, cols)``.
    ``rows`` is the size of the conceptual tensor (it bounds ``row_begin + n_rows``);
    a row's values do not depend on ``rows``, so any slice of a tensor can be drawn
    on its own and matches the same rows of the whole tensor.
    """
    if n_rows is None:
        n_rows = rows - row_begin
    if row_begin < 0 or n_rows < 0 or row_begin + n_rows > rows:
        raise ValueError("row range outside the tensor")
    if out is None:
        out = np.empty((n_rows, cols), dtype=np.uint16)
    if out.dtype != np.uint16 or out.size != n_rows * cols or not out.flags["C_CONTIGUOUS"]:
        raise ValueError("out must be a C-contiguous uint16 array of n_rows*cols elements")
    rc = _load().synth_normal_bf16(seed, tensor_id, row_begin, n_rows, cols, float(sigma),
                                   1 if unit_rms_rows else 0, out.ctypes.data,
                                   threads or default_threads())
    if rc != 0:
        raise RuntimeError("synth_normal_bf16 failed")
    return out


def normal_at(seed: int, tensor_id: int, j: int) -> float:
    """Normal number ``j`` (fp64, before scaling and rounding) of stream (seed, tensor_id)."""
    lib = _load()
    return lib.synth_normal_at(lib.synth_stream_key(seed, tensor_id), j)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_to_bf16_bits(values) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns bit patterns."""
    u = np.ascontiguousarray(np.asarray(values, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


# --- the router workloads ---------------------------------------------------

def router_inputs(N: int, h: int, r: int, M: int, seed: int = 0, x_unit_rms: bool = False,
                  row_begin: int = 0, n_rows: int | None = None, threads: int | None = None):
    """X (rows of N x h), R1 (h x r), R2 (r x M) as bf16 bit patterns.

    X ~ N(0, 1) (rows optionally rescaled to unit RMS), R1 ~ N(0, 1/h), R2 ~ N(0, 1/r),
    each from its own substream of ``seed``.
    """
    X = normal_bf16(seed, TENSOR_X, N, h, 1.0, x_unit_rms, row_begin, n_rows, threads=threads)
    R1 = normal_bf16(seed, TENSOR_R1, h, r, 1.0 / np.sqrt(h), threads=threads)
    R2 = normal_bf16(seed, TENSOR_R2, r, M, 1.0 / np.sqrt(r), threads=threads)
    return X, R1, R2
