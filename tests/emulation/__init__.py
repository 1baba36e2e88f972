"""Test-only host emulation of the library's CUDA-core kernels.

The kernel sources in ``mixture_experts_rank_b200/csrc`` are compiled unchanged with g++ after a
textual rewrite of the few CUDA-only constructs:
- ``kernel<<<grid, block, smem, stream>>>(args)`` becomes a call of the fiber runtime;
- shared memory, dynamic and static, comes from the runtime, one copy per CTA;
- the cooperative-groups header is replaced by the runtime's cluster calls.

The runtime (``fibers.cpp``) runs each CTA's threads, or each cluster's, as fibers: barriers, warp
shuffles and DSMEM maps switch between them.  This is checking infrastructure for kernels that
use no tensor-core, TMA or asynchronous-barrier instructions (those cannot be emulated), the way
the oracle checks results.  It is not a way to run the library: the package loads only the
nvcc-built sm_100a library and has no CPU path.
"""
from __future__ import annotations

import ctypes
import os
import re
import shutil
import subprocess
import tempfile

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
CSRC = os.path.join(ROOT, "mixture_experts_rank_b200", "csrc")
KERNELS = ("backward.cu", "route_cluster.cu", "route_small.cu", "dispatch.cu", "route_unfused.cu",
           "route_scores_topk.cu")


def _split_top(s: str) -> list[str]:
    parts, depth, cur = [], 0, ""
    for ch in s:
        depth += ch in "(["
        depth -= ch in ")]"
        if ch == "," and depth == 0:
            parts.append(cur.strip())
            cur = ""
        else:
            cur += ch
    return parts + [cur.strip()]


def _balanced(s: str, i: int) -> int:
    depth = 0
    for j in range(i, len(s)):
        depth += s[j] == "("
        depth -= s[j] == ")"
        if depth == 0:
            return j + 1
    raise ValueError("unbalanced parentheses")


def _shared_decls(src: str) -> str:
    """Block-scope shared-memory declarations become per-CTA storage of the runtime:
    ``extern __shared__ T name[];`` the CTA's dynamic shared memory, and each declarator of
    ``__shared__ T a[..], b[..];`` a buffer of its own (one id per declarator)."""
    src = re.sub(r"extern\s+__shared__\s+(?:__align__\(\d+\)\s+)?([\w:]+)\s+(\w+)\[\];",
                 r"\1* \2 = reinterpret_cast<\1*>(::emu::smem());", src)
    counter = [0]

    def one(m):
        indent, typ, decls = m.group(1), m.group(2), m.group(3)
        out = []
        for d in _split_top(decls):
            name, dims = re.match(r"(\w+)((?:\[[^\]]+\])*)$", d.strip()).groups()
            counter[0] += 1
            out.append(f"{indent}auto& {name} = ::emu::shared_static<{typ}{dims}>({counter[0]});")
        return "\n".join(out)

    return re.sub(r"^([ \t]*)__shared__\s+(?:__align__\(\d+\)\s+)?([\w:]+)\s+([^;]+);", one, src, flags=re.M)


def transform(src: str) -> str:
    """The emulated form of one kernel source."""
    src = src.replace('#include "more_internal.cuh"',
                      '#include "prelude.h"\n#include "more_internal.cuh"\n#include "postlude.h"')
    src = src.replace("#include <cooperative_groups.h>", "")
    src = _shared_decls(src)
    out, pos = "", 0
    for m in re.finditer(r"([A-Za-z_]\w*(?:<\w+>)?)<<<", src):
        if m.start() < pos:
            continue
        cfg_end = src.index(">>>", m.end())
        cfg = _split_top(src[m.end():cfg_end])
        a0 = cfg_end + 3
        a1 = _balanced(src, a0)
        smem = cfg[2] if len(cfg) > 2 else "0"
        out += (src[pos:m.start()] +
                f"::emu::launch(dim3({cfg[0]}), dim3({cfg[1]}), {smem}, [&]() {{ {m.group(1)}({src[a0 + 1:a1 - 1]}); }})")
        pos = a1
    return out + src[pos:]


def available() -> str | None:
    """None when the emulation can be built here, else the reason it cannot."""
    if not shutil.which("g++"):
        return "g++ not found"
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    if not os.path.exists(os.path.join(cuda_inc, "cuda_bf16.h")):
        return "CUDA headers not found"
    return None


def build(out_dir: str | None = None, mutate: dict | None = None) -> str:
    """Compile the emulated kernels; returns the shared library's path.  ``mutate`` maps a kernel
    file name to (text, replacement): a planted mistake, for the tests that show one is caught."""
    out_dir = out_dir or tempfile.mkdtemp(prefix="more_emulation_")
    os.makedirs(out_dir, exist_ok=True)
    srcs = [os.path.join(HERE, "fibers.cpp"), os.path.join(HERE, "entry.cpp")]
    for name in KERNELS:
        with open(os.path.join(CSRC, name)) as f:
            text = f.read()
        if mutate and name in mutate:
            old, new = mutate[name]
            if text.count(old) != 1:
                raise ValueError(f"mutation anchor not found once in {name}: {old!r}")
            text = text.replace(old, new)
        dst = os.path.join(out_dir, name.replace(".cu", "_emulated.cpp"))
        with open(dst, "w") as g:
            g.write(transform(text))
        srcs.append(dst)
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    lib = os.path.join(out_dir, "libmore_emulated.so")
    cmd = ["g++", "-O1", "-std=c++17", "-fPIC", "-shared", "-I", cuda_inc, "-I", os.path.join(ROOT, "include"),
           "-I", CSRC, "-I", HERE, *srcs, "-o", lib]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"emulation build failed:\n{res.stderr[-4000:]}")
    return lib


class Emulated:
    """The emulated library, with host arrays that end against an inaccessible page."""

    def __init__(self, path: str):
        P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        self.lib = lib = ctypes.CDLL(path)
        lib.emu_alloc.restype = P
        lib.emu_alloc.argtypes = [ctypes.c_size_t]
        lib.emu_free.argtypes = [P]
        lib.emu_backward_scratch_bytes.restype = ctypes.c_long
        lib.emu_backward_scratch_bytes.argtypes = [I64, I, I, I]
        lib.emu_backward.restype = I
        lib.emu_backward.argtypes = [P, P, P, I64, I, I, I, I] + [P] * 11
        lib.emu_route_cluster.restype = I
        lib.emu_route_cluster.argtypes = [P, P, P, I64, I, I, I, I, P, P, P, P, P]
        lib.emu_route_small.restype = I
        lib.emu_route_small.argtypes = [P, P, P, I64, I, I, I, I, P, P, P, P, P]
        lib.emu_unfused_scratch_bytes.restype = ctypes.c_long
        lib.emu_unfused_scratch_bytes.argtypes = [I64, I, I]
        lib.emu_route_unfused.restype = I
        lib.emu_route_unfused.argtypes = [P, P, P, I64, I, I, I, I, P, P, P, P, P, P]
        lib.emu_route_cluster_self_zero.restype = I
        lib.emu_route_cluster_self_zero.argtypes = [P, P, P, I64, I, I, I, I, P, P, P, P, P]
        lib.emu_route_small_self_zero.restype = I
        lib.emu_route_small_self_zero.argtypes = [P, P, P, I, I, I, I, P, P, P, P, P]
        lib.emu_threshold_topk.restype = I
        lib.emu_threshold_topk.argtypes = [P, I64, I, I, P, P, P, P, P]
        lib.emu_train_stats.restype = I
        lib.emu_train_stats.argtypes = [P, P, P, I64, I, I, I, P, P, P, P]
        lib.emu_dispatch_scratch_bytes.restype = ctypes.c_long
        lib.emu_dispatch_scratch_bytes.argtypes = [I64, I]
        lib.emu_dispatch.restype = I
        lib.emu_dispatch.argtypes = [P, I64, I, P, P, P, P]
        lib.emu_dispatch_shared.restype = I
        lib.emu_dispatch_shared.argtypes = [P, I64, I, P, P, P, P]
        self._live = []

    def put(self, a) -> int | None:
        if a is None:
            return None
        a = np.ascontiguousarray(a)
        p = self.lib.emu_alloc(max(a.nbytes, 16))
        ctypes.memmove(p, a.ctypes.data, a.nbytes)
        self._live.append(p)
        return p

    def empty(self, nbytes: int) -> int:
        p = self.lib.emu_alloc(max(nbytes, 16))
        self._live.append(p)
        return p

    @staticmethod
    def get(p: int, shape, dtype) -> np.ndarray:
        out = np.empty(shape, dtype)
        ctypes.memmove(out.ctypes.data, p, out.nbytes)
        return out

    def free_all(self):
        for p in self._live:
            self.lib.emu_free(p)
        self._live = []
