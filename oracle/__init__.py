"""fp64 oracle of the MoRE low-rank router — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The routing library (``mixture_experts_rank_b200``) never
does, and shares no code with it.  The arithmetic lives in ``more_oracle.c``
(plain C loops in double precision); this module only marshals numpy arrays.

Source: "MoRE: Scaling mixture of experts with hardware-aware low-rank routing"
(arXiv 2609.36301), §2 "MoRE layer", App. F eq. (5) and Algorithm 1; the standard
(full-rank) router that App. H.3 fuses the same way (``route_fullrank``).
Parity status of every function: pinned by ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import NamedTuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "more_oracle.c")
_LIB = os.path.join(_HERE, "libmore_oracle.so")


def build(force: bool = False) -> str:
    """Compile ``libmore_oracle.so`` next to its source.

    -O2 without -ffast-math, so the loops keep IEEE double arithmetic in source order.
    """
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None
_P = ctypes.c_void_p


def _bind(lib):
    lib.oracle_route.restype = ctypes.c_int
    lib.oracle_route.argtypes = [_P, _P, _P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_int, _P, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P,
                                 ctypes.c_int]
    lib.oracle_route_fullrank.restype = ctypes.c_int
    lib.oracle_route_fullrank.argtypes = [_P, _P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          _P, ctypes.c_int64, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int]
    lib.oracle_logits_at_fullrank.restype = ctypes.c_int
    lib.oracle_logits_at_fullrank.argtypes = [_P, _P, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int64, _P, _P, _P]
    lib.oracle_logits.restype = ctypes.c_int
    lib.oracle_logits.argtypes = [_P, _P, _P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                  _P, ctypes.c_int64, _P]
    lib.oracle_projection.restype = ctypes.c_int
    lib.oracle_projection.argtypes = [_P, _P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, _P,
                                      ctypes.c_int64, _P]
    lib.oracle_logits_at.restype = ctypes.c_int
    lib.oracle_logits_at.argtypes = [_P, _P, _P, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_int64, _P, _P, _P]
    lib.oracle_train_stats.restype = ctypes.c_int
    lib.oracle_train_stats.argtypes = [_P, _P, _P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       _P, ctypes.c_int64, _P, _P, _P, ctypes.c_int]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _u16(a, shape):
    a = np.ascontiguousarray(a, dtype=np.uint16)
    if a.size != int(np.prod(shape)):
        raise ValueError(f"expected {shape} bf16 elements, got {a.shape}")
    return a


def _rows(rows, N):
    if rows is None:
        return None, N
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    return rows, rows.size


@dataclass
class OracleResult:
    idx: np.ndarray      # (n, k) int32, routing order
    gate: np.ndarray     # (n, k) float64
    logit: np.ndarray    # (n, k) float64, logits of idx
    margin: np.ndarray   # (n,) l_(k) - l_(k+1); inf when k == M
    gaps: np.ndarray     # (n, k) l_(j) - l_(j+1); gaps[:, k-1] == margin
    rms: np.ndarray      # (n,) sqrt(mean_e l_e^2)
    counts: np.ndarray   # (M,) int64 selections per expert over these rows


def route(X, R1, R2, N: int, h: int, r: int, M: int, k: int, rows=None,
          threads: int | None = None) -> OracleResult:
    """Route tokens ``rows`` (default: all N) of bf16 X (N x h) with R1 (h x r), R2 (r x M)."""
    X = _u16(X, (N, h))
    R1 = _u16(R1, (h, r))
    R2 = _u16(R2, (r, M))
    rows, n = _rows(rows, N)
    idx = np.empty((n, k), np.int32)
    gate = np.empty((n, k))
    logit = np.empty((n, k))
    margin = np.empty(n)
    gaps = np.empty((n, k))
    rms = np.empty(n)
    counts = np.empty(M, np.int64)
    rc = _load().oracle_route(X.ctypes.data, R1.ctypes.data, R2.ctypes.data, N, h, r, M, k,
                              None if rows is None else rows.ctypes.data, n, idx.ctypes.data,
                              gate.ctypes.data, logit.ctypes.data, margin.ctypes.data, gaps.ctypes.data,
                              rms.ctypes.data, counts.ctypes.data,
                              threads or max(1, min(64, os.cpu_count() or 1)))
    if rc != 0:
        raise ValueError("oracle_route: invalid arguments")
    return OracleResult(idx, gate, logit, margin, gaps, rms, counts)


def route_fullrank(X, W, N: int, h: int, M: int, k: int, rows=None, threads: int | None = None) -> OracleResult:
    """The standard router of App. H.3 on tokens ``rows`` (default: all N): logits x . W with a
    full-rank bf16 W (h x M), then the selection, gates and statistics of :func:`route`."""
    X = _u16(X, (N, h))
    W = _u16(W, (h, M))
    rows, n = _rows(rows, N)
    idx = np.empty((n, k), np.int32)
    gate = np.empty((n, k))
    logit = np.empty((n, k))
    margin = np.empty(n)
    gaps = np.empty((n, k))
    rms = np.empty(n)
    counts = np.empty(M, np.int64)
    rc = _load().oracle_route_fullrank(X.ctypes.data, W.ctypes.data, N, h, M, k,
                                       None if rows is None else rows.ctypes.data, n, idx.ctypes.data,
                                       gate.ctypes.data, logit.ctypes.data, margin.ctypes.data,
                                       gaps.ctypes.data, rms.ctypes.data, counts.ctypes.data,
                                       threads or max(1, min(64, os.cpu_count() or 1)))
    if rc != 0:
        raise ValueError("oracle_route_fullrank: invalid arguments")
    return OracleResult(idx, gate, logit, margin, gaps, rms, counts)


def logits_at_fullrank(X, W, N: int, h: int, M: int, rows, experts) -> np.ndarray:
    """Full-rank logits x_n . W[:, e] of single (row, expert) pairs, fp64."""
    X = _u16(X, (N, h))
    W = _u16(W, (h, M))
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    experts = np.ascontiguousarray(experts, dtype=np.int32)
    out = np.empty(rows.size)
    if _load().oracle_logits_at_fullrank(X.ctypes.data, W.ctypes.data, N, h, M, rows.size, rows.ctypes.data,
                                         experts.ctypes.data, out.ctypes.data) != 0:
        raise ValueError("oracle_logits_at_fullrank: invalid arguments")
    return out


def logits(X, R1, R2, N: int, h: int, r: int, M: int, rows=None) -> np.ndarray:
    """All M logits of tokens ``rows`` (n x M, float64)."""
    X = _u16(X, (N, h))
    R1 = _u16(R1, (h, r))
    R2 = _u16(R2, (r, M))
    rows, n = _rows(rows, N)
    out = np.empty((n, M))
    rc = _load().oracle_logits(X.ctypes.data, R1.ctypes.data, R2.ctypes.data, N, h, r, M,
                               None if rows is None else rows.ctypes.data, n, out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_logits: invalid arguments")
    return out


def projection(X, R1, N: int, h: int, r: int, rows=None) -> np.ndarray:
    """z = x . R1 of tokens ``rows`` (n x r, float64)."""
    X = _u16(X, (N, h))
    R1 = _u16(R1, (h, r))
    rows, n = _rows(rows, N)
    out = np.empty((n, r))
    rc = _load().oracle_projection(X.ctypes.data, R1.ctypes.data, N, h, r,
                                   None if rows is None else rows.ctypes.data, n, out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_projection: invalid arguments")
    return out


def logits_at(X, R1, R2, N: int, h: int, r: int, M: int, rows, experts) -> np.ndarray:
    """Logit of each (rows[p], experts[p]) pair (float64)."""
    X = _u16(X, (N, h))
    R1 = _u16(R1, (h, r))
    R2 = _u16(R2, (r, M))
    rows = np.ascontiguousarray(rows, dtype=np.int64).ravel()
    experts = np.ascontiguousarray(experts, dtype=np.int32).ravel()
    if rows.size != experts.size:
        raise ValueError("rows and experts differ in length")
    out = np.empty(rows.size)
    rc = _load().oracle_logits_at(X.ctypes.data, R1.ctypes.data, R2.ctypes.data, N, h, r, M, rows.size,
                                  rows.ctypes.data, experts.ctypes.data, out.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_logits_at: invalid arguments")
    return out


class TrainStats(NamedTuple):
    m: np.ndarray     # (n,) largest logit of each token
    Z: np.ndarray     # (n,) sum_j exp(l_j - m)
    psum: np.ndarray  # (M,) sum over the tokens of the full-softmax probabilities


def train_stats(X, R1, R2, N: int, h: int, r: int, M: int, rows=None, threads: int | None = None) -> TrainStats:
    """m, Z and psum of tokens ``rows`` (default: all N): App. F, Algorithm 2, eqs. (6)-(7)."""
    X = _u16(X, (N, h))
    R1 = _u16(R1, (h, r))
    R2 = _u16(R2, (r, M))
    rows, n = _rows(rows, N)
    m = np.empty(n)
    Z = np.empty(n)
    psum = np.empty(M)
    rc = _load().oracle_train_stats(X.ctypes.data, R1.ctypes.data, R2.ctypes.data, N, h, r, M,
                                    None if rows is None else rows.ctypes.data, n, m.ctypes.data,
                                    Z.ctypes.data, psum.ctypes.data,
                                    threads or max(1, min(64, os.cpu_count() or 1)))
    if rc != 0:
        raise ValueError("oracle_train_stats: invalid arguments")
    return TrainStats(m, Z, psum)


class Dispatch(NamedTuple):
    offsets: np.ndarray  # (M + 1,) int64: expert e owns sorted[offsets[e]:offsets[e + 1]]
    sorted: np.ndarray   # (N k,) int64: flat slot ids n k + j, grouped by expert, in slot order


def dispatch(idx, M: int) -> Dispatch:
    """Dispatch bookkeeping after routing ("MoRE", App. E, Fig. 9, "Sort + Count"): the
    (N, k) expert indices flattened to N k slots, stably sorted by expert, and the
    per-expert offsets (exclusive prefix sum of the counts, M + 1 entries).  A library
    stable sort and cumulative sum are the steps; nothing else is done to them."""
    flat = np.ascontiguousarray(idx, dtype=np.int64).ravel()
    if flat.size and (flat.min() < 0 or flat.max() >= M):
        raise ValueError("expert index outside [0, M)")
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=M)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return Dispatch(offsets, order.astype(np.int64))


class RouterGrads(NamedTuple):
    X: np.ndarray   # (N, h) gradient of the loss with respect to X
    R1: np.ndarray  # (h, r) ... to R1
    R2: np.ndarray  # (r, M) ... to R2
    g: np.ndarray   # (N,) g_n = sum_i pbar_i P_ni of eq. (12)


def router_backward_f64(X, R1, R2, top_idx, top_vals_bar, pbar) -> RouterGrads:
    """Backward of the low-rank router ("MoRE", App. F, F.2.2, Algorithm 3 and eqs. (10)-(12)),
    fp64 throughout, for float inputs (the bf16 entry point widens and calls this).

    Two gradients arrive: ``top_vals_bar`` (N x k), the gradient of the loss with respect to
    the selected logits l[n, top_idx[n, j]], and ``pbar`` (M), the gradient with respect to
    psum (eq. (7)).  In the steps of Algorithm 3: z = X R1; the logits l = z R2 and the full
    softmax P over all M experts; g_n = sum_i pbar_i P_ni; the logit gradient
    ybar = P (pbar - g) (eq. (12)) plus top_vals_bar scattered into the selected columns;
    zbar = ybar R2^T and the R2 gradient z^T ybar; the X gradient zbar R1^T and the R1
    gradient X^T zbar.  Matrix products are library matmuls.
    """
    X = np.asarray(X, dtype=np.float64)
    R1 = np.asarray(R1, dtype=np.float64)
    R2 = np.asarray(R2, dtype=np.float64)
    top_idx = np.asarray(top_idx, dtype=np.int64)
    top_vals_bar = np.asarray(top_vals_bar, dtype=np.float64)
    pbar = np.asarray(pbar, dtype=np.float64)
    N = X.shape[0]
    z = X @ R1
    logits = z @ R2
    m = logits.max(axis=1, keepdims=True)
    E = np.exp(logits - m)
    P = E / E.sum(axis=1, keepdims=True)
    g = P @ pbar
    ybar = P * (pbar[None, :] - g[:, None])
    np.add.at(ybar, (np.repeat(np.arange(N), top_idx.shape[1]), top_idx.ravel()), top_vals_bar.ravel())
    zbar = ybar @ R2.T
    return RouterGrads(zbar @ R1.T, X.T @ zbar, z.T @ ybar, g)


def router_backward(X, R1, R2, N: int, h: int, r: int, M: int, top_idx, top_vals_bar, pbar) -> RouterGrads:
    """:func:`router_backward_f64` on bf16 inputs (raw bit patterns, widened exactly)."""
    wide = lambda a, shape: ((_u16(a, shape).astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    return router_backward_f64(wide(X, (N, h)), wide(R1, (h, r)), wide(R2, (r, M)), top_idx, top_vals_bar, pbar)
