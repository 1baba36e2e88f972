"""Fused low-rank MoE router (MoRE) for NVIDIA B200 — Python binding of the C ABI.

Every step of the routing path runs in this package's CUDA library
(``libmore_route.so``, built from ``csrc/`` for sm_100a); this module only
marshals arguments.  PyTorch provides device memory and streams.  There is no
CPU fallback: if the library cannot be loaded, importing raises.

The operation: "MoRE: Scaling mixture of experts with hardware-aware low-rank
routing", §2 "MoRE layer" and App. F, Algorithm 1 — for each token x,
z = x . R1 (h x r), logits z . R2 (r x M), the top-k experts with softmax gates
over the k selected logits, and per-expert selection counts.  The C declarations
are in ``include/more_route.h``.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import _build

__all__ = ["route", "auto_variant", "route_fullrank", "selftest_wait_timeout", "route_train", "route_backward", "route_backward_scratch_bytes", "dispatch",
           "dispatch_scratch_bytes", "route_unfused", "route_unfused_tc", "route_unfused_static", "unfused_scratch_bytes", "device_status",
           "Router", "MoreError", "VARIANTS", "library_path", "abi_version", "KMAX", "STATS_MMAX"]

KMAX = 16
STATS_MMAX = 32768
VARIANTS = {"auto": 0, "fused_tc": 1, "small_n": 2, "cluster": 3}
DISPATCH_VARIANTS = {"auto": 0, "global": 1, "shared": 2}
STATUS = {0: "MORE_OK", 1: "MORE_ERR_INVALID_ARG", 2: "MORE_ERR_UNSUPPORTED", 3: "MORE_ERR_CUDA",
          4: "MORE_ERR_DEVICE"}


class MoreError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


def _load_library() -> ctypes.CDLL:
    path = _build.build()  # rebuilds only when a source is newer than the library
    lib = ctypes.CDLL(path)
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    route_args = [P, P, P, I64, I, I, I, I, P, P, P, P]
    lib.more_route.restype = I
    lib.more_route.argtypes = route_args + [P]
    lib.more_route_variant.restype = I
    lib.more_route_variant.argtypes = route_args + [I, P]
    lib.more_route_unfused.restype = I
    lib.more_route_unfused.argtypes = route_args + [P, ctypes.c_size_t, P]
    lib.more_route_fullrank.restype = I
    lib.more_route_fullrank.argtypes = [P, P, I64, I, I, I, P, P, P, P, P]
    lib.more_selftest_wait_timeout.restype = I
    lib.more_selftest_wait_timeout.argtypes = [P, P]
    lib.more_route_auto_variant.restype = I
    lib.more_route_auto_variant.argtypes = [I64, I, I, I, I]
    lib.more_route_unfused_tc.restype = I
    lib.more_route_unfused_tc.argtypes = route_args + [P, ctypes.c_size_t, P]
    lib.more_route_unfused_static.restype = I
    lib.more_route_unfused_static.argtypes = route_args + [P]
    lib.more_dispatch_scratch_bytes.restype = ctypes.c_size_t
    lib.more_dispatch_scratch_bytes.argtypes = [I64, I, I]
    lib.more_dispatch.restype = I
    lib.more_dispatch.argtypes = [P, I64, I, I, P, P, P, ctypes.c_size_t, P]
    lib.more_dispatch_variant.restype = I
    lib.more_dispatch_variant.argtypes = [P, I64, I, I, P, P, P, ctypes.c_size_t, I, P]
    lib.more_route_train.restype = I
    lib.more_route_train.argtypes = route_args + [P, P, P, P]
    lib.more_route_backward_scratch_bytes.restype = ctypes.c_size_t
    lib.more_route_backward_scratch_bytes.argtypes = [I64, I, I, I]
    lib.more_route_backward.restype = I
    lib.more_route_backward.argtypes = [P, P, P, I64, I, I, I, I] + [P] * 10 + [ctypes.c_size_t, P]
    lib.more_route_unfused_scratch_bytes.restype = ctypes.c_size_t
    lib.more_route_unfused_scratch_bytes.argtypes = [I64, I, I]
    lib.more_device_status.restype = I
    lib.more_device_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.more_status_string.restype = ctypes.c_char_p
    lib.more_status_string.argtypes = [I]
    lib.more_abi_version.restype = I
    lib.more_abi_version.argtypes = []
    return lib


_lib = _load_library()


def library_path() -> str:
    return _build.LIB


def abi_version() -> int:
    return _lib.more_abi_version()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != 0:
        raise MoreError(status, what)


def _as_bf16(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")
    return t


def _outputs(N, k, M, device, out_idx, out_gate, out_count, out_logits, want_logits):
    if out_idx is None:
        out_idx = torch.empty((N, k), dtype=torch.int32, device=device)
    if out_gate is None:
        out_gate = torch.empty((N, k), dtype=torch.float32, device=device)
    if out_count is None:
        out_count = torch.empty((M,), dtype=torch.int32, device=device)
    if out_logits is None and want_logits:
        out_logits = torch.empty((N, k), dtype=torch.float32, device=device)
    return out_idx, out_gate, out_count, out_logits


def route(X: torch.Tensor, R1: torch.Tensor, R2: torch.Tensor, k: int, *, out_idx=None, out_gate=None,
          out_expert_count=None, out_logits=None, return_logits: bool = True, variant: str = "auto",
          stream=None):
    """Route the rows of X (N x h, bf16) with R1 (h x r) and R2 (r x M).

    Returns ``(idx int32 [N,k], gate fp32 [N,k], expert_count int32 [M], logits fp32 [N,k] or None)``.
    Outputs may be passed in to avoid allocation.  Runs asynchronously on ``stream``
    (default: the current stream).
    """
    X, R1, R2 = _as_bf16(X, "X"), _as_bf16(R1, "R1"), _as_bf16(R2, "R2")
    N, h = X.shape
    h1, r = R1.shape
    r1, M = R2.shape
    if h1 != h or r1 != r:
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, R1 {tuple(R1.shape)}, R2 {tuple(R2.shape)}")
    outs = _outputs(N, k, M, X.device, out_idx, out_gate, out_expert_count, out_logits, return_logits)
    st = _lib.more_route_variant(_ptr(X), _ptr(R1), _ptr(R2), N, h, r, M, k, _ptr(outs[0]), _ptr(outs[1]),
                                 _ptr(outs[2]), _ptr(outs[3]), VARIANTS[variant], _stream_handle(stream))
    _check(st, "more_route")
    return outs


def route_train(X: torch.Tensor, R1: torch.Tensor, R2: torch.Tensor, k: int, *, out_idx=None, out_gate=None,
                out_expert_count=None, out_logits=None, out_m=None, out_Z=None, out_psum=None,
                return_logits: bool = True, stream=None):
    """:func:`route` plus the training statistics of the full softmax over all M experts.

    Returns ``(idx, gate, expert_count, logits, m, Z, psum)``: ``m`` [N] the largest logit of
    each token, ``Z`` [N] the sum of exp(logit - m) over all M experts, ``psum`` [M] the
    column sum of the full softmax over the tokens (all fp32).
    """
    X, R1, R2 = _as_bf16(X, "X"), _as_bf16(R1, "R1"), _as_bf16(R2, "R2")
    N, h = X.shape
    h1, r = R1.shape
    r1, M = R2.shape
    if h1 != h or r1 != r:
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, R1 {tuple(R1.shape)}, R2 {tuple(R2.shape)}")
    outs = _outputs(N, k, M, X.device, out_idx, out_gate, out_expert_count, out_logits, return_logits)
    if out_m is None:
        out_m = torch.empty((N,), dtype=torch.float32, device=X.device)
    if out_Z is None:
        out_Z = torch.empty((N,), dtype=torch.float32, device=X.device)
    if out_psum is None:
        out_psum = torch.empty((M,), dtype=torch.float32, device=X.device)
    st = _lib.more_route_train(_ptr(X), _ptr(R1), _ptr(R2), N, h, r, M, k, _ptr(outs[0]), _ptr(outs[1]),
                               _ptr(outs[2]), _ptr(outs[3]), _ptr(out_m), _ptr(out_Z), _ptr(out_psum),
                               _stream_handle(stream))
    _check(st, "more_route_train")
    return (*outs, out_m, out_Z, out_psum)


def route_backward_scratch_bytes(N: int, h: int, r: int, M: int) -> int:
    return int(_lib.more_route_backward_scratch_bytes(N, h, r, M))


def _as_f32(t, name, shape):
    if t is None:
        return None
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != shape:
        raise ValueError(f"{name} must be a contiguous float32 CUDA tensor of shape {shape}")
    return t


def route_backward(X: torch.Tensor, R1: torch.Tensor, R2: torch.Tensor, k: int, *, top_idx=None,
                   top_vals_bar=None, pbar=None, m=None, Z=None, scratch: torch.Tensor | None = None,
                   out_Xbar=None, out_R1bar=None, out_R2bar=None, out_g=None, stream=None):
    """Backward of the router (App. F, Algorithm 3) with z recomputed from X.

    ``top_idx`` (int32 [N, k]) and ``top_vals_bar`` (fp32 [N, k]): the forward's selections and
    the gradient on the selected logits; ``pbar`` (fp32 [M]): the gradient on psum, with ``m``
    and ``Z`` (fp32 [N]) as :func:`route_train` returns them.  Either gradient may be None.
    Returns ``(Xbar fp32 [N, h], R1bar fp32 [h, r], R2bar fp32 [r, M], g fp32 [N])``.
    """
    X, R1, R2 = _as_bf16(X, "X"), _as_bf16(R1, "R1"), _as_bf16(R2, "R2")
    N, h = X.shape
    h1, r = R1.shape
    r1, M = R2.shape
    if h1 != h or r1 != r:
        raise ValueError(f"shape mismatch: X {tuple(X.shape)}, R1 {tuple(R1.shape)}, R2 {tuple(R2.shape)}")
    if top_vals_bar is not None:
        if top_idx is None or top_idx.dtype != torch.int32 or not top_idx.is_cuda or \
                not top_idx.is_contiguous() or tuple(top_idx.shape) != (N, k):
            raise ValueError("top_idx must be a contiguous int32 CUDA tensor of shape [N, k]")
        _as_f32(top_vals_bar, "top_vals_bar", (N, k))
    else:
        top_idx = None
    if pbar is not None:
        _as_f32(pbar, "pbar", (M,))
        if m is None or Z is None:
            raise ValueError("pbar needs the forward's m and Z")
        _as_f32(m, "m", (N,))
        _as_f32(Z, "Z", (N,))
    else:
        m = Z = None
    dev = X.device
    if scratch is None:
        scratch = torch.empty(max(route_backward_scratch_bytes(N, h, r, M), 16), dtype=torch.uint8, device=dev)
    out_Xbar = torch.empty((N, h), dtype=torch.float32, device=dev) if out_Xbar is None else out_Xbar
    out_R1bar = torch.empty((h, r), dtype=torch.float32, device=dev) if out_R1bar is None else out_R1bar
    out_R2bar = torch.empty((r, M), dtype=torch.float32, device=dev) if out_R2bar is None else out_R2bar
    out_g = torch.empty((N,), dtype=torch.float32, device=dev) if out_g is None else out_g
    st = _lib.more_route_backward(_ptr(X), _ptr(R1), _ptr(R2), N, h, r, M, k, _ptr(top_idx), _ptr(top_vals_bar),
                                  _ptr(pbar), _ptr(m), _ptr(Z), _ptr(out_Xbar), _ptr(out_R1bar), _ptr(out_R2bar),
                                  _ptr(out_g), _ptr(scratch), scratch.numel(), _stream_handle(stream))
    _check(st, "more_route_backward")
    return out_Xbar, out_R1bar, out_R2bar, out_g


def dispatch_scratch_bytes(N: int, k: int, M: int) -> int:
    return int(_lib.more_dispatch_scratch_bytes(N, k, M))


def dispatch(idx: torch.Tensor, M: int, *, scratch: torch.Tensor | None = None, out_offsets=None,
             out_sorted=None, variant: str = "auto", stream=None):
    """Dispatch bookkeeping for routing indices ``idx`` (int32 [N, k], CUDA): returns
    ``(offsets int32 [M + 1], sorted int32 [N k])``; expert e owns ``sorted[offsets[e]:offsets[e+1]]``,
    the flat slots n k + j naming it, in increasing order."""
    if idx.dtype != torch.int32 or not idx.is_cuda or not idx.is_contiguous() or idx.dim() != 2:
        raise ValueError("idx must be a contiguous int32 CUDA tensor of shape [N, k]")
    N, k = idx.shape
    if scratch is None:
        scratch = torch.empty(max(dispatch_scratch_bytes(N, k, M), 16), dtype=torch.uint8, device=idx.device)
    if out_offsets is None:
        out_offsets = torch.empty((M + 1,), dtype=torch.int32, device=idx.device)
    if out_sorted is None:
        out_sorted = torch.empty((N * k,), dtype=torch.int32, device=idx.device)
    st = _lib.more_dispatch_variant(_ptr(idx), N, k, M, _ptr(out_offsets), _ptr(out_sorted), _ptr(scratch),
                                    scratch.numel(), DISPATCH_VARIANTS[variant], _stream_handle(stream))
    _check(st, "more_dispatch")
    return out_offsets, out_sorted


def auto_variant(N: int, h: int, r: int, M: int, k: int) -> str | None:
    """The kernel ``route(..., variant="auto")`` runs for this shape (``more_route_auto_variant``),
    or None if the shape fails the argument requirements."""
    v = int(_lib.more_route_auto_variant(N, h, r, M, k))
    return {value: name for name, value in VARIANTS.items()}[v] if v else None


def route_fullrank(X, W, k: int, *, out_idx=None, out_gate=None, out_expert_count=None, out_logits=None,
                   return_logits: bool = True, stream=None):
    """The standard full-rank router x . W (W: h x M), fused (``more_route_fullrank``; App. H.3).
    Same outputs as :func:`route`."""
    X, W = _as_bf16(X, "X"), _as_bf16(W, "W")
    N, h = X.shape
    if W.shape[0] != h:
        raise ValueError(f"W has {W.shape[0]} rows, X has {h} columns")
    M = W.shape[1]
    outs = _outputs(N, k, M, X.device, out_idx, out_gate, out_expert_count, out_logits, return_logits)
    st = _lib.more_route_fullrank(_ptr(X), _ptr(W), N, h, M, k, _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]),
                                  _ptr(outs[3]), _stream_handle(stream))
    _check(st, "more_route_fullrank")
    return outs


def unfused_scratch_bytes(N: int, r: int, M: int) -> int:
    return int(_lib.more_route_unfused_scratch_bytes(N, r, M))


def route_unfused(X, R1, R2, k: int, *, scratch: torch.Tensor | None = None, out_idx=None, out_gate=None,
                  out_expert_count=None, out_logits=None, return_logits: bool = True, stream=None):
    """The materialise-then-top-k comparison path; same results as :func:`route`."""
    X, R1, R2 = _as_bf16(X, "X"), _as_bf16(R1, "R1"), _as_bf16(R2, "R2")
    N, h = X.shape
    r, M = R2.shape
    need = unfused_scratch_bytes(N, r, M)
    if scratch is None:
        scratch = torch.empty(max(need, 16), dtype=torch.uint8, device=X.device)
    outs = _outputs(N, k, M, X.device, out_idx, out_gate, out_expert_count, out_logits, return_logits)
    st = _lib.more_route_unfused(_ptr(X), _ptr(R1), _ptr(R2), N, h, r, M, k, _ptr(outs[0]), _ptr(outs[1]),
                                 _ptr(outs[2]), _ptr(outs[3]), _ptr(scratch), scratch.numel(),
                                 _stream_handle(stream))
    _check(st, "more_route_unfused")
    return outs


def route_unfused_tc(X, R1, R2, k: int, *, scratch: torch.Tensor | None = None, out_idx=None, out_gate=None,
                     out_expert_count=None, out_logits=None, return_logits: bool = True, stream=None):
    """The materialise-then-top-k comparison with the scores written by the fused kernel's
    tensor-core products (``more_route_unfused_tc``); same results as :func:`route`."""
    X, R1, R2 = _as_bf16(X, "X"), _as_bf16(R1, "R1"), _as_bf16(R2, "R2")
    N, h = X.shape
    r, M = R2.shape
    need = unfused_scratch_bytes(N, r, M)
    if scratch is None:
        scratch = torch.empty(max(need, 16), dtype=torch.uint8, device=X.device)
    outs = _outputs(N, k, M, X.device, out_idx, out_gate, out_expert_count, out_logits, return_logits)
    st = _lib.more_route_unfused_tc(_ptr(X), _ptr(R1), _ptr(R2), N, h, r, M, k, _ptr(outs[0]), _ptr(outs[1]),
                                    _ptr(outs[2]), _ptr(outs[3]), _ptr(scratch), scratch.numel(),
                                    _stream_handle(stream))
    _check(st, "more_route_unfused_tc")
    return outs


STATIC_SCRATCH_BYTES = 32 << 20


def route_unfused_static(X, R1, R2, k: int, *, out_idx=None, out_gate=None, out_expert_count=None,
                         out_logits=None, return_logits: bool = True, stream=None):
    """:func:`route_unfused` without a scratch tensor: the library's fixed scratch
    (``STATIC_SCRATCH_BYTES``) is used, so nothing is allocated for it.  For callers that
    may not allocate device memory; calls that overlap on the GPU share the scratch and race.
    """
    X, R1, R2 = _as_bf16(X, "X"), _as_bf16(R1, "R1"), _as_bf16(R2, "R2")
    N, h = X.shape
    r, M = R2.shape
    outs = _outputs(N, k, M, X.device, out_idx, out_gate, out_expert_count, out_logits, return_logits)
    st = _lib.more_route_unfused_static(_ptr(X), _ptr(R1), _ptr(R2), N, h, r, M, k, _ptr(outs[0]),
                                        _ptr(outs[1]), _ptr(outs[2]), _ptr(outs[3]), _stream_handle(stream))
    _check(st, "more_route_unfused_static")
    return outs


def selftest_wait_timeout(stream=None) -> torch.Tensor:
    """Run the failure-path self-test (``more_selftest_wait_timeout``): one bounded wait that
    nothing completes.  Returns the device int32 result (2 once the wait gave up); the device
    error word then holds MORE_DEVERR_WAIT_TIMEOUT (read it with :func:`device_status`)."""
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(_lib.more_selftest_wait_timeout(_ptr(out), _stream_handle(stream)), "more_selftest_wait_timeout")
    return out


def device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the library's device error word."""
    detail = ctypes.c_uint32(0)
    st = _lib.more_device_status(_stream_handle(stream), ctypes.byref(detail))
    if st not in (0, 4):
        _check(st, "more_device_status")
    return int(detail.value)


class Router:
    """Routes host-resident batches: copies X in, routes, copies the results out.

    Device buffers are allocated once for ``max_tokens`` tokens, so repeated calls
    allocate nothing.  ``route_host`` takes a (preferably pinned) CPU bf16 tensor
    and returns CPU tensors (idx, gate, counts, logits).  ``variant`` is the routing
    kernel, as for :func:`route`.
    """

    def __init__(self, R1: torch.Tensor, R2: torch.Tensor, k: int, max_tokens: int, device="cuda",
                 return_logits: bool = True, variant: str = "auto"):
        if variant not in VARIANTS:
            raise ValueError(f"unknown variant {variant!r}")
        self.variant = variant
        self.R1 = R1.to(device=device, dtype=torch.bfloat16).contiguous()
        self.R2 = R2.to(device=device, dtype=torch.bfloat16).contiguous()
        self.h, self.r = self.R1.shape
        self.M = self.R2.shape[1]
        self.k = k
        self.max_tokens = max_tokens
        self.X = torch.empty((max_tokens, self.h), dtype=torch.bfloat16, device=device)
        self.idx = torch.empty((max_tokens, k), dtype=torch.int32, device=device)
        self.gate = torch.empty((max_tokens, k), dtype=torch.float32, device=device)
        self.count = torch.empty((self.M,), dtype=torch.int32, device=device)
        self.logits = torch.empty((max_tokens, k), dtype=torch.float32, device=device) if return_logits else None
        self.h_idx = torch.empty((max_tokens, k), dtype=torch.int32, pin_memory=True)
        self.h_gate = torch.empty((max_tokens, k), dtype=torch.float32, pin_memory=True)
        self.h_count = torch.empty((self.M,), dtype=torch.int32, pin_memory=True)
        self.h_logits = torch.empty((max_tokens, k), dtype=torch.float32, pin_memory=True) \
            if return_logits else None

    def route_host(self, X_host: torch.Tensor, stream=None, synchronize: bool = True):
        N = X_host.shape[0]
        if N > self.max_tokens:
            raise ValueError("batch larger than max_tokens")
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            self.X[:N].copy_(X_host, non_blocking=True)
            logits = None if self.logits is None else self.logits[:N]
            route(self.X[:N], self.R1, self.R2, self.k, out_idx=self.idx[:N], out_gate=self.gate[:N],
                  out_expert_count=self.count, out_logits=logits, variant=self.variant, stream=s)
            self.h_idx[:N].copy_(self.idx[:N], non_blocking=True)
            self.h_gate[:N].copy_(self.gate[:N], non_blocking=True)
            self.h_count.copy_(self.count, non_blocking=True)
            if logits is not None:
                self.h_logits[:N].copy_(logits, non_blocking=True)
        if synchronize:
            s.synchronize()
        return (self.h_idx[:N], self.h_gate[:N], self.h_count,
                None if self.h_logits is None else self.h_logits[:N])

    def bytes_per_call(self, N: int) -> tuple[int, int]:
        """(host-to-device, device-to-host) bytes moved by one ``route_host`` of N tokens."""
        h2d = N * self.h * 2
        d2h = N * self.k * (4 + 4 + (4 if self.logits is not None else 0)) + self.M * 4
        return h2d, d2h
