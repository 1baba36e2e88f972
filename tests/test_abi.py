"""The C ABI library loads, exports every declared symbol, and rejects bad arguments
before touching a GPU (these calls return before any CUDA runtime call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


def declared_functions():
    names = []
    for fn in sorted(os.listdir(HEADER_DIR)):
        if fn.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(more_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    import mixture_experts_rank_b200 as m
    return m._lib


def test_header_declares_the_route_entry_points():
    names = declared_functions()
    for required in ("more_route", "more_route_variant", "more_route_train", "more_route_backward",
                     "more_route_backward_scratch_bytes", "more_route_unfused", "more_route_unfused_tc", "more_route_fullrank",
                     "more_route_unfused_scratch_bytes", "more_device_status", "more_status_string",
                     "more_abi_version"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_abi_version_and_status_strings(lib):
    assert lib.more_abi_version() == 1
    for code in range(5):
        assert lib.more_status_string(code).startswith(b"MORE_")
    assert lib.more_status_string(99) == b"unknown more_status"


def call(lib, N=16, h=64, r=32, M=64, k=4, X=16, R1=16, R2=16, idx=16, gate=16, cnt=16, logits=None,
         variant=0):
    P = ctypes.c_void_p
    return lib.more_route_variant(P(X) if X else None, P(R1) if R1 else None, P(R2) if R2 else None, N, h,
                                  r, M, k, P(idx) if idx else None, P(gate) if gate else None,
                                  P(cnt) if cnt else None, P(logits) if logits else None, variant, None)


@pytest.mark.parametrize("kwargs,expected", [
    (dict(k=0), 1), (dict(k=65), 1), (dict(N=-1), 1), (dict(h=4), 1), (dict(h=66), 1),
    (dict(M=4), 1), (dict(M=70), 1), (dict(X=0), 1), (dict(R1=0), 1), (dict(R2=0), 1),
    (dict(idx=0), 1), (dict(gate=0), 1), (dict(cnt=0), 1), (dict(X=24), 1), (dict(gate=40), 1),
    (dict(logits=8), 1), (dict(variant=7), 1),
    (dict(k=17, M=64), 2), (dict(r=24), 2), (dict(r=8), 2), (dict(r=144), 2), (dict(M=262152), 2),
])
def test_invalid_arguments_are_rejected(lib, kwargs, expected):
    assert call(lib, **kwargs) == expected


def test_unfused_scratch_size_and_checks(lib):
    n = lib.more_route_unfused_scratch_bytes(1000, 32, 256)
    assert n >= 1000 * 32 * 2 + 1000 * 256 * 4
    assert lib.more_route_unfused_scratch_bytes(-1, 32, 256) == 0
    P = ctypes.c_void_p
    # too little scratch
    st = lib.more_route_unfused(P(16), P(16), P(16), 1000, 64, 32, 256, 4, P(16), P(16), P(16), None, P(16),
                                n - 1, None)
    assert st == 1


@pytest.mark.parametrize("shape,expected", [
    ((1, 2048, 16, 4096, 4), "small_n"), ((148, 2048, 16, 4096, 4), "small_n"),
    ((1, 2048, 32, 4096, 8), "cluster"), ((64, 2048, 32, 4096, 8), "cluster"),   # r (h + M) = 196608
    ((65, 2048, 32, 4096, 8), "small_n"), ((148, 2048, 32, 4096, 8), "small_n"),
    ((1, 2048, 32, 4088, 8), "small_n"),            # just below 196608
    ((148, 2048, 128, 4096, 16), "cluster"),        # r (h + M) >= 393216 at any N
    ((149, 2048, 32, 4096, 8), "cluster"), ((1024, 2048, 32, 4096, 8), "cluster"),
    ((2048, 2048, 32, 4096, 8), "fused_tc"), ((262144, 2048, 32, 4096, 8), "fused_tc"),
    ((1900, 2048, 16, 4096, 4), "cluster"), ((1940, 2048, 16, 4096, 4), "fused_tc"),
    ((1430, 2048, 32, 4096, 8), "cluster"), ((1450, 2048, 32, 4096, 8), "fused_tc"),
    ((4096, 2048, 16, 4096, 4), "fused_tc"),
    ((262144, 2048, 128, 4096, 16), "cluster"),     # the fused kernel's plan does not hold r = 128, k > 8
    ((262144, 2048, 128, 8192, 8), "fused_tc"), ((262144, 2048, 128, 65536, 8), "fused_tc"),
    ((262144, 2048, 48, 4096, 8), "cluster"),       # r outside the fused kernel's ranks
    ((32768, 4096, 64, 65536, 8), "fused_tc"),
    ((16, 64, 32, 64, 0), None), ((16, 64, 24, 64, 4), None),
])
def test_auto_variant_follows_the_measured_crossovers(shape, expected):
    """AUTO's choice (host-only, no GPU): small-N up to 148 tokens unless the weights one CTA
    would read are large (then the cluster kernel), the cluster kernel up to the
    fused kernel's one-tile floor, the fused kernel beyond, and the cluster kernel for shapes the
    fused kernel's shared-memory plan cannot hold."""
    import mixture_experts_rank_b200 as m
    assert m.auto_variant(*shape) == expected


@pytest.mark.parametrize("kwargs,expected", [
    (dict(k=0), 1), (dict(k=65), 1), (dict(N=-1), 1), (dict(h=4), 1), (dict(h=66), 1), (dict(M=70), 1),
    (dict(X=0), 1), (dict(W=0), 1), (dict(idx=0), 1), (dict(cnt=0), 1), (dict(W=24), 1), (dict(logits=8), 1),
    (dict(k=17, M=64), 2), (dict(M=262152), 2),
])
def test_fullrank_rejects_invalid_arguments(lib, kwargs, expected):
    P = ctypes.c_void_p
    args = dict(N=16, h=64, M=64, k=4, X=16, W=16, idx=16, gate=16, cnt=16, logits=None)
    args.update(kwargs)
    opt = lambda v: P(v) if v else None
    st = lib.more_route_fullrank(opt(args["X"]), opt(args["W"]), args["N"], args["h"], args["M"], args["k"],
                                 opt(args["idx"]), opt(args["gate"]), opt(args["cnt"]), opt(args["logits"]), None)
    assert st == expected


def test_selftest_checks_its_output_pointer(lib):
    P = ctypes.c_void_p
    assert lib.more_selftest_wait_timeout(None, None) == 1
    assert lib.more_selftest_wait_timeout(P(18), None) == 1   # not 4-byte aligned


def test_unfused_tc_checks_rank_and_scratch(lib):
    """The tensor-core materialisation takes r in {16, 32, 64, 128} and the unfused scratch size."""
    n = lib.more_route_unfused_scratch_bytes(1000, 32, 256)
    P = ctypes.c_void_p
    args = lambda r, nbytes: (P(16), P(16), P(16), 1000, 64, r, 256, 4, P(16), P(16), P(16), None, P(16), nbytes,
                              None)
    assert lib.more_route_unfused_tc(*args(32, n - 1)) == 1
    assert lib.more_route_unfused_tc(*args(48, 1 << 30)) == 2
    assert lib.more_route_unfused_tc(*args(96, 1 << 30)) == 2
    assert lib.more_route_unfused_tc(*args(24, 1 << 30)) == 2   # not a multiple of 16: outside every path


@pytest.mark.parametrize("kwargs,expected", [
    (dict(psum=0), 1), (dict(m=0), 1), (dict(Z=0), 1), (dict(psum=8), 1), (dict(m=40), 1),
    (dict(k=0), 1), (dict(M=32776), 2),
])
def test_train_entry_rejects_invalid_arguments(lib, kwargs, expected):
    P = ctypes.c_void_p
    args = dict(N=16, h=64, r=32, M=64, k=4, m=16, Z=16, psum=16)
    args.update(kwargs)
    opt = lambda v: P(v) if v else None
    st = lib.more_route_train(P(16), P(16), P(16), args["N"], args["h"], args["r"], args["M"], args["k"], P(16),
                              P(16), P(16), None, opt(args["m"]), opt(args["Z"]), opt(args["psum"]), None)
    assert st == expected


@pytest.mark.parametrize("kwargs,expected", [
    (dict(k=0), 1), (dict(M=0), 1), (dict(N=-1), 1), (dict(offsets=0), 1), (dict(offsets=8), 1),
    (dict(idx=0), 1), (dict(sorted_=0), 1), (dict(scratch=0), 1), (dict(scratch_bytes=-1), 1),
    (dict(k=17), 2), (dict(M=262152), 2),
])
def test_dispatch_rejects_invalid_arguments(lib, kwargs, expected):
    P = ctypes.c_void_p
    a = dict(N=100, k=4, M=64, idx=16, offsets=16, sorted_=16, scratch=16, scratch_bytes=0)
    a.update(kwargs)
    need = lib.more_dispatch_scratch_bytes(max(a["N"], 0), max(a["k"], 1), max(a["M"], 1))
    nbytes = need + a["scratch_bytes"] if kwargs.get("scratch_bytes") is not None else need
    opt = lambda v: P(v) if v else None
    st = lib.more_dispatch(opt(a["idx"]), a["N"], a["k"], a["M"], opt(a["offsets"]), opt(a["sorted_"]),
                           opt(a["scratch"]), nbytes, None)
    assert st == expected


def test_dispatch_scratch_size():
    import mixture_experts_rank_b200 as m
    assert m.dispatch_scratch_bytes(262144, 8, 4096) >= (262144 * 8 // 2048) * 4096 * 4
    assert m.dispatch_scratch_bytes(-1, 8, 64) == 0
    assert m.dispatch_scratch_bytes(1 << 28, 16, 64) == 0  # N k beyond 2^31 slots


def test_package_refuses_to_run_without_the_library(monkeypatch, tmp_path):
    """The binding has no fallback: a missing nvcc and library means import fails."""
    import importlib
    import sys
    import mixture_experts_rank_b200._build as b
    monkeypatch.setattr(b, "LIB", str(tmp_path / "missing.so"))
    monkeypatch.setenv("NVCC", str(tmp_path / "no-nvcc"))
    monkeypatch.setattr(b.shutil, "which", lambda _: None)
    monkeypatch.setattr(b.os.path, "exists", lambda p: False)
    saved = sys.modules.pop("mixture_experts_rank_b200")
    try:
        with pytest.raises(RuntimeError):
            importlib.import_module("mixture_experts_rank_b200")
    finally:
        sys.modules["mixture_experts_rank_b200"] = saved


@pytest.mark.parametrize("kwargs,expected", [
    (dict(k=0), 1), (dict(N=-1), 1), (dict(h=4), 1), (dict(M=70), 1), (dict(X=0), 1), (dict(R1=0), 1),
    (dict(R1bar=0), 1), (dict(R2bar=0), 1), (dict(Xbar=0), 1), (dict(scratch=0), 1), (dict(idx=0), 1),
    (dict(m=0), 1), (dict(Z=0), 1), (dict(pbar=8), 1), (dict(g=40), 1), (dict(short=1), 1),
    (dict(r=24), 2), (dict(r=144), 2), (dict(k=17, M=64), 2), (dict(M=262152), 2),
])
def test_backward_rejects_invalid_arguments(lib, kwargs, expected):
    P = ctypes.c_void_p
    a = dict(N=100, h=64, r=32, M=64, k=4, X=16, R1=16, R2=16, idx=16, tvb=16, pbar=16, m=16, Z=16, Xbar=16,
             R1bar=16, R2bar=16, g=None, scratch=16, short=0)
    a.update(kwargs)
    need = lib.more_route_backward_scratch_bytes(max(a["N"], 0), a["h"], a["r"], a["M"])
    opt = lambda v: P(v) if v else None
    st = lib.more_route_backward(opt(a["X"]), opt(a["R1"]), opt(a["R2"]), a["N"], a["h"], a["r"], a["M"], a["k"],
                                 opt(a["idx"]), opt(a["tvb"]), opt(a["pbar"]), opt(a["m"]), opt(a["Z"]),
                                 opt(a["Xbar"]), opt(a["R1bar"]), opt(a["R2bar"]), opt(a["g"]), opt(a["scratch"]),
                                 need - a["short"], None)
    assert st == expected


def test_backward_scratch_size():
    import mixture_experts_rank_b200 as m
    # z and zbar ([N][r padded to a power of two >= 16], fp32), g, and the per-split partial sums
    assert m.route_backward_scratch_bytes(262144, 2048, 32, 4096) >= 2 * 262144 * 32 * 4 + 262144 * 4
    assert m.route_backward_scratch_bytes(1000, 64, 48, 64) >= 2 * 1000 * 64 * 4
    assert m.route_backward_scratch_bytes(0, 64, 32, 64) >= 0
    assert m.route_backward_scratch_bytes(-1, 64, 32, 64) == 0
    assert m.route_backward_scratch_bytes(10, 64, 144, 64) == 0


@pytest.mark.parametrize("variant,M,expected", [(3, 64, 1), (-1, 64, 1), (2, 32776, 2), (1, 262152, 2)])
def test_dispatch_variant_rejects_invalid_arguments(lib, variant, M, expected):
    P = ctypes.c_void_p
    need = lib.more_dispatch_scratch_bytes(100, 4, min(M, 262144))
    st = lib.more_dispatch_variant(P(16), 100, 4, M, P(16), P(16), P(16), need, variant, None)
    assert st == expected


def test_static_entry_point_checks_arguments_before_its_size_limit(lib):
    """A call with bad arguments returns MORE_ERR_INVALID_ARG even when the problem would also
    be too large for the fixed scratch (the arguments are checked first, as for
    more_route_unfused); a valid but too-large problem is MORE_ERR_UNSUPPORTED only then."""
    P = ctypes.c_void_p
    N, h, r, M, k = 1 << 20, 64, 32, 4096, 4           # far beyond the 32 MiB scratch
    assert lib.more_route_unfused_scratch_bytes(N, r, M) > (32 << 20)
    # null X
    assert lib.more_route_unfused_static(None, P(16), P(16), N, h, r, M, k, P(16), P(16), P(16), None,
                                         None) == 1
    # h not a multiple of 8, k > M
    assert lib.more_route_unfused_static(P(16), P(16), P(16), N, 66, r, M, k, P(16), P(16), P(16), None,
                                         None) == 1
    assert lib.more_route_unfused_static(P(16), P(16), P(16), N, h, r, 16, 17, P(16), P(16), P(16), None,
                                         None) == 1
    # misaligned output
    assert lib.more_route_unfused_static(P(16), P(16), P(16), N, h, r, M, k, P(20), P(16), P(16), None,
                                         None) == 1
