"""The CUDA-core kernels of the backward and of the cluster routing variant, run on the CPU under
the test-only thread emulation (tests/emulation), against the fp64 oracle.

The sources are the library's own (``csrc/backward.cu``, ``csrc/route_cluster.cu``), compiled
with g++; each CTA's threads, or each cluster's, run as fibers.  Checks, with the tolerances of
the GPU tests:
- the backward's gradients ("MoRE: Scaling mixture of experts with hardware-aware low-rank
  routing", App. F, Algorithm 3) within 2e-3 of the magnitude bound S
  (tests/test_gpu_training_backward.py);
- the cluster variant's routing (App. F, Algorithm 1, Fig. 12) by the parity rules
  (tests/parity.py).
Every host array ends against an inaccessible page, and the runtime aborts on a deadlock, a write
past a CTA's shared memory, or a DSMEM address outside it.  These checks catch the kernels'
index, barrier and arithmetic mistakes before any GPU runs them; the GPU tests remain the
parity tests proper.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synthetic as syn
from tests import emulation, parity
from tests import test_gpu_training_backward as B


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    reason = emulation.available()
    if reason:
        pytest.skip(reason)
    e = emulation.Emulated(emulation.build(str(tmp_path_factory.mktemp("emulation"))))
    yield e
    e.free_all()


def backward(e, N, h, r, M, k, seed, balance=True, selected=True, idx=None):
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=seed)
    if idx is None:
        idx = oracle.route(X, R1, R2, N, h, r, M, k).idx.astype(np.int32) if N else np.zeros((0, k), np.int32)
    tvb, pbar = B.gradients(N, M, k, seed, balance, selected)
    m, Z = B.saved_stats(X, R1, R2, N, h, r, M)
    status = ctypes.c_uint(0)
    out = {"Xbar": e.empty(N * h * 4), "R1bar": e.empty(h * r * 4), "R2bar": e.empty(r * M * 4), "g": e.empty(N * 4)}
    rc = e.lib.emu_backward(e.put(X), e.put(R1), e.put(R2), N, h, r, M, k,
                            e.put(np.asarray(idx, np.int32)) if selected else None, e.put(tvb), e.put(pbar),
                            e.put(m) if balance else None, e.put(Z) if balance else None, out["Xbar"], out["R1bar"],
                            out["R2bar"], out["g"], e.empty(e.lib.emu_backward_scratch_bytes(N, h, r, M)),
                            ctypes.addressof(status))
    assert rc == 0
    got = {"Xbar": e.get(out["Xbar"], (N, h), np.float32), "R1bar": e.get(out["R1bar"], (h, r), np.float32),
           "R2bar": e.get(out["R2bar"], (r, M), np.float32), "g": e.get(out["g"], (N,), np.float32)}
    ref, S = B.reference(X, R1, R2, N, h, r, M, k, idx, tvb, pbar)
    B.compare(got, ref, S)
    e.free_all()
    return status.value


@pytest.mark.parametrize("N,h,r,M,k", [(300, 128, 32, 192, 4), (97, 256, 16, 256, 16), (65, 200, 48, 200, 8),
                                       (33, 64, 128, 1024, 8), (1, 64, 32, 64, 1)])
def test_backward_kernels_match_oracle(emu, N, h, r, M, k):
    assert backward(emu, N, h, r, M, k, seed=N) == 0


@pytest.mark.parametrize("balance,selected", [(False, True), (True, False), (False, False)])
def test_backward_kernels_with_one_gradient_absent(emu, balance, selected):
    assert backward(emu, 70, 128, 32, 192, 4, seed=3, balance=balance, selected=selected) == 0


def test_backward_kernels_skip_out_of_range_selections(emu):
    idx = np.tile(np.array([[5, 5, 200, -1]], np.int32), (40, 1))
    idx[::3, 1] = 191
    assert backward(emu, 40, 128, 32, 192, 4, seed=4, idx=idx) == 4  # MORE_DEVERR_BAD_INPUT


def test_backward_kernels_empty_batch(emu):
    assert backward(emu, 0, 64, 32, 64, 4, seed=0) == 0


def cluster(e, X, R1, R2, N, h, r, M, k, exact=False):
    out = [e.empty(N * k * 4), e.empty(N * k * 4), e.empty(M * 4), e.empty(N * k * 4)]
    status = ctypes.c_uint(0)
    assert e.lib.emu_route_cluster(e.put(X), e.put(R1), e.put(R2), N, h, r, M, k, *out, ctypes.addressof(status)) == 0
    idx, gate = e.get(out[0], (N, k), np.int32), e.get(out[1], (N, k), np.float32)
    cnt, logits = e.get(out[2], (M,), np.int32), e.get(out[3], (N, k), np.float32)
    e.free_all()
    assert status.value == 0
    return parity.compare(X, R1, R2, N, h, r, M, k, idx, gate, cnt, logits, exact=exact)


@pytest.mark.parametrize("N,h,r,M,k", [
    (8, 2048, 32, 4096, 8),   # decode shape
    (13, 256, 32, 512, 8),    # ragged last cluster
    (9, 64, 16, 8, 8),        # M = 8: seven of the eight CTAs hold no expert; k = M
    (20, 200, 48, 200, 1),    # r = 48, ragged M, k = 1
    (5, 64, 128, 16, 16),     # r = 128, k = M = 16
])
def test_cluster_routing_matches_oracle(emu, N, h, r, M, k):
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=N)
    cluster(emu, X, R1, R2, N, h, r, M, k)


def test_cluster_routing_tie_heavy_exact(emu):
    """Integer logits with many exact ties (R1 = R2 = I): the lower expert must win across CTAs."""
    M, N, k = 64, 100, 8
    X = syn.f32_to_bf16_bits(np.random.default_rng(8).integers(-3, 4, size=(N, M)).astype(np.float32))
    eye = syn.f32_to_bf16_bits(np.eye(M, dtype=np.float32))
    cluster(emu, X, eye, eye, N, M, M, M, k, exact=True)


@pytest.mark.parametrize("name,old,new", [
    ("backward.cu", "(pbt[e] - tg[t])", "(pbt[e] + tg[t])"),                   # the sign of g in ybar
    ("route_cluster.cu", "for (int p = 0; p < kCluster; ++p) z +=", "for (int p = 1; p < kCluster; ++p) z +="),
])
def test_planted_kernel_mistake_is_caught(tmp_path, name, old, new):
    """A mistake planted in a kernel source fails these checks (a dropped partial z, a sign)."""
    reason = emulation.available()
    if reason:
        pytest.skip(reason)
    e = emulation.Emulated(emulation.build(str(tmp_path), mutate={name: (old, new)}))
    with pytest.raises(AssertionError):
        if name == "backward.cu":
            backward(e, 70, 128, 32, 192, 4, seed=3)
        else:
            X, R1, R2 = syn.router_inputs(13, 256, 32, 512, seed=13)
            cluster(e, X, R1, R2, 13, 256, 32, 512, 8)
    e.free_all()
