"""The library's CUDA-core kernels run on the CPU under the test-only thread emulation
(tests/emulation), against the fp64 oracle.

The sources are the library's own, compiled with g++: backward, cluster and small-N routing,
training statistics, dispatch, and the unfused path.  Each CTA's threads, or each cluster's, run
as fibers.  Checks, with the tolerances of the GPU tests:
- the backward's gradients ("MoRE: Scaling mixture of experts with hardware-aware low-rank
  routing", App. F, Algorithm 3) within 2e-3 of the magnitude bound S
  (tests/test_gpu_training_backward.py);
- routing (App. F, Algorithm 1, Fig. 12) by the parity rules (tests/parity.py);
- the training statistics (Algorithm 2) within the bounds of tests/test_gpu_train_stats.py;
- dispatch (Fig. 9) bit-exact.
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
    (1, 2048, 32, 4096, 8),   # one token
    (3, 4096, 64, 1024, 4),   # 512 hidden rows per CTA: two staged chunks
    (7, 136, 16, 64, 2),      # 24-row slices: the last CTAs hold no hidden row
    (2, 64, 32, 8192, 8),     # 1024 experts per CTA: two 512-expert passes
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
    ("route_cluster.cu", "acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], 16);", "acc[t] += 0.f;"),  # half-warp rows lost
    ("route_scores_topk.cu", "lane < k && lv >= xv", "lane < k && lv > xv"),  # equal values: later expert first
    ("route_scores_topk.cu", "first ? lmax >= floor0", "first ? lmax > floor0"),  # drops values at the floor
])
def test_planted_kernel_mistake_is_caught(tmp_path, name, old, new):
    """A mistake planted in a kernel source fails these checks (a dropped partial z, the lost rows
    of a half warp, a sign, the order of equal scores, a first-chunk filter that drops values at
    its floor)."""
    reason = emulation.available()
    if reason:
        pytest.skip(reason)
    e = emulation.Emulated(emulation.build(str(tmp_path), mutate={name: (old, new)}))
    with pytest.raises(AssertionError):
        if name == "backward.cu":
            backward(e, 70, 128, 32, 192, 4, seed=3)
        elif name == "route_scores_topk.cu":
            ties = np.random.default_rng(0).integers(-3, 4, size=(40, 520)).astype(np.float32)
            check_threshold_topk(e, ties, 4)
        else:
            X, R1, R2 = syn.router_inputs(13, 256, 48, 512, seed=13)  # r = 48: a full and a half column block
            cluster(e, X, R1, R2, 13, 256, 48, 512, 8)
    e.free_all()


def route_with(e, entry, X, R1, R2, N, h, r, M, k, exact=False):
    out = [e.empty(N * k * 4), e.empty(N * k * 4), e.empty(M * 4), e.empty(N * k * 4)]
    status = ctypes.c_uint(0)
    args = [e.put(X), e.put(R1), e.put(R2), N, h, r, M, k, *out]
    if entry == "unfused":
        args.append(e.empty(e.lib.emu_unfused_scratch_bytes(N, r, M)))
    fn = e.lib.emu_route_unfused if entry == "unfused" else e.lib.emu_route_small
    assert fn(*args, ctypes.addressof(status)) == 0
    idx, gate = e.get(out[0], (N, k), np.int32), e.get(out[1], (N, k), np.float32)
    cnt, logits = e.get(out[2], (M,), np.int32), e.get(out[3], (N, k), np.float32)
    e.free_all()
    assert status.value == 0
    return parity.compare(X, R1, R2, N, h, r, M, k, idx, gate, cnt, logits, exact=exact)


@pytest.mark.parametrize("entry", ["small_n", "unfused"])
@pytest.mark.parametrize("N,h,r,M,k", [(7, 2048, 32, 4096, 8), (33, 136, 48, 64, 8), (20, 72, 16, 200, 1),
                                       (9, 256, 64, 16, 16), (11, 128, 32, 304, 3), (13, 96, 16, 128, 5),
                                       (6, 64, 32, 512, 12)])
def test_routing_kernels_match_oracle(emu, entry, N, h, r, M, k):
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=N)
    route_with(emu, entry, X, R1, R2, N, h, r, M, k)


@pytest.mark.parametrize("entry", ["small_n", "unfused"])
def test_routing_kernels_tie_heavy_exact(emu, entry):
    M, N, k = 64, 60, 8
    X = syn.f32_to_bf16_bits(np.random.default_rng(9).integers(-3, 4, size=(N, M)).astype(np.float32))
    eye = syn.f32_to_bf16_bits(np.eye(M, dtype=np.float32))
    route_with(emu, entry, X, eye, eye, N, M, M, M, k, exact=True)


def threshold_topk(e, scores, k):
    N, M = scores.shape
    out = (e.empty(N * k * 4), e.empty(N * k * 4), e.empty(M * 4), e.empty(N * k * 4))
    status = ctypes.c_uint(0)
    assert e.lib.emu_threshold_topk(e.put(np.asarray(scores, np.float32)), N, M, k, *out,
                                    ctypes.addressof(status)) == 0
    got = (e.get(out[0], (N, k), np.int32), e.get(out[1], (N, k), np.float32), e.get(out[2], (M,), np.int32),
           e.get(out[3], (N, k), np.float32))
    e.free_all()
    assert status.value == 0
    return got


def check_threshold_topk(e, scores, k):
    """The selection is fixed by the fp32 scores themselves: the k largest in routing order
    (larger value first, lower expert first on equal values), softmax over them, counts."""
    N, M = scores.shape
    idx, gate, cnt, logits = threshold_topk(e, scores, k)
    order = np.lexsort((np.broadcast_to(np.arange(M), (N, M)), -scores.astype(np.float64)), axis=1)[:, :k]
    np.testing.assert_array_equal(idx, order)
    sel = np.take_along_axis(scores, order, axis=1)
    np.testing.assert_array_equal(logits, sel)
    ex = np.exp(sel.astype(np.float64) - sel[:, :1])
    np.testing.assert_allclose(gate, ex / ex.sum(axis=1, keepdims=True), rtol=0, atol=2e-6)
    np.testing.assert_array_equal(cnt, np.bincount(order.ravel(), minlength=M))


@pytest.mark.parametrize("N,M,k", [(50, 8, 8), (64, 40, 3), (33, 128, 16), (40, 200, 1), (25, 1000, 8),
                                   (6, 4096, 8), (9, 4104, 5), (3, 520, 16)])
def test_threshold_topk_kernel_on_oracle_scores(emu, N, M, k):
    """The tensor-core unfused path's top-k kernel on fp32 scores taken from the oracle's logits
    (ragged chunks: M = 40, 200, 1000, 4104; k = 1 .. 16)."""
    X, R1, R2 = syn.router_inputs(N, 64, 16, M, seed=M + k)
    check_threshold_topk(emu, oracle.logits(X, R1, R2, N, 64, 16, M).astype(np.float32), k)


@pytest.mark.parametrize("k", [1, 4, 16])
def test_threshold_topk_kernel_ties_and_orders(emu, k):
    """Small integers (ties inside and across chunks), then rows in ascending order (every value
    enters the list), descending order (only the first chunk does), and constant rows."""
    rng = np.random.default_rng(k)
    M = 520
    rows = [rng.integers(-3, 4, size=(40, M)).astype(np.float32),
            np.tile(np.arange(M, dtype=np.float32), (3, 1)),
            np.tile(np.arange(M, dtype=np.float32)[::-1].copy(), (3, 1)),
            np.full((3, M), 2.5, np.float32)]
    check_threshold_topk(emu, np.concatenate(rows), k)


@pytest.mark.parametrize("h,r,M,k", [(2048, 32, 4096, 8), (136, 48, 64, 8), (72, 16, 200, 1)])
def test_small_n_single_token_zeroes_its_counts(emu, h, r, M, k):
    """A one-token call runs on one CTA, which zeroes the counts itself (no memset is issued):
    counts that start as garbage end as the bincount of the token's k selections."""
    e = emu
    X, R1, R2 = syn.router_inputs(1, h, r, M, seed=h + r)
    out = [e.empty(k * 4), e.empty(k * 4), e.empty(M * 4), e.empty(k * 4)]
    status = ctypes.c_uint(0)
    assert e.lib.emu_route_small_self_zero(e.put(X), e.put(R1), e.put(R2), h, r, M, k, *out,
                                           ctypes.addressof(status)) == 0
    idx, gate = e.get(out[0], (1, k), np.int32), e.get(out[1], (1, k), np.float32)
    cnt, logits = e.get(out[2], (M,), np.int32), e.get(out[3], (1, k), np.float32)
    e.free_all()
    assert status.value == 0
    parity.compare(X, R1, R2, 1, h, r, M, k, idx, gate, cnt, logits)


@pytest.mark.parametrize("N,h,r,M,k", [(1, 2048, 32, 4096, 8), (8, 136, 48, 64, 8), (5, 72, 16, 200, 1)])
def test_cluster_single_cluster_zeroes_its_counts(emu, N, h, r, M, k):
    """Up to 8 tokens run on one cluster, whose CTAs zero the counts themselves (no memset is
    issued): counts that start as garbage end as the bincount of the selections."""
    e = emu
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=N + h)
    out = [e.empty(N * k * 4), e.empty(N * k * 4), e.empty(M * 4), e.empty(N * k * 4)]
    status = ctypes.c_uint(0)
    assert e.lib.emu_route_cluster_self_zero(e.put(X), e.put(R1), e.put(R2), N, h, r, M, k, *out,
                                             ctypes.addressof(status)) == 0
    idx, gate = e.get(out[0], (N, k), np.int32), e.get(out[1], (N, k), np.float32)
    cnt, logits = e.get(out[2], (M,), np.int32), e.get(out[3], (N, k), np.float32)
    e.free_all()
    assert status.value == 0
    parity.compare(X, R1, R2, N, h, r, M, k, idx, gate, cnt, logits)


@pytest.mark.parametrize("N,h,r,M", [(23, 128, 32, 192), (6, 512, 16, 1000), (1, 64, 128, 64)])
def test_train_stats_kernel_matches_oracle(emu, N, h, r, M):
    e = emu
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=N + 1)
    pm, pz, pp = e.empty(N * 4), e.empty(N * 4), e.empty(M * 4)
    status = ctypes.c_uint(0)
    assert e.lib.emu_train_stats(e.put(X), e.put(R1), e.put(R2), N, h, r, M, pm, pz, pp,
                                 ctypes.addressof(status)) == 0
    gm, gz, gp = e.get(pm, (N,), np.float32), e.get(pz, (N,), np.float32), e.get(pp, (M,), np.float32)
    e.free_all()
    o = oracle.train_stats(X, R1, R2, N, h, r, M)
    tol = parity.LOGIT_TOL * oracle.route(X, R1, R2, N, h, r, M, 1).rms
    assert np.all(np.abs(gm - o.m) <= tol)
    assert np.all(np.abs(np.log(gz.astype(np.float64)) - np.log(o.Z)) <= 2 * tol + 1e-5)
    assert np.all(np.abs(gp - o.psum) / o.psum <= 4 * tol.max() + 1e-5)


@pytest.mark.parametrize("variant", ["global", "shared"])
@pytest.mark.parametrize("N,k,M,seed", [(1, 1, 8, 0), (37, 3, 16, 1), (3000, 8, 1000, 2), (700, 4, 4096, 3),
                                        (9000, 8, 64, 5)])
def test_dispatch_kernels_match_oracle(emu, variant, N, k, M, seed):
    e = emu
    idx = np.random.default_rng(seed).integers(0, M, size=(N, k)).astype(np.int32)
    S = N * k
    off, srt = e.empty((M + 1) * 4), e.empty(S * 4)
    status = ctypes.c_uint(0)
    fn = e.lib.emu_dispatch_shared if variant == "shared" else e.lib.emu_dispatch
    assert fn(e.put(idx), S, M, off, srt, e.empty(e.lib.emu_dispatch_scratch_bytes(S, M)),
              ctypes.addressof(status)) == 0
    got_off, got_srt = e.get(off, (M + 1,), np.int32), e.get(srt, (S,), np.int32)
    e.free_all()
    o = oracle.dispatch(idx, M)
    np.testing.assert_array_equal(got_off, o.offsets)
    np.testing.assert_array_equal(got_srt, o.sorted)
    assert status.value == 0


def test_shared_dispatch_at_its_chunk_cap(emu):
    """700,000 slots: the shared-memory variant's full 296 chunks, several batches each."""
    test_dispatch_kernels_match_oracle(emu, "shared", 87500, 8, 4096, 11)


@pytest.mark.parametrize("variant", ["global", "shared"])
def test_dispatch_kernels_skip_out_of_range(emu, variant):
    e = emu
    M = 16
    idx = np.random.default_rng(4).integers(0, M, size=(50, 4)).astype(np.int32)
    bad = idx.copy()
    bad[::7, 1] = M + 3
    bad[::11, 2] = -1
    S = bad.size
    off, srt = e.empty((M + 1) * 4), e.empty(S * 4)
    status = ctypes.c_uint(0)
    fn = e.lib.emu_dispatch_shared if variant == "shared" else e.lib.emu_dispatch
    assert fn(e.put(bad), S, M, off, srt, e.empty(e.lib.emu_dispatch_scratch_bytes(S, M)),
              ctypes.addressof(status)) == 0
    got_off = e.get(off, (M + 1,), np.int32)
    ok = (bad >= 0) & (bad < M)
    expect = np.concatenate([[0], np.cumsum(np.bincount(bad[ok], minlength=M))])
    np.testing.assert_array_equal(got_off, expect)
    valid_slots = np.flatnonzero(ok.ravel())
    got_srt = e.get(srt, (S,), np.int32)[: got_off[M]]
    e.free_all()
    np.testing.assert_array_equal(np.sort(got_srt), valid_slots)
    assert status.value == 4  # MORE_DEVERR_BAD_INPUT
