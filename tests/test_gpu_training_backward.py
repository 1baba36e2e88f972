"""GPU backward of the router (more_route_backward) vs the fp64 oracle, through the C ABI.

"MoRE: Scaling mixture of experts with hardware-aware low-rank routing", App. F, F.2.2,
Algorithm 3 and eqs. (10)-(12): with z = X R1, l = z R2 and P the full softmax over the M
experts, g_n = sum_i pbar_i P_ni, ybar = P (pbar - g) plus the selected-logit gradients,
and the gradients Xbar = ybar R2^T R1^T, R1bar = X^T ybar R2^T, R2bar = z^T ybar.

Tolerance.  The pages give none for the backward, so it is derived from the arithmetic.
The kernels compute in fp32 from exact bf16 inputs, and every output is a sum of products.
Replacing every factor by its magnitude gives a bound S on the sum of the magnitudes of
an output's terms:
  S_ybar = P (|pbar| + |g|) + |selected gradients|,   S_zbar = S_ybar |R2|^T,
  S_Xbar = S_zbar |R1|^T,   S_R1bar = |X|^T S_zbar,   S_g = P |pbar|,
  S_R2bar = |z|^T S_ybar + (|X| |R1|)^T |ybar|   (the second term covers the error of z).
A chain of K fp32 multiply-adds is off by at most about K u S (u = 2^-24).  The chains here
are at most a few thousand terms (h, M, or the tokens of one split), so every element is
required within TAU = 2e-3 of S.  The planted mistakes this must catch (the sign of g, a
dropped selected gradient, a wrong column) move elements by 1e-2 S or more.

At the full prefill size, the oracle checks sampled rows of Xbar and g.  R1bar and R2bar are
checked against the oracle at a mid size, where the splits are thousands of tokens long.  At
full size they are checked by the identity <Xbar, X> = <R1bar, R1> = <R2bar, R2>: each side
equals sum_n <ybar_n, l_n>.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from tests import parity
from tests.test_gpu_parity import inputs

pytestmark = pytest.mark.gpu

TAU = 2e-3
IDENTITY_TOL = 1e-4


def selections(N, M, k, seed):
    """Seeded expert ids, distinct per token: (a_n + j s_n) mod M with 1 <= s_n <= M // k."""
    rng = np.random.default_rng(seed)
    a = rng.integers(0, M, N)
    s = rng.integers(1, M // k + 1, N)
    return ((a[:, None] + np.arange(k)[None, :] * s[:, None]) % M).astype(np.int32)


def gradients(N, M, k, seed, balance=True, selected=True):
    rng = np.random.default_rng(seed + 101)
    tvb = rng.standard_normal((N, k)).astype(np.float32) if selected else None
    pbar = rng.standard_normal(M).astype(np.float32) if balance else None
    return tvb, pbar


def reference(X, R1, R2, N, h, r, M, k, idx, tvb, pbar):
    """The oracle's gradients and the magnitude bounds S, fp64.  Absent gradients are zeros;
    selections outside [0, M) are dropped (the kernels skip them)."""
    idx = np.asarray(idx, dtype=np.int64).reshape(N, k)
    tvb = np.zeros((N, k)) if tvb is None else np.asarray(tvb, dtype=np.float64).reshape(N, k)
    pbar = np.zeros(M) if pbar is None else np.asarray(pbar, dtype=np.float64)
    ok = (idx >= 0) & (idx < M)
    idx, tvb = np.where(ok, idx, 0), np.where(ok, tvb, 0.0)
    o = oracle.router_backward(X, R1, R2, N, h, r, M, idx, tvb, pbar)
    Xf, R1f, R2f = (syn.bf16_bits_to_f64(a) for a in (X, R1, R2))
    Xf = Xf.reshape(N, h)
    z = Xf @ R1f
    l = z @ R2f
    if N:
        P = np.exp(l - l.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
    else:
        P = l
    sel = np.zeros((N, M))
    np.add.at(sel, (np.repeat(np.arange(N), k), idx.ravel()), np.abs(tvb).ravel())
    S_y = P * (np.abs(pbar)[None, :] + np.abs(o.g)[:, None]) + sel
    ybar_abs = np.abs(P * (pbar[None, :] - o.g[:, None])) + sel
    S_zb = S_y @ np.abs(R2f).T
    S = {"Xbar": S_zb @ np.abs(R1f).T, "R1bar": np.abs(Xf).T @ S_zb,
         "R2bar": np.abs(z).T @ S_y + (np.abs(Xf) @ np.abs(R1f)).T @ ybar_abs, "g": P @ np.abs(pbar)}
    return {"Xbar": o.X, "R1bar": o.R1, "R2bar": o.R2, "g": o.g}, S


def compare(got, ref, S, names=("Xbar", "R1bar", "R2bar", "g")):
    """Every element within TAU S of the oracle (exactly equal where S is zero)."""
    worst = {}
    for name in names:
        g = np.asarray(got[name], dtype=np.float64)
        assert g.shape == ref[name].shape, f"{name}: shape {g.shape} != {ref[name].shape}"
        assert np.all(np.isfinite(g)), f"{name}: non-finite values"
        err = np.abs(g - ref[name])
        bad = err > TAU * S[name]
        ratio = err / np.where(S[name] > 0, S[name], 1.0)
        assert not bad.any(), f"{name}: {int(bad.sum())} elements beyond {TAU} S (worst err/S {ratio.max():.3g})"
        worst[name] = float(ratio.max()) if ratio.size else 0.0
    return worst


def check_identity(xbar_dot_x, r1bar_dot_r1, r2bar_dot_r2):
    """<Xbar, X> = <R1bar, R1> = <R2bar, R2> (= sum_n <ybar_n, l_n>), relative to the first."""
    a = float(xbar_dot_x)
    assert a != 0.0
    for other in (r1bar_dot_r1, r2bar_dot_r2):
        assert abs(float(other) - a) <= IDENTITY_TOL * abs(a), f"identity: {a} vs {float(other)}"


def dev(a, dtype):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, dtype=dtype)).cuda()


def run_gpu(Xd, R1d, R2d, k, idx, tvb, pbar, m, Z):
    import mixture_experts_rank_b200 as mm
    out = mm.route_backward(Xd, R1d, R2d, k, top_idx=dev(idx, np.int32), top_vals_bar=dev(tvb, np.float32),
                            pbar=dev(pbar, np.float32), m=dev(m, np.float32) if pbar is not None else None,
                            Z=dev(Z, np.float32) if pbar is not None else None)
    torch.cuda.synchronize()
    return dict(zip(("Xbar", "R1bar", "R2bar", "g"), out)), mm.device_status()


def saved_stats(X, R1, R2, N, h, r, M):
    if N == 0:
        return np.zeros(0, np.float32), np.zeros(0, np.float32)
    st = oracle.train_stats(X, R1, R2, N, h, r, M)
    return st.m.astype(np.float32), st.Z.astype(np.float32)


def check_case(N, h, r, M, k, seed=0, balance=True, selected=True, top_k=True, idx=None):
    X, R1, R2, Xd, R1d, R2d = inputs(N, h, r, M, seed)
    if idx is None:
        idx = oracle.route(X, R1, R2, N, h, r, M, k).idx.astype(np.int32) if (top_k and N) else \
            selections(N, M, k, seed)
    tvb, pbar = gradients(N, M, k, seed, balance, selected)
    m, Z = saved_stats(X, R1, R2, N, h, r, M)
    got, status = run_gpu(Xd, R1d, R2d, k, idx, tvb, pbar, m, Z)
    ref, S = reference(X, R1, R2, N, h, r, M, k, idx, tvb, pbar)
    worst = compare({n: t.cpu().numpy() for n, t in got.items()}, ref, S)
    return worst, status


@pytest.mark.parametrize("N,h,r,M,k", [
    (300, 128, 32, 192, 4),    # ragged token block, three expert tiles
    (97, 256, 16, 256, 16),    # r = 16, k = 16
    (65, 200, 48, 200, 8),     # r = 48 (padded to 64), ragged hidden and expert tiles
    (33, 64, 128, 1024, 8),    # r = 128
    (1000, 512, 64, 2048, 8),
    (1, 64, 32, 64, 1),        # one token, one selection
])
def test_backward_matches_oracle(N, h, r, M, k):
    _, status = check_case(N, h, r, M, k)
    assert status == 0


@pytest.mark.parametrize("balance,selected", [(False, True), (True, False), (False, False)])
def test_backward_with_one_gradient_absent(balance, selected):
    _, status = check_case(200, 128, 32, 192, 4, seed=3, balance=balance, selected=selected)
    assert status == 0


def test_backward_repeated_and_out_of_range_selections():
    N, M, k = 40, 192, 4
    idx = np.tile(np.array([[5, 5, 200, -1]], np.int32), (N, 1))
    idx[::3, 1] = 191
    _, status = check_case(N, 128, 32, M, k, seed=4, idx=idx)
    assert status == 4  # MORE_DEVERR_BAD_INPUT; the out-of-range selections were skipped


def test_backward_empty_batch():
    import mixture_experts_rank_b200 as mm
    _, _, _, Xd, R1d, R2d = inputs(0, 64, 32, 64)
    Xbar, R1bar, R2bar, g = mm.route_backward(Xd, R1d, R2d, 4, pbar=torch.ones(64, device="cuda"),
                                              m=torch.zeros(0, device="cuda"), Z=torch.ones(0, device="cuda"))
    torch.cuda.synchronize()
    assert Xbar.shape == (0, 64) and g.shape == (0,)
    assert torch.count_nonzero(R1bar) == 0 and torch.count_nonzero(R2bar) == 0


def test_backward_is_deterministic():
    N, h, r, M, k = 3000, 256, 32, 1024, 8
    X, R1, R2, Xd, R1d, R2d = inputs(N, h, r, M, 6)
    idx = selections(N, M, k, 6)
    tvb, pbar = gradients(N, M, k, 6)
    m, Z = saved_stats(X, R1, R2, N, h, r, M)
    a, _ = run_gpu(Xd, R1d, R2d, k, idx, tvb, pbar, m, Z)
    b, _ = run_gpu(Xd, R1d, R2d, k, idx, tvb, pbar, m, Z)
    for name in a:
        assert torch.equal(a[name], b[name]), name


def test_backward_mid_size_long_splits():
    """N = 32768: the R1 / R2 splits run over ~900 and ~1700 tokens each."""
    _, status = check_case(32768, 512, 32, 1024, 8, seed=7, top_k=False)
    assert status == 0


def test_backward_full_prefill():
    """N = 262144, h = 2048, r = 32, M = 4096, k = 8: sampled rows vs the oracle, and the identity."""
    import mixture_experts_rank_b200 as mm
    N, h, r, M, k = 262144, 2048, 32, 4096, 8
    X, R1, R2, Xd, R1d, R2d = inputs(N, h, r, M, 0)
    m, Z = saved_stats(X, R1, R2, N, h, r, M)
    rows = parity.sample_rows(N, 256, 0)

    # sampled rows of Xbar and g against the oracle on those rows (per-token quantities)
    idx = selections(N, M, k, 8)
    tvb, pbar = gradients(N, M, k, 8)
    got, status = run_gpu(Xd, R1d, R2d, k, idx, tvb, pbar, m, Z)
    assert status == 0
    Xr = np.ascontiguousarray(np.asarray(X).reshape(N, h)[rows])
    ref, S = reference(Xr, R1, R2, len(rows), h, r, M, k, idx[rows], tvb[rows], pbar)
    rows_d = torch.from_numpy(rows.astype(np.int64)).cuda()
    compare({"Xbar": got["Xbar"][rows_d].cpu().numpy(), "g": got["g"][rows_d].cpu().numpy()}, ref, S,
            names=("Xbar", "g"))
    del got

    # the identity, with the forward's own top-k and positive selected-logit gradients so that
    # sum_n <ybar_n, l_n> does not cancel
    idx_d = mm.route(Xd, R1d, R2d, k)[0]
    rng = np.random.default_rng(9)
    tvb_d = torch.from_numpy(rng.uniform(0.5, 1.5, (N, k)).astype(np.float32)).cuda()
    Xbar, R1bar, R2bar, _ = mm.route_backward(Xd, R1d, R2d, k, top_idx=idx_d, top_vals_bar=tvb_d,
                                              pbar=dev(pbar, np.float32), m=dev(m, np.float32), Z=dev(Z, np.float32))
    torch.cuda.synchronize()
    assert mm.device_status() == 0
    a = sum(float((Xbar[i:i + 16384].double() * Xd[i:i + 16384].double()).sum()) for i in range(0, N, 16384))
    b = float((R1bar.double() * R1d.double()).sum())
    c = float((R2bar.double() * R2d.double()).sum())
    check_identity(a, b, c)
