"""Pins of the fp64 oracle against facts the MoRE pages and plain mathematics fix.

Source: "MoRE: Scaling mixture of experts with hardware-aware low-rank routing"
(arXiv 2609.36301).  Every check here is independent of the oracle's own code:
explicit W = R1 R2 products, brute-force ranks, closed-form constructions from
App. J, symmetry (Lemma 3), limiting cases of the softmax, and statistics
(Proposition 1, Lemma 1).  ``test_oracle_mutations.py`` shows that plausible
mistakes planted in a copy of the oracle fail these pins.
"""
import os

import numpy as np
import pytest

import oracle
import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(values):
    v = np.asarray(values, dtype=np.float64)
    bits = syn.f32_to_bf16_bits(v.astype(np.float32))
    assert np.array_equal(syn.bf16_bits_to_f64(bits), v), "value not exact in bf16"
    return bits


def identity_router(values):
    """h = r = M and R1 = R2 = I, so the logits equal the (bf16-exact) inputs."""
    X = bf16(np.atleast_2d(values))
    M = X.shape[1]
    eye = bf16(np.eye(M))
    return X, eye, eye


def route_values(values, k):
    X, R1, R2 = identity_router(values)
    N, M = X.shape
    return oracle.route(X, R1, R2, N, M, M, M, k, threads=2)


def brute_force_order(l):
    """Routing order by counting, for each expert, the experts that beat it."""
    M = len(l)
    rank = np.array([sum(1 for b in range(M) if l[b] > l[a] or (l[b] == l[a] and b < a))
                     for a in range(M)])
    order = np.empty(M, dtype=np.int64)
    order[rank] = np.arange(M)
    return order


def read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([part.split() for part in line.split("|")])
    return rows


# --- factorisation: standard router with W = R1 R2 (MoRE §2, A1 == A2) -----------

def test_logits_equal_explicit_W_product():
    N, h, r, M = 37, 48, 16, 72
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=11)
    Xf, R1f, R2f = (syn.bf16_bits_to_f64(a) for a in (X, R1, R2))
    W = R1f @ R2f                                   # h x M, formed explicitly
    expected = Xf @ W                               # standard router x W
    got = oracle.logits(X, R1, R2, N, h, r, M)
    np.testing.assert_allclose(got, expected, rtol=1e-11, atol=1e-12)
    res = oracle.route(X, R1, R2, N, h, r, M, 5)
    np.testing.assert_allclose(res.logit, np.take_along_axis(expected, res.idx.astype(np.int64), 1),
                               rtol=1e-11, atol=1e-12)


def test_projection_and_pairs_agree_with_matmul():
    N, h, r, M = 9, 40, 24, 30
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=5)
    Xf, R1f, R2f = (syn.bf16_bits_to_f64(a) for a in (X, R1, R2))
    np.testing.assert_allclose(oracle.projection(X, R1, N, h, r), Xf @ R1f, rtol=1e-12, atol=1e-13)
    rows = np.array([0, 3, 3, 8, 1])
    experts = np.array([29, 0, 7, 15, 2])
    np.testing.assert_allclose(oracle.logits_at(X, R1, R2, N, h, r, M, rows, experts),
                               (Xf @ R1f @ R2f)[rows, experts], rtol=1e-11, atol=1e-12)
    sub = oracle.logits(X, R1, R2, N, h, r, M, rows=rows)
    np.testing.assert_allclose(sub, (Xf @ R1f @ R2f)[rows], rtol=1e-11, atol=1e-12)


# --- the standard (full-rank) router of App. H.3 -----------------------------------

def test_fullrank_matches_the_factored_router_when_W_is_their_product():
    """W = R1 R2 with small integer factors is exact in bf16 (|W| <= 4r < 256), so the full-rank
    router on W and the low-rank router on (R1, R2) define the same logits: the two oracle
    paths (x . W against (x . R1) . R2) must agree to fp64 rounding and select the same
    experts."""
    N, h, r, M, k = 40, 48, 16, 72, 5
    rng = np.random.default_rng(3)
    R1f = rng.integers(-2, 3, size=(h, r)).astype(np.float32)
    R2f = rng.integers(-2, 3, size=(r, M)).astype(np.float32)
    W = syn.f32_to_bf16_bits(R1f @ R2f)
    R1, R2 = syn.f32_to_bf16_bits(R1f), syn.f32_to_bf16_bits(R2f)
    assert np.array_equal(syn.bf16_bits_to_f64(W), (R1f @ R2f).astype(np.float64))
    X = syn.normal_bf16(7, syn.TENSOR_X, N, h)
    full = oracle.route_fullrank(X, W, N, h, M, k)
    low = oracle.route(X, R1, R2, N, h, r, M, k)
    np.testing.assert_allclose(full.logit, low.logit, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(full.rms, low.rms, rtol=1e-12)
    np.testing.assert_allclose(full.margin, low.margin, rtol=1e-9, atol=1e-9)
    clear = low.margin > 1e-9 * low.rms
    assert clear.mean() > 0.9
    np.testing.assert_array_equal(full.idx[clear], low.idx[clear])
    np.testing.assert_array_equal(full.counts, low.counts)
    rows = np.array([0, 5, 5, 39])
    experts = np.array([71, 0, 33, 12])
    np.testing.assert_allclose(oracle.logits_at_fullrank(X, W, N, h, M, rows, experts),
                               oracle.logits_at(X, R1, R2, N, h, r, M, rows, experts), rtol=1e-12, atol=1e-12)


def test_fullrank_tie_order_and_brute_force_ranks():
    """Small integer logits (x one-hot rows times integer W): many exact ties, which the
    full-rank router must break towards the lower expert, as brute-force ranks do."""
    N, h, M, k = 30, 16, 24, 6
    rng = np.random.default_rng(9)
    X = syn.f32_to_bf16_bits(np.eye(h, dtype=np.float32)[rng.integers(0, h, N)])
    Wf = rng.integers(-2, 3, size=(h, M)).astype(np.float32)
    res = oracle.route_fullrank(X, syn.f32_to_bf16_bits(Wf), N, h, M, k)
    L = syn.bf16_bits_to_f64(X) @ Wf.astype(np.float64)
    for n in range(N):
        rank = [int(np.sum((L[n] > L[n, e]) | ((L[n] == L[n, e]) & (np.arange(M) < e)))) for e in range(M)]
        expected = sorted(range(M), key=lambda e: rank[e])[:k]
        assert res.idx[n].tolist() == expected


# --- selection: brute force, ties, relabelling ----------------------------------

@pytest.mark.parametrize("M", [1, 2, 7, 13, 33])
def test_topk_matches_brute_force_random(M):
    rng = np.random.default_rng(M)
    vals = syn.bf16_bits_to_f64(syn.f32_to_bf16_bits(rng.standard_normal((6, M)).astype(np.float32)))
    for k in range(1, M + 1):
        res = route_values(vals, k)
        for n in range(vals.shape[0]):
            assert list(res.idx[n]) == list(brute_force_order(vals[n])[:k])


@pytest.mark.parametrize("M", [5, 16, 40])
def test_topk_matches_brute_force_tie_heavy(M):
    rng = np.random.default_rng(100 + M)
    vals = rng.integers(-2, 3, size=(8, M)).astype(np.float64)   # many equal logits
    for k in sorted({1, 2, M // 2, M - 1, M}):
        if k < 1:
            continue
        res = route_values(vals, k)
        for n in range(vals.shape[0]):
            assert list(res.idx[n]) == list(brute_force_order(vals[n])[:k])


def test_golden_tie_order():
    for (mk, logits, expected) in read_golden("tie_order.txt"):
        M, k = int(mk[0]), int(mk[1])
        vals = [float(v) for v in logits]
        assert len(vals) == M
        res = route_values([vals], k)
        assert list(res.idx[0]) == [int(e) for e in expected]


def test_relabelling_equivariance():
    """Lemma 3 (App. J): permuting the experts permutes the selected set (no ties)."""
    N, h, r, M, k = 64, 32, 16, 96, 7
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=3)
    base = oracle.route(X, R1, R2, N, h, r, M, k)
    perm = np.random.default_rng(0).permutation(M)            # new column j is old expert perm[j]
    R2p = np.ascontiguousarray(R2[:, perm])
    moved = oracle.route(X, R1, R2p, N, h, r, M, k)
    assert np.array_equal(perm[moved.idx], base.idx)
    np.testing.assert_array_equal(moved.logit, base.logit)
    np.testing.assert_array_equal(moved.counts[np.argsort(perm)], base.counts)


# --- gates, margin, rms, counts --------------------------------------------------

def test_k_equals_M_gives_full_softmax():
    N, h, r, M = 20, 24, 16, 12
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=8)
    res = oracle.route(X, R1, R2, N, h, r, M, M)
    full = oracle.logits(X, R1, R2, N, h, r, M)
    e = np.exp(full - full.max(axis=1, keepdims=True))
    softmax = e / e.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(res.gate, np.take_along_axis(softmax, res.idx.astype(np.int64), 1),
                               rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(res.gate.sum(axis=1), 1.0, rtol=0, atol=1e-13)
    assert np.all(np.isinf(res.margin))


def test_gate_special_cases():
    vals = np.array([[0.5, 3.0, -1.0, 2.25, 0.0]])
    one = route_values(vals, 1)
    assert one.gate[0, 0] == 1.0
    two = route_values(vals, 2)
    d = 3.0 - 2.25                                       # k = 2: softmax is the logistic function
    np.testing.assert_allclose(two.gate[0], [1 / (1 + np.exp(-d)), 1 / (1 + np.exp(d))], rtol=1e-15)


def test_margin_gaps_and_rms_against_sorted_logits():
    N, h, r, M, k = 25, 32, 16, 50, 6
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=21)
    res = oracle.route(X, R1, R2, N, h, r, M, k)
    full = oracle.logits(X, R1, R2, N, h, r, M)
    s = -np.sort(-full, axis=1)
    np.testing.assert_allclose(res.logit, s[:, :k], rtol=0, atol=0)
    np.testing.assert_allclose(res.margin, s[:, k - 1] - s[:, k], rtol=0, atol=0)
    np.testing.assert_allclose(res.gaps, s[:, :k] - s[:, 1:k + 1], rtol=0, atol=0)
    np.testing.assert_allclose(res.rms, np.linalg.norm(full, axis=1) / np.sqrt(M), rtol=1e-14)


def test_counts_are_the_bincount_of_indices():
    N, h, r, M, k = 300, 32, 16, 40, 3
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=2)
    res = oracle.route(X, R1, R2, N, h, r, M, k, threads=3)
    assert res.counts.sum() == N * k
    np.testing.assert_array_equal(res.counts, np.bincount(res.idx.ravel(), minlength=M))
    rows = np.array([7, 299, 0, 7])
    part = oracle.route(X, R1, R2, N, h, r, M, k, rows=rows)
    np.testing.assert_array_equal(part.idx, res.idx[rows])
    np.testing.assert_array_equal(part.counts, np.bincount(res.idx[rows].ravel(), minlength=M))
    # each row's selected experts are distinct
    for n in range(N):
        assert len(set(res.idx[n])) == k


# --- closed forms from App. J -----------------------------------------------------

def test_golden_jl_construction():
    for (mk, S, margin, gate) in read_golden("jl_construction.txt"):
        M, k = int(mk[0]), int(mk[1])
        S = [int(s) for s in S]
        x = np.full(M, -float(k))
        x[S] = float(M - k)
        X, R1, R2 = identity_router([x])
        res = oracle.route(X, R1, R2, 1, M, M, M, k)
        assert list(res.idx[0]) == S
        assert res.margin[0] == float(margin[0])
        np.testing.assert_allclose(res.gate[0], float(gate[0]), rtol=0, atol=1e-15)


def hypercube_router(h, r):
    """R1 selects the first r coordinates; column a of R2 is the sign vector of a."""
    M = 2 ** r
    R1 = np.zeros((h, r))
    R1[:r, :r] = np.eye(r)
    signs = np.array([[1.0 if (a >> l) & 1 else -1.0 for a in range(M)] for l in range(r)])
    return bf16(R1), bf16(signs), M


def test_golden_hypercube_top1_is_sign_pattern():
    R1, R2, M = hypercube_router(8, 8)
    for (z, expected) in read_golden("hypercube_k1.txt"):
        x = bf16([[float(v) for v in z]])
        res = oracle.route(x, R1, R2, 1, 8, 8, M, 1)
        assert res.idx[0, 0] == int(expected[0])


def test_hypercube_top1_random_inputs():
    h, r = 12, 8
    R1, R2, M = hypercube_router(h, r)
    X = syn.normal_bf16(4, syn.TENSOR_X, 500, h)
    xf = syn.bf16_bits_to_f64(X)[:, :r]
    res = oracle.route(X, R1, R2, 500, h, r, M, 1)
    expected = ((xf > 0) * (1 << np.arange(r))).sum(axis=1)
    np.testing.assert_array_equal(res.idx[:, 0], expected)


@pytest.mark.parametrize("k", [1, 4])
def test_hypercube_load_balance_bound(k):
    """Proposition 1: with M = 2^r sign-vector experts each is chosen w.p. exactly k/M,
    and max_a |N_a - nk/M| <= sqrt(2 n k L / M) + (2/3) L, L = log(2M/delta), w.p. 1 - delta."""
    h, r, n, delta = 10, 6, 20000, 1e-6
    R1, R2, M = hypercube_router(h, r)
    X = syn.normal_bf16(9, syn.TENSOR_X, n, h)
    res = oracle.route(X, R1, R2, n, h, r, M, k)
    L = np.log(2 * M / delta)
    bound = np.sqrt(2 * n * k * L / M) + 2.0 / 3.0 * L
    assert np.max(np.abs(res.counts - n * k / M)) <= bound
    assert res.counts.sum() == n * k


def test_logit_variance_matches_lemma_1():
    """Lemma 1 (App. D.2): Var([R1 R2 x]_e) = r s1^2 s2^2 |x|^2; with R1 ~ N(0, 1/h) and
    R2 ~ N(0, 1/r) this is |x|^2 / h.  Averaged over tokens, experts and three seeds."""
    h, r, M, N = 128, 32, 192, 512
    ratios = []
    for seed in (0, 1, 2):
        X, R1, R2 = syn.router_inputs(N, h, r, M, seed=seed)
        l = oracle.logits(X, R1, R2, N, h, r, M)
        xf = syn.bf16_bits_to_f64(X)
        ratios.append(np.mean(l ** 2 / (np.sum(xf ** 2, axis=1, keepdims=True) / h)))
    assert abs(np.mean(ratios) - 1.0) < 0.08


# --- argument checks --------------------------------------------------------------

def test_oracle_rejects_invalid_arguments():
    X, R1, R2 = syn.router_inputs(4, 8, 4, 6)
    with pytest.raises(ValueError):
        oracle.route(X, R1, R2, 4, 8, 4, 6, 7)           # k > M
    with pytest.raises(ValueError):
        oracle.route(X, R1, R2, 4, 8, 4, 6, 0)           # k < 1
    with pytest.raises(ValueError):
        oracle.route(X, R1, R2, 4, 8, 4, 6, 2, rows=[4])  # row out of range
    empty = oracle.route(X, R1, R2, 4, 8, 4, 6, 2, rows=np.zeros(0, np.int64))
    assert empty.idx.shape == (0, 2) and empty.counts.sum() == 0


# --- training statistics (App. F, Algorithm 2, eqs. (6)-(7)) ----------------------------------

def test_train_stats_closed_forms():
    """Equal logits: m is that value, Z = M, every probability 1/M.  One logit 1 above
    M - 1 zeros: Z = 1 + (M - 1) e^-1 and that expert's probability is 1 / Z."""
    M, n = 16, 3
    X, R1, R2 = identity_router(np.full((n, M), 2.0))
    st = oracle.train_stats(X, R1, R2, n, M, M, M, threads=2)
    np.testing.assert_array_equal(st.m, np.full(n, 2.0))
    np.testing.assert_allclose(st.Z, np.full(n, float(M)), rtol=1e-15)
    np.testing.assert_allclose(st.psum, np.full(M, n / M), rtol=1e-14)
    vals = np.zeros((n, M))
    vals[:, 5] = 1.0
    X, R1, R2 = identity_router(vals)
    st = oracle.train_stats(X, R1, R2, n, M, M, M, threads=2)
    Z = 1.0 + (M - 1) * np.exp(-1.0)
    np.testing.assert_array_equal(st.m, np.ones(n))
    np.testing.assert_allclose(st.Z, np.full(n, Z), rtol=1e-14)
    np.testing.assert_allclose(st.psum[5], n / Z, rtol=1e-14)
    np.testing.assert_allclose(np.delete(st.psum, 5), n * np.exp(-1.0) / Z, rtol=1e-14)


def test_train_stats_against_library_softmax():
    """m, m + log Z and psum equal numpy's max, scipy's logsumexp and the column sum of
    scipy's softmax, applied to the independently pinned logits."""
    from scipy.special import logsumexp, softmax

    N, h, r, M = 50, 96, 16, 80
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=11)
    rows = np.array([0, 3, 17, 18, 49])
    st = oracle.train_stats(X, R1, R2, N, h, r, M, rows=rows, threads=3)
    lg = oracle.logits(X, R1, R2, N, h, r, M, rows=rows)
    np.testing.assert_array_equal(st.m, lg.max(axis=1))
    np.testing.assert_allclose(st.m + np.log(st.Z), logsumexp(lg, axis=1), rtol=1e-13)
    np.testing.assert_allclose(st.psum, softmax(lg, axis=1).sum(axis=0), rtol=1e-12, atol=1e-15)
    assert abs(st.psum.sum() - rows.size) < 1e-12  # every softmax row sums to one


def test_train_stats_shift_and_relabelling():
    """A per-token constant added to all logits (an R2 row of equal entries times that
    token's z) moves m only; permuting R2's columns permutes psum."""
    N, h, r, M = 40, 64, 16, 48
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=12)
    R2a = R2.copy()
    R2a[0, :] = syn.f32_to_bf16_bits(np.zeros(M, np.float32))
    R2b = R2.copy()
    R2b[0, :] = syn.f32_to_bf16_bits(np.full(M, 0.75, np.float32))
    a = oracle.train_stats(X, R1, R2a, N, h, r, M, threads=2)
    b = oracle.train_stats(X, R1, R2b, N, h, r, M, threads=2)
    z0 = oracle.projection(X, R1, N, h, r)[:, 0]
    np.testing.assert_allclose(b.m - a.m, 0.75 * z0, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(b.Z, a.Z, rtol=1e-12)
    np.testing.assert_allclose(b.psum, a.psum, rtol=1e-11)
    perm = np.random.default_rng(5).permutation(M)
    c = oracle.train_stats(X, R1, np.ascontiguousarray(R2[:, perm]), N, h, r, M, threads=2)
    d = oracle.train_stats(X, R1, R2, N, h, r, M, threads=2)
    np.testing.assert_allclose(c.psum, d.psum[perm], rtol=1e-12)
    np.testing.assert_array_equal(c.m, d.m)


# --- dispatch bookkeeping (App. E, Fig. 9 "Sort + Count") -------------------------------------

def brute_force_dispatch(idx, M):
    """Expert by expert, the slots naming it in increasing slot order."""
    flat = [int(v) for v in np.asarray(idx).ravel()]
    sorted_slots, offsets = [], [0]
    for e in range(M):
        sorted_slots += [s for s, v in enumerate(flat) if v == e]
        offsets.append(len(sorted_slots))
    return np.array(offsets), np.array(sorted_slots, dtype=np.int64)


@pytest.mark.parametrize("N,k,M", [(1, 1, 8), (7, 3, 8), (50, 4, 16), (33, 8, 64)])
def test_dispatch_matches_brute_force(N, k, M):
    rng = np.random.default_rng(N * 100 + k)
    idx = rng.integers(0, M, size=(N, k))
    d = oracle.dispatch(idx, M)
    off, srt = brute_force_dispatch(idx, M)
    np.testing.assert_array_equal(d.offsets, off)
    np.testing.assert_array_equal(d.sorted, srt)


def test_dispatch_invariants_on_routing_output():
    """On real routing output: a permutation of the slots, grouped by expert, increasing
    within each expert, with offsets equal to the cumulative routing counts."""
    N, h, r, M, k = 200, 64, 16, 48, 6
    X, R1, R2 = syn.router_inputs(N, h, r, M, seed=21)
    o = oracle.route(X, R1, R2, N, h, r, M, k, threads=2)
    d = oracle.dispatch(o.idx, M)
    assert np.array_equal(np.sort(d.sorted), np.arange(N * k))
    flat = o.idx.ravel()
    np.testing.assert_array_equal(np.diff(d.offsets), o.counts)
    for e in range(M):
        seg = d.sorted[d.offsets[e]:d.offsets[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0)
    with pytest.raises(ValueError):
        oracle.dispatch(np.array([[0, M]]), M)


# --- backward (App. F, F.2.2, Algorithm 3) -------------------------------------------------------

def _backward_case(seed, N=3, h=7, r=4, M=9, k=2):
    rng = np.random.default_rng(seed)
    X, R1, R2 = rng.standard_normal((N, h)), rng.standard_normal((h, r)) / 2, rng.standard_normal((r, M)) / 2
    top_idx = np.argsort(-(X @ R1 @ R2), axis=1, kind="stable")[:, :k]
    return X, R1, R2, top_idx, rng.standard_normal((N, k)), rng.standard_normal(M)


def _loss(X, R1, R2, top_idx, tvb, pbar):
    """sum tvb * selected logits + pbar . psum: the loss whose gradients Algorithm 3 returns."""
    logits = X @ R1 @ R2
    E = np.exp(logits - logits.max(axis=1, keepdims=True))
    P = E / E.sum(axis=1, keepdims=True)
    return float((tvb * np.take_along_axis(logits, top_idx, axis=1)).sum() + P.sum(axis=0) @ pbar)


def test_backward_matches_finite_differences():
    X, R1, R2, ti, tvb, pbar = _backward_case(1)
    gr = oracle.router_backward_f64(X, R1, R2, ti, tvb, pbar)
    for name, A, G in (("X", X, gr.X), ("R1", R1, gr.R1), ("R2", R2, gr.R2)):
        fd = np.zeros_like(A)
        for idx in np.ndindex(A.shape):
            d = 1e-6
            A[idx] += d
            up = _loss(X, R1, R2, ti, tvb, pbar)
            A[idx] -= 2 * d
            dn = _loss(X, R1, R2, ti, tvb, pbar)
            A[idx] += d
            fd[idx] = (up - dn) / (2 * d)
        np.testing.assert_allclose(G, fd, rtol=1e-6, atol=1e-8, err_msg=name)


def test_backward_matches_torch_autograd():
    import torch

    X, R1, R2, ti, tvb, pbar = _backward_case(2, N=5, h=12, r=6, M=20, k=3)
    gr = oracle.router_backward_f64(X, R1, R2, ti, tvb, pbar)
    tX, tR1, tR2 = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (X, R1, R2))
    logits = tX @ tR1 @ tR2
    loss = (torch.tensor(tvb) * torch.gather(logits, 1, torch.tensor(ti))).sum() + \
        torch.softmax(logits, dim=1).sum(dim=0) @ torch.tensor(pbar)
    loss.backward()
    np.testing.assert_allclose(gr.X, tX.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(gr.R1, tR1.grad.numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(gr.R2, tR2.grad.numpy(), rtol=1e-12, atol=1e-13)


def test_backward_constant_pbar_and_bf16_entry():
    """A constant pbar adds the same to every psum_i's weight, and sum_i psum_i = N does not
    depend on the logits: the balancing term's gradient vanishes, and g_n equals that constant."""
    X, R1, R2, ti, tvb, _ = _backward_case(3)
    with_c = oracle.router_backward_f64(X, R1, R2, ti, tvb, np.full(R2.shape[1], 0.37))
    without = oracle.router_backward_f64(X, R1, R2, ti, tvb, np.zeros(R2.shape[1]))
    np.testing.assert_allclose(with_c.g, 0.37, rtol=1e-14)
    np.testing.assert_allclose(with_c.X, without.X, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(with_c.R2, without.R2, rtol=1e-12, atol=1e-14)
    N, h, r, M = 4, 16, 8, 24
    Xb, R1b, R2b = syn.router_inputs(N, h, r, M, seed=4)
    ti = oracle.route(Xb, R1b, R2b, N, h, r, M, 2, threads=1).idx
    gb = oracle.router_backward(Xb, R1b, R2b, N, h, r, M, ti, np.ones((N, 2)), np.zeros(M))
    gf = oracle.router_backward_f64(syn.bf16_bits_to_f64(Xb), syn.bf16_bits_to_f64(R1b), syn.bf16_bits_to_f64(R2b), ti,
                                    np.ones((N, 2)), np.zeros(M))
    np.testing.assert_array_equal(gb.R1, gf.R1)
