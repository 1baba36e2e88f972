"""GPU routing vs the fp64 oracle, through the C ABI (Python binding).

Configurations: the five workloads of the MoRE router benchmark (tiny, expert sweep,
prefill, many experts, decode) at their full sizes, compared on sampled tokens; ragged
and degenerate shapes compared on every token; tie-heavy and closed-form inputs
compared exactly (their logits are exact in fp32).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from tests import parity

pytestmark = pytest.mark.gpu

VARIANTS = ["small_n", "fused_tc"]
UNFUSED = ["unfused", "unfused_tc"]   # materialise-then-top-k: CUDA-core and tensor-core scores
TC_RANKS = (16, 32, 64, 128)          # ranks of the tensor-core kernels

_cache = {}


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def inputs(N, h, r, M, seed=0, unit_rms=False):
    key = (N, h, r, M, seed, unit_rms)
    if key not in _cache:
        if len(_cache) > 3:
            _cache.clear()
        X, R1, R2 = syn.router_inputs(N, h, r, M, seed=seed, x_unit_rms=unit_rms)
        _cache[key] = (X, R1, R2, dev_bf16(X), dev_bf16(R1), dev_bf16(R2))
    return _cache[key]


def lib():
    import mixture_experts_rank_b200 as m
    return m


def supported(variant, N, h, r, M, k):
    m = lib()
    if variant == "unfused_tc":
        return r in TC_RANKS
    if variant == "fused_tc":
        try:
            X = torch.zeros((max(N, 1), h), dtype=torch.bfloat16, device="cuda")
            m.route(X[:0] if N == 0 else X[:1], torch.zeros((h, r), dtype=torch.bfloat16, device="cuda"),
                    torch.zeros((r, M), dtype=torch.bfloat16, device="cuda"), k, variant=variant)
        except m.MoreError as e:
            if e.status == 2:
                return False
            raise
    return True


def run(variant, Xd, R1d, R2d, k):
    m = lib()
    if variant == "unfused":
        out = m.route_unfused(Xd, R1d, R2d, k)
    elif variant == "unfused_tc":
        out = m.route_unfused_tc(Xd, R1d, R2d, k)
    else:
        out = m.route(Xd, R1d, R2d, k, variant=variant)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    return [None if t is None else t.cpu().numpy() for t in out]


def check(variant, N, h, r, M, k, seed=0, unit_rms=False, n_sample=None, near_scan=0, near_count=0):
    """Route on the GPU and compare with the oracle.  With ``n_sample`` the comparison takes
    that many rows: the first and last rows, three whole 128-token tiles from the middle of
    the batch, random rows, and the ``near_count`` rows with the smallest oracle margins
    among ``near_scan`` scanned rows (all N when near_scan >= N)."""
    if not supported(variant, N, h, r, M, k):
        pytest.skip(f"{variant} does not take this shape")
    X, R1, R2, Xd, R1d, R2d = inputs(N, h, r, M, seed, unit_rms)
    idx, gate, cnt, logits = run(variant, Xd, R1d, R2d, k)
    rows = None
    if n_sample is not None:
        extra = ()
        if near_count:
            scan = None if near_scan >= N else np.random.default_rng(seed + 1).choice(N, near_scan, replace=False)
            extra = parity.near_tie_rows(X, R1, R2, N, h, r, M, k, near_count, scan=scan)
        tiles = (N // 256, N // 384 + 1, (5 * N) // 768) if N >= 1024 else ()
        rows = parity.sample_rows(N, n_sample, seed, tiles=tiles, extra=extra)
    return parity.compare(X, R1, R2, N, h, r, M, k, idx, gate, cnt, logits, rows=rows)


# --- the benchmark workloads --------------------------------------------------------

@pytest.mark.parametrize("variant", VARIANTS + UNFUSED)
def test_tiny_full_oracle(variant):
    rep = check(variant, 4096, 128, 32, 192, 4)
    assert rep.set_fraction > 0.8


@pytest.mark.parametrize("variant", VARIANTS + UNFUSED)
@pytest.mark.parametrize("M", [1024, 2048, 4096, 8192, 16384])
def test_expert_sweep_sampled(variant, M):
    check(variant, 65536, 512, 32, M, 8, n_sample=4096, near_scan=16384, near_count=256)


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("r", [16, 32, 64, 128])
def test_prefill_sampled(variant, r):
    # the headline shape (r = 32) scans every token's margin for the 1024 closest near-ties
    check(variant, 262144, 2048, r, 4096, 8, unit_rms=True, n_sample=8192,
          near_scan=262144 if r == 32 else 32768, near_count=1024 if r == 32 else 256)


def test_prefill_unfused_sampled():
    check("unfused", 262144, 2048, 32, 4096, 8, unit_rms=True, n_sample=256)


@pytest.mark.parametrize("r", [16, 32, 64, 128])
def test_prefill_unfused_tc_sampled(r):
    check("unfused_tc", 262144, 2048, r, 4096, 8, unit_rms=True, n_sample=4096,
          near_scan=32768, near_count=256)


@pytest.mark.parametrize("variant", VARIANTS + UNFUSED)
def test_many_experts_sampled(variant):
    check(variant, 32768, 4096, 64, 65536, 8, n_sample=1024, near_scan=4096, near_count=128)


@pytest.mark.parametrize("variant", VARIANTS + UNFUSED)
@pytest.mark.parametrize("N", [1, 8, 64, 256])
def test_decode_full_oracle(variant, N):
    check(variant, N, 2048, 32, 4096, 8)


# --- ragged and degenerate shapes ------------------------------------------------------

@pytest.mark.parametrize("variant", VARIANTS + UNFUSED)
@pytest.mark.parametrize("N,h,r,M,k", [
    (127, 72, 16, 200, 1),
    (129, 136, 48, 64, 8),
    (1000, 512, 128, 1000, 16),
    (300, 256, 64, 16, 16),      # k == M == KMAX
    (513, 64, 32, 4104, 5),     # M one tile past a multiple of 32
    (2049, 1032, 32, 96, 3),
])
def test_ragged_shapes_full_oracle(variant, N, h, r, M, k):
    check(variant, N, h, r, M, k, seed=N)


@pytest.mark.parametrize("variant", VARIANTS + UNFUSED)
def test_empty_batch_zeroes_counts(variant):
    m = lib()
    h, r, M, k = 64, 32, 128, 4
    X = torch.zeros((0, h), dtype=torch.bfloat16, device="cuda")
    R1 = torch.zeros((h, r), dtype=torch.bfloat16, device="cuda")
    R2 = torch.zeros((r, M), dtype=torch.bfloat16, device="cuda")
    cnt = torch.full((M,), 7, dtype=torch.int32, device="cuda")
    if variant == "unfused":
        m.route_unfused(X, R1, R2, k, out_expert_count=cnt)
    elif variant == "unfused_tc":
        m.route_unfused_tc(X, R1, R2, k, out_expert_count=cnt)
    else:
        if not supported(variant, 0, h, r, M, k):
            pytest.skip("variant does not take this shape")
        m.route(X, R1, R2, k, out_expert_count=cnt, variant=variant)
    torch.cuda.synchronize()
    assert int(cnt.abs().sum()) == 0


# --- exact inputs: ties, closed forms --------------------------------------------------

def identity_weights(M):
    eye = syn.f32_to_bf16_bits(np.eye(M, dtype=np.float32))
    return eye, eye


@pytest.mark.parametrize("variant", VARIANTS + UNFUSED)
@pytest.mark.parametrize("k", [1, 3, 8, 16])
def test_tie_heavy_exact(variant, k):
    """Small-integer logits (R1 = R2 = I): many exact ties; lower index wins (Alg. 1)."""
    M, N = 64, 777
    rng = np.random.default_rng(k)
    X = syn.f32_to_bf16_bits(rng.integers(-3, 4, size=(N, M)).astype(np.float32))
    R1, R2 = identity_weights(M)
    if not supported(variant, N, M, M, M, k):
        pytest.skip("variant does not take this shape")
    idx, gate, cnt, logits = run(variant, dev_bf16(X), dev_bf16(R1), dev_bf16(R2), k)
    parity.compare(X, R1, R2, N, M, M, M, k, idx, gate, cnt, logits, exact=True)


@pytest.mark.parametrize("variant", VARIANTS + UNFUSED)
def test_jl_construction_exact(variant):
    """App. J, Theorem 4 (uncompressed): x_S = (M-k) on S, -k elsewhere; top-k is S."""
    M, k, N = 64, 4, 600
    rng = np.random.default_rng(1)
    X = np.full((N, M), -float(k), dtype=np.float32)
    sets = np.array([np.sort(rng.choice(M, size=k, replace=False)) for _ in range(N)])
    for n in range(N):
        X[n, sets[n]] = M - k
    Xb = syn.f32_to_bf16_bits(X)
    R1, R2 = identity_weights(M)
    if not supported(variant, N, M, M, M, k):
        pytest.skip("variant does not take this shape")
    idx, gate, cnt, logits = run(variant, dev_bf16(Xb), dev_bf16(R1), dev_bf16(R2), k)
    np.testing.assert_array_equal(idx, sets)
    np.testing.assert_allclose(gate, 1.0 / k, rtol=0, atol=1e-6)
    parity.compare(Xb, R1, R2, N, M, M, M, k, idx, gate, cnt, logits, exact=True)


def hypercube(h, r, r_impl=None):
    """Rank-r hypercube router embedded in rank r_impl >= r (zero padding leaves the logits unchanged)."""
    r_impl = r if r_impl is None else r_impl
    M = 2 ** r
    R1 = np.zeros((h, r_impl), dtype=np.float32)
    R1[:r, :r] = np.eye(r)
    R2 = np.zeros((r_impl, M), dtype=np.float32)
    R2[:r] = np.array([[1.0 if (a >> l) & 1 else -1.0 for a in range(M)] for l in range(r)])
    return syn.f32_to_bf16_bits(R1), syn.f32_to_bf16_bits(R2), M


@pytest.mark.parametrize("variant", VARIANTS + UNFUSED)
def test_hypercube_top1_is_sign_pattern(variant):
    """Prop. 1 proof (App. J): the k = 1 winner is the sign pattern of z."""
    h, r = 64, 16
    R1, R2, M = hypercube(h, r)
    N = 2000
    if not supported(variant, N, h, r, M, 1):
        pytest.skip("variant does not take this shape")
    X = syn.normal_bf16(5, syn.TENSOR_X, N, h)
    idx, gate, cnt, logits = run(variant, dev_bf16(X), dev_bf16(R1), dev_bf16(R2), 1)
    z = syn.bf16_bits_to_f64(X)[:, :r]
    expected = ((z > 0) * (1 << np.arange(r))).sum(axis=1)
    np.testing.assert_array_equal(idx[:, 0], expected)
    assert np.all(gate == 1.0)


@pytest.mark.parametrize("variant", VARIANTS)
def test_hypercube_load_balance_bound(variant):
    """Prop. 1: every count within sqrt(2nkL/M) + 2L/3 of nk/M (delta = 1e-6)."""
    h, r, n, k, delta = 64, 8, 200000, 4, 1e-6
    R1, R2, M = hypercube(h, r, r_impl=16)
    if not supported(variant, n, h, 16, M, k):
        pytest.skip("variant does not take this shape")
    X = syn.normal_bf16(6, syn.TENSOR_X, n, h)
    idx, gate, cnt, logits = run(variant, dev_bf16(X), dev_bf16(R1), dev_bf16(R2), k)
    L = np.log(2 * M / delta)
    assert np.max(np.abs(cnt - n * k / M)) <= np.sqrt(2 * n * k * L / M) + 2 * L / 3
    assert cnt.sum() == n * k


def test_variants_agree_on_selections():
    """The fused and small-N kernels select the same experts where margins are clear."""
    if not supported("fused_tc", 8192, 512, 32, 2048, 8):
        pytest.skip("fused kernel unavailable for this shape")
    X, R1, R2, Xd, R1d, R2d = inputs(8192, 512, 32, 2048, seed=3)
    a = run("fused_tc", Xd, R1d, R2d, 8)
    b = run("small_n", Xd, R1d, R2d, 8)
    o = oracle.route(X, R1, R2, 8192, 512, 32, 2048, 8, rows=np.arange(0, 8192, 7))
    clear = o.margin > 2e-2 * o.rms
    rows = np.arange(0, 8192, 7)[clear]
    np.testing.assert_array_equal(np.sort(a[0][rows], 1), np.sort(b[0][rows], 1))
