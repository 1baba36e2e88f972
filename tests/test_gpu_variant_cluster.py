"""The cluster variant of the router (MORE_VARIANT_CLUSTER) vs the fp64 oracle, through the C ABI.

Eight tokens per cluster of eight CTAs: the experts are split over the cluster and the partial
top-k lists are merged through distributed shared memory ("MoRE: Scaling mixture of experts
with hardware-aware low-rank routing", App. F, Algorithm 1 and Fig. 12).  The checks are the
parity suite's: the same tolerances, the benchmark's decode and tiny workloads, ragged and
degenerate shapes, and the exact tie-heavy and closed-form inputs.
"""
import pytest

import tests.test_gpu_parity as P

pytestmark = pytest.mark.gpu

V = "cluster"


@pytest.mark.parametrize("N", [1, 8, 64, 256])
def test_decode_full_oracle(N):
    P.test_decode_full_oracle(V, N)


def test_tiny_full_oracle():
    P.test_tiny_full_oracle(V)


def test_expert_sweep_sampled():
    P.test_expert_sweep_sampled(V, 1024)


def test_many_experts_sampled():
    """M = 65,536: 8,192 experts per CTA, 16 passes of 512 with a running top-k."""
    P.test_many_experts_sampled(V)


@pytest.mark.parametrize("N,h,r,M,k", [
    (127, 72, 16, 200, 1),
    (129, 136, 48, 64, 8),
    (1000, 512, 128, 1000, 16),
    (300, 256, 64, 16, 16),      # k == M == KMAX: six of the eight CTAs hold no expert
    (513, 64, 32, 4104, 5),
    (13, 8, 16, 8, 8),           # h == M == 8: one hidden row and at most one expert tile per CTA
])
def test_ragged_shapes_full_oracle(N, h, r, M, k):
    P.test_ragged_shapes_full_oracle(V, N, h, r, M, k)


def test_empty_batch_zeroes_counts():
    P.test_empty_batch_zeroes_counts(V)


@pytest.mark.parametrize("k", [1, 3, 8, 16])
def test_tie_heavy_exact(k):
    P.test_tie_heavy_exact(V, k)


def test_jl_construction_exact():
    P.test_jl_construction_exact(V)


def test_hypercube_top1_is_sign_pattern():
    P.test_hypercube_top1_is_sign_pattern(V)
