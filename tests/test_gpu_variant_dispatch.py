"""The shared-memory dispatch variant (MORE_DISPATCH_SHARED) vs the oracle, bit-exact.

"MoRE: Scaling mixture of experts with hardware-aware low-rank routing", App. E, Fig. 9
("Sort + Count").  The checks of tests/test_gpu_dispatch.py, with about two chunks per SM
counted in shared-memory histograms; experts up to MORE_DISPATCH_SHARED_MMAX.
"""
import numpy as np
import pytest
import torch

import tests.test_gpu_dispatch as D

pytestmark = pytest.mark.gpu

V = "shared"


@pytest.mark.parametrize("N,k,M,seed", [(1, 1, 8, 0), (37, 3, 16, 1), (3000, 8, 4096, 2), (70000, 8, 1000, 3),
                                        (262144, 8, 4096, 6), (5000, 16, 32768, 4), (20000, 2, 8, 5)])
def test_dispatch_random_indices(N, k, M, seed):
    D.check_random_indices(N, k, M, seed, V)


def test_dispatch_one_expert_and_routing_output():
    D.check_one_expert_and_routing_output(V)


def test_dispatch_empty_and_out_of_range():
    D.check_empty_and_out_of_range(V)


def test_dispatch_rejects_too_many_experts():
    import mixture_experts_rank_b200 as m
    idx = torch.zeros((4, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(m.MoreError) as e:
        m.dispatch(idx, 32776, variant=V)
    assert e.value.status == 2
