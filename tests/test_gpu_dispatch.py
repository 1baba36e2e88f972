"""GPU dispatch bookkeeping (more_dispatch) vs the oracle, bit-exact.

"MoRE: Scaling mixture of experts with hardware-aware low-rank routing", App. E, Fig. 9
("Sort + Count"): the N k routing slots stably sorted by expert, and per-expert offsets.
Integer work, so every output must equal the oracle's exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.test_gpu_parity import inputs

pytestmark = pytest.mark.gpu


def run_dispatch(idx_np, M, variant="auto"):
    import mixture_experts_rank_b200 as m
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    off, srt = m.dispatch(idx, M, variant=variant)
    torch.cuda.synchronize()
    return off.cpu().numpy(), srt.cpu().numpy(), m.device_status()


def check_random_indices(N, k, M, seed, variant="auto"):
    idx = np.random.default_rng(seed).integers(0, M, size=(N, k))
    off, srt, status = run_dispatch(idx, M, variant)
    assert status == 0
    o = oracle.dispatch(idx, M)
    np.testing.assert_array_equal(off, o.offsets)
    np.testing.assert_array_equal(srt, o.sorted)


def check_one_expert_and_routing_output(variant="auto"):
    N, k, M = 9000, 4, 64
    off, srt, status = run_dispatch(np.full((N, k), 17), M, variant)
    o = oracle.dispatch(np.full((N, k), 17), M)
    np.testing.assert_array_equal(off, o.offsets)
    np.testing.assert_array_equal(srt, o.sorted)
    # routing output: the oracle's selections, dispatched by both sides
    import mixture_experts_rank_b200 as m
    X, R1, R2, Xd, R1d, R2d = inputs(4096, 128, 32, 192)
    sel = oracle.route(X, R1, R2, 4096, 128, 32, 192, 4).idx
    off, srt, status = run_dispatch(sel, 192, variant)
    o = oracle.dispatch(sel, 192)
    np.testing.assert_array_equal(off, o.offsets)
    np.testing.assert_array_equal(srt, o.sorted)
    # and the GPU's own routing: the offsets' differences are its counts
    idx, _, cnt, _ = m.route(Xd, R1d, R2d, 4)
    off, srt = m.dispatch(idx, 192, variant=variant)
    np.testing.assert_array_equal(np.diff(off.cpu().numpy()), cnt.cpu().numpy())


def check_empty_and_out_of_range(variant="auto"):
    off, srt, status = run_dispatch(np.zeros((0, 4)), 32, variant)
    assert status == 0 and np.all(off == 0) and srt.size == 0
    idx = np.array([[3, 40], [1, 3]])  # 40 is outside [0, 32): skipped and flagged
    off, srt, status = run_dispatch(idx, 32, variant)
    assert status & 0x4
    assert off[-1] == 3
    np.testing.assert_array_equal(srt[:3], [2, 0, 3])


@pytest.mark.parametrize("N,k,M,seed", [(1, 1, 8, 0), (37, 3, 16, 1), (3000, 8, 4096, 2), (70000, 8, 1000, 3),
                                        (5000, 16, 262144, 4), (20000, 2, 8, 5)])
def test_dispatch_random_indices(N, k, M, seed):
    check_random_indices(N, k, M, seed)


def test_dispatch_one_expert_and_routing_output():
    check_one_expert_and_routing_output()


def test_dispatch_empty_and_out_of_range():
    check_empty_and_out_of_range()
