"""GPU training statistics (more_route_train) vs the fp64 oracle, through the C ABI.

"MoRE: Scaling mixture of experts with hardware-aware low-rank routing", App. F,
Algorithm 2 and eqs. (6)-(8): per token m = max_j l_j and Z = sum_j exp(l_j - m); per
expert psum_i = sum_n exp(l_ni - m_n) / Z_n.

Tolerances follow from the logit tolerance tol_n = 1e-2 x rms_n of the routing parity
checks (every GPU logit within tol_n of the oracle's): m is a logit, so |dm| <= tol_n;
log Z moves by at most max_j |dl_j - dm| <= 2 tol_n; each probability's relative error
is at most |dl - dm| + |d log Z| <= 4 tol_n, and so is each psum_i's (a sum of positive
terms), up to fp32 rounding of the sums (relative 1e-5 here).
"""
import numpy as np
import pytest
import torch

import oracle
from tests import parity
from tests.test_gpu_parity import inputs

pytestmark = pytest.mark.gpu


def run_train(Xd, R1d, R2d, k):
    import mixture_experts_rank_b200 as m
    out = m.route_train(Xd, R1d, R2d, k)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    return [None if t is None else t.cpu().numpy() for t in out]


def check_stats(N, h, r, M, k, seed=0, unit_rms=False):
    import mixture_experts_rank_b200 as m
    X, R1, R2, Xd, R1d, R2d = inputs(N, h, r, M, seed, unit_rms)
    idx, gate, cnt, logits, gm, gZ, gpsum = run_train(Xd, R1d, R2d, k)
    # the routing outputs are those of more_route
    ri, rg, rc, rl = (t.cpu().numpy() for t in m.route(Xd, R1d, R2d, k))
    np.testing.assert_array_equal(idx, ri)
    np.testing.assert_array_equal(cnt, rc)
    np.testing.assert_array_equal(gate, rg)
    parity.compare(X, R1, R2, N, h, r, M, k, idx, gate, cnt, logits, rows=parity.sample_rows(N, 256, seed)
                   if N > 4096 else None)
    o = oracle.train_stats(X, R1, R2, N, h, r, M)
    rms = oracle.route(X, R1, R2, N, h, r, M, min(k, M)).rms
    tol = parity.LOGIT_TOL * rms
    assert np.all(np.abs(gm - o.m) <= tol), f"m: max err / rms {np.max(np.abs(gm - o.m) / rms):.3g}"
    dlogZ = np.abs(np.log(gZ.astype(np.float64)) - np.log(o.Z))
    assert np.all(dlogZ <= 2 * tol + 1e-5), f"log Z: max err {dlogZ.max():.3g}"
    rel = np.abs(gpsum - o.psum) / o.psum
    assert np.all(rel <= 4 * tol.max() + 1e-5), f"psum: max relative err {rel.max():.3g}"
    assert abs(gpsum.astype(np.float64).sum() - N) <= 1e-4 * N  # every softmax row sums to one
    return float(np.max(np.abs(gm - o.m) / rms)), float(dlogZ.max()), float(rel.max())


def test_tiny_train_stats():
    check_stats(4096, 128, 32, 192, 4)


def test_sweep_shape_train_stats():
    check_stats(16384, 512, 32, 2048, 8)


@pytest.mark.parametrize("N,h,r,M,k", [(37, 72, 16, 200, 1), (300, 256, 64, 16, 16), (513, 128, 128, 1000, 8),
                                       (129, 136, 48, 64, 8)])   # r = 48: the CUDA-core statistics kernel
def test_ragged_train_stats(N, h, r, M, k):
    check_stats(N, h, r, M, k)


def test_empty_batch_train_stats():
    import mixture_experts_rank_b200 as m
    _, _, _, _, R1d, R2d = inputs(8, 64, 32, 64)
    X = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    out = m.route_train(X, R1d, R2d, 4)
    torch.cuda.synchronize()
    assert int(out[2].sum()) == 0 and float(out[6].abs().sum()) == 0.0
