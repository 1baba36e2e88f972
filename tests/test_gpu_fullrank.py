"""GPU full-rank router (``more_route_fullrank``; "MoRE: Scaling mixture of experts with
hardware-aware low-rank routing", App. H.3, the standard router fused like the low-rank one)
against the fp64 oracle's ``route_fullrank``, through the C ABI.

Shapes: ragged N, h not a multiple of the 64-element stage, M not a multiple of the 128-expert
tile, k from 1 to 16 (k == M included); the Fig. 20 prefill shape (N = 262,144, h = 2048,
M = 4096, k = 4) and a many-experts shape, both on sampled rows with near-tie tokens; exact
integer inputs with many ties; the empty batch.
"""
import numpy as np
import pytest
import torch

import synthetic as syn
from tests import parity

pytestmark = pytest.mark.gpu


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def weights(h, M, seed):
    """W ~ N(0, 1/h): logits of unit-RMS rows at about unit scale, as the low-rank router's."""
    return syn.normal_bf16(seed, syn.TENSOR_R2, h, M, 1.0 / np.sqrt(h))


def run(X, W, k):
    import mixture_experts_rank_b200 as m
    out = m.route_fullrank(dev_bf16(X), dev_bf16(W), k)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    return [t.cpu().numpy() for t in out]


@pytest.mark.parametrize("N,h,M,k", [
    (300, 256, 200, 4),
    (129, 72, 64, 8),
    (1000, 520, 1000, 16),
    (2049, 1032, 96, 3),
    (64, 64, 16, 16),        # k == M == KMAX
    (513, 136, 4104, 5),     # M one tile past a multiple of 128
    (1, 2048, 4096, 1),
])
def test_fullrank_matches_oracle(N, h, M, k):
    X = syn.normal_bf16(N, syn.TENSOR_X, N, h)
    W = weights(h, M, N + 1)
    idx, gate, cnt, logits = run(X, W, k)
    parity.compare_fullrank(X, W, N, h, M, k, idx, gate, cnt, logits)


def test_fullrank_prefill_sampled():
    """The Fig. 20 prefill shape at h = 2048, M = 4096, k = 4: rows at unit RMS, 2048 sampled
    rows (first and last, three whole middle tiles, random) plus the 256 closest near-ties of
    8192 scanned rows."""
    N, h, M, k = 262144, 2048, 4096, 4
    X = syn.normal_bf16(0, syn.TENSOR_X, N, h, 1.0, True)
    W = weights(h, M, 0)
    idx, gate, cnt, logits = run(X, W, k)
    scan = np.random.default_rng(1).choice(N, 8192, replace=False)
    near = parity.near_tie_rows_fullrank(X, W, N, h, M, k, 256, scan=scan)
    rows = parity.sample_rows(N, 2048, 0, tiles=(N // 256, N // 384 + 1, (5 * N) // 768), extra=near)
    rep = parity.compare_fullrank(X, W, N, h, M, k, idx, gate, cnt, logits, rows=rows)
    assert rep.fine_set_compared > 0.9 * rows.size


def test_fullrank_many_experts_sampled():
    N, h, M, k = 4096, 1024, 65536, 8
    X = syn.normal_bf16(3, syn.TENSOR_X, N, h)
    W = weights(h, M, 3)
    idx, gate, cnt, logits = run(X, W, k)
    rows = parity.sample_rows(N, 192, 3, tiles=(17,))
    parity.compare_fullrank(X, W, N, h, M, k, idx, gate, cnt, logits, rows=rows)


@pytest.mark.parametrize("k", [1, 3, 8, 16])
def test_fullrank_tie_heavy_exact(k):
    """One-hot rows times a small-integer W: every logit is a small integer, with many exact
    ties, which must go to the lower expert."""
    N, h, M = 777, 64, 192
    rng = np.random.default_rng(k)
    X = syn.f32_to_bf16_bits(np.eye(h, dtype=np.float32)[rng.integers(0, h, N)])
    W = syn.f32_to_bf16_bits(rng.integers(-3, 4, size=(h, M)).astype(np.float32))
    idx, gate, cnt, logits = run(X, W, k)
    parity.compare_fullrank(X, W, N, h, M, k, idx, gate, cnt, logits, exact=True)


def test_fullrank_empty_batch_zeroes_counts():
    import mixture_experts_rank_b200 as m
    h, M, k = 64, 128, 4
    cnt = torch.full((M,), 7, dtype=torch.int32, device="cuda")
    m.route_fullrank(torch.zeros((0, h), dtype=torch.bfloat16, device="cuda"),
                     torch.zeros((h, M), dtype=torch.bfloat16, device="cuda"), k, out_expert_count=cnt)
    torch.cuda.synchronize()
    assert int(cnt.abs().sum()) == 0
