"""The multi-rank host path on CPU: two gloo ranks split a token batch by rows.

Routing is independent per token ("MoRE: Scaling mixture of experts with
hardware-aware low-rank routing", App. F), so each rank routes its own rows.  Only
batch-wide sums cross ranks: the per-expert counts (App. F eq. (9)), the softmax
column sums psum (eq. (7)), and the R1 and R2 gradients of the backward
(Algorithm 3).  On CPU the fp64 oracle stands in for each rank's calls; what is
tested is the sharding, those all-reduces, and the max-over-ranks timing reduction.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, n_total, shape, out_dir):
    import sys

    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle
    import synthetic as syn
    from mixture_experts_rank_b200 import shard

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        h, r, M, k = shape
        begin, count = shard.shard_range(n_total, world, rank)
        X, R1, R2 = syn.router_inputs(n_total, h, r, M, seed=0, row_begin=begin, n_rows=count)
        res = oracle.route(X, R1, R2, count, h, r, M, k, threads=2)
        local = torch.from_numpy(res.counts.astype(np.int32))
        total = shard.global_expert_counts(local)
        st = oracle.train_stats(X, R1, R2, count, h, r, M, threads=2)
        psum = shard.global_psum(torch.from_numpy(st.psum.astype(np.float32)))
        slowest = shard.max_over_ranks(1.5 + rank, torch.device("cpu"))
        # backward of this rank's rows (the same pbar everywhere), R1 and R2 gradients summed
        rng = np.random.default_rng(5)
        tvb_all, pbar = rng.standard_normal((n_total, k)), rng.standard_normal(M)
        g = oracle.router_backward(X, R1, R2, count, h, r, M, res.idx, tvb_all[begin:begin + count], pbar)
        r1bar, r2bar = shard.global_router_grads(torch.from_numpy(g.R1.astype(np.float32)),
                                                 torch.from_numpy(g.R2.astype(np.float32)))
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), begin=begin, count=count, idx=res.idx,
                 total=total.numpy(), slowest=slowest, psum=psum.numpy(), xbar=g.X, r1bar=r1bar.numpy(),
                 r2bar=r2bar.numpy())
    finally:
        dist.destroy_process_group()


def test_shard_range_partitions_rows():
    from mixture_experts_rank_b200 import shard

    for n_total in (0, 1, 7, 64, 1001):
        for world in (1, 2, 3, 8):
            ranges = [shard.shard_range(n_total, world, i) for i in range(world)]
            assert ranges[0][0] == 0
            for (b0, c0), (b1, _) in zip(ranges, ranges[1:]):
                assert b0 + c0 == b1
            assert sum(c for _, c in ranges) == n_total
            assert max(c for _, c in ranges) - min(c for _, c in ranges) <= 1
    with pytest.raises(ValueError):
        shard.shard_range(10, 2, 2)


def test_two_gloo_ranks_match_single_batch(tmp_path):
    n_total, shape = 37, (128, 32, 192, 4)  # ragged: 19 + 18 rows
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), n_total, shape, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    parts = [np.load(tmp_path / f"rank{i}.npz") for i in range(world)]

    import oracle
    import synthetic as syn

    h, r, M, k = shape
    X, R1, R2 = syn.router_inputs(n_total, h, r, M, seed=0)
    whole = oracle.route(X, R1, R2, n_total, h, r, M, k, threads=2)
    idx = np.concatenate([p["idx"] for p in parts])
    np.testing.assert_array_equal(idx, whole.idx)                  # shards cover the batch in order
    whole_stats = oracle.train_stats(X, R1, R2, n_total, h, r, M, threads=2)
    for p in parts:
        np.testing.assert_array_equal(p["total"], whole.counts)    # all-reduced counts = whole batch
        assert float(p["slowest"]) == 2.5                          # max over ranks
        # all-reduced softmax column sums = the whole batch's (fp32 per rank, then summed)
        np.testing.assert_allclose(p["psum"], whole_stats.psum, rtol=1e-6)
    assert int(parts[0]["total"].sum()) == n_total * k
    # backward: per-rank X gradients are the whole batch's rows; R1 and R2 gradients all-reduced
    rng = np.random.default_rng(5)
    tvb_all, pbar = rng.standard_normal((n_total, k)), rng.standard_normal(M)
    gw = oracle.router_backward(X, R1, R2, n_total, h, r, M, whole.idx, tvb_all, pbar)
    np.testing.assert_allclose(np.concatenate([p["xbar"] for p in parts]), gw.X, rtol=1e-12, atol=1e-15)
    for p in parts:  # fp32 per rank, then summed: relative 1e-6 of the largest entry
        np.testing.assert_allclose(p["r1bar"], gw.R1, rtol=0, atol=1e-6 * np.abs(gw.R1).max())
        np.testing.assert_allclose(p["r2bar"], gw.R2, rtol=0, atol=1e-6 * np.abs(gw.R2).max())
