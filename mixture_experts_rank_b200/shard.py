"""Token sharding of the router across ranks (one process per GPU).

Routing is independent per token ("MoRE: Scaling mixture of experts with
hardware-aware low-rank routing", App. F: every token's top-k depends only on its
own row of X and the shared R1, R2), so N tokens split into contiguous row
ranges, one per rank, with R1 and R2 replicated.  No collective is needed on the
data path; the helpers below are the host-side bookkeeping around it:

* ``shard_range``: the row range of a rank;
* ``global_expert_counts``: the sum over ranks of the per-rank expert counts
  (the per-expert load statistic f of App. F eq. (9) over the whole batch), one
  all-reduce of M integers, outside the routing call;
* ``global_psum``: the same for the softmax column sums psum of the training call
  (App. F eq. (7)), so the balancing loss of eq. (9) covers the whole batch;
* ``global_router_grads``: the sum over ranks of the R1 and R2 gradients of the backward
  (App. F, Algorithm 3), each rank's a sum over its own tokens: one all-reduce of
  h r + r M values; the X gradient stays with the rank whose rows it is;
* ``max_over_ranks``: the slowest rank's time, which sets the batch's time.
"""
from __future__ import annotations

import torch


def shard_range(n_total: int, world: int, rank: int) -> tuple[int, int]:
    """Rows ``[begin, begin + count)`` of ``rank``: contiguous, sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world or n_total < 0:
        raise ValueError(f"bad shard request: n_total={n_total} world={world} rank={rank}")
    base, extra = divmod(n_total, world)
    begin = rank * base + min(rank, extra)
    return begin, base + (1 if rank < extra else 0)


def global_expert_counts(local_counts: torch.Tensor, group=None) -> torch.Tensor:
    """Sum of every rank's ``out_expert_count`` (int32 [M]); returns a new int64 tensor."""
    import torch.distributed as dist

    total = local_counts.to(torch.int64).clone()
    dist.all_reduce(total, op=dist.ReduceOp.SUM, group=group)
    return total


def global_psum(local_psum: torch.Tensor, group=None) -> torch.Tensor:
    """Sum of every rank's ``out_psum`` (fp32 [M], from ``route_train``) in fp64: the column
    sum of the full softmax over the whole batch (App. F eq. (7)), for the balancing loss."""
    import torch.distributed as dist

    total = local_psum.to(torch.float64).clone()
    dist.all_reduce(total, op=dist.ReduceOp.SUM, group=group)
    return total


def global_router_grads(R1bar: torch.Tensor, R2bar: torch.Tensor, group=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Sum over ranks of ``out_R1bar`` [h, r] and ``out_R2bar`` [r, M] (fp32, from
    ``route_backward`` on each rank's token shard, with the same pbar on every rank), summed
    in fp64 in one all-reduce; returns new fp64 tensors of the same shapes."""
    import torch.distributed as dist

    n1 = R1bar.numel()
    flat = torch.cat([R1bar.reshape(-1), R2bar.reshape(-1)]).to(torch.float64)
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return flat[:n1].view(R1bar.shape), flat[n1:].view(R2bar.shape)


def max_over_ranks(value: float, device, group=None) -> float:
    """The largest of the ranks' values (used for per-step times)."""
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
