"""Data-parallel replicas of the forward pass, one process per GPU.

The rows of a batch are independent sequences ("The Mathematics of Karpathy's
nanochat", §Data Loading and Batching: B rows of T tokens each), so N ranks
run N replicas of the same weights on disjoint rows with no collective on the
data path.  The ranks meet only in three host-side reductions:
  * the timing: the slowest rank's elapsed time defines the step time;
  * the throughput: tokens of all ranks divided by that time;
  * the mean loss of the global batch ([Math] §Cross-Entropy Loss: the mean
    over every valid target of every row), one all-reduce of the pair
    (sum of per-token losses, count of valid targets).
Everything here is plumbing over torch.distributed; no arithmetic of the
forward pass lives in this module.
"""
from __future__ import annotations


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic rows (distinct rows per rank, same weights)."""
    return seed + 1000 * rank


def _dist():
    import torch.distributed as dist
    return dist if dist.is_available() and dist.is_initialized() else None


def _device():
    import torch
    dist = _dist()
    if dist is not None and dist.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def max_over_ranks(x: float) -> float:
    """The largest value of x over all ranks (x itself without a process group)."""
    import torch
    dist = _dist()
    if dist is None or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def global_mean_loss(loss_sum: float, count: int) -> float:
    """Mean per-token loss of the global batch from each rank's (sum, count);
    NaN when no rank has a valid target."""
    import torch
    dist = _dist()
    t = torch.tensor([float(loss_sum), float(count)], dtype=torch.float64, device=_device())
    if dist is not None and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    s, n = float(t[0].item()), float(t[1].item())
    return s / n if n > 0 else float("nan")


def aggregate_throughput(tokens_per_rank: int, world: int, steps: int, seconds_max: float) -> float:
    """Whole-job tokens per second: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world * steps / seconds_max
