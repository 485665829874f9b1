"""Host-side helpers for runs with one process per GPU (torchrun).

The convolution's rows are independent, so the data path needs no
collective: each rank runs its own workload and only the timings are combined
(max over ranks, the slowest rank bounds the job).
"""
import os


def rank_env():
    """(rank, world_size, local_rank) from the torchrun environment (1 process default)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value, dist=None, device=None):
    """Max of a float over all ranks of the default process group (identity when single)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(outputs_per_rank, world, max_seconds):
    """Whole-job outputs per second: every rank's outputs over the slowest rank's time."""
    return outputs_per_rank * world / max_seconds
