"""Host-side helpers for runs with one process per GPU (torchrun).

The convolution's rows are independent and every channel's spectrum is
read-only, so the data path needs no collective: the channels are split into
contiguous blocks, one per rank, each rank computes its own spectrum slice and
its own output slice, and only the timings are combined (max over ranks, the
slowest rank bounds the job).  A caller that needs one logical output tensor
gathers the slices along the channel axis.
"""
import os


def rank_env():
    """(rank, world_size, local_rank) from the torchrun environment (1 process default)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_channels(H, world, rank):
    """Channel block [h0, h1) of `rank` when H channels are split over `world`
    ranks: contiguous, in rank order, sizes differing by at most one (the first
    H % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    base, rem = divmod(int(H), int(world))
    h0 = rank * base + min(rank, rem)
    return h0, h0 + base + (1 if rank < rem else 0)


def slice_channels_1d(wl, h0, h1):
    """The channels [h0, h1) of a 1-D workload as a workload of its own
    (u, v, w [:, h0:h1], k [h0:h1], D [h0:h1]): a rank's shard."""
    from dataclasses import replace
    sl = slice(h0, h1)
    return replace(wl, name=f"{wl.name}[h{h0}:{h1}]", H=h1 - h0, u=wl.u[:, sl].copy(), k=wl.k[sl].copy(),
                   D=None if wl.D is None else wl.D[sl].copy(),
                   v=None if wl.v is None else wl.v[:, sl].copy(), w=None if wl.w is None else wl.w[:, sl].copy())


def slice_channels_2d(wl, c0, c1):
    """The channels [c0, c1) of a 2-D workload (u [:, c0:c1], k [c0:c1])."""
    from dataclasses import replace
    sl = slice(c0, c1)
    return replace(wl, name=f"{wl.name}[c{c0}:{c1}]", C=c1 - c0, u=wl.u[:, sl].copy(), k=wl.k[sl].copy())


def max_over_ranks(value, dist=None, device=None):
    """Max of a float over all ranks of the default process group (identity when single)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value, dist=None, device=None):
    """Sum of a float over all ranks of the default process group (identity when single)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_throughput(outputs_per_rank, world, max_seconds):
    """Whole-job outputs per second: every rank's outputs over the slowest rank's time."""
    return outputs_per_rank * world / max_seconds
