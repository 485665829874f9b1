"""The multi-rank timing logic of bench.py on world_size-2 gloo ranks (CPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from fft_long_convolution_causal_b200 import dist as fdist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as d
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    d.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, _ = fdist.rank_env()
        mx = fdist.max_over_ranks(1.5 + r, d)
        # uneven shards: rank r holds 1000 + 7 r outputs; the job holds their sum
        total = fdist.sum_over_ranks(1000 + 7 * r, d)
        q.put((r, w, mx, fdist.job_throughput(1000, w, mx), total))
    finally:
        d.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[0] for g in got] == [0, 1]
    for _, w, mx, thr, total in got:
        assert w == 2 and mx == pytest.approx(2.5) and thr == pytest.approx(2000 / 2.5)
        assert total == 2007.0


def test_single_process_is_identity():
    assert fdist.max_over_ranks(3.25) == 3.25
    assert fdist.sum_over_ranks(3.25) == 3.25
    assert fdist.job_throughput(10, 1, 2.0) == 5.0


@pytest.mark.parametrize("H,world", [(768, 8), (10, 3), (5, 2), (3, 4), (1, 1)])
def test_shard_channels_partition(H, world):
    blocks = [fdist.shard_channels(H, world, r) for r in range(world)]
    assert blocks[0][0] == 0 and blocks[-1][1] == H
    for (a0, a1), (b0, b1) in zip(blocks, blocks[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in blocks]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == H


def _shard_worker(rank, world, port, q, spec):
    """One gloo rank: its channel shard of a small workload through the oracle,
    all-gathered; rank 0 reports the gathered output."""
    import numpy as np
    import torch
    import torch.distributed as d
    import oracle
    from fft_long_convolution_causal_b200 import workloads as wlmod
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    d.init_process_group("gloo", rank=rank, world_size=world)
    try:
        kind, args = spec
        if kind == "1d":
            wl = wlmod.make_1d(**args)
            h0, h1 = fdist.shard_channels(wl.H, world, rank)
            sh = fdist.slice_channels_1d(wl, h0, h1)
            y = oracle.causal_conv1d(sh.u, sh.k, D=sh.D, w=sh.w, v=sh.v)
            axis_len = wl.H
        else:
            wl = wlmod.make_2d(**args)
            c0, c1 = fdist.shard_channels(wl.C, world, rank)
            sh = fdist.slice_channels_2d(wl, c0, c1)
            y = oracle.causal_conv2d(sh.u, sh.k)
            axis_len = wl.C
        # uneven shards: pad to the largest before the all-gather, crop after
        most = -(-axis_len // world)
        pad = np.zeros((y.shape[0], most) + y.shape[2:])
        pad[:, :y.shape[1]] = y
        parts = [torch.zeros_like(torch.from_numpy(pad)) for _ in range(world)]
        d.all_gather(parts, torch.from_numpy(pad))
        if rank == 0:
            pieces = []
            for r, t in enumerate(parts):
                a, b = fdist.shard_channels(axis_len, world, r)
                pieces.append(t.numpy()[:, :b - a])
            q.put(np.concatenate(pieces, axis=1))
    finally:
        d.destroy_process_group()


@pytest.mark.parametrize("spec", [
    ("1d", dict(B=3, H=5, N=256, dtype="bf16", gated=True, seed=41, with_D=True)),
    ("1d", dict(B=2, H=4, N=512, dtype="f32", seed=42)),
    ("2d", dict(B=3, C=3, Hs=16, Ws=32, dtype="f32", seed=43, sigma=8.0)),
])
def test_channel_shards_reproduce_the_whole(spec):
    """Two gloo ranks each convolve their channel block (the index arithmetic
    bench.py and a multi-GPU caller use); the gathered result equals the
    whole-workload oracle output exactly (same fp64 sums, same order)."""
    import numpy as np
    import oracle
    from fft_long_convolution_causal_b200 import workloads as wlmod
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q, spec)) for r in range(2)]
    for p in procs:
        p.start()
    got = q.get(timeout=120)
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    kind, args = spec
    if kind == "1d":
        wl = wlmod.make_1d(**args)
        want = oracle.causal_conv1d(wl.u, wl.k, D=wl.D, w=wl.w, v=wl.v)
    else:
        wl = wlmod.make_2d(**args)
        want = oracle.causal_conv2d(wl.u, wl.k)
    assert got.shape == want.shape
    assert np.array_equal(got, want)
