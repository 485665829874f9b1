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
        q.put((r, w, mx, fdist.job_throughput(1000, w, mx)))
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
    for _, w, mx, thr in got:
        assert w == 2 and mx == pytest.approx(2.5) and thr == pytest.approx(2000 / 2.5)


def test_single_process_is_identity():
    assert fdist.max_over_ranks(3.25) == 3.25
    assert fdist.job_throughput(10, 1, 2.0) == 5.0
