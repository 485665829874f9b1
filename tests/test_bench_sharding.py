"""bench.py's per-rank workloads: weak sharding gives every rank the named
shape (rank 0 exactly the named draw), strong sharding splits the named
workload's channels so that the blocks put back together are the whole."""
import importlib.util
import os

import numpy as np
import pytest

from fft_long_convolution_causal_b200 import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_shard", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def test_weak_shards_have_the_named_shape():
    b = _bench()
    named = workloads.make_config("pr1_b1_h4_n1024_f32")
    r0 = b.build_workload("pr1_b1_h4_n1024_f32", rank=0, world=2, shard="weak")
    r1 = b.build_workload("pr1_b1_h4_n1024_f32", rank=1, world=2, shard="weak")
    assert np.array_equal(r0.u, named.u) and np.array_equal(r0.k, named.k) and np.array_equal(r0.D, named.D)
    assert r1.u.shape == named.u.shape and not np.array_equal(r1.u, named.u)


@pytest.mark.parametrize("world", [2, 3, 4])
def test_strong_shards_reassemble_the_workload(world):
    b = _bench()
    name = "pr1_b1_h4_n1024_f32"
    whole = workloads.make_config(name)
    parts = [b.build_workload(name, rank=r, world=world, shard="strong") for r in range(world)]
    assert sum(p.H for p in parts) == whole.H
    assert np.array_equal(np.concatenate([p.u for p in parts], axis=1), whole.u)
    assert np.array_equal(np.concatenate([p.k for p in parts], axis=0), whole.k)
    assert np.array_equal(np.concatenate([p.D for p in parts], axis=0), whole.D)


def test_strong_2d_shards_reassemble_the_workload():
    b = _bench()
    name = "conv2d_b4_c256_256x256_bf16"
    whole = b.build_workload(name, channels=6)
    parts = [b.build_workload(name, channels=6, rank=r, world=4, shard="strong") for r in range(4)]
    assert [p.C for p in parts] == [2, 2, 1, 1]
    assert np.array_equal(np.concatenate([p.u for p in parts], axis=1), whole.u)
    assert np.array_equal(np.concatenate([p.k for p in parts], axis=0), whole.k)


def test_strong_sharding_refuses_more_ranks_than_channels():
    b = _bench()
    with pytest.raises(SystemExit):
        b.build_workload("pr1_b1_h4_n1024_f32", rank=0, world=8, shard="strong")
