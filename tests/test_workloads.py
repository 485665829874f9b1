"""The seeded input generators both sides consume: bf16 rounding, the named
recipes' shapes, dtypes and seeds, and the sampled-position sets."""
import numpy as np
import pytest
import torch

from fft_long_convolution_causal_b200 import workloads as wl


def test_round_bf16_matches_torch_and_ties_to_even():
    r = np.random.default_rng(0)
    x = np.concatenate([r.standard_normal(100_000).astype(np.float32) * 10.0 ** r.integers(-6, 6, 100_000),
                        np.array([0.0, -0.0, 1.0, -2.5, 3.0e38, 1e-40], np.float32)]).astype(np.float32)
    got = wl.round_bf16(x)
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(got, want)
    assert np.all(got.view(np.uint32) & 0xFFFF == 0)          # representable in bf16
    assert np.array_equal(wl.round_bf16(got), got)             # idempotent
    # halfway cases go to the even neighbour: 1 + 2^-8 -> 1, 1 + 3 * 2^-8 -> 1 + 2^-6
    halves = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8], np.float32)
    assert list(wl.round_bf16(halves)) == [1.0, 1 + 2.0 ** -6]


@pytest.mark.parametrize("name", ["pr1_b1_h4_n1024_f32", "hyena_b8_h768_n4096_bf16"])
def test_named_recipes(name):
    c = wl.CONFIGS[name]
    w = wl.make_config(name)
    assert (w.B, w.H, w.N, w.dtype, w.gated, w.seed) == (c["B"], c["H"], c["N"], c["dtype"], c["gated"], c["seed"])
    assert w.u.shape == (c["B"], c["H"], c["N"]) and w.u.dtype == np.float32
    assert w.k.shape == (c["H"], c["N"]) and w.k.dtype == np.float32
    assert (w.D is not None) == c["with_D"] and w.D.shape == (c["H"],)
    if c["dtype"] == "bf16":
        assert np.array_equal(wl.round_bf16(w.u), w.u)
    again = wl.make_config(name)
    assert np.array_equal(again.u, w.u) and np.array_equal(again.k, w.k) and np.array_equal(again.D, w.D)
    assert abs(float(w.u.mean())) < 0.01 and abs(float(w.u.std()) - 1.0) < 0.01


def test_gated_recipe_at_reduced_size():
    """The gated workload's recipe (u, v, w drawn, bf16-rounded, no D) on fewer channels."""
    c = dict(wl.CONFIGS["gated_b4_h1024_n16384_bf16"])
    c.pop("kind")
    c["H"] = 8
    w = wl.make_1d(**c)
    assert w.D is None and w.v is not None and w.w is not None
    for a in (w.u, w.v, w.w):
        assert a.shape == (4, 8, 16384) and np.array_equal(wl.round_bf16(a), a)
    assert not np.array_equal(w.u, w.v) and not np.array_equal(w.v, w.w)
    # decaying filters: the tail of every channel is smaller than its head on average
    head = np.sqrt((w.k[:, :1024].astype(np.float64) ** 2).mean(axis=1))
    tail = np.sqrt((w.k[:, -1024:].astype(np.float64) ** 2).mean(axis=1))
    assert np.all(tail < head)


def test_different_seeds_differ_and_2d_recipe():
    a = wl.make_1d(2, 3, 256, seed=1)
    b = wl.make_1d(2, 3, 256, seed=2)
    assert not np.array_equal(a.u, b.u)
    w = wl.make_2d(2, 3, 32, 16, dtype="bf16", seed=4, sigma=8.0)
    assert w.u.shape == (2, 3, 32, 16) and w.k.shape == (3, 32, 16)
    assert np.array_equal(wl.round_bf16(w.u), w.u)
    # the window anchored at (0, 0): the far corner's taps are the smallest on average
    assert np.abs(w.k[:, :4, :4]).mean() > 10 * np.abs(w.k[:, -4:, -4:]).mean()


def test_sample_points_1d_fixed_set_plus_uniform_draws():
    B, H, N, n = 2, 3, 4096, 12
    b, h, t = wl.sample_points_1d(B, H, N, n, seed=5)
    fixed = {0, 1, N // 2 - 1, N // 2, N - 1} | {1 << i for i in range(12)}
    per_row = len(fixed) + n
    assert b.size == h.size == t.size == B * H * per_row
    for bi in range(B):
        for hi in range(H):
            tt = t[(b == bi) & (h == hi)]
            assert tt.size == per_row and fixed <= set(tt.tolist())
    assert t.min() >= 0 and t.max() < N
    again = wl.sample_points_1d(B, H, N, n, seed=5)
    assert all(np.array_equal(x, y) for x, y in zip((b, h, t), again))


def test_sample_points_2d_corners_and_range():
    b, c, i, j = wl.sample_points_2d(4, 5, 256, 128, 64, seed=1)
    assert b.size == c.size == i.size == j.size == 64
    pts = set(zip(i[:5].tolist(), j[:5].tolist()))
    assert pts == {(0, 0), (0, 127), (255, 0), (255, 127), (128, 64)}
    assert b.max() < 4 and c.max() < 5 and i.max() < 256 and j.max() < 128 and min(i.min(), j.min()) >= 0
