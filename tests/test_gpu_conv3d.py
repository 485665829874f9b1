"""GPU parity of the 3-D causal convolution (first-octant crop of the
zero-padded linear convolution, "Native Multi-Dimensional Subquadratic
Operators via Input Dependent Long Convolutions", abstract: N-D geometry)
through the C ABI against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from fft_long_convolution_causal_b200 import workloads as wlmod
from parity import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_causal_b200 import binding
    binding.load_library()


def _volume(B, C, Dd, Hs, Ws, Kd, Kh, Kw, dtype, seed, sigma):
    """u ~ N(0,1); k[c,e,p,q] = N(0,1) exp(-(e^2 + p^2 + q^2) / (2 sigma^2))."""
    r = np.random.default_rng(seed)
    u = r.standard_normal((B, C, Dd, Hs, Ws)).astype(np.float32)
    if dtype == "bf16":
        u = wlmod.round_bf16(u)
    e = np.arange(Kd, dtype=np.float64)[:, None, None]
    p = np.arange(Kh, dtype=np.float64)[None, :, None]
    q = np.arange(Kw, dtype=np.float64)[None, None, :]
    win = np.exp(-(e * e + p * p + q * q) / (2.0 * sigma * sigma))
    k = (r.standard_normal((C, Kd, Kh, Kw)) * win[None]).astype(np.float32)
    return u, k


def _scale(u, k, b_idx=None, c_idx=None):
    """Per-volume scale RMS(u[b, c]) * ||k[c]||."""
    s = np.sqrt(np.mean(u.astype(np.float64) ** 2, axis=(2, 3, 4))) * np.sqrt(
        np.sum(k.astype(np.float64) ** 2, axis=(1, 2, 3)))[None, :]
    if b_idx is None:
        return np.broadcast_to(s[:, :, None, None, None], u.shape)
    return s[b_idx, c_idx]


def _run(u, k, dtype, **kw):
    from fft_long_convolution_causal_b200 import binding
    B, C, Dd, Hs, Ws = u.shape
    plan = binding.Plan3D(B, C, Dd, Hs, Ws, dtype)
    assert plan.path == "3d"
    khat = plan.kernel_spectrum(torch.from_numpy(k).cuda())
    y = to_host(plan.fwd(to_dev(u, dtype), khat))
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    return y, plan


@pytest.mark.parametrize("B,C,Dd,Hs,Ws,Kd,Kh,Kw,dtype", [
    (3, 2, 16, 16, 16, 16, 16, 16, "f32"), (2, 3, 16, 32, 16, 5, 20, 16, "f32"), (1, 2, 32, 16, 32, 32, 3, 7, "f32"),
    (4, 1, 16, 16, 64, 9, 16, 33, "bf16"), (3, 2, 16, 16, 16, 1, 1, 1, "f32")])
def test_conv3d_full_compare(B, C, Dd, Hs, Ws, Kd, Kh, Kw, dtype):
    """Every output: odd and even B, B = 1, filters shorter than the volume
    along each axis, the single-tap filter (y = k u), bf16 I/O."""
    u, k = _volume(B, C, Dd, Hs, Ws, Kd, Kh, Kw, dtype, seed=Dd + 3 * Hs + 7 * Ws + B, sigma=Dd / 2)
    y, _ = _run(u, k, dtype)
    want = oracle.causal_conv3d(u, k)
    assert_close(y, want, dtype, f"3d B={B} C={C} {Dd}x{Hs}x{Ws} k{Kd}x{Kh}x{Kw} {dtype}", scale=_scale(u, k))


def test_conv3d_sampled_larger():
    """64 x 64 x 64 volumes, full-size filters: 2048 sampled voxels."""
    B, C, Dd, Hs, Ws = 2, 2, 64, 64, 64
    u, k = _volume(B, C, Dd, Hs, Ws, Dd, Hs, Ws, "f32", seed=91, sigma=16.0)
    y, _ = _run(u, k, "f32")
    r = np.random.default_rng(92)
    n = 2048
    idx = (r.integers(0, B, n), r.integers(0, C, n), r.integers(0, Dd, n), r.integers(0, Hs, n),
           r.integers(0, Ws, n))
    ref = oracle.causal_conv3d_points(u, k, *idx)
    assert_close(y[idx], ref, "f32", "3d 64^3 sampled", scale=_scale(u, k, idx[0], idx[1]))


def test_conv3d_several_groups():
    """256 x 256 x 128 volumes: the 1 GiB workspace holds two channels' slice
    spectra (402 MB each), so three channels run as groups of 2 and 1; 2048
    sampled voxels (8 x 8 x 8 filters)."""
    from fft_long_convolution_causal_b200 import binding
    B, C, Dd, Hs, Ws = 1, 3, 256, 256, 128
    u, k = _volume(B, C, Dd, Hs, Ws, 8, 8, 8, "f32", seed=93, sigma=4.0)
    plan = binding.Plan3D(B, C, Dd, Hs, Ws, "f32")
    assert plan.workspace_bytes == 2 * Dd * (Hs + 2 * Hs) * 2 * Ws * 8
    khat = plan.kernel_spectrum(torch.from_numpy(k).cuda())
    y = to_host(plan.fwd(to_dev(u, "f32"), khat))
    r = np.random.default_rng(94)
    n = 2048
    idx = (r.integers(0, B, n), r.integers(0, C, n), r.integers(0, Dd, n), r.integers(0, Hs, n),
           r.integers(0, Ws, n))
    ref = oracle.causal_conv3d_points(u, k, *idx)
    assert_close(y[idx], ref, "f32", "3d groups", scale=_scale(u, k, idx[0], idx[1]))


@pytest.mark.parametrize("B,dtype", [(1, "f32"), (2, "bf16")])
def test_conv3d_max_side_full_filters(B, dtype):
    """256 x 256 x 256 volumes, the largest side on every axis, with filters
    as large as the volume: the eight corners of each volume (the far corner
    sums all 256^3 taps) plus uniformly drawn voxels."""
    C, S = 1, 256
    u, k = _volume(B, C, S, S, S, S, S, S, dtype, seed=95, sigma=48.0)
    y, _ = _run(u, k, dtype)
    r = np.random.default_rng(96)
    corners = np.array([(d, h, w) for d in (0, S - 1) for h in (0, S - 1) for w in (0, S - 1)])
    n = 96
    bi = np.concatenate([np.repeat(np.arange(B), len(corners)), r.integers(0, B, n)])
    di = np.concatenate([np.tile(corners[:, 0], B), r.integers(0, S, n)])
    hi = np.concatenate([np.tile(corners[:, 1], B), r.integers(0, S, n)])
    wi = np.concatenate([np.tile(corners[:, 2], B), r.integers(0, S, n)])
    ci = np.zeros_like(bi)
    ref = oracle.causal_conv3d_points(u, k, bi, ci, di, hi, wi)
    assert_close(y[bi, ci, di, hi, wi], ref, dtype, f"3d 256^3 {dtype}", scale=_scale(u, k, bi, ci))


def test_conv3d_errors():
    from fft_long_convolution_causal_b200 import binding
    with pytest.raises(binding.FFTConvError):
        binding.Plan3D(1, 1, 8, 16, 16, "f32")  # depth below the minimum
    plan = binding.Plan3D(1, 1, 16, 16, 16, "f32")
    u = torch.zeros(1, 1, 16, 16, 16, device="cuda")
    with pytest.raises(binding.FFTConvError):
        plan.fwd(u, plan.new_spectrum())  # spectrum not computed
    with pytest.raises(binding.FFTConvError):
        plan.kernel_spectrum(torch.zeros(1, 17, 1, 1, device="cuda"))  # Kd > Dd
