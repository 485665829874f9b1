"""GPU parity of the forward with input-dependent filters (one per batch row,
transformed in the same launch; one per 2-D image, transformed in the same
call) through the C ABI against the fp64 oracle."""
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


def _filters(B, H, L, seed):
    """Per-row decaying filters k[b,h,t] = N(0,1) exp(-a_bh t), a_bh ~ U(1e-4, 1e-2)."""
    r = np.random.default_rng(seed)
    a = r.uniform(1e-4, 1e-2, size=(B, H, 1))
    t = np.arange(L)[None, None, :]
    return (r.standard_normal((B, H, L)) * np.exp(-a * t)).astype(np.float32)


def _row_scale(wl, k):
    x = wl.u.astype(np.float64) * (wl.w if wl.gated else 1.0)
    kn = np.sqrt(np.sum(k.astype(np.float64) ** 2, axis=2))
    if wl.D is not None:
        kn = kn + np.abs(wl.D.astype(np.float64))[None, :]
    return np.broadcast_to((np.sqrt(np.mean(x * x, axis=2)) * kn)[:, :, None], wl.u.shape)


@pytest.mark.parametrize("N,dtype,gated,with_D,B,L", [
    (64, "f32", False, True, 3, None), (1024, "f32", True, True, 2, 500), (4096, "f32", False, False, 5, None),
    (4096, "bf16", False, True, 4, None), (2048, "bf16", True, True, 3, 77), (512, "bf16", False, True, 1, None)])
def test_dynamic_full_compare(N, dtype, gated, with_D, B, L):
    from fft_long_convolution_causal_b200 import binding
    wl = wlmod.make_1d(B, 3, N, dtype=dtype, gated=gated, seed=N + B, with_D=with_D)
    k = _filters(B, 3, L or N, seed=N + 11)
    plan = binding.Plan(B, 3, N, dtype, gated=gated)
    D = torch.from_numpy(wl.D).cuda() if wl.D is not None else None
    y = plan.fwd_dynamic(to_dev(wl.u, dtype), torch.from_numpy(k).cuda(), D=D, v=to_dev(wl.v, dtype),
                         w=to_dev(wl.w, dtype))
    torch.cuda.synchronize()
    want = oracle.causal_conv1d_dynamic(wl.u, k, D=wl.D, w=wl.w, v=wl.v)
    # the whole transform runs in fp32 (bf16 only at the I/O): the fp32 bound,
    # plus the bf16 output rounding for bf16 plans
    assert_close(to_host(y), want, dtype, f"dynamic N={N} {dtype} gated={gated} B={B} L={L}",
                 gate=wl.v if gated else None, scale=_row_scale(wl, k))


def test_dynamic_equals_shared_filter_path():
    """Every row carrying its channel's filter gives the shared-filter forward's result."""
    from fft_long_convolution_causal_b200 import binding
    wl = wlmod.make_1d(4, 3, 1024, dtype="f32", seed=5, with_D=True)
    plan = binding.Plan(4, 3, 1024, "f32")
    khat = plan.kernel_spectrum(torch.from_numpy(wl.k).cuda())
    u, D = to_dev(wl.u, "f32"), torch.from_numpy(wl.D).cuda()
    y_shared = plan.fwd(u, khat, D=D)
    kk = torch.from_numpy(np.broadcast_to(wl.k[None], (4, 3, 1024)).copy()).cuda()
    y_dyn = plan.fwd_dynamic(u, kk, D=D)
    torch.cuda.synchronize()
    assert_close(to_host(y_dyn), to_host(y_shared).astype(np.float64), "f32", "dynamic vs shared")


def test_dynamic_refuses_long_sequences():
    from fft_long_convolution_causal_b200 import binding
    plan = binding.Plan(2, 1, 8192, "f32")
    u = torch.zeros(2, 1, 8192, device="cuda")
    with pytest.raises(binding.FFTConvError) as e:
        plan.fwd_dynamic(u, torch.zeros(2, 1, 8192, device="cuda"))
    assert e.value.status == 2


def _filters_2d(B, C, Kh, Kw, sigma, seed):
    """Per-image filters k[b,c,p,q] = N(0,1) exp(-(p^2 + q^2) / (2 sigma^2))."""
    r = np.random.default_rng(seed)
    p = np.arange(Kh, dtype=np.float64)[:, None]
    q = np.arange(Kw, dtype=np.float64)[None, :]
    win = np.exp(-(p * p + q * q) / (2.0 * sigma * sigma))
    return (r.standard_normal((B, C, Kh, Kw)) * win[None, None]).astype(np.float32)


def _scale_2d(u, k, b_idx=None, c_idx=None):
    """Per-image scale RMS(u[b, c]) * ||k[b, c]|| (the 2-D analogue of the row scale)."""
    s = np.sqrt(np.mean(u.astype(np.float64) ** 2, axis=(2, 3))) * np.sqrt(
        np.sum(k.astype(np.float64) ** 2, axis=(2, 3)))
    if b_idx is None:
        return np.broadcast_to(s[:, :, None, None], u.shape)
    return s[b_idx, c_idx]


@pytest.mark.parametrize("B,C,Hs,Ws,dtype,Kh,Kw", [
    (3, 2, 16, 16, "f32", 16, 16), (2, 3, 64, 32, "bf16", 40, 9), (1, 2, 128, 128, "f32", 128, 128),
    (3, 2, 256, 64, "bf16", 100, 64), (2, 2, 256, 256, "bf16", 256, 256)])
def test_dynamic_2d_full_compare(B, C, Hs, Ws, dtype, Kh, Kw):
    """One filter per image (fftconv2d_fwd_dynamic): the SIMT passes and the
    tensor-core passes (256 rows, bf16), odd and even B; every output
    compared with the oracle's per-image convolution."""
    from fft_long_convolution_causal_b200 import binding
    wl = wlmod.make_2d(B, C, Hs, Ws, dtype=dtype, seed=Hs + 3 * Ws + B, sigma=Hs / 4)
    k = _filters_2d(B, C, Kh, Kw, Hs / 4, seed=Hs * 7 + C)
    plan = binding.Plan2DDynamic(B, C, Hs, Ws, dtype)
    y = to_host(plan.fwd(to_dev(wl.u, dtype), torch.from_numpy(k).cuda()))
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    want = oracle.causal_conv2d_dynamic(wl.u, k)
    assert_close(y, want, dtype, f"2d dynamic B={B} C={C} {Hs}x{Ws} {dtype} k{Kh}x{Kw}", scale=_scale_2d(wl.u, k))


def test_dynamic_2d_filters_differ_per_image():
    """Two images of one channel with different filters: each output follows
    its own filter (a path that shared one filter per channel would fail)."""
    from fft_long_convolution_causal_b200 import binding
    wl = wlmod.make_2d(2, 1, 64, 64, dtype="f32", seed=5, sigma=16.0)
    k = _filters_2d(2, 1, 8, 8, 16.0, seed=6)
    k[1] *= -3.0
    y = to_host(binding.Plan2DDynamic(2, 1, 64, 64, "f32").fwd(to_dev(wl.u, "f32"), torch.from_numpy(k).cuda()))
    want = oracle.causal_conv2d_dynamic(wl.u, k)
    assert_close(y, want, "f32", "2d dynamic, different filters", scale=_scale_2d(wl.u, k))
    shared = oracle.causal_conv2d(wl.u, k[0])
    assert np.max(np.abs(y[1] - shared[1])) > 1.0


def test_dynamic_2d_sampled_at_named_size():
    """Per-image filters at the 2-D workload's image size (256 x 256 bf16,
    full-size filters), 2048 sampled pixels against the oracle."""
    from fft_long_convolution_causal_b200 import binding
    B, C = 4, 6
    wl = wlmod.make_2d(B, C, 256, 256, dtype="bf16", seed=41, sigma=64.0)
    k = _filters_2d(B, C, 256, 256, 64.0, seed=42)
    y = to_host(binding.Plan2DDynamic(B, C, 256, 256, "bf16").fwd(to_dev(wl.u, "bf16"), torch.from_numpy(k).cuda()))
    idx = wlmod.sample_points_2d(B, C, 256, 256, 2048, seed=43)
    ref = oracle.causal_conv2d_dynamic_points(wl.u, k, *idx)
    assert_close(y[idx], ref, "bf16", "2d dynamic 256x256 sampled", scale=_scale_2d(wl.u, k, idx[0], idx[1]))


def test_dynamic_2d_rejects_other_plans():
    from fft_long_convolution_causal_b200 import binding
    plan = binding.Plan2D(2, 2, 16, 16, "f32")
    lib = binding.load_library()
    u = torch.zeros(2, 2, 16, 16, device="cuda")
    k = torch.zeros(2, 2, 4, 4, device="cuda")
    ws = plan.new_workspace()
    st = lib.fftconv2d_fwd_dynamic(plan._handle, u.data_ptr(), k.data_ptr(), 4, 4, torch.empty_like(u).data_ptr(),
                                   ws.data_ptr() if ws is not None else None, None)
    assert st == 1  # FFTCONV_ERR_INVALID_ARG: not a plan with one filter per image
