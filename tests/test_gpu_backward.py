"""GPU parity of the backward pass (gradients du, dv, dw, dk, dD) through the
C ABI against the fp64 oracle's chain-rule gradients.

The data gradient runs through the plan's own forward kernel with the
conjugated spectrum, so every forward path is exercised (fp32 fused, bf16
tensor-core kernels, the two-stage tcgen05 kernel, multi-pass); the filter
gradient through the fp32 pair-transform kernel (N <= 8192)."""
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


def run_bwd(wl, dy, filter_grad=True, **plan_kw):
    from fft_long_convolution_causal_b200 import binding
    plan = binding.Plan(wl.B, wl.H, wl.N, wl.dtype, gated=wl.gated, **plan_kw)
    khat = plan.kernel_spectrum(torch.from_numpy(wl.k).cuda())
    kc = plan.spectrum_conjugate(khat)
    D = torch.from_numpy(wl.D).cuda() if wl.D is not None else None
    g = plan.bwd(to_dev(dy, wl.dtype), to_dev(wl.u, wl.dtype), khat, kc, D=D, v=to_dev(wl.v, wl.dtype),
                 w=to_dev(wl.w, wl.dtype), L=wl.L, filter_grad=filter_grad)
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    return {k: (None if v is None else to_host(v)) for k, v in g.items()}, plan


def _row_scale(wl, a):
    """(||k_h||_2 + |D_h|) RMS(a_{b,h}) per element: the expected RMS of a
    convolution (or correlation) of the row a with the channel's filter, the
    per-row scale of the per-element bound (as for the forward outputs)."""
    knorm = np.sqrt(np.sum(wl.k.astype(np.float64) ** 2, axis=1))
    if wl.D is not None:
        knorm = knorm + np.abs(wl.D.astype(np.float64))
    a = np.asarray(a, dtype=np.float64)
    return np.broadcast_to((np.sqrt(np.mean(a * a, axis=2)) * knorm[None, :])[:, :, None], a.shape)


def check(wl, dy, got, what, filter_grad=True):
    """Each gradient against the oracle with the forward's tolerance rule: its
    own row scale (the filter applied to g = dy v for du and dw, to x = u w for
    dv) and the gate factor of the elementwise product it ends with (w for du,
    u for dw, dy for dv)."""
    want = oracle.causal_conv1d_bwd(wl.u, wl.k, dy, D=wl.D, w=wl.w, v=wl.v)
    g = dy * wl.v if wl.gated else dy
    x = wl.u * wl.w if wl.gated else wl.u
    assert_close(got["du"], want["du"], wl.dtype, f"{what} du", gate=wl.w if wl.gated else None,
                 scale=_row_scale(wl, g))
    if wl.gated:
        assert_close(got["dw"], want["dw"], wl.dtype, f"{what} dw", gate=wl.u, scale=_row_scale(wl, g))
        assert_close(got["dv"], want["dv"], wl.dtype, f"{what} dv", gate=dy, scale=_row_scale(wl, x))
    if filter_grad:
        # the filter gradient is an fp32 transform of the exact (widened) inputs
        assert_close(got["dk"], want["dk"], "f32", f"{what} dk")
        if wl.D is not None:
            assert_close(got["dD"], want["dD"], "f32", f"{what} dD")


def _dy(wl, seed):
    a = np.random.default_rng(seed).standard_normal(wl.u.shape, dtype=np.float32)
    return wlmod.round_bf16(a) if wl.dtype == "bf16" else a


@pytest.mark.parametrize("N,dtype,gated,with_D,L", [
    (64, "f32", False, True, None), (1024, "f32", False, True, 300), (1024, "f32", True, True, None),
    (8192, "f32", False, False, None), (4096, "bf16", False, True, None), (4096, "bf16", True, True, 1000),
    (2048, "bf16", True, False, None), (8192, "bf16", False, True, None), (512, "bf16", True, True, None)])
def test_backward_full_compare(N, dtype, gated, with_D, L):
    wl = wlmod.make_1d(3, 2, N, dtype=dtype, gated=gated, seed=N + 7 * gated, with_D=with_D, L=L)
    dy = _dy(wl, N + 1)
    got, plan = run_bwd(wl, dy)
    check(wl, dy, got, f"bwd N={N} {dtype} gated={gated} D={with_D} L={L} ({plan.path})")


@pytest.mark.parametrize("kernel", ["tcgen05", "mma_sync", "simt"])
def test_backward_every_forward_kernel(kernel):
    """The data gradient through each forward kernel family at 2N = 8192."""
    wl = wlmod.make_1d(4, 3, 4096, dtype="bf16", gated=False, seed=71, with_D=True)
    dy = _dy(wl, 72)
    got, plan = run_bwd(wl, dy, kernel=kernel)
    check(wl, dy, got, f"bwd kernel={kernel} ({plan.path})")


def test_backward_multipass_data_gradient():
    """N = 32768 (multi-pass forward): du through the conjugated spectrum;
    the filter gradient is unsupported there and refused with status 2."""
    from fft_long_convolution_causal_b200 import binding
    wl = wlmod.make_1d(3, 2, 32768, dtype="f32", gated=False, seed=73, with_D=True, alpha=1e-4)
    dy = _dy(wl, 74)
    got, plan = run_bwd(wl, dy, filter_grad=False)
    assert plan.path == "multipass"
    want = oracle.causal_conv1d_bwd(wl.u, wl.k, dy, D=wl.D)
    assert_close(got["du"], want["du"], "f32", "bwd multipass du")
    with pytest.raises(binding.FFTConvError) as e:
        run_bwd(wl, dy, filter_grad=True)
    assert e.value.status == 2


def test_conjugate_twice_is_identity():
    from fft_long_convolution_causal_b200 import binding
    for N, dtype, kernel in ((1024, "f32", "auto"), (4096, "bf16", "mma_sync"), (4096, "bf16", "tcgen05"),
                             (1 << 15, "f32", "auto")):
        plan = binding.Plan(2, 3, N, dtype, kernel=kernel)
        khat = plan.kernel_spectrum(torch.randn(3, N, device="cuda"))
        back = plan.spectrum_conjugate(plan.spectrum_conjugate(khat))
        torch.cuda.synchronize()
        assert torch.equal(back, khat), plan.path
