"""GPU parity of the partial-convolution path (filters much shorter than the
rows, overlap-save in chunks on chip) through the C ABI against the fp64
oracle's direct causal sum with the short filter."""
import numpy as np
import pytest
import torch

import oracle
from fft_long_convolution_causal_b200 import workloads as wlmod
from parity import assert_close, row_scale_1d, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_causal_b200 import binding
    binding.load_library()


def run(wl, L_max=None):
    from fft_long_convolution_causal_b200 import binding
    plan = binding.PartialPlan(wl.B, wl.H, wl.N, wl.dtype, gated=wl.gated, L_max=L_max or wl.L)
    assert plan.path == "partial_chunked"
    khat = plan.kernel_spectrum(torch.from_numpy(wl.k).cuda())
    D = torch.from_numpy(wl.D).cuda() if wl.D is not None else None
    y = plan.fwd(to_dev(wl.u, wl.dtype), khat, D=D, v=to_dev(wl.v, wl.dtype), w=to_dev(wl.w, wl.dtype))
    torch.cuda.synchronize()
    return to_host(y)


@pytest.mark.parametrize("B,H,N,L,dtype,gated,with_D", [
    (3, 2, 4096, 100, "f32", False, True), (2, 3, 65536, 1000, "f32", True, True),
    (1, 2, 16384, 8192, "f32", False, False), (4, 2, 8192, 64, "bf16", True, False),
    (5, 1, 32768, 2048, "bf16", False, True)])
def test_partial_full_compare(B, H, N, L, dtype, gated, with_D):
    wl = wlmod.make_1d(B, H, N, dtype=dtype, gated=gated, seed=N + L, with_D=with_D, L=L)
    y = run(wl)
    want = oracle.causal_conv1d(wl.u, wl.k, D=wl.D, w=wl.w, v=wl.v)
    assert_close(y, want, dtype, f"partial B={B} H={H} N={N} L={L} {dtype} gated={gated}",
                 gate=wl.v if gated else None, scale=row_scale_1d(wl))


def test_partial_long_rows_sampled():
    """N = 2^20 with a 4096-tap filter (256 chunks per row), sampled outputs."""
    wl = wlmod.make_1d(2, 4, 1 << 20, dtype="f32", seed=91, L=4096, alpha=1e-3)
    y = run(wl)
    b, h, t = wlmod.sample_points_1d(wl.B, wl.H, wl.N, 128, seed=91)
    want = oracle.causal_conv1d_points(wl.u, wl.k, b, h, t, D=wl.D)
    assert_close(y[b, h, t], want, "f32", "partial N=2^20 L=4096", scale=row_scale_1d(wl, b, h))


def test_partial_rejects_long_filters():
    from fft_long_convolution_causal_b200 import binding
    plan = binding.PartialPlan(2, 2, 4096, "f32", L_max=300)   # chunk 512
    with pytest.raises(binding.FFTConvError):
        plan.kernel_spectrum(torch.zeros(2, 600, device="cuda"))
    with pytest.raises(binding.FFTConvError):
        binding.PartialPlan(2, 2, 4096, "f32", L_max=10000)      # chunk above the on-chip limit
