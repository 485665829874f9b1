"""fftconv_fwd_static_workspace: the forward for callers that cannot allocate.

Callers that may not call cudaMalloc while they convolve (allocation forbidden
or too costly at that point, or all device memory owned by another pool) use
this entry point; its scratch is a fixed device array inside the library.  It
must give the same result as fftconv_fwd with a caller workspace.  The test
calls it twice in a row on different inputs (the array keeps the previous
call's contents, which must not leak into the next result) and compares each
call with fftconv_fwd on the same input, within the parity tolerance, and the
first call also with the fp64 oracle on sampled outputs.  One case has more
row pairs than the static array holds at once and a short last group (10
pairs of 2 MiB in groups of 8), a split that only this entry point makes.

The file is named to be collected last, and it needs nothing from the other
tests, so it passes alone in a fresh process as well as after them.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from fft_long_convolution_causal_b200 import workloads as wlmod
from parity import assert_close, row_scale_1d, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_causal_b200 import binding
    return binding.load_library()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("N,dtype,gated,B,H", [(1 << 16, "f32", False, 3, 2), (1 << 15, "bf16", True, 3, 2),
                                               (1 << 20, "f32", False, 3, 2), (1 << 17, "f32", False, 3, 5)])
def test_static_workspace_matches_fftconv_fwd(lib, N, dtype, gated, B, H):
    from fft_long_convolution_causal_b200 import binding
    plan = binding.Plan(B, H, N, dtype, gated=gated)
    assert plan.path == "multipass"
    first = wlmod.make_1d(B, H, N, dtype=dtype, gated=gated, seed=N, alpha=1e-4)
    khat = plan.kernel_spectrum(torch.from_numpy(first.k).cuda())
    D = torch.from_numpy(first.D).cuda()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((N + 1, N + 2)):
        wl = wlmod.make_1d(B, H, N, dtype=dtype, gated=gated, seed=seed, alpha=1e-4)
        wl.k, wl.D = first.k, first.D  # same filters: the cached spectrum stays valid
        u, v, w = to_dev(wl.u, dtype), to_dev(wl.v, dtype), to_dev(wl.w, dtype)
        y_ref = plan.fwd(u, khat, D=D, v=v, w=w)
        y = torch.full_like(y_ref, float("nan"))
        st = lib.fftconv_fwd_static_workspace(plan._handle, _p(u), _p(v), _p(w), _p(khat), _p(D), _p(y), stream)
        assert st == 0, binding.status_string(st)
        torch.cuda.synchronize()
        a, b = to_host(y), to_host(y_ref)
        assert np.all(np.isfinite(a)), f"call {call}: unwritten outputs"
        assert_close(a, b, dtype, f"static workspace call {call} N={N} {dtype}",
                     gate=wl.v if gated else None, scale=row_scale_1d(wl))
        if call == 0:
            bi, hi, ti = wlmod.sample_points_1d(B, H, N, 48, seed=N)
            ref = oracle.causal_conv1d_points(wl.u, wl.k, bi, hi, ti, D=wl.D, w=wl.w, v=wl.v)
            assert_close(a[bi, hi, ti], ref, dtype, f"static workspace vs oracle N={N} {dtype}",
                         gate=wl.v[bi, hi, ti] if gated else None, scale=row_scale_1d(wl, bi, hi))


def test_static_workspace_rejects_non_multipass_plans(lib):
    from fft_long_convolution_causal_b200 import binding
    plan = binding.Plan(2, 2, 4096, "f32")
    assert plan.path == "fused"
    k = torch.randn(2, 4096, device="cuda")
    khat = plan.kernel_spectrum(k)
    u = torch.randn(2, 2, 4096, device="cuda")
    y = torch.empty_like(u)
    st = lib.fftconv_fwd_static_workspace(plan._handle, _p(u), None, None, _p(khat), None, _p(y), None)
    assert st == 2  # FFTCONV_ERR_UNSUPPORTED
    assert lib.fftconv_static_workspace_bytes() == 16 << 20
