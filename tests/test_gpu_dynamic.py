"""GPU parity of the forward with input-dependent filters (one per batch row,
transformed in the same launch) through the C ABI against the fp64 oracle."""
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
