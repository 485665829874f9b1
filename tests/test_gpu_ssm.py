"""GPU parity of the chunked state-passing path (filters of a diagonal
state-space model) through the C ABI against the fp64 oracle: the filter
k[h,t] = Re(sum_j c lam^t) materialised over the whole row in fp64, then
the direct causal sum."""
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


def ssm_params(H, d, seed, rmin=0.999, rmax=0.99999):
    """Slowly decaying complex poles (state carried across many chunks)."""
    r = np.random.default_rng(seed)
    lam = r.uniform(rmin, rmax, (H, d)) * np.exp(1j * r.uniform(-0.2, 0.2, (H, d)))
    c = (r.standard_normal((H, d)) + 1j * r.standard_normal((H, d))) / np.sqrt(d)
    # the GPU sees fp32 parameters: give the oracle exactly those values
    lam = lam.real.astype(np.float32) + 1j * lam.imag.astype(np.float32)
    c = c.real.astype(np.float32) + 1j * c.imag.astype(np.float32)
    return lam, c


def run(B, H, N, dtype, d, T, seed, with_D=True):
    from fft_long_convolution_causal_b200 import binding
    lam, c = ssm_params(H, d, seed)
    r = np.random.default_rng(seed + 1)
    u = r.standard_normal((B, H, N), dtype=np.float32)
    if dtype == "bf16":
        u = wlmod.round_bf16(u)
    D = r.standard_normal(H, dtype=np.float32) if with_D else None
    plan = binding.SSMPlan(B, H, N, dtype, d_state=d, chunk=T)
    assert plan.path == "ssm_chunked"
    khat = plan.set_filters(torch.from_numpy(lam), torch.from_numpy(c))
    y = plan.fwd(to_dev(u, dtype), khat, D=None if D is None else torch.from_numpy(D).cuda())
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    k = oracle.ssm_kernel(lam, c, N)
    wl = wlmod.Workload1D("ssm", B, H, N, dtype, False, u, k.astype(np.float32), D)
    return to_host(y), u, k, D, wl


@pytest.mark.parametrize("B,H,N,dtype,d,T", [(2, 3, 1024, "f32", 4, 256), (3, 2, 4096, "f32", 8, 4096),
                                             (1, 2, 16384, "bf16", 8, 1024), (2, 2, 8192, "f32", 64, 64)])
def test_ssm_full_compare(B, H, N, dtype, d, T):
    y, u, k, D, wl = run(B, H, N, dtype, d, T, seed=N + d)
    want = oracle.causal_conv1d(u, k, D=D)
    assert_close(y, want, dtype, f"ssm B={B} H={H} N={N} {dtype} d={d} T={T}", scale=row_scale_1d(wl))


@pytest.mark.parametrize("N,T,d", [(1 << 16, 8192, 16), (1 << 20, 8192, 16)])
def test_ssm_long_sampled(N, T, d):
    """Up to 2^20 (128 chunks of 8192): sampled outputs, uniform draws plus edges."""
    B, H = 2, 3
    y, u, k, D, wl = run(B, H, N, "f32", d, T, seed=d + T)
    b, h, t = wlmod.sample_points_1d(B, H, N, 64, seed=N)
    want = oracle.causal_conv1d_points(u, k, b, h, t, D=D)
    assert_close(y[b, h, t], want, "f32", f"ssm N={N} T={T} d={d}", scale=row_scale_1d(wl, b, h))


@pytest.mark.parametrize("B,H,N", [(3, 2, 16384), (2, 3, 4096)])
def test_ssm_bf16_tensor_core_chunks(B, H, N):
    """bf16 plans with chunks of 4096 run the chunk convolutions on the
    two-stage tcgen05 kernel (chunks of one channel share its spectrum); every
    output compared, odd B, a single chunk."""
    y, u, k, D, wl = run(B, H, N, "bf16", 16, 4096, seed=N + B)
    want = oracle.causal_conv1d(u, k, D=D)
    assert_close(y, want, "bf16", f"ssm bf16 tensor-core chunks B={B} H={H} N={N}", scale=row_scale_1d(wl))


def test_ssm_bf16_tensor_core_chunks_long():
    """2^20 bf16 (256 chunks of 4096 on the tensor cores), sampled outputs."""
    B, H, N = 2, 3, 1 << 20
    y, u, k, D, wl = run(B, H, N, "bf16", 16, 4096, seed=17)
    b, h, t = wlmod.sample_points_1d(B, H, N, 64, seed=N + 1)
    want = oracle.causal_conv1d_points(u, k, b, h, t, D=D)
    assert_close(y[b, h, t], want, "bf16", "ssm bf16 2^20 tensor-core chunks", scale=row_scale_1d(wl, b, h))


def test_ssm_rejects_bad_shapes():
    from fft_long_convolution_causal_b200 import binding
    for args in ((2, 2, 1000, "f32", 4, 256), (2, 2, 4096, "f32", 4, 16384), (2, 2, 4096, "f32", 0, 256),
                 (2, 2, 4096, "f32", 65, 256)):
        with pytest.raises(binding.FFTConvError):
            binding.SSMPlan(*args[:4], d_state=args[4], chunk=args[5])
