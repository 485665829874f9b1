"""GPU parity of frequency-sparse convolutions (multi-pass plans with spectrum
rows dropped by a block mask) through the C ABI against the fp64 oracle's
masked FFT formula; the dropped rows' work is skipped in all three passes."""
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


def symmetric_mask(G, frac, seed):
    """Keep flags over the outer frequency digit, keep[j] == keep[(G - j) % G]."""
    r = np.random.default_rng(seed)
    keep = np.ones(G, bool)
    for j in range(1, G // 2 + 1):
        if r.random() < frac:
            keep[j] = keep[(G - j) % G] = False
    return keep


@pytest.mark.parametrize("N,dtype,gated,frac", [(16384, "f32", False, 0.5), (32768, "f32", True, 0.75),
                                                (32768, "bf16", False, 0.25), (65536, "f32", False, 0.9)])
def test_sparse_full_compare(N, dtype, gated, frac):
    from fft_long_convolution_causal_b200 import binding
    wl = wlmod.make_1d(3, 2, N, dtype=dtype, gated=gated, seed=N + 3, with_D=True, alpha=1e-4)
    plan = binding.Plan(wl.B, wl.H, wl.N, dtype, gated=gated)
    assert plan.path == "multipass"
    G = plan.spectrum_blocks
    keep = symmetric_mask(G, frac, seed=N)
    khat = plan.kernel_spectrum(torch.from_numpy(wl.k).cuda())
    plan.sparsify(khat, keep)
    D = torch.from_numpy(wl.D).cuda()
    y = to_host(plan.fwd(to_dev(wl.u, dtype), khat, D=D, v=to_dev(wl.v, dtype), w=to_dev(wl.w, dtype)))
    x = wl.u * wl.w if gated else wl.u
    want = oracle.freq_sparse_conv1d(x, wl.k, keep, D=wl.D)
    if gated:
        want = want * wl.v
    # the masked output is a band-limited part of the full one: scale the bound by
    # the RMS of the masked reference row instead of the full filter's
    sc = np.broadcast_to(np.sqrt(np.mean(want ** 2, axis=2, keepdims=True)), want.shape)
    assert_close(y, want, dtype, f"sparse N={N} {dtype} gated={gated} frac={frac}", gate=wl.v if gated else None,
                 scale=sc)
    # a dense plan again (after recomputing the spectrum) gives the ordinary convolution
    plan.sparsify(khat, None)
    khat = plan.kernel_spectrum(torch.from_numpy(wl.k).cuda(), khat=khat)
    y2 = to_host(plan.fwd(to_dev(wl.u, dtype), khat, D=D, v=to_dev(wl.v, dtype), w=to_dev(wl.w, dtype)))
    b, h, t = wlmod.sample_points_1d(wl.B, wl.H, N, 32, seed=1)
    ref = oracle.causal_conv1d_points(wl.u, wl.k, b, h, t, D=wl.D, w=wl.w, v=wl.v)
    assert_close(y2[b, h, t], ref, dtype, "dense again", gate=None if wl.v is None else wl.v[b, h, t],
                 scale=row_scale_1d(wl, b, h))


def test_sparse_rejects_asymmetric_and_fused():
    from fft_long_convolution_causal_b200 import binding
    plan = binding.Plan(2, 1, 16384, "f32")
    khat = plan.kernel_spectrum(torch.randn(1, 16384, device="cuda"))
    keep = np.ones(plan.spectrum_blocks, bool)
    keep[1] = False  # its partner G - 1 kept: not Hermitian
    with pytest.raises(binding.FFTConvError) as e:
        plan.sparsify(khat, keep)
    assert e.value.status == 1
    fused = binding.Plan(2, 1, 4096, "f32")
    assert fused.spectrum_blocks == 0
    with pytest.raises(binding.FFTConvError) as e:
        fused.sparsify(fused.kernel_spectrum(torch.randn(1, 4096, device="cuda")), [True] * 8)
    assert e.value.status == 2
