"""Metamorphic checks on the GPU that need no oracle, at full sequence length:
the delta filter returns its input, and delaying the input by s delays the
output by s (the convolution is shift-invariant and causal).  They follow
from the defining formula, "FlashFFTConv: Efficient Convolutions for Long
Sequences with Tensor Cores" (abstract: the FFT convolution of a sequence
with a long filter), with zero padding keeping it causal ("RubiConv", Caracal
abstract)."""
import pytest
import torch

from fft_long_convolution_causal_b200 import binding

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = {"f32": 1e-5, "bf16": 2e-2}


def _rel(a, b):
    a, b = a.double(), b.double()
    return (torch.linalg.vector_norm(a - b) / torch.linalg.vector_norm(b)).item()


CASES = [
    (1, 2, 1 << 20, "f32", False, "multipass"),
    (3, 8, 4096, "bf16", False, "fused_t2"),
    (2, 4, 16384, "bf16", True, "fused_tc"),
    (2, 3, 1 << 16, "bf16", False, "multipass"),
]


def _inputs(B, H, N, dtype, gated, seed):
    td = binding.TORCH_DTYPES[dtype]
    g = torch.Generator().manual_seed(seed)
    u = torch.randn(B, H, N, generator=g).to(td).to(DEV)
    v = torch.randn(B, H, N, generator=g).to(td).to(DEV) if gated else None
    w = torch.randn(B, H, N, generator=g).to(td).to(DEV) if gated else None
    return u, v, w


@pytest.mark.parametrize("B,H,N,dtype,gated,path", CASES)
def test_delta_filter_returns_the_input(B, H, N, dtype, gated, path):
    plan = binding.Plan(B, H, N, dtype, gated=gated)
    assert plan.path == path
    u, v, w = _inputs(B, H, N, dtype, gated, 21)
    k = torch.zeros(H, N, device=DEV)
    k[:, 0] = 1.0
    y = plan.fwd(u, plan.kernel_spectrum(k), v=v, w=w)
    x = u.double() * w.double() if gated else u.double()
    want = v.double() * x if gated else x
    assert _rel(y, want) <= TOL[dtype]
    assert plan.device_status() == 0


@pytest.mark.parametrize("B,H,N,dtype,gated,path", CASES)
def test_delayed_input_gives_delayed_output(B, H, N, dtype, gated, path):
    plan = binding.Plan(B, H, N, dtype, gated=gated)
    assert plan.path == path
    u, v, w = _inputs(B, H, N, dtype, gated, 22)
    g = torch.Generator().manual_seed(23)
    decay = torch.exp(-torch.arange(N, dtype=torch.float32) / (N / 8))
    k = (torch.randn(H, N, generator=g) * decay / (N ** 0.5)).to(DEV)
    D = torch.randn(H, generator=g).to(DEV)
    kh = plan.kernel_spectrum(k)
    s = N // 8 + 3
    y = plan.fwd(u, kh, D=D, v=v, w=w).double()
    us = torch.zeros_like(u)
    us[..., s:] = u[..., :N - s]
    if gated:
        # delay the whole layer input: x = u w and the gate v move together
        vs, ws = torch.zeros_like(v), torch.zeros_like(w)
        vs[..., s:] = v[..., :N - s]
        ws[..., s:] = w[..., :N - s]
    else:
        vs = ws = None
    ys = plan.fwd(us, kh, D=D, v=vs, w=ws).double()
    assert _rel(ys[..., s:], y[..., :N - s]) <= TOL[dtype]
    # before the delay the output is zero up to the transform's rounding: its
    # RMS within the path's tolerance of the output's, no value far beyond it
    rms = y.pow(2).mean().sqrt().item()
    head = ys[..., :s]
    assert head.pow(2).mean().sqrt().item() <= TOL[dtype] * rms
    assert head.abs().max().item() <= 8 * TOL[dtype] * rms
    assert plan.device_status() == 0
