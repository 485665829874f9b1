"""Degenerate inputs on every path family: a zero input, or a zero filter with
no skip term, gives exactly zero at every output.

The transforms are linear, so the exact result is 0; any nonzero or NaN
output would come from storage the kernel did not write this call (shared or
tensor memory, a workspace, a stale spectrum).  The outputs are first filled
with a nonzero pattern so that an output the kernel skipped also shows.
"""
import pytest
import torch

from fft_long_convolution_causal_b200 import binding

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _poison(y):
    y.fill_(3.0)
    return y


def _zero(y):
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0, f"{torch.count_nonzero(y).item()} nonzero outputs"


@pytest.mark.parametrize("B,H,N,dtype,gated,path", [
    (3, 5, 4096, "bf16", False, "fused_t2"),
    (2, 3, 16384, "bf16", True, "fused_tc"),
    (3, 2, 1024, "f32", False, "fused"),
    (3, 2, 1 << 16, "f32", True, "multipass"),
])
def test_1d_zero_input_and_zero_filter(B, H, N, dtype, gated, path):
    plan = binding.Plan(B, H, N, dtype, gated=gated)
    assert plan.path == path
    td = binding.TORCH_DTYPES[dtype]
    g = torch.Generator().manual_seed(N + B)
    rnd = lambda *s: torch.randn(*s, generator=g).to(td).to(DEV)  # noqa: E731
    u, v, w = rnd(B, H, N), (rnd(B, H, N) if gated else None), (rnd(B, H, N) if gated else None)
    D = torch.randn(H, generator=g).to(DEV)
    kh = plan.kernel_spectrum(torch.randn(H, N, generator=g).to(DEV) * 0.02)
    y = torch.empty(B, H, N, dtype=td, device=DEV)
    # zero input (the skip term D u is zero too)
    plan.fwd(torch.zeros_like(u), kh, D=D, v=v, w=w, y=_poison(y))
    _zero(y)
    # zero filter, no skip term
    kz = plan.kernel_spectrum(torch.zeros(H, N, device=DEV))
    plan.fwd(u, kz, v=v, w=w, y=_poison(y))
    _zero(y)
    assert plan.device_status() == 0


def test_2d_zero_input_and_zero_filter():
    plan = binding.Plan2D(2, 2, 256, 256, "bf16")
    assert plan.path == "2d_tc"
    g = torch.Generator().manual_seed(11)
    u = torch.randn(2, 2, 256, 256, generator=g).to(torch.bfloat16).to(DEV)
    kh = plan.kernel_spectrum(torch.randn(2, 256, 256, generator=g).to(DEV) * 0.01)
    y = torch.empty_like(u)
    plan.fwd(torch.zeros_like(u), kh, y=_poison(y))
    _zero(y)
    kz = plan.kernel_spectrum(torch.zeros(2, 256, 256, device=DEV))
    plan.fwd(u, kz, y=_poison(y))
    _zero(y)


def test_3d_zero_input_and_zero_filter():
    plan = binding.Plan3D(2, 2, 16, 32, 16, "f32")
    g = torch.Generator().manual_seed(12)
    u = torch.randn(2, 2, 16, 32, 16, generator=g).to(DEV)
    kh = plan.kernel_spectrum(torch.randn(2, 16, 32, 16, generator=g).to(DEV))
    y = torch.empty_like(u)
    plan.fwd(torch.zeros_like(u), kh, y=_poison(y))
    _zero(y)
    kz = plan.kernel_spectrum(torch.zeros(2, 16, 32, 16, device=DEV))
    plan.fwd(u, kz, y=_poison(y))
    _zero(y)


@pytest.mark.parametrize("dtype,chunk", [("f32", 8192), ("bf16", 4096)])
def test_state_passing_zero_input_and_zero_filter(dtype, chunk):
    B, H, N, d = 2, 2, 32768, 4
    plan = binding.SSMPlan(B, H, N, dtype, d_state=d, chunk=chunk)
    td = binding.TORCH_DTYPES[dtype]
    g = torch.Generator().manual_seed(13)
    lam = torch.polar(1.0 - torch.rand(H, d, generator=g) * 1e-2, torch.rand(H, d, generator=g) * 0.2)
    c = torch.complex(torch.randn(H, d, generator=g), torch.randn(H, d, generator=g)) * 0.1
    u = torch.randn(B, H, N, generator=g).to(td).to(DEV)
    D = torch.randn(H, generator=g).to(DEV)
    y = torch.empty_like(u)
    kh = plan.set_filters(lam, c)
    plan.fwd(torch.zeros_like(u), kh, D=D, y=_poison(y))
    _zero(y)
    # c = 0: every filter tap is zero, and so is the state carried between chunks
    kz = plan.set_filters(lam, torch.zeros_like(c))
    plan.fwd(u, kz, y=_poison(y))
    _zero(y)
