"""CUDA graph capture of every forward path family and of the backward pass.

The entry points enqueue only kernel launches on the caller's stream (the
one-time per-process launch set-up happens on the first eager call), so a
captured call must replay to the same bytes as the eager call, and must read
the buffers it was given at capture time: the tests overwrite the outputs
before each replay (a replay that wrote nothing would fail) and change the
inputs in place between replays (a graph that had kept a copy would fail).
Eager results themselves are checked against the oracle by the parity tests.
"""
import pytest
import torch

from fft_long_convolution_causal_b200 import binding

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _rand(shape, dtype, g, scale=1.0):
    return (torch.randn(*shape, generator=g) * scale).to(dtype).to(DEV)


def _check_graph(inputs, run):
    """run() writes into preallocated outputs and returns them (a tuple)."""
    eager = [t.clone() for t in run()]
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        outs = run()
    for o in outs:
        o.zero_()
    gr.replay()
    torch.cuda.synchronize()
    for o, e in zip(outs, eager):
        assert torch.equal(o, e)
    # new input values in the same buffers: the replay follows them
    g = torch.Generator().manual_seed(99)
    for t in inputs:
        t.copy_(torch.randn(*t.shape, generator=g).to(t.dtype))
    fresh = [t.clone() for t in run()]
    torch.cuda.synchronize()
    assert any(not torch.equal(f, e) for f, e in zip(fresh, eager))
    for o in outs:
        o.zero_()
    gr.replay()
    torch.cuda.synchronize()
    for o, f in zip(outs, fresh):
        assert torch.equal(o, f)
    del gr


@pytest.mark.parametrize("B,H,N,dtype,gated,path", [
    (3, 40, 4096, "bf16", False, "fused_t2"),
    (2, 8, 16384, "bf16", True, "fused_tc"),
    (2, 4, 1024, "f32", False, "fused"),
    (2, 2, 1 << 16, "f32", False, "multipass"),
])
def test_graph_1d(B, H, N, dtype, gated, path):
    plan = binding.Plan(B, H, N, dtype, gated=gated)
    assert plan.path == path
    g = torch.Generator().manual_seed(B * 131 + H)
    td = binding.TORCH_DTYPES[dtype]
    u = _rand((B, H, N), td, g)
    v = _rand((B, H, N), td, g) if gated else None
    w = _rand((B, H, N), td, g) if gated else None
    k = _rand((H, N), torch.float32, g, 0.02)
    D = _rand((H,), torch.float32, g)
    kh = plan.kernel_spectrum(k)
    y = torch.empty(B, H, N, dtype=td, device=DEV)
    _check_graph([u] + ([v, w] if gated else []), lambda: (plan.fwd(u, kh, D=D, v=v, w=w, y=y),))


def test_graph_2d_tensor_core():
    plan = binding.Plan2D(2, 2, 256, 256, "bf16")
    assert plan.path == "2d_tc"
    g = torch.Generator().manual_seed(5)
    u = _rand((2, 2, 256, 256), torch.bfloat16, g)
    kh = plan.kernel_spectrum(_rand((2, 256, 256), torch.float32, g, 0.01))
    y = torch.empty_like(u)
    _check_graph([u], lambda: (plan.fwd(u, kh, y=y),))


def test_graph_3d():
    plan = binding.Plan3D(1, 2, 16, 16, 16, "f32")
    g = torch.Generator().manual_seed(6)
    u = _rand((1, 2, 16, 16, 16), torch.float32, g)
    kh = plan.kernel_spectrum(_rand((2, 16, 16, 16), torch.float32, g, 0.05))
    y = torch.empty_like(u)
    _check_graph([u], lambda: (plan.fwd(u, kh, y=y),))


def test_graph_state_passing_bf16_chunks():
    B, H, N, d = 1, 2, 16384, 4
    plan = binding.SSMPlan(B, H, N, "bf16", d_state=d, chunk=4096)
    g = torch.Generator().manual_seed(7)
    lam = torch.polar(1.0 - torch.rand(H, d, generator=g) * 1e-2, torch.rand(H, d, generator=g) * 0.2)
    c = torch.complex(torch.randn(H, d, generator=g), torch.randn(H, d, generator=g)) * 0.1
    kh = plan.set_filters(lam, c)
    u = _rand((B, H, N), torch.bfloat16, g)
    D = _rand((H,), torch.float32, g)
    y = torch.empty_like(u)
    _check_graph([u], lambda: (plan.fwd(u, kh, D=D, y=y),))


def test_graph_backward():
    B, H, N = 2, 4, 4096
    plan = binding.Plan(B, H, N, "bf16")
    g = torch.Generator().manual_seed(8)
    u = _rand((B, H, N), torch.bfloat16, g)
    dy = _rand((B, H, N), torch.bfloat16, g)
    D = _rand((H,), torch.float32, g)
    kh = plan.kernel_spectrum(_rand((H, N), torch.float32, g, 0.02))
    khc = plan.spectrum_conjugate(kh)
    outs = {}

    def run():
        r = plan.bwd(dy, u, kh, khc, D=D)
        outs.update(r)
        return (r["du"], r["dk"], r["dD"])

    _check_graph([u, dy], run)
