"""GPU parity: the CUDA path (through the C ABI) against the CPU fp64 oracle.

Small sizes are compared element by element over the whole output; the five
named workloads run at full size in the launch configuration bench.py times
and are compared on seeded samples of outputs that the oracle computes one by
one, plus properties that hold at any size.
"""
import numpy as np
import pytest
import scipy.signal
import torch

import oracle
from fft_long_convolution_causal_b200 import workloads as wlmod
from parity import assert_close, row_scale_1d, row_scale_2d, to_dev, to_host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_causal_b200 import binding
    binding.load_library()


def run_1d(wl, **plan_kw):
    """One forward through the C ABI; returns (y, plan).  The device status
    word of the plan that launched is read (and must be clear) after the
    launch, so every parity case also checks that no bounded device wait of
    its kernel gave up."""
    from fft_long_convolution_causal_b200 import binding
    plan = binding.Plan(wl.B, wl.H, wl.N, wl.dtype, gated=wl.gated, **plan_kw)
    k = torch.from_numpy(wl.k).cuda()
    khat = plan.kernel_spectrum(k)
    u = to_dev(wl.u, wl.dtype)
    v = to_dev(wl.v, wl.dtype)
    w = to_dev(wl.w, wl.dtype)
    D = torch.from_numpy(wl.D).cuda() if wl.D is not None else None
    y = plan.fwd(u, khat, D=D, v=v, w=w)
    torch.cuda.synchronize()
    assert plan.device_status() == 0, f"{plan.path}: a bounded device wait gave up"
    return to_host(y), plan


def oracle_full(wl):
    return oracle.causal_conv1d(wl.u, wl.k, D=wl.D, w=wl.w, v=wl.v)


# ------------------------------------------------------------- small, full
FUSED_N = [64, 128, 256, 512, 1024, 2048, 4096, 8192]


@pytest.mark.parametrize("N", FUSED_N)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fused_full_compare(N, dtype):
    wl = wlmod.make_1d(3, 2, N, dtype=dtype, gated=False, seed=N, kernel="decay")
    y, plan = run_1d(wl)
    want = "fused_tc" if (dtype == "bf16" and 2048 <= N <= 16384) else "fused"
    if dtype == "bf16" and N == 4096:
        want = "fused_t2"  # the two-stage tcgen05 kernel is the default at 2N = 8192
    assert plan.path == want
    assert_close(y, oracle_full(wl), dtype, f"fused N={N} {dtype}", scale=row_scale_1d(wl))


@pytest.mark.parametrize("N", [256, 4096, 8192])
def test_fused_gated_full_compare(N):
    wl = wlmod.make_1d(3, 3, N, dtype="bf16", gated=True, seed=7 + N, with_D=True)
    y, _ = run_1d(wl)
    assert_close(y, oracle_full(wl), "bf16", f"fused gated N={N}", gate=wl.v, scale=row_scale_1d(wl))
    wl = wlmod.make_1d(2, 2, N, dtype="f32", gated=True, seed=8 + N, with_D=False)
    y, _ = run_1d(wl)
    assert_close(y, oracle_full(wl), "f32", f"fused gated f32 N={N}", gate=wl.v, scale=row_scale_1d(wl))


@pytest.mark.parametrize("N,L", [(1024, 1), (1024, 100), (4096, 4095), (32768, 777), (65536, 40000)])
def test_partial_kernel(N, L):
    """k shorter than the sequence (a partial convolution): taps past L are zero."""
    wl = wlmod.make_1d(2, 2, N, dtype="f32", seed=L, L=L, kernel="normal")
    y, _ = run_1d(wl)
    if N <= 32768:
        ref = oracle_full(wl)
        assert_close(y, ref, "f32", f"partial N={N} L={L}", scale=row_scale_1d(wl))
    else:
        b, h, t = wlmod.sample_points_1d(wl.B, wl.H, N, 256, seed=L)
        ref = oracle.causal_conv1d_points(wl.u, wl.k, b, h, t, D=wl.D)
        assert_close(y[b, h, t], ref, "f32", f"partial N={N} L={L}", scale=row_scale_1d(wl, b, h))


@pytest.mark.parametrize("N", [2048, 4096, 8192, 16384])
@pytest.mark.parametrize("B,gated,with_D,L", [(1, False, True, None), (5, True, True, None),
                                             (2, False, False, 333), (3, True, False, None)])
def test_tensor_core_path(N, B, gated, with_D, L):
    """bf16 tensor-core fused kernel: odd/even/single batch, gate, skip term, partial kernel."""
    wl = wlmod.make_1d(B, 3, N, dtype="bf16", gated=gated, seed=N + B, with_D=with_D, L=L)
    y, plan = run_1d(wl, kernel="mma_sync")
    assert plan.path == "fused_tc"
    assert_close(y, oracle_full(wl), "bf16", f"tc N={N} B={B} gated={gated} D={with_D} L={L}",
                 gate=wl.v if gated else None, scale=row_scale_1d(wl))


@pytest.mark.parametrize("N", [2048, 4096])
@pytest.mark.parametrize("B,gated,with_D,L", [(1, False, True, None), (5, True, True, None),
                                             (2, False, False, 333), (3, True, False, None), (8, False, True, None)])
def test_tcgen05_path(N, B, gated, with_D, L):
    """bf16 fused kernels on tcgen05 (plan option kernel="tcgen05"): the
    two-stage kernel for 2N = 8192 ungated, else the kernel with the mma.sync
    kernel's factorisation; same cases as the mma.sync kernel.  run_1d checks
    the status word of the plan that launched."""
    wl = wlmod.make_1d(B, 5, N, dtype="bf16", gated=gated, seed=3 * N + B, with_D=with_D, L=L)
    y, plan = run_1d(wl, kernel="tcgen05")
    assert plan.path == ("fused_t2" if (N == 4096 and not gated) else "fused_umma")
    assert_close(y, oracle_full(wl), "bf16", f"umma N={N} B={B} gated={gated} D={with_D} L={L}",
                 gate=wl.v if gated else None, scale=row_scale_1d(wl))


@pytest.mark.parametrize("B,H,with_D,L", [(1, 3, True, None), (3, 4, True, None), (6, 5, False, None),
                                         (7, 2, True, 1000), (4, 300, True, None), (2, 1, False, 1)])
def test_two_stage_kernel(B, H, with_D, L):
    """The two-stage tcgen05 kernel (2N = 8192): a missing last row (odd B),
    CTAs whose second slot has no pair (few pairs), many pairs per slot
    (H = 300), partial kernels, no skip term; every output compared."""
    wl = wlmod.make_1d(B, H, 4096, dtype="bf16", gated=False, seed=17 * B + H, with_D=with_D, L=L)
    y, plan = run_1d(wl, kernel="tcgen05")
    assert plan.path == "fused_t2"
    assert_close(y, oracle_full(wl), "bf16", f"t2 B={B} H={H} D={with_D} L={L}", scale=row_scale_1d(wl))


def test_two_stage_kernel_named_full():
    """The Hyena-style workload through the two-stage kernel, every output."""
    wl = _named("hyena_b8_h768_n4096_bf16")
    y, plan = run_1d(wl, kernel="tcgen05")
    assert plan.path == "fused_t2"
    assert_close(y, oracle_full(wl), "bf16", wl.name + " (t2, full)", scale=row_scale_1d(wl))


def test_tensor_core_large_dynamic_range():
    """Inputs far from unit scale: the bf16 path keeps fp32's exponent range."""
    wl = wlmod.make_1d(2, 2, 4096, dtype="bf16", seed=11)
    wl.u = wlmod.round_bf16(wl.u * np.float32(3.0e4))
    wl.k = (wl.k * np.float32(1.0e-3)).astype(np.float32)
    y, _ = run_1d(wl)
    assert_close(y, oracle_full(wl), "bf16", "tc scaled inputs", scale=row_scale_1d(wl))


def test_no_skip_term_and_single_row():
    wl = wlmod.make_1d(1, 5, 2048, dtype="f32", seed=3, with_D=False)
    y, _ = run_1d(wl)
    assert_close(y, oracle_full(wl), "f32", "B=1 no D", scale=row_scale_1d(wl))


@pytest.mark.parametrize("N,dtype,gated", [(16384, "f32", False), (32768, "f32", False), (16384, "f32", True),
                                           (32768, "bf16", True), (32768, "bf16", False)])
def test_multipass_full_compare(N, dtype, gated):
    wl = wlmod.make_1d(3, 2, N, dtype=dtype, gated=gated, seed=N + gated, with_D=True)
    y, plan = run_1d(wl)
    assert plan.path == "multipass"
    assert_close(y, oracle_full(wl), dtype, f"multipass N={N} {dtype} gated={gated}",
                 gate=wl.v if gated else None, scale=row_scale_1d(wl))


@pytest.mark.parametrize("log2N", [16, 17, 18, 19, 20])
def test_multipass_sampled(log2N):
    N = 1 << log2N
    wl = wlmod.make_1d(3, 1, N, dtype="f32", seed=log2N, alpha=1e-5)
    y, plan = run_1d(wl)
    assert plan.path == "multipass"
    b, h, t = wlmod.sample_points_1d(wl.B, wl.H, N, 400, seed=log2N)
    ref = oracle.causal_conv1d_points(wl.u, wl.k, b, h, t, D=wl.D)
    assert_close(y[b, h, t], ref, "f32", f"multipass N=2^{log2N}", scale=row_scale_1d(wl, b, h))


def test_multipass_ragged_groups():
    """More pairs than one workspace group holds, with a short last group."""
    N = 1 << 20
    wl = wlmod.make_1d(3, 5, N, dtype="bf16", seed=99, alpha=1e-5)
    y, plan = run_1d(wl, group_bytes=64 << 20)  # 4 pairs of 16 MiB per group: groups of 4, 4, 2
    assert plan.workspace_bytes == 64 << 20
    b, h, t = wlmod.sample_points_1d(wl.B, wl.H, N, 64, seed=99)
    ref = oracle.causal_conv1d_points(wl.u, wl.k, b, h, t, D=wl.D)
    assert_close(y[b, h, t], ref, "bf16", "ragged groups", scale=row_scale_1d(wl, b, h))


@pytest.mark.parametrize("N", [4096, 1 << 20])
def test_geometric_kernel_recursion_full_length(N):
    """k[t] = c a^t gives y[t] = a y[t-1] + c u[t] (+ D u[t]): every output of a
    full-length launch is checked against this O(N) recursion in fp64."""
    rng = np.random.default_rng(5)
    B, H = 2, 2
    u = rng.standard_normal((B, H, N), dtype=np.float32)
    a = np.array([0.9999, 0.99])
    c = np.array([0.5, -1.5])
    t = np.arange(N)
    k = (c[:, None] * a[:, None] ** t[None, :]).astype(np.float32)
    D = np.array([0.25, -2.0], dtype=np.float32)
    wl = wlmod.Workload1D("geometric", B, H, N, "f32", False, u, k, D)
    y, _ = run_1d(wl)
    ref = np.empty((B, H, N))
    for h in range(H):
        # y[t] = a y[t-1] + c u[t], run as a first-order IIR filter in fp64
        ref[:, h, :] = scipy.signal.lfilter([c[h]], [1.0, -a[h]], u[:, h, :].astype(np.float64), axis=-1)
    ref += D[None, :, None].astype(np.float64) * u.astype(np.float64)
    # k was rounded to fp32 (<= 2^-24 relative per tap); the error that induces
    # in y is orders of magnitude inside the fp32 tolerance.
    assert_close(y, ref, "f32", f"geometric recursion N={N}")


# ------------------------------------------------ the named workloads, full size
def _named(name):
    return wlmod.make_config(name)


def test_pr1_full():
    wl = _named("pr1_b1_h4_n1024_f32")
    y, plan = run_1d(wl)
    assert plan.path == "fused"
    assert_close(y, oracle_full(wl), "f32", wl.name, scale=row_scale_1d(wl))


def test_named_hyena_full():
    """The Hyena-style workload at full size through the mma.sync kernel
    (persistent CTAs, several row pairs each): every one of its 25,165,824
    outputs against the oracle (the default two-stage kernel has its own
    full-size test)."""
    wl = _named("hyena_b8_h768_n4096_bf16")
    y, _ = run_1d(wl, kernel="mma_sync")
    assert_close(y, oracle_full(wl), "bf16", wl.name + " (full)", scale=row_scale_1d(wl))


def test_named_gated_rows_full():
    """The gated workload at full size: 512 whole rows (seeded draw of (b, h))
    against the oracle, plus sampled positions with uniform draws in every row."""
    wl = _named("gated_b4_h1024_n16384_bf16")
    y, _ = run_1d(wl)
    rng = np.random.default_rng(77)
    rows = rng.choice(wl.B * wl.H, size=512, replace=False)
    bi, hi = rows // wl.H, rows % wl.H
    # the chosen rows as one [1, 512, N] workload with their own filters
    ref = oracle.causal_conv1d(wl.u[bi, hi][None], wl.k[hi], w=wl.w[bi, hi][None], v=wl.v[bi, hi][None])[0]
    sub = wlmod.Workload1D("rows", 1, 512, wl.N, wl.dtype, True, wl.u[bi, hi][None], wl.k[hi], None,
                           wl.v[bi, hi][None], wl.w[bi, hi][None])
    assert_close(y[bi, hi], ref, "bf16", wl.name + " (512 rows)", gate=wl.v[bi, hi],
                 scale=row_scale_1d(sub)[0])
    b, h, t = wlmod.sample_points_1d(wl.B, wl.H, wl.N, 8, seed=1)
    ref = oracle.causal_conv1d_points(wl.u, wl.k, b, h, t, D=wl.D, w=wl.w, v=wl.v)
    assert_close(y[b, h, t], ref, wl.dtype, wl.name + " (sampled)", gate=wl.v[b, h, t],
                 scale=row_scale_1d(wl, b, h))


def test_named_long_sampled():
    wl = _named("long_b2_h64_n1048576_f32")
    y, _ = run_1d(wl)
    b, h, t = wlmod.sample_points_1d(wl.B, wl.H, wl.N, 96, seed=1)
    ref = oracle.causal_conv1d_points(wl.u, wl.k, b, h, t, D=wl.D, w=wl.w, v=wl.v)
    assert_close(y[b, h, t], ref, wl.dtype, wl.name, scale=row_scale_1d(wl, b, h))


@pytest.mark.parametrize("N,kernel", [(2048, "tcgen05"), (4096, "tcgen05"), (16384, "auto")])  # umma, t2, P = 128
def test_wait_limit_timeout_then_recovers(N, kernel):
    """A wait limit of 0 makes the first bounded device wait of every CTA give
    up: the launch drains its products, frees its tensor memory and reports
    FFTCONV_ERR_TIMEOUT once; the same plan, back at the default limit, then
    runs a normal launch that matches the oracle.  Nothing hangs or faults:
    the products do complete, the wait just stops looking."""
    from fft_long_convolution_causal_b200 import binding
    wl = wlmod.make_1d(3, 3, N, dtype="bf16", gated=False, seed=5 * N, with_D=True)
    plan = binding.Plan(wl.B, wl.H, wl.N, "bf16", kernel=kernel)
    assert plan.path in ("fused_umma", "fused_t2", "fused_tc"), plan.path
    khat = plan.kernel_spectrum(torch.from_numpy(wl.k).cuda())
    u, D = to_dev(wl.u, "bf16"), torch.from_numpy(wl.D).cuda()
    plan.set_wait_limit(0)
    plan.fwd(u, khat, D=D)
    assert plan.device_status() == 6  # FFTCONV_ERR_TIMEOUT, once
    assert plan.device_status() == 0
    plan.set_wait_limit()
    y = plan.fwd(u, khat, D=D)
    torch.cuda.synchronize()
    assert plan.device_status() == 0
    assert_close(to_host(y), oracle_full(wl), "bf16", f"after timeout N={N}", scale=row_scale_1d(wl))


def test_mma_flops_reported():
    from fft_long_convolution_causal_b200 import binding
    assert binding.Plan(2, 2, 1024, "f32").mma_flops == 0.0
    assert binding.Plan(2, 2, 1 << 16, "f32").mma_flops == 0.0
    # mma.sync kernel, 2N = 8192 (P = 32): 1536 m16n8k16 products per pair
    assert binding.Plan(4, 3, 4096, "bf16", kernel="mma_sync").mma_flops == 2 * 3 * 1536 * 2 * 16 * 8 * 16


# ------------------------------------------------------------------ 2-D
def run_2d(wl, **plan_kw):
    from fft_long_convolution_causal_b200 import binding
    plan = binding.Plan2D(wl.B, wl.C, wl.Hs, wl.Ws, wl.dtype, **plan_kw)
    khat = plan.kernel_spectrum(torch.from_numpy(wl.k).cuda())
    y = plan.fwd(to_dev(wl.u, wl.dtype), khat)
    torch.cuda.synchronize()
    return to_host(y)


@pytest.mark.parametrize("Hs,Ws", [(16, 16), (32, 64), (64, 32), (128, 128)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_conv2d_full_compare(Hs, Ws, dtype):
    wl = wlmod.make_2d(3, 2, Hs, Ws, dtype=dtype, seed=Hs + Ws, sigma=Hs / 4)
    y = run_2d(wl)
    assert_close(y, oracle.causal_conv2d(wl.u, wl.k), dtype, f"2d {Hs}x{Ws} {dtype}", scale=row_scale_2d(wl))


def test_conv2d_small_kernel():
    wl = wlmod.make_2d(2, 3, 64, 64, dtype="f32", seed=2, Kh=5, Kw=17)
    y = run_2d(wl)
    assert_close(y, oracle.causal_conv2d(wl.u, wl.k), "f32", "2d small kernel", scale=row_scale_2d(wl))


def test_conv2d_tensor_core_groups():
    """2-D on the tensor cores with several workspace groups (the last one short)."""
    wl = wlmod.make_2d(4, 3, 256, 256, dtype="bf16", seed=31, Kh=12, Kw=20, sigma=64.0)
    y = run_2d(wl, group_bytes=4 << 20)  # 4 pairs of 1 MiB per group: groups of 4, 2 (6 pairs)
    idx = wlmod.sample_points_2d(wl.B, wl.C, wl.Hs, wl.Ws, 2048, seed=31)
    ref = oracle.causal_conv2d_points(wl.u, wl.k, *idx)
    assert_close(y[idx], ref, "bf16", "2d tc groups", scale=row_scale_2d(wl, idx[0], idx[1]))


@pytest.mark.parametrize("Ws,Kh,Kw", [(256, 24, 24), (64, 256, 9)])
def test_conv2d_tensor_core_columns(Ws, Kh, Kw):
    """bf16 images of 256 rows: the column pass runs on the tensor cores (every output compared)."""
    from fft_long_convolution_causal_b200 import binding
    wl = wlmod.make_2d(3, 2, 256, Ws, dtype="bf16", seed=Ws + Kh, Kh=Kh, Kw=Kw, sigma=64.0)
    assert binding.Plan2D(wl.B, wl.C, wl.Hs, wl.Ws, "bf16").path == "2d_tc"
    y = run_2d(wl)
    assert_close(y, oracle.causal_conv2d(wl.u, wl.k), "bf16", f"2d tc 256x{Ws} k{Kh}x{Kw}", scale=row_scale_2d(wl))


@pytest.mark.parametrize("Hs,Ws,dtype,Kh,Kw", [(16, 16, "f32", 16, 16), (64, 32, "bf16", 40, 32),
                                              (256, 256, "bf16", 256, 256), (256, 64, "bf16", 100, 64)])
@pytest.mark.parametrize("frac", [(0.5, 0.5), (1.0, 1.0), (0.5, 0.0), (0.0, 0.25)])
def test_conv2d_crop_offset(Hs, Ws, dtype, Kh, Kw, frac):
    """Crop windows other than the first quadrant (fftconv2d_fwd_offset): the
    centred reading (Hs/2, Ws/2), the far window, and one-sided shifts, on
    the SIMT passes and on the tensor-core passes (256 rows, bf16); every
    output against the oracle's window of the full linear convolution."""
    oy, ox = 8 * int(Hs * frac[0] / 8), 8 * int(Ws * frac[1] / 8)  # offsets are multiples of 8
    from fft_long_convolution_causal_b200 import binding
    wl = wlmod.make_2d(3, 2, Hs, Ws, dtype=dtype, seed=Hs + Ws + oy + ox, Kh=Kh, Kw=Kw, sigma=Hs / 4)
    plan = binding.Plan2D(wl.B, wl.C, wl.Hs, wl.Ws, dtype)
    khat = plan.kernel_spectrum(torch.from_numpy(wl.k).cuda())
    y = to_host(plan.fwd(to_dev(wl.u, dtype), khat, offset=(oy, ox)))
    want = oracle.causal_conv2d_offset(wl.u, wl.k, oy, ox)
    assert_close(y, want, dtype, f"2d offset {Hs}x{Ws} {dtype} ({oy},{ox}) path={plan.path}", scale=row_scale_2d(wl))


def test_conv2d_named_sampled():
    wl = _named("conv2d_b4_c256_256x256_bf16")
    y = run_2d(wl)
    idx = wlmod.sample_points_2d(wl.B, wl.C, wl.Hs, wl.Ws, 4096, seed=4)
    ref = oracle.causal_conv2d_points(wl.u, wl.k, *idx)
    assert_close(y[idx], ref, "bf16", wl.name, scale=row_scale_2d(wl, idx[0], idx[1]))


# ------------------------------------------------------------------ API on GPU
def test_fwd_before_spectrum_is_not_ready():
    from fft_long_convolution_causal_b200 import binding
    plan = binding.Plan(2, 2, 1024, "f32")
    u = torch.zeros(2, 2, 1024, device="cuda")
    khat = plan.new_spectrum()
    with pytest.raises(binding.FFTConvError) as e:
        plan.fwd(u, khat)
    assert e.value.status == 3


def test_misaligned_and_aliased_pointers_rejected():
    from fft_long_convolution_causal_b200 import binding
    plan = binding.Plan(1, 1, 1024, "f32")
    k = torch.randn(1, 1024, device="cuda")
    khat = plan.kernel_spectrum(k)
    buf = torch.zeros(1025 + 4, device="cuda")
    lib = binding.load_library()
    import ctypes
    bad = ctypes.c_void_p(buf.data_ptr() + 4)
    ok = ctypes.c_void_p(buf.data_ptr())
    st = lib.fftconv_fwd(plan._handle, bad, None, None, ctypes.c_void_p(khat.data_ptr()), None, ok, None,
                         None)
    assert st == 1
    st = lib.fftconv_fwd(plan._handle, ok, None, None, ctypes.c_void_p(khat.data_ptr()), None, ok, None, None)
    assert st == 1


def test_repeated_calls_are_deterministic():
    wl = wlmod.make_1d(4, 8, 4096, dtype="bf16", seed=17)
    y1, _ = run_1d(wl)
    y2, _ = run_1d(wl)
    assert np.array_equal(y1, y2)
