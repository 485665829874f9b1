"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

from fft_long_convolution_causal_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fftconv.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"FFTCONV_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for n in ("fftconv_plan_create", "fftconv_kernel_spectrum", "fftconv_fwd", "fftconv2d_plan_create",
              "fftconv2d_kernel_spectrum", "fftconv2d_fwd", "fftconv_plan_destroy", "fftconv_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
        assert n in binding._SIGS, f"binding does not declare {n}"


def test_no_internal_symbols_leak(lib):
    # C++ internals are hidden; only the fftconv_* C names are exported.
    out = os.popen(f"nm -D --defined-only {build.LIB}").read()
    exported = [l.split()[-1] for l in out.splitlines() if l.split() and l.split()[1] in "TtWw"]
    assert exported and all(n.startswith("fftconv") for n in exported), exported


def test_status_strings(lib):
    for code in range(7):
        assert binding.status_string(code) == binding.STATUS[code]
    assert lib.fftconv_version() >= 100


def _create(lib, B, H, N, dtype=0, gated=0, null_out=False):
    h = ctypes.c_void_p()
    ref = None if null_out else ctypes.byref(h)
    return lib.fftconv_plan_create(ref, B, H, N, dtype, gated), h


@pytest.mark.parametrize("B,H,N,dtype,want", [
    (0, 4, 1024, 0, 1), (1, 0, 1024, 0, 1), (1, 4, 1024, 7, 1),
    (1, 4, 1000, 0, 2), (1, 4, 32, 0, 2), (1, 4, 1 << 21, 0, 2), (1, 4, 0, 0, 2), (1, 4, -1024, 0, 2),
])
def test_plan_create_rejects_before_any_cuda_call(lib, B, H, N, dtype, want):
    st, h = _create(lib, B, H, N, dtype)
    assert st == want
    assert not h.value


def test_plan_create_null_out(lib):
    st, _ = _create(lib, 1, 4, 1024, null_out=True)
    assert st == 1


@pytest.mark.parametrize("B,C,Hs,Ws,want", [
    (0, 1, 16, 16, 1), (1, 0, 16, 16, 1), (1, 1, 8, 16, 2), (1, 1, 16, 512, 2), (1, 1, 48, 64, 2),
])
def test_plan2d_create_rejects(lib, B, C, Hs, Ws, want):
    h = ctypes.c_void_p()
    assert lib.fftconv2d_plan_create(ctypes.byref(h), B, C, Hs, Ws, 1) == want
    assert not h.value


def test_null_plan_calls(lib):
    assert lib.fftconv_fwd(None, None, None, None, None, None, None, None, None) == 1
    assert lib.fftconv_kernel_spectrum(None, None, 1, None, None, None) == 1
    assert lib.fftconv2d_fwd(None, None, None, None, None, None) == 1
    assert lib.fftconv2d_kernel_spectrum(None, None, 1, 1, None, None, None) == 1
    assert lib.fftconv_spectrum_bytes(None) == 0
    assert lib.fftconv_workspace_bytes(None) == 0
    assert lib.fftconv_plan_path(None) == b"none"
    assert lib.fftconv_plan_destroy(None) == 0


def test_binding_refuses_missing_library(tmp_path, monkeypatch):
    monkeypatch.setattr(build, "LIB", str(tmp_path / "absent.so"))
    monkeypatch.setattr(binding, "_LIB", None)
    with pytest.raises(FileNotFoundError):
        binding.load_library()


def test_plan_options_defaults_and_validation(lib):
    o = binding.PlanOptions()
    o.kernel, o.group_bytes = 7, 123
    lib.fftconv_plan_options_init(ctypes.byref(o))
    assert (o.kernel, o.group_bytes) == (0, 0)
    h = ctypes.c_void_p()
    for bad in (-1, 4, 99):
        o.kernel = bad
        assert lib.fftconv_plan_create_ex(ctypes.byref(h), 1, 4, 1024, 0, 0, ctypes.byref(o)) == 1
        assert lib.fftconv2d_plan_create_ex(ctypes.byref(h), 1, 1, 16, 16, 1, ctypes.byref(o)) == 1
        assert not h.value
    # size errors are reported the same way with or without options
    o.kernel = 0
    assert lib.fftconv_plan_create_ex(ctypes.byref(h), 1, 4, 1000, 0, 0, ctypes.byref(o)) == 2
    assert lib.fftconv_plan_create_ex(ctypes.byref(h), 1, 4, 1000, 0, 0, None) == 2


def test_null_plan_option_calls(lib):
    assert lib.fftconv_plan_set_wait_limit(None, 0) == 1
    assert lib.fftconv_plan_mma_flops(None) == 0.0
    assert lib.fftconv_device_status(None, None) == 1
    assert lib.fftconv_fwd_static_workspace(None, None, None, None, None, None, None, None) == 1


def _out():
    h = ctypes.c_void_p()
    return h, ctypes.byref(h)


@pytest.mark.parametrize("B,H,N,dtype,d,chunk,want", [
    (0, 4, 1 << 16, 0, 16, 8192, 1),          # no rows
    (1, 4, 1 << 16, 2, 16, 8192, 1),          # fp16 is not a state-passing dtype
    (1, 4, 1 << 16, 0, 0, 8192, 1),           # no state
    (1, 4, 1 << 16, 0, 65, 8192, 1),          # state above the largest supported
    (1, 4, 1 << 16, 0, 16, 6144, 2),          # chunk not a power of two
    (1, 4, 1 << 16, 0, 16, 32, 2),            # chunk below the smallest
    (1, 4, 1 << 16, 0, 16, 16384, 2),         # chunk above the largest
    (1, 4, 4096, 0, 16, 8192, 2),             # sequence shorter than one chunk
    (1, 4, 12288, 0, 16, 8192, 2),            # sequence not a whole number of chunks
    (1, 64, 1 << 20, 0, 16, 64, 2),           # channels x chunks past the launch grid
])
def test_ssm_plan_create_rejects(lib, B, H, N, dtype, d, chunk, want):
    h, ref = _out()
    assert lib.fftconv_ssm_plan_create(ref, B, H, N, dtype, d, chunk) == want
    assert not h.value
    assert lib.fftconv_ssm_plan_create(None, 1, 4, 1 << 16, 0, 16, 8192) == 1


@pytest.mark.parametrize("B,H,N,dtype,L,want", [
    (0, 4, 1 << 16, 0, 1024, 1), (1, 4, 1 << 16, 2, 1024, 1), (1, 4, 1 << 16, 0, 0, 1),
    (1, 4, 1 << 16, 0, 16384, 2),   # the on-chip chunk would exceed 8192
    (1, 4, 1024, 0, 2048, 2),       # sequence shorter than the chunk
])
def test_partial_plan_create_rejects(lib, B, H, N, dtype, L, want):
    h, ref = _out()
    assert lib.fftconv_partial_plan_create(ref, B, H, N, dtype, 0, L) == want
    assert not h.value


@pytest.mark.parametrize("B,C,Hs,Ws,want", [
    (0, 1, 64, 64, 1), (1, 0, 64, 64, 1), (1 << 16, 1 << 15, 64, 64, 1),
    (1, 1, 8, 64, 2), (1, 1, 64, 512, 2), (1, 1, 48, 64, 2),
])
def test_plan2d_dynamic_create_rejects(lib, B, C, Hs, Ws, want):
    h, ref = _out()
    assert lib.fftconv2d_dynamic_plan_create(ref, B, C, Hs, Ws, 1) == want
    assert not h.value


@pytest.mark.parametrize("B,C,Dd,Hs,Ws,dtype,want", [
    (0, 1, 16, 16, 16, 0, 1), (1, 0, 16, 16, 16, 0, 1), (1, 1, 16, 16, 16, 2, 1),
    (1, 1 << 25, 64, 16, 16, 0, 1),   # C x Dd slices past 2^30
    (1, 1, 8, 16, 16, 0, 2), (1, 1, 16, 48, 16, 0, 2), (1, 1, 16, 16, 512, 0, 2),
])
def test_plan3d_create_rejects(lib, B, C, Dd, Hs, Ws, dtype, want):
    h, ref = _out()
    assert lib.fftconv3d_plan_create(ref, B, C, Dd, Hs, Ws, dtype) == want
    assert not h.value
    assert lib.fftconv3d_plan_create(None, 1, 1, 16, 16, 16, 0) == 1


def test_null_plan_calls_of_the_extended_paths(lib):
    """Every entry point beyond the four core calls reports a NULL plan as an
    invalid argument (sizes as 0) without touching the device."""
    assert lib.fftconv_fwd_dynamic(None, None, None, None, None, 1, None, None, None) == 1
    assert lib.fftconv_spectrum_blocks(None) == 0
    assert lib.fftconv_spectrum_sparsify(None, None, None, 0, None) == 1
    assert lib.fftconv_ssm_spectrum(None, None, None, None, None, None, None, None) == 1
    assert lib.fftconv2d_fwd_offset(None, None, None, None, None, None, 0, 0) == 1
    assert lib.fftconv2d_fwd_dynamic(None, None, None, 1, 1, None, None, None) == 1
    assert lib.fftconv3d_kernel_spectrum(None, None, 1, 1, 1, None, None, None) == 1
    assert lib.fftconv3d_fwd(None, None, None, None, None, None) == 1
    assert lib.fftconv_spectrum_conjugate(None, None, None, None) == 1
    assert lib.fftconv_bwd_workspace_bytes(None) == 0
    assert lib.fftconv_bwd(*([None] * 8), 1, *([None] * 7)) == 1
