"""ctypes binding of libfftconv_b200.so (the C ABI in include/fftconv.h).

Argument marshalling only: every step of the convolution runs in the CUDA
library.  torch supplies device memory and the current stream.  If the
library is missing the calls raise -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

_LIB = None

STATUS = {
    0: "ok", 1: "invalid argument", 2: "unsupported size", 3: "kernel spectrum not computed for this plan",
    4: "out of device memory", 5: "CUDA error", 6: "device wait timed out",
}
DTYPES = {"f32": 0, "bf16": 1}
TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}
KERNELS = {"auto": 0, "simt": 1, "mma_sync": 2, "tcgen05": 3}  # fftconv_kernel
DEFAULT_WAIT_PROBES = 65536


class PlanOptions(ctypes.Structure):
    """fftconv_plan_options."""
    _fields_ = [("kernel", ctypes.c_int), ("group_bytes", ctypes.c_size_t)]


# name -> (restype, argtypes); mirrors include/fftconv.h
_vp = ctypes.c_void_p
_optp = ctypes.POINTER(PlanOptions)
_SIGS = {
    "fftconv_plan_options_init": (None, [_optp]),
    "fftconv_plan_create_ex": (ctypes.c_int, [ctypes.POINTER(_vp), ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                              ctypes.c_int, ctypes.c_int, _optp]),
    "fftconv2d_plan_create_ex": (ctypes.c_int, [ctypes.POINTER(_vp), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, _optp]),
    "fftconv_plan_set_wait_limit": (ctypes.c_int, [_vp, ctypes.c_uint32]),
    "fftconv_spectrum_conjugate": (ctypes.c_int, [_vp, _vp, _vp, _vp]),
    "fftconv_fwd_dynamic": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, ctypes.c_int64, _vp, _vp, _vp]),
    "fftconv_ssm_plan_create": (ctypes.c_int, [ctypes.POINTER(_vp), ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int64]),
    "fftconv_ssm_spectrum": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fftconv_spectrum_blocks": (ctypes.c_int, [_vp]),
    "fftconv_spectrum_sparsify": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, _vp]),
    "fftconv_partial_plan_create": (ctypes.c_int, [ctypes.POINTER(_vp), ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                                   ctypes.c_int, ctypes.c_int, ctypes.c_int64]),
    "fftconv_bwd_workspace_bytes": (ctypes.c_size_t, [_vp]),
    "fftconv_bwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int64, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _vp]),
    "fftconv_plan_mma_flops": (ctypes.c_double, [_vp]),
    "fftconv_plan_create": (ctypes.c_int, [ctypes.POINTER(_vp), ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                           ctypes.c_int, ctypes.c_int]),
    "fftconv2d_plan_create": (ctypes.c_int, [ctypes.POINTER(_vp), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int]),
    "fftconv_plan_destroy": (ctypes.c_int, [_vp]),
    "fftconv_spectrum_bytes": (ctypes.c_size_t, [_vp]),
    "fftconv_workspace_bytes": (ctypes.c_size_t, [_vp]),
    "fftconv_plan_path": (ctypes.c_char_p, [_vp]),
    "fftconv_kernel_spectrum": (ctypes.c_int, [_vp, _vp, ctypes.c_int64, _vp, _vp, _vp]),
    "fftconv_fwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fftconv2d_kernel_spectrum": (ctypes.c_int, [_vp, _vp, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp]),
    "fftconv2d_fwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp]),
    "fftconv2d_fwd_offset": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int, ctypes.c_int]),
    "fftconv3d_plan_create": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "fftconv3d_kernel_spectrum": (ctypes.c_int, [_vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp]),
    "fftconv3d_fwd": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp]),
    "fftconv2d_dynamic_plan_create": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int, ctypes.c_int,
                                                     ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "fftconv2d_fwd_dynamic": (ctypes.c_int, [_vp, _vp, _vp, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp]),
    "fftconv_fwd_static_workspace": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fftconv_static_workspace_bytes": (ctypes.c_size_t, []),
    "fftconv_device_status": (ctypes.c_int, [_vp, _vp]),
    "fftconv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "fftconv_version": (ctypes.c_int, []),
}


class FFTConvError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, 'unknown')} (status {status})")
        self.status = status


def library_path() -> str:
    return _build.LIB


def load_library(build_if_missing: bool = False) -> ctypes.CDLL:
    """Load the CUDA library; raises if it is not built."""
    global _LIB
    if _LIB is None:
        path = _build.LIB
        if not os.path.exists(path):
            if not build_if_missing:
                raise FileNotFoundError(
                    f"{path} is missing: build it with `python -m fft_long_convolution_causal_b200.build`")
            _build.build()
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def status_string(status: int) -> str:
    return load_library().fftconv_status_string(status).decode()


def _check(status: int, what: str):
    if status != 0:
        raise FFTConvError(status, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, shape, dtype):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class _PlanBase:
    _handle: ctypes.c_void_p

    def __del__(self):
        h = getattr(self, "_handle", None)
        if h is not None and h.value and _LIB is not None:
            _LIB.fftconv_plan_destroy(h)
            self._handle = None

    def destroy(self):
        self.__del__()

    @property
    def spectrum_bytes(self) -> int:
        return int(self.lib.fftconv_spectrum_bytes(self._handle))

    @property
    def workspace_bytes(self) -> int:
        return int(self.lib.fftconv_workspace_bytes(self._handle))

    @property
    def path(self) -> str:
        return self.lib.fftconv_plan_path(self._handle).decode()

    @property
    def mma_flops(self) -> float:
        """Tensor-core flops of one forward call (0 for SIMT paths)."""
        return float(self.lib.fftconv_plan_mma_flops(self._handle))

    def set_wait_limit(self, probes: int = DEFAULT_WAIT_PROBES):
        """Probes per bounded device wait (0: give up at the first check)."""
        _check(self.lib.fftconv_plan_set_wait_limit(self._handle, int(probes)), "fftconv_plan_set_wait_limit")

    def device_status(self, stream=None) -> int:
        """Synchronise the stream; 0, or 6 (timed out) once after a launch whose device wait gave up."""
        return int(self.lib.fftconv_device_status(self._handle, _stream(stream)))

    def new_spectrum(self, device=None) -> torch.Tensor:
        return torch.empty(self.spectrum_bytes, dtype=torch.uint8, device=device or "cuda")

    def new_workspace(self, device=None) -> Optional[torch.Tensor]:
        n = self.workspace_bytes
        return torch.empty(n, dtype=torch.uint8, device=device or "cuda") if n else None

    def _ws(self, workspace):
        if workspace is None and self.workspace_bytes:
            if self._workspace is None:
                self._workspace = self.new_workspace()
            workspace = self._workspace
        if workspace is not None and workspace.numel() * workspace.element_size() < self.workspace_bytes:
            raise ValueError("workspace too small")
        return workspace


def _options(lib, kernel: str, group_bytes: int) -> PlanOptions:
    o = PlanOptions()
    lib.fftconv_plan_options_init(ctypes.byref(o))
    o.kernel = KERNELS[kernel]
    o.group_bytes = int(group_bytes)
    return o


class Plan(_PlanBase):
    """1-D plan: fftconv_plan_create_ex(B, H, N, dtype, gated, options).

    kernel: "auto" (default), "simt", "mma_sync" or "tcgen05"; group_bytes:
    multi-pass workspace per group of row pairs (0 = the library default)."""

    def __init__(self, B: int, H: int, N: int, dtype: str = "bf16", gated: bool = False, kernel: str = "auto",
                 group_bytes: int = 0):
        self.lib = load_library()
        self.B, self.H, self.N, self.dtype, self.gated = B, H, N, dtype, bool(gated)
        self.torch_dtype = TORCH_DTYPES[dtype]
        h = ctypes.c_void_p()
        opts = _options(self.lib, kernel, group_bytes)
        _check(self.lib.fftconv_plan_create_ex(ctypes.byref(h), B, H, N, DTYPES[dtype], int(bool(gated)),
                                               ctypes.byref(opts)), "fftconv_plan_create_ex")
        self._handle = h
        self._workspace = None

    def kernel_spectrum(self, k: torch.Tensor, khat: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """khat <- spectrum of k [H, L] (fp32, L <= N)."""
        if k.dim() != 2:
            raise ValueError("k must be [H, L]")
        _need(k, "k", (self.H, k.shape[1]), torch.float32)
        if khat is None:
            khat = self.new_spectrum(k.device)
        workspace = self._ws(workspace)
        _check(self.lib.fftconv_kernel_spectrum(self._handle, _ptr(k), k.shape[1], _ptr(khat), _ptr(workspace),
                                                _stream(stream)), "fftconv_kernel_spectrum")
        return khat

    def fwd(self, u: torch.Tensor, khat: torch.Tensor, D: Optional[torch.Tensor] = None,
            v: Optional[torch.Tensor] = None, w: Optional[torch.Tensor] = None,
            y: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
            stream=None) -> torch.Tensor:
        """y = v * ((u*w) conv k + D (u*w)) (gated) or (u conv k) + D u."""
        shape = (self.B, self.H, self.N)
        _need(u, "u", shape, self.torch_dtype)
        if self.gated:
            _need(v, "v", shape, self.torch_dtype)
            _need(w, "w", shape, self.torch_dtype)
        elif v is not None or w is not None:
            raise ValueError("v and w are only for a gated plan")
        if D is not None:
            _need(D, "D", (self.H,), torch.float32)
        if y is None:
            y = torch.empty(shape, dtype=self.torch_dtype, device=u.device)
        _need(y, "y", shape, self.torch_dtype)
        workspace = self._ws(workspace)
        _check(self.lib.fftconv_fwd(self._handle, _ptr(u), _ptr(v), _ptr(w), _ptr(khat), _ptr(D), _ptr(y),
                                    _ptr(workspace), _stream(stream)), "fftconv_fwd")
        return y


    def fwd_dynamic(self, u: torch.Tensor, k: torch.Tensor, D: Optional[torch.Tensor] = None,
                    v: Optional[torch.Tensor] = None, w: Optional[torch.Tensor] = None,
                    y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """y with one filter per batch row: k [B, H, L] fp32, transformed in the same launch."""
        shape = (self.B, self.H, self.N)
        _need(u, "u", shape, self.torch_dtype)
        if k.dim() != 3:
            raise ValueError("k must be [B, H, L]")
        _need(k, "k", (self.B, self.H, k.shape[2]), torch.float32)
        if self.gated:
            _need(v, "v", shape, self.torch_dtype)
            _need(w, "w", shape, self.torch_dtype)
        if D is not None:
            _need(D, "D", (self.H,), torch.float32)
        if y is None:
            y = torch.empty(shape, dtype=self.torch_dtype, device=u.device)
        _check(self.lib.fftconv_fwd_dynamic(self._handle, _ptr(u), _ptr(v), _ptr(w), _ptr(k), k.shape[2], _ptr(D),
                                            _ptr(y), _stream(stream)), "fftconv_fwd_dynamic")
        return y

    @property
    def spectrum_blocks(self) -> int:
        """Outer frequency blocks a frequency-sparse mask has (0: not a multi-pass plan)."""
        return int(self.lib.fftconv_spectrum_blocks(self._handle))

    def sparsify(self, khat: torch.Tensor, keep, stream=None):
        """Frequency-sparse: zero khat on the outer frequency rows k1 with keep[k1] false (None: dense)."""
        if keep is None:
            _check(self.lib.fftconv_spectrum_sparsify(self._handle, _ptr(khat), None, 0, _stream(stream)),
                   "fftconv_spectrum_sparsify")
            return khat
        arr = (ctypes.c_uint8 * len(keep))(*[1 if x else 0 for x in keep])
        _check(self.lib.fftconv_spectrum_sparsify(self._handle, _ptr(khat), ctypes.cast(arr, ctypes.c_void_p),
                                                  len(keep), _stream(stream)), "fftconv_spectrum_sparsify")
        return khat

    def spectrum_conjugate(self, khat: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """conj(khat) in the plan's layout: the spectrum of the correlation with k."""
        if out is None:
            out = torch.empty_like(khat)
        _check(self.lib.fftconv_spectrum_conjugate(self._handle, _ptr(khat), _ptr(out), _stream(stream)),
               "fftconv_spectrum_conjugate")
        return out

    @property
    def bwd_workspace_bytes(self) -> int:
        return int(self.lib.fftconv_bwd_workspace_bytes(self._handle))

    def bwd(self, dy: torch.Tensor, u: torch.Tensor, khat: torch.Tensor, khat_conj: torch.Tensor,
            D: Optional[torch.Tensor] = None, v: Optional[torch.Tensor] = None, w: Optional[torch.Tensor] = None,
            L: int = 0, filter_grad: bool = True, stream=None) -> dict:
        """Gradients of y = fwd(u, khat, D, v, w) for the upstream gradient dy:
        du (dv, dw gated) of the plan's dtype, dk [H, L] and dD [H] fp32
        (dk only with filter_grad, dD only with D)."""
        shape = (self.B, self.H, self.N)
        _need(dy, "dy", shape, self.torch_dtype)
        _need(u, "u", shape, self.torch_dtype)
        if self.gated:
            _need(v, "v", shape, self.torch_dtype)
            _need(w, "w", shape, self.torch_dtype)
        du = torch.empty_like(u)
        dv = torch.empty_like(u) if self.gated else None
        dw = torch.empty_like(u) if self.gated else None
        L = L or self.N
        dk = torch.empty(self.H, L, dtype=torch.float32, device=u.device) if filter_grad else None
        dD = torch.empty(self.H, dtype=torch.float32, device=u.device) if (filter_grad and D is not None) else None
        n = self.bwd_workspace_bytes
        ws = torch.empty(n, dtype=torch.uint8, device=u.device) if n else None
        _check(self.lib.fftconv_bwd(self._handle, _ptr(dy), _ptr(u), _ptr(v), _ptr(w), _ptr(khat), _ptr(khat_conj),
                                    _ptr(D), L, _ptr(du), _ptr(dv), _ptr(dw), _ptr(dk), _ptr(dD), _ptr(ws),
                                    _stream(stream)), "fftconv_bwd")
        return {"du": du, "dv": dv, "dw": dw, "dk": dk, "dD": dD}


class Plan2D(_PlanBase):
    """2-D plan: fftconv2d_plan_create_ex(B, C, Hs, Ws, dtype, options)."""

    def __init__(self, B: int, C: int, Hs: int, Ws: int, dtype: str = "bf16", kernel: str = "auto",
                 group_bytes: int = 0):
        self.lib = load_library()
        self.B, self.C, self.Hs, self.Ws, self.dtype = B, C, Hs, Ws, dtype
        self.torch_dtype = TORCH_DTYPES[dtype]
        h = ctypes.c_void_p()
        opts = _options(self.lib, kernel, group_bytes)
        _check(self.lib.fftconv2d_plan_create_ex(ctypes.byref(h), B, C, Hs, Ws, DTYPES[dtype], ctypes.byref(opts)),
               "fftconv2d_plan_create_ex")
        self._handle = h
        self._workspace = None

    def kernel_spectrum(self, k: torch.Tensor, khat: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        if k.dim() != 3:
            raise ValueError("k must be [C, Kh, Kw]")
        _need(k, "k", (self.C, k.shape[1], k.shape[2]), torch.float32)
        if khat is None:
            khat = self.new_spectrum(k.device)
        workspace = self._ws(workspace)
        _check(self.lib.fftconv2d_kernel_spectrum(self._handle, _ptr(k), k.shape[1], k.shape[2], _ptr(khat),
                                                  _ptr(workspace), _stream(stream)), "fftconv2d_kernel_spectrum")
        return khat

    def fwd(self, u: torch.Tensor, khat: torch.Tensor, y: Optional[torch.Tensor] = None,
            workspace: Optional[torch.Tensor] = None, stream=None, offset=(0, 0)) -> torch.Tensor:
        """y = window [oy, oy+Hs) x [ox, ox+Ws) of the full linear convolution
        (offset (0, 0): the first-quadrant crop; (Hs/2, Ws/2): the centred one)."""
        shape = (self.B, self.C, self.Hs, self.Ws)
        _need(u, "u", shape, self.torch_dtype)
        if y is None:
            y = torch.empty(shape, dtype=self.torch_dtype, device=u.device)
        _need(y, "y", shape, self.torch_dtype)
        workspace = self._ws(workspace)
        oy, ox = (int(offset[0]), int(offset[1]))
        _check(self.lib.fftconv2d_fwd_offset(self._handle, _ptr(u), _ptr(khat), _ptr(y), _ptr(workspace),
                                             _stream(stream), oy, ox), "fftconv2d_fwd_offset")
        return y


class Plan2DDynamic(_PlanBase):
    """2-D plan with one filter per image: fftconv2d_dynamic_plan_create(B, C, Hs, Ws, dtype)."""

    def __init__(self, B: int, C: int, Hs: int, Ws: int, dtype: str = "bf16"):
        self.lib = load_library()
        self.B, self.C, self.Hs, self.Ws, self.dtype = B, C, Hs, Ws, dtype
        self.torch_dtype = TORCH_DTYPES[dtype]
        h = ctypes.c_void_p()
        _check(self.lib.fftconv2d_dynamic_plan_create(ctypes.byref(h), B, C, Hs, Ws, DTYPES[dtype]),
               "fftconv2d_dynamic_plan_create")
        self._handle = h
        self._workspace = None

    def fwd(self, u: torch.Tensor, k: torch.Tensor, y: Optional[torch.Tensor] = None,
            workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """y[b, c] = first-quadrant crop of u[b, c] convolved with k[b, c] ([B, C, Kh, Kw] fp32)."""
        shape = (self.B, self.C, self.Hs, self.Ws)
        _need(u, "u", shape, self.torch_dtype)
        if k.dim() != 4:
            raise ValueError("k must be [B, C, Kh, Kw]")
        _need(k, "k", (self.B, self.C, k.shape[2], k.shape[3]), torch.float32)
        if y is None:
            y = torch.empty(shape, dtype=self.torch_dtype, device=u.device)
        _need(y, "y", shape, self.torch_dtype)
        workspace = self._ws(workspace)
        _check(self.lib.fftconv2d_fwd_dynamic(self._handle, _ptr(u), _ptr(k), k.shape[2], k.shape[3], _ptr(y),
                                              _ptr(workspace), _stream(stream)), "fftconv2d_fwd_dynamic")
        return y


class Plan3D(_PlanBase):
    """3-D plan: fftconv3d_plan_create(B, C, Dd, Hs, Ws, dtype)."""

    def __init__(self, B: int, C: int, Dd: int, Hs: int, Ws: int, dtype: str = "f32"):
        self.lib = load_library()
        self.B, self.C, self.Dd, self.Hs, self.Ws, self.dtype = B, C, Dd, Hs, Ws, dtype
        self.torch_dtype = TORCH_DTYPES[dtype]
        h = ctypes.c_void_p()
        _check(self.lib.fftconv3d_plan_create(ctypes.byref(h), B, C, Dd, Hs, Ws, DTYPES[dtype]),
               "fftconv3d_plan_create")
        self._handle = h
        self._workspace = None

    def kernel_spectrum(self, k: torch.Tensor, khat: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """khat <- spectrum of k [C, Kd, Kh, Kw] (fp32)."""
        if k.dim() != 4:
            raise ValueError("k must be [C, Kd, Kh, Kw]")
        _need(k, "k", (self.C, k.shape[1], k.shape[2], k.shape[3]), torch.float32)
        if khat is None:
            khat = self.new_spectrum(k.device)
        workspace = self._ws(workspace)
        _check(self.lib.fftconv3d_kernel_spectrum(self._handle, _ptr(k), k.shape[1], k.shape[2], k.shape[3],
                                                  _ptr(khat), _ptr(workspace), _stream(stream)),
               "fftconv3d_kernel_spectrum")
        return khat

    def fwd(self, u: torch.Tensor, khat: torch.Tensor, y: Optional[torch.Tensor] = None,
            workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        shape = (self.B, self.C, self.Dd, self.Hs, self.Ws)
        _need(u, "u", shape, self.torch_dtype)
        if y is None:
            y = torch.empty(shape, dtype=self.torch_dtype, device=u.device)
        _need(y, "y", shape, self.torch_dtype)
        workspace = self._ws(workspace)
        _check(self.lib.fftconv3d_fwd(self._handle, _ptr(u), _ptr(khat), _ptr(y), _ptr(workspace), _stream(stream)),
               "fftconv3d_fwd")
        return y


class PartialPlan(Plan):
    """Partial convolution, filters of at most L_max taps:
    fftconv_partial_plan_create(B, H, N, dtype, gated, L_max); kernel_spectrum
    and fwd as a 1-D plan."""

    def __init__(self, B: int, H: int, N: int, dtype: str = "f32", gated: bool = False, L_max: int = 1024):
        self.lib = load_library()
        self.B, self.H, self.N, self.dtype, self.gated = B, H, N, dtype, bool(gated)
        self.torch_dtype = TORCH_DTYPES[dtype]
        h = ctypes.c_void_p()
        _check(self.lib.fftconv_partial_plan_create(ctypes.byref(h), B, H, N, DTYPES[dtype], int(bool(gated)),
                                                    int(L_max)), "fftconv_partial_plan_create")
        self._handle = h
        self._workspace = None


class SSMPlan(_PlanBase):
    """Chunked state passing: fftconv_ssm_plan_create(B, H, N, dtype, d_state, chunk)."""

    def __init__(self, B: int, H: int, N: int, dtype: str = "f32", d_state: int = 16, chunk: int = 8192):
        self.lib = load_library()
        self.B, self.H, self.N, self.dtype, self.d, self.chunk = B, H, N, dtype, d_state, chunk
        self.torch_dtype = TORCH_DTYPES[dtype]
        h = ctypes.c_void_p()
        _check(self.lib.fftconv_ssm_plan_create(ctypes.byref(h), B, H, N, DTYPES[dtype], d_state, chunk),
               "fftconv_ssm_plan_create")
        self._handle = h
        self._workspace = None

    def set_filters(self, lam: torch.Tensor, c: torch.Tensor, khat: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
        """k[h,t] = Re(sum_j c[h,j] lam[h,j]^t); lam, c complex [H, d] (any device)."""
        shape = (self.H, self.d)
        if tuple(lam.shape) != shape or tuple(c.shape) != shape:
            raise ValueError(f"lam and c must be {shape}")
        parts = [t.real.to(torch.float32).contiguous().cuda() for t in (lam, c)] + \
                [t.imag.to(torch.float32).contiguous().cuda() for t in (lam, c)]
        lr, cr, li, ci = parts
        if khat is None:
            khat = self.new_spectrum()
        ws = self._ws(None)
        _check(self.lib.fftconv_ssm_spectrum(self._handle, _ptr(lr), _ptr(li), _ptr(cr), _ptr(ci), _ptr(khat),
                                             _ptr(ws), _stream(stream)), "fftconv_ssm_spectrum")
        self._keep = parts  # alive until the launch has read them
        return khat

    def fwd(self, u: torch.Tensor, khat: torch.Tensor, D: Optional[torch.Tensor] = None,
            y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        shape = (self.B, self.H, self.N)
        _need(u, "u", shape, self.torch_dtype)
        if D is not None:
            _need(D, "D", (self.H,), torch.float32)
        if y is None:
            y = torch.empty(shape, dtype=self.torch_dtype, device=u.device)
        ws = self._ws(None)
        _check(self.lib.fftconv_fwd(self._handle, _ptr(u), None, None, _ptr(khat), _ptr(D), _ptr(y), _ptr(ws),
                                    _stream(stream)), "fftconv_fwd")
        return y


def fftconv(u: torch.Tensor, k: torch.Tensor, D: Optional[torch.Tensor] = None,
            v: Optional[torch.Tensor] = None, w: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One-shot causal long convolution (plan + spectrum + forward)."""
    B, H, N = u.shape
    dtype = {torch.float32: "f32", torch.bfloat16: "bf16"}[u.dtype]
    plan = Plan(B, H, N, dtype, gated=v is not None)
    khat = plan.kernel_spectrum(k.contiguous())
    y = plan.fwd(u, khat, D=D, v=v, w=w)
    torch.cuda.current_stream().synchronize()  # the plan's tables are freed on return
    return y


def fftconv2d(u: torch.Tensor, k: torch.Tensor) -> torch.Tensor:
    """One-shot 2-D causal convolution (plan + spectrum + forward)."""
    B, C, Hs, Ws = u.shape
    dtype = {torch.float32: "f32", torch.bfloat16: "bf16"}[u.dtype]
    plan = Plan2D(B, C, Hs, Ws, dtype)
    khat = plan.kernel_spectrum(k.contiguous())
    y = plan.fwd(u, khat)
    torch.cuda.current_stream().synchronize()  # the plan's tables are freed on return
    return y
