"""CPU fp64 oracle for the causal FFT long convolution (ctypes wrapper).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this package.  The CUDA library never imports it and shares no code with it.

Definitions (see fftconv_oracle.c for the page citations):

* ``causal_conv1d``: y[b,h,t] = sum_{s<=t, s<L} k[h,s] x[b,h,t-s] (+ D[h] x[b,h,t]),
  x = u (ungated) or u*w (gated, then y *= v).  This is
  irfft(rfft(x,2N) * rfft(k,2N))[:N] (+ D x) evaluated as the direct sum.
* ``causal_conv1d_dynamic``: the same with one filter per batch row, k [B,H,L].
* ``freq_sparse_conv1d``: the formula with the filter's spectrum zeroed on
  blocks of frequencies (numpy FFT as the library step).
* ``ssm_kernel``: filters of a diagonal state-space model, k = Re(sum c lam^t);
  the convolution itself is causal_conv1d (or _points) with that k.
* ``causal_conv1d_bwd``: the gradients du (dv, dw), dk, dD of that y for an
  upstream gradient dy, by the chain rule written as direct sums.
* ``causal_conv2d``: y[b,c,i,j] = sum_{p<=i,q<=j} k[c,p,q] u[b,c,i-p,j-q].
* ``causal_conv2d_offset``: the same convolution, crop window moved by (oy, ox).
* ``dft_causal_conv1d`` / ``dft_causal_conv2d``: the same results through an
  explicit O(M^2) DFT product (tiny sizes only), the independent second route.
"""
import ctypes

import numpy as np

from . import build as _build

_lib = None
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i64 = ctypes.c_int64


def bind(path):
    """Open an oracle shared library at ``path`` and declare its signatures."""
    lib = ctypes.CDLL(path)
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_causal_conv1d.argtypes = [_i64] * 4 + [_f64p] * 6
    lib.oracle_causal_conv1d_points.argtypes = [_i64] * 4 + [_f64p] * 5 + [_i64] + [_i64p] * 3 + [_f64p]
    lib.oracle_causal_conv1d_bwd.argtypes = [_i64] * 4 + [_f64p] * 11
    lib.oracle_causal_conv1d_dynamic.argtypes = [_i64] * 4 + [_f64p] * 6
    lib.oracle_ssm_kernel.argtypes = [_i64] * 3 + [_f64p] * 5
    lib.oracle_causal_conv2d.argtypes = [_i64] * 6 + [_f64p] * 3
    lib.oracle_causal_conv2d_offset.argtypes = [_i64] * 8 + [_f64p] * 3
    lib.oracle_causal_conv2d_points.argtypes = [_i64] * 6 + [_f64p] * 2 + [_i64] + [_i64p] * 4 + [_f64p]
    lib.oracle_causal_conv3d.argtypes = [_i64] * 8 + [_f64p] * 3
    lib.oracle_causal_conv3d_points.argtypes = [_i64] * 8 + [_f64p] * 2 + [_i64] + [_i64p] * 5 + [_f64p]
    lib.oracle_dft_causal_conv1d.argtypes = [_i64, _i64, _f64p, _f64p, _f64p]
    lib.oracle_dft_causal_conv2d.argtypes = [_i64] * 4 + [_f64p] * 3
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(_build.build())
    return _lib


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a):
    return None if a is None else a.ctypes.data_as(_f64p)


def _ip(a):
    return a.ctypes.data_as(_i64p)


def num_threads() -> int:
    """OpenMP threads the oracle runs with."""
    return int(_load().oracle_num_threads())


def _check_1d(u, k, D, w, v):
    u = _f64(u)
    k = _f64(k)
    if u.ndim != 3 or k.ndim != 2:
        raise ValueError("u must be [B,H,N] and k [H,L]")
    B, H, N = u.shape
    if k.shape[0] != H or k.shape[1] > N or k.shape[1] < 1:
        raise ValueError("k must be [H,L] with 1 <= L <= N")
    if (w is None) != (v is None):
        raise ValueError("gated form needs both w and v")
    w, v, D = _f64(w), _f64(v), _f64(D)
    for a in (w, v):
        if a is not None and a.shape != u.shape:
            raise ValueError("w, v must have u's shape")
    if D is not None and D.shape != (H,):
        raise ValueError("D must be [H]")
    return u, k, D, w, v


def causal_conv1d(u, k, D=None, w=None, v=None) -> np.ndarray:
    """Full fp64 direct-sum oracle; returns y [B,H,N]."""
    u, k, D, w, v = _check_1d(u, k, D, w, v)
    B, H, N = u.shape
    y = np.empty_like(u)
    _load().oracle_causal_conv1d(B, H, N, k.shape[1], _p(u), _p(w), _p(v), _p(k), _p(D), _p(y))
    return y


def causal_conv1d_points(u, k, b_idx, h_idx, t_idx, D=None, w=None, v=None) -> np.ndarray:
    """fp64 oracle at the sampled outputs y[b_idx[i], h_idx[i], t_idx[i]]."""
    u, k, D, w, v = _check_1d(u, k, D, w, v)
    B, H, N = u.shape
    bi = np.ascontiguousarray(b_idx, dtype=np.int64)
    hi = np.ascontiguousarray(h_idx, dtype=np.int64)
    ti = np.ascontiguousarray(t_idx, dtype=np.int64)
    if not (bi.shape == hi.shape == ti.shape) or bi.ndim != 1:
        raise ValueError("index arrays must be 1-D and of equal length")
    if bi.size and (bi.min() < 0 or bi.max() >= B or hi.min() < 0 or hi.max() >= H
                    or ti.min() < 0 or ti.max() >= N):
        raise ValueError("sample index out of range")
    out = np.empty(bi.size, dtype=np.float64)
    _load().oracle_causal_conv1d_points(B, H, N, k.shape[1], _p(u), _p(w), _p(v), _p(k), _p(D),
                                        bi.size, _ip(bi), _ip(hi), _ip(ti), _p(out))
    return out


def causal_conv1d_dynamic(u, k, D=None, w=None, v=None) -> np.ndarray:
    """fp64 oracle with one filter per batch row: k [B,H,L]; returns y [B,H,N]."""
    k = _f64(k)
    if k.ndim != 3 or k.shape[:2] != np.shape(u)[:2]:
        raise ValueError("k must be [B,H,L]")
    u, _, D, w, v = _check_1d(u, k[0], D, w, v)
    B, H, N = u.shape
    y = np.empty_like(u)
    _load().oracle_causal_conv1d_dynamic(B, H, N, k.shape[2], _p(u), _p(w), _p(v), _p(k), _p(D), _p(y))
    return y


def ssm_kernel(lam, c, L) -> np.ndarray:
    """fp64 filters of a diagonal state-space model: k[h,t] = Re(sum_j c[h,j]
    lam[h,j]^t) for t < L; lam, c complex [H, d].  Returns [H, L]."""
    lam = np.ascontiguousarray(np.asarray(lam, dtype=np.complex128))
    c = np.ascontiguousarray(np.asarray(c, dtype=np.complex128))
    if lam.ndim != 2 or lam.shape != c.shape:
        raise ValueError("lam and c must be [H, d]")
    H, d = lam.shape
    parts = [np.ascontiguousarray(a) for a in (lam.real, lam.imag, c.real, c.imag)]
    k = np.empty((H, int(L)))
    _load().oracle_ssm_kernel(H, d, int(L), *[_p(a) for a in parts], _p(k))
    return k


def freq_sparse_conv1d(u, k, keep, D=None) -> np.ndarray:
    """Frequency-sparse causal convolution ("FlashFFTConv", abstract): the
    defining formula with the filter's spectrum (skip term included) zeroed on
    blocks of frequencies,
        y = Re(iDFT_M(DFT_M(pad u) . (DFT_M(pad k) + D) . m))[:N],  M = 2N,
    m[f] = keep[f mod G] for a block mask keep of G entries (f = k1 + G k2:
    the outer frequency digit k1 of the split M = G x (M / G)).  numpy's FFT is
    the library step; fp64.  u [B,H,N], k [H,L], keep [G] bool."""
    u = np.asarray(u, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    keep = np.asarray(keep, dtype=bool)
    B, H, N = u.shape
    M = 2 * N
    if M % keep.size:
        raise ValueError("the mask length must divide 2N")
    m = keep[np.arange(M) % keep.size].astype(np.float64)
    K = np.fft.fft(k, M, axis=-1)
    if D is not None:
        K = K + np.asarray(D, dtype=np.float64)[:, None]
    Y = np.fft.fft(u, M, axis=-1) * (K * m)[None]
    return np.real(np.fft.ifft(Y, axis=-1))[..., :N]


def causal_conv1d_bwd(u, k, dy, D=None, w=None, v=None) -> dict:
    """fp64 gradients of y = causal_conv1d(u, k, D, w, v) for the upstream
    gradient dy [B,H,N]: du (and dv, dw when gated) [B,H,N], dk [H,L],
    dD [H] (when D is given).  The chain rule of the forward definition,
    evaluated as direct sums (see fftconv_oracle.c)."""
    u, k, D, w, v = _check_1d(u, k, D, w, v)
    dy = _f64(dy)
    if dy.shape != u.shape:
        raise ValueError("dy must have u's shape")
    B, H, N = u.shape
    L = k.shape[1]
    du = np.empty_like(u)
    dv = np.empty_like(u) if w is not None else None
    dw = np.empty_like(u) if w is not None else None
    dk = np.empty((H, L))
    dD = np.empty(H) if D is not None else None
    _load().oracle_causal_conv1d_bwd(B, H, N, L, _p(u), _p(w), _p(v), _p(k), _p(D), _p(dy), _p(du), _p(dv),
                                     _p(dw), _p(dk), _p(dD))
    return {"du": du, "dv": dv, "dw": dw, "dk": dk, "dD": dD}


def _check_2d(u, k):
    u = _f64(u)
    k = _f64(k)
    if u.ndim != 4 or k.ndim != 3:
        raise ValueError("u must be [B,C,Hs,Ws] and k [C,Kh,Kw]")
    B, C, Hs, Ws = u.shape
    if k.shape[0] != C or not (1 <= k.shape[1] <= Hs) or not (1 <= k.shape[2] <= Ws):
        raise ValueError("k must be [C,Kh,Kw] with Kh <= Hs, Kw <= Ws")
    return u, k


def causal_conv2d(u, k) -> np.ndarray:
    """Full fp64 2-D oracle (first-quadrant crop of the zero-padded linear conv)."""
    u, k = _check_2d(u, k)
    B, C, Hs, Ws = u.shape
    y = np.empty_like(u)
    _load().oracle_causal_conv2d(B, C, Hs, Ws, k.shape[1], k.shape[2], _p(u), _p(k), _p(y))
    return y


def _check_3d(u, k):
    u = _f64(u)
    k = _f64(k)
    if u.ndim != 5 or k.ndim != 4:
        raise ValueError("u must be [B,C,Dd,Hs,Ws] and k [C,Kd,Kh,Kw]")
    B, C, Dd, Hs, Ws = u.shape
    if k.shape[0] != C or not (1 <= k.shape[1] <= Dd and 1 <= k.shape[2] <= Hs and 1 <= k.shape[3] <= Ws):
        raise ValueError("k must be [C,Kd,Kh,Kw] with Kd <= Dd, Kh <= Hs, Kw <= Ws")
    return u, k


def causal_conv3d(u, k) -> np.ndarray:
    """Full fp64 3-D oracle: the first-octant crop of the zero-padded linear
    convolution (the 3-D analogue of [:N]), by direct sums."""
    u, k = _check_3d(u, k)
    B, C, Dd, Hs, Ws = u.shape
    y = np.empty_like(u)
    _load().oracle_causal_conv3d(B, C, Dd, Hs, Ws, k.shape[1], k.shape[2], k.shape[3], _p(u), _p(k), _p(y))
    return y


def causal_conv3d_points(u, k, b_idx, c_idx, d_idx, i_idx, j_idx) -> np.ndarray:
    """fp64 3-D oracle at sampled voxels."""
    u, k = _check_3d(u, k)
    B, C, Dd, Hs, Ws = u.shape
    idx = [np.ascontiguousarray(a, dtype=np.int64) for a in (b_idx, c_idx, d_idx, i_idx, j_idx)]
    n = idx[0].size
    if any(a.shape != (n,) for a in idx):
        raise ValueError("index arrays must be 1-D and of equal length")
    if n and any(a.min() < 0 or a.max() >= m for a, m in zip(idx, (B, C, Dd, Hs, Ws))):
        raise ValueError("sample index out of range")
    out = np.empty(n, dtype=np.float64)
    _load().oracle_causal_conv3d_points(B, C, Dd, Hs, Ws, k.shape[1], k.shape[2], k.shape[3], _p(u), _p(k), n,
                                        *[_ip(a) for a in idx], _p(out))
    return out


def causal_conv2d_dynamic(u, k) -> np.ndarray:
    """fp64 2-D oracle with one filter per image ("Native Multi-Dimensional
    Subquadratic Operators via Input Dependent Long Convolutions", abstract):
    y[b, c] = first-quadrant crop of u[b, c] convolved with k[b, c]; k is
    [B][C][Kh][Kw].  Every image is its own channel of a one-image batch."""
    u = np.asarray(u, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    if u.ndim != 4 or k.ndim != 4 or k.shape[:2] != u.shape[:2]:
        raise ValueError("u must be [B, C, Hs, Ws] and k [B, C, Kh, Kw]")
    B, C, Hs, Ws = u.shape
    y = causal_conv2d(u.reshape(1, B * C, Hs, Ws), k.reshape(B * C, k.shape[2], k.shape[3]))
    return y.reshape(B, C, Hs, Ws)


def causal_conv2d_dynamic_points(u, k, b_idx, c_idx, i_idx, j_idx) -> np.ndarray:
    """causal_conv2d_dynamic at sampled pixels."""
    u = np.asarray(u, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    B, C, Hs, Ws = u.shape
    flat = np.asarray(b_idx, dtype=np.int64) * C + np.asarray(c_idx, dtype=np.int64)
    return causal_conv2d_points(u.reshape(1, B * C, Hs, Ws), k.reshape(B * C, k.shape[2], k.shape[3]),
                                np.zeros_like(flat), flat, i_idx, j_idx)


def causal_conv2d_offset(u, k, oy, ox) -> np.ndarray:
    """fp64 2-D oracle, crop window [oy, oy+Hs) x [ox, ox+Ws) of the full linear
    convolution (0, 0: the first-quadrant crop; Hs/2, Ws/2: the centred one)."""
    u, k = _check_2d(u, k)
    B, C, Hs, Ws = u.shape
    if not (0 <= oy <= Hs and 0 <= ox <= Ws):
        raise ValueError("offset outside [0, Hs] x [0, Ws]")
    y = np.empty_like(u)
    _load().oracle_causal_conv2d_offset(B, C, Hs, Ws, k.shape[1], k.shape[2], int(oy), int(ox), _p(u), _p(k), _p(y))
    return y


def causal_conv2d_points(u, k, b_idx, c_idx, i_idx, j_idx) -> np.ndarray:
    """fp64 2-D oracle at sampled pixels."""
    u, k = _check_2d(u, k)
    B, C, Hs, Ws = u.shape
    idx = [np.ascontiguousarray(a, dtype=np.int64) for a in (b_idx, c_idx, i_idx, j_idx)]
    n = idx[0].size
    if any(a.shape != (n,) for a in idx):
        raise ValueError("index arrays must be 1-D and of equal length")
    lims = (B, C, Hs, Ws)
    if n and any(a.min() < 0 or a.max() >= m for a, m in zip(idx, lims)):
        raise ValueError("sample index out of range")
    out = np.empty(n, dtype=np.float64)
    _load().oracle_causal_conv2d_points(B, C, Hs, Ws, k.shape[1], k.shape[2], _p(u), _p(k), n,
                                        *[_ip(a) for a in idx], _p(out))
    return out


def dft_causal_conv1d(x, k) -> np.ndarray:
    """Second route (tiny N): explicit length-2N DFT product, inverse, crop."""
    x = _f64(x)
    k = _f64(k)
    if x.ndim != 1 or k.ndim != 1 or not (1 <= k.size <= x.size):
        raise ValueError("x [N], k [L] with L <= N")
    y = np.empty_like(x)
    _load().oracle_dft_causal_conv1d(x.size, k.size, _p(x), _p(k), _p(y))
    return y


def dft_causal_conv2d(x, k) -> np.ndarray:
    """Second route for 2-D (tiny sizes): explicit (2Hs x 2Ws) DFT product, crop."""
    x = _f64(x)
    k = _f64(k)
    if x.ndim != 2 or k.ndim != 2 or k.shape[0] > x.shape[0] or k.shape[1] > x.shape[1]:
        raise ValueError("x [Hs,Ws], k [Kh,Kw] with Kh <= Hs, Kw <= Ws")
    y = np.empty_like(x)
    _load().oracle_dft_causal_conv2d(x.shape[0], x.shape[1], k.shape[0], k.shape[1],
                                     _p(x), _p(k), _p(y))
    return y


__all__ = ["causal_conv1d", "causal_conv1d_points", "causal_conv1d_bwd", "causal_conv1d_dynamic", "ssm_kernel", "freq_sparse_conv1d", "causal_conv2d", "causal_conv2d_points", "causal_conv2d_offset",
           "dft_causal_conv1d", "dft_causal_conv2d", "num_threads"]
