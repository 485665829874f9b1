"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each check raises AssertionError on failure.  They are collected as tests in
test_oracle_pins.py and re-run against deliberately broken copies of the
oracle in test_oracle_mutants.py, which shows that a plausible mistake anywhere
in the oracle fails at least one of them.

What pins what:
* the numpy FFT route of the defining formula y = irfft(rfft(x,2N) rfft(k,2N))[:N]
  (+ D x), written literally with numpy.fft ("FlashFFTConv: Efficient
  Convolutions for Long Sequences with Tensor Cores", abstract; causal padding:
  "RubiConv -- Efficient Boundary-Respecting Convolutions", Caracal abstract);
* numpy.convolve / scipy.signal.convolve2d, the library linear convolutions;
* closed forms (geometric kernel on a constant input; the first-order
  recursion that a geometric kernel satisfies, exact at any N);
* identities the definition fixes: delta kernel / delta input, linearity,
  commutativity, causality, shift invariance, 2-D separability;
* hand-derived fixtures in tests/golden/hand_examples.json.
"""
import json
import os

import numpy as np
import scipy.signal

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_examples.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _fft_formula_1d(x, k, D=None):
    """The defining formula with numpy's FFT as the library step (fp64)."""
    N = x.shape[-1]
    M = 2 * N
    y = np.fft.irfft(np.fft.rfft(x, M) * np.fft.rfft(k, M), M)[..., :N]
    if D is not None:
        y = y + D * x
    return y


def check_golden_1d():
    cases = json.load(open(GOLDEN))["cases_1d"]
    for c in cases:
        u = np.array(c["u"], float)[None, None]
        k = np.array(c["k"], float)[None]
        D = None if c["D"] is None else np.array([c["D"]], float)
        w = None if c["w"] is None else np.array(c["w"], float)[None, None]
        v = None if c["v"] is None else np.array(c["v"], float)[None, None]
        y = oracle.causal_conv1d(u, k, D=D, w=w, v=v)[0, 0]
        assert np.array_equal(y, np.array(c["y"], float)), (c["name"], y, c["y"])


def check_golden_2d():
    for c in json.load(open(GOLDEN))["cases_2d"]:
        u = np.array(c["u"], float)[None, None]
        k = np.array(c["k"], float)[None]
        y = oracle.causal_conv2d(u, k)[0, 0]
        assert np.array_equal(y, np.array(c["y"], float)), (c["name"], y, c["y"])


def check_fft_formula_1d():
    """Direct sum == the FFT formula written with numpy.fft, ungated and gated,
    L = N and L < N, with and without D, several N (powers of two and not)."""
    r = _rng(11)
    for (B, H, N, L) in [(2, 3, 64, 64), (1, 2, 1000, 1000), (2, 2, 256, 37), (1, 1, 1024, 1024)]:
        u = r.standard_normal((B, H, N))
        k = r.standard_normal((H, L)) * np.exp(-0.01 * np.arange(L))
        D = r.standard_normal(H)
        got = oracle.causal_conv1d(u, k, D=D)
        kp = np.zeros((H, N))
        kp[:, :L] = k
        want = np.stack([_fft_formula_1d(u[b], kp, D[:, None]) for b in range(B)])
        assert np.allclose(got, want, rtol=1e-11, atol=1e-11 * np.abs(want).max()), (B, H, N, L)
        got0 = oracle.causal_conv1d(u, k)
        want0 = np.stack([_fft_formula_1d(u[b], kp) for b in range(B)])
        assert np.allclose(got0, want0, rtol=1e-11, atol=1e-11 * np.abs(want0).max())
        # gated: y = v * ((u*w) conv k + D (u*w))
        w = r.standard_normal((B, H, N))
        v = r.standard_normal((B, H, N))
        gotg = oracle.causal_conv1d(u, k, D=D, w=w, v=v)
        wantg = np.stack([v[b] * _fft_formula_1d(u[b] * w[b], kp, D[:, None]) for b in range(B)])
        assert np.allclose(gotg, wantg, rtol=1e-11, atol=1e-11 * np.abs(wantg).max())


def check_numpy_convolve_1d():
    r = _rng(12)
    for N, L in [(1, 1), (5, 3), (64, 64), (300, 17)]:
        x = r.standard_normal(N)
        k = r.standard_normal(L)
        got = oracle.causal_conv1d(x[None, None], k[None])[0, 0]
        want = np.convolve(x, k)[:N]
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12), (N, L)


def check_dft_route_1d():
    """The oracle's explicit-DFT route equals numpy's FFT formula and the direct sum."""
    r = _rng(13)
    for N, L in [(1, 1), (4, 4), (16, 9), (64, 64), (33, 33)]:
        x = r.standard_normal(N)
        k = r.standard_normal(L)
        kp = np.zeros(N)
        kp[:L] = k
        d = oracle.dft_causal_conv1d(x, k)
        f = _fft_formula_1d(x, kp)
        s = oracle.causal_conv1d(x[None, None], k[None])[0, 0]
        scale = max(1.0, np.abs(f).max())
        assert np.allclose(d, f, rtol=0, atol=1e-12 * scale * N), (N, L)
        assert np.allclose(d, s, rtol=0, atol=1e-12 * scale * N), (N, L)


def check_delta_identities():
    r = _rng(14)
    B, H, N = 2, 3, 97
    u = r.standard_normal((B, H, N))
    k = r.standard_normal((H, N))
    delta_k = np.zeros((H, N))
    delta_k[:, 0] = 1.0
    assert np.array_equal(oracle.causal_conv1d(u, delta_k), u)
    D = r.standard_normal(H)
    assert np.allclose(oracle.causal_conv1d(u, delta_k, D=D), u * (1.0 + D[:, None]), rtol=1e-15, atol=0)
    delta_u = np.zeros((B, H, N))
    delta_u[:, :, 0] = 1.0
    assert np.array_equal(oracle.causal_conv1d(delta_u, k), np.broadcast_to(k, (B, H, N)))
    # kernel shorter than the sequence: u = delta returns k followed by zeros
    ks = r.standard_normal((H, 40))
    want = np.zeros((B, H, N))
    want[:, :, :40] = ks
    assert np.array_equal(oracle.causal_conv1d(delta_u, ks), want)


def check_linearity_commutativity():
    r = _rng(15)
    B, H, N = 1, 2, 128
    u1, u2 = r.standard_normal((2, B, H, N))
    k1, k2 = r.standard_normal((2, H, N))
    a, b = 0.75, -1.25
    lhs = oracle.causal_conv1d(a * u1 + b * u2, k1)
    rhs = a * oracle.causal_conv1d(u1, k1) + b * oracle.causal_conv1d(u2, k1)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-12)
    lhs = oracle.causal_conv1d(u1, a * k1 + b * k2)
    rhs = a * oracle.causal_conv1d(u1, k1) + b * oracle.causal_conv1d(u1, k2)
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-12)
    # commutativity u*k = k*u (both length N, one row per channel)
    yk = oracle.causal_conv1d(u1, k1)
    ku = oracle.causal_conv1d(k1[None], u1[0])
    assert np.allclose(yk, ku, rtol=1e-12, atol=1e-12)


def check_causality_shift():
    r = _rng(16)
    H, N = 2, 200
    u = r.standard_normal((1, H, N))
    k = r.standard_normal((H, N))
    y = oracle.causal_conv1d(u, k)
    for t0 in (0, 1, 57, N - 1):
        up = u.copy()
        up[:, :, t0] += 3.0
        yp = oracle.causal_conv1d(up, k)
        assert np.array_equal(yp[:, :, :t0], y[:, :, :t0]), t0
        assert not np.array_equal(yp[:, :, t0], y[:, :, t0]), t0
    # delaying u by s delays y by s
    s = 13
    us = np.zeros_like(u)
    us[:, :, s:] = u[:, :, :N - s]
    ys = oracle.causal_conv1d(us, k)
    assert np.allclose(ys[:, :, s:], y[:, :, :N - s], rtol=1e-12, atol=1e-12)
    assert np.array_equal(ys[:, :, :s], np.zeros((1, H, s)))


def check_closed_forms():
    # k[t] = a^t on u = 1: y[t] = (1 - a^(t+1)) / (1 - a)
    N, a = 500, 0.97
    t = np.arange(N)
    y = oracle.causal_conv1d(np.ones((1, 1, N)), (a ** t)[None])[0, 0]
    assert np.allclose(y, (1 - a ** (t + 1)) / (1 - a), rtol=1e-12, atol=0)
    # k[t] = c a^t on any u: y[t] = a y[t-1] + c u[t]  (exact at any N)
    r = _rng(17)
    N, a, c = 4096, 0.999, -0.7
    u = r.standard_normal(N)
    y = oracle.causal_conv1d(u[None, None], (c * a ** np.arange(N))[None])[0, 0]
    rec = np.empty(N)
    acc = 0.0
    for i in range(N):
        acc = a * acc + c * u[i]
        rec[i] = acc
    assert np.allclose(y, rec, rtol=1e-9, atol=1e-9 * np.abs(rec).max())


def check_points_match_full_1d():
    r = _rng(18)
    B, H, N = 3, 4, 150
    u, w, v = r.standard_normal((3, B, H, N))
    k = r.standard_normal((H, 120))
    D = r.standard_normal(H)
    full = oracle.causal_conv1d(u, k, D=D, w=w, v=v)
    bi = r.integers(0, B, 200)
    hi = r.integers(0, H, 200)
    ti = r.integers(0, N, 200)
    pts = oracle.causal_conv1d_points(u, k, bi, hi, ti, D=D, w=w, v=v)
    assert np.array_equal(pts, full[bi, hi, ti])


def check_conv2d_library():
    r = _rng(19)
    for (Hs, Ws, Kh, Kw) in [(1, 1, 1, 1), (7, 5, 7, 5), (16, 16, 16, 16), (12, 20, 5, 9)]:
        u = r.standard_normal((2, 2, Hs, Ws))
        k = r.standard_normal((2, Kh, Kw))
        got = oracle.causal_conv2d(u, k)
        for b in range(2):
            for c in range(2):
                want = scipy.signal.convolve2d(u[b, c], k[c], mode="full")[:Hs, :Ws]
                assert np.allclose(got[b, c], want, rtol=1e-12, atol=1e-12), (Hs, Ws, Kh, Kw)


def check_conv2d_separable_and_dft():
    r = _rng(20)
    Hs, Ws = 12, 10
    u1, k1 = r.standard_normal((2, Hs))
    u2, k2 = r.standard_normal((2, Ws))
    y = oracle.causal_conv2d(np.outer(u1, u2)[None, None], np.outer(k1, k2)[None])[0, 0]
    y1 = oracle.causal_conv1d(u1[None, None], k1[None])[0, 0]
    y2 = oracle.causal_conv1d(u2[None, None], k2[None])[0, 0]
    assert np.allclose(y, np.outer(y1, y2), rtol=1e-12, atol=1e-12)
    x = r.standard_normal((6, 5))
    k = r.standard_normal((4, 5))
    d = oracle.dft_causal_conv2d(x, k)
    s = oracle.causal_conv2d(x[None, None], k[None])[0, 0]
    f = np.fft.irfft2(np.fft.rfft2(x, (12, 10)) * np.fft.rfft2(k, (12, 10)), (12, 10))[:6, :5]
    assert np.allclose(d, f, rtol=0, atol=1e-11)
    assert np.allclose(s, f, rtol=0, atol=1e-11)


def check_points_match_full_2d():
    r = _rng(21)
    u = r.standard_normal((2, 3, 9, 11))
    k = r.standard_normal((3, 9, 11))
    full = oracle.causal_conv2d(u, k)
    idx = [r.integers(0, m, 100) for m in (2, 3, 9, 11)]
    pts = oracle.causal_conv2d_points(u, k, *idx)
    assert np.array_equal(pts, full[tuple(idx)])


def _loss(u, k, D, w, v, dy):
    """The scalar <dy, y> of the forward oracle: its gradients are the backward."""
    return float(np.sum(dy * oracle.causal_conv1d(u, k, D=D, w=w, v=v)))


def check_bwd_central_differences():
    """The backward oracle against central differences of the (pinned) forward
    oracle.  The loss <dy, y> is linear in each of u, k, D, v and w separately,
    so a central difference has no truncation error: the two agree to
    rounding, for every gradient entry, gated and ungated, L < N."""
    r = _rng(61)
    for gated, L in ((False, 9), (True, 12), (True, 5)):
        B, H, N = 2, 2, 12
        u = r.standard_normal((B, H, N))
        k = r.standard_normal((H, L))
        D = r.standard_normal(H)
        dy = r.standard_normal((B, H, N))
        w = r.standard_normal((B, H, N)) if gated else None
        v = r.standard_normal((B, H, N)) if gated else None
        g = oracle.causal_conv1d_bwd(u, k, dy, D=D, w=w, v=v)
        eps = 0.5
        args = {"u": u, "k": k, "D": D, "w": w, "v": v}
        for name in ("u", "k", "D") + (("w", "v") if gated else ()):
            base = args[name]
            num = np.empty_like(base)
            for idx in np.ndindex(base.shape):
                plus, minus = base.copy(), base.copy()
                plus[idx] += eps
                minus[idx] -= eps
                lp = _loss(**{**args, name: plus}, dy=dy)
                lm = _loss(**{**args, name: minus}, dy=dy)
                num[idx] = (lp - lm) / (2 * eps)
            got = g["d" + name]
            assert np.allclose(got, num, rtol=1e-9, atol=1e-9), (name, gated, np.abs(got - num).max())


def check_bwd_numpy_correlate():
    """dx and dk against numpy.correlate (the library cross-correlation):
    dx[t] = sum_j k[j] g[t+j] is correlate(g, k) at lags 0..N-1, and
    dk[j] = sum_b sum_t g[t] x[t-j] is sum_b correlate(g_b, x_b) at lags 0..L-1."""
    r = _rng(62)
    B, H, N, L = 3, 2, 40, 17
    u = r.standard_normal((B, H, N))
    k = r.standard_normal((H, L))
    dy = r.standard_normal((B, H, N))
    g = oracle.causal_conv1d_bwd(u, k, dy)
    for b in range(B):
        for h in range(H):
            full = np.correlate(dy[b, h], k[h], mode="full")  # index N-1+lag? see below
            # numpy: c[n] = sum_m a[n+m-(len(v)-1)] v[m]; lag 0 of a against v is n = L-1
            want = full[L - 1:L - 1 + N]
            assert np.allclose(g["du"][b, h], want, rtol=1e-12, atol=1e-12)
    for h in range(H):
        acc = np.zeros(L)
        for b in range(B):
            c = np.correlate(dy[b, h], u[b, h], mode="full")  # lag j of dy against u at N-1+j
            acc += c[N - 1:N - 1 + L]
        assert np.allclose(g["dk"][h], acc, rtol=1e-12, atol=1e-11)


def check_bwd_delta_kernel():
    """k = delta, D = 0: y = u, so du = dy exactly and dk[j] = sum_b <dy, u shifted by j>."""
    r = _rng(63)
    B, H, N = 2, 1, 10
    u = r.standard_normal((B, H, N))
    dy = r.standard_normal((B, H, N))
    k = np.zeros((H, 4))
    k[:, 0] = 1.0
    g = oracle.causal_conv1d_bwd(u, k, dy, D=np.zeros(H))
    assert np.array_equal(g["du"], dy)
    for j in range(4):
        assert np.isclose(g["dk"][0, j], float(np.sum(dy[:, 0, j:] * u[:, 0, :N - j])), rtol=1e-13)
    assert np.isclose(g["dD"][0], float(np.sum(dy * u)), rtol=1e-13)


def check_dynamic_kernels():
    """Per-row filters: numpy.convolve row by row (the library routine), the
    shared-filter oracle when every row carries its channel's filter, and row
    independence (changing one row's filter changes only that row)."""
    r = _rng(64)
    B, H, N, L = 3, 2, 33, 20
    u = r.standard_normal((B, H, N))
    k = r.standard_normal((B, H, L))
    D = r.standard_normal(H)
    y = oracle.causal_conv1d_dynamic(u, k, D=D)
    for b in range(B):
        for h in range(H):
            want = np.convolve(u[b, h], k[b, h])[:N] + D[h] * u[b, h]
            assert np.allclose(y[b, h], want, rtol=1e-12, atol=1e-12)
    shared = np.broadcast_to(k[0][None], k.shape).copy()
    w = r.standard_normal((B, H, N))
    v = r.standard_normal((B, H, N))
    assert np.array_equal(oracle.causal_conv1d_dynamic(u, shared, D=D, w=w, v=v),
                          oracle.causal_conv1d(u, k[0], D=D, w=w, v=v))
    k2 = k.copy()
    k2[1, 0] += 1.0
    y2 = oracle.causal_conv1d_dynamic(u, k2, D=D)
    changed = np.any(y2 != y, axis=2)
    assert changed[1, 0] and changed.sum() == 1


def check_ssm_kernel():
    """State-space filters: numpy's complex power (the library routine); the
    conjugate-pair closed form 2 |c| |lam|^t cos(t arg lam + arg c); and the
    state-space recursion itself -- s_j[t] = lam_j s_j[t-1] + x[t],
    y[t] = Re(sum_j c_j s_j[t]) + D x[t], run in fp64 -- equal to the causal
    convolution oracle with the materialised filter (the state-space view a
    chunked computation passes between chunks)."""
    r = _rng(65)
    H, d, L = 2, 4, 300
    lam = (r.uniform(0.9, 0.999, (H, d)) * np.exp(1j * r.uniform(-1.0, 1.0, (H, d))))
    c = r.standard_normal((H, d)) + 1j * r.standard_normal((H, d))
    k = oracle.ssm_kernel(lam, c, L)
    t = np.arange(L)
    want = np.real(np.sum(c[:, :, None] * lam[:, :, None] ** t[None, None, :], axis=1))
    assert np.allclose(k, want, rtol=1e-11, atol=1e-11)
    lam1 = np.array([[0.97 * np.exp(0.3j), 0.97 * np.exp(-0.3j)]])
    c1 = np.array([[0.5 - 0.25j, 0.5 + 0.25j]])
    want1 = 2 * abs(c1[0, 0]) * 0.97 ** t * np.cos(0.3 * t + np.angle(c1[0, 0]))
    assert np.allclose(oracle.ssm_kernel(lam1, c1, L)[0], want1, rtol=1e-11, atol=1e-12)
    B, N = 2, 300
    x = r.standard_normal((B, H, N))
    D = r.standard_normal(H)
    y = oracle.causal_conv1d(x, k, D=D)
    s = np.zeros((B, H, d), dtype=np.complex128)
    rec = np.empty((B, H, N))
    for tt in range(N):
        s = lam[None] * s + x[:, :, tt:tt + 1]
        rec[:, :, tt] = np.real(np.sum(c[None] * s, axis=2)) + D[None] * x[:, :, tt]
    assert np.allclose(y, rec, rtol=1e-9, atol=1e-9)


def check_freq_sparse():
    """Frequency-sparse form: an all-true mask gives the direct sum; a masked
    case equals the same formula written with explicit O(M^2) DFT matrices
    (no FFT library); a Hermitian-symmetric mask keeps the result real and
    linear in u."""
    r = _rng(66)
    B, H, N, L = 2, 2, 32, 20
    u = r.standard_normal((B, H, N))
    k = r.standard_normal((H, L))
    D = r.standard_normal(H)
    G = 8
    full = oracle.freq_sparse_conv1d(u, k, np.ones(G, bool), D=D)
    assert np.allclose(full, oracle.causal_conv1d(u, k, D=D), rtol=1e-11, atol=1e-11)
    keep = np.array([1, 0, 1, 1, 0, 1, 1, 0], bool)  # keep[j] == keep[(G - j) % G]
    assert all(keep[j] == keep[(G - j) % G] for j in range(G))
    y = oracle.freq_sparse_conv1d(u, k, keep, D=D)
    M = 2 * N
    f = np.arange(M)
    F = np.exp(-2j * np.pi * np.outer(f, f) / M)            # explicit DFT matrix
    up = np.zeros((B, H, M)); up[..., :N] = u
    kp = np.zeros((H, M)); kp[:, :L] = k
    Kf = (F @ kp.T).T + D[:, None]
    Yf = np.einsum("fm,bhm->bhf", F, up) * (Kf * keep[f % G])[None]
    want = np.einsum("nf,bhf->bhn", np.conj(F), Yf)[..., :N] / M
    assert np.allclose(want.imag, 0, atol=1e-9)
    assert np.allclose(y, want.real, rtol=1e-10, atol=1e-10)
    y2 = oracle.freq_sparse_conv1d(2.0 * u, k, keep, D=D)
    assert np.allclose(y2, 2.0 * y, rtol=1e-12, atol=1e-12)


def check_conv2d_dynamic():
    """Per-image 2-D filters: filters equal across the batch give the
    shared-filter oracle; every image is scipy.signal.convolve2d's full linear
    convolution of its own image and filter, cropped to the first quadrant;
    the sampled entry point matches the full one."""
    from scipy.signal import convolve2d
    r = _rng(68)
    B, C, Hs, Ws, Kh, Kw = 3, 2, 8, 16, 5, 7
    u = r.standard_normal((B, C, Hs, Ws))
    kc = r.standard_normal((C, Kh, Kw))
    same = oracle.causal_conv2d_dynamic(u, np.broadcast_to(kc, (B, C, Kh, Kw)))
    assert np.allclose(same, oracle.causal_conv2d(u, kc), rtol=1e-12, atol=1e-12)
    k = r.standard_normal((B, C, Kh, Kw))
    y = oracle.causal_conv2d_dynamic(u, k)
    for b in range(B):
        for c in range(C):
            want = convolve2d(u[b, c], k[b, c])[:Hs, :Ws]
            assert np.allclose(y[b, c], want, rtol=1e-11, atol=1e-11), (b, c)
    bi, ci = np.array([0, 2, 1, 2]), np.array([1, 0, 1, 1])
    ii, jj = np.array([0, 7, 3, 5]), np.array([15, 0, 9, 4])
    pts = oracle.causal_conv2d_dynamic_points(u, k, bi, ci, ii, jj)
    assert np.allclose(pts, y[bi, ci, ii, jj], rtol=1e-12, atol=1e-12)


def check_conv3d():
    """3-D first-octant crop: scipy.signal.convolve's full N-D linear
    convolution (direct method) cropped; one depth slice is the 2-D oracle;
    a separable volume and filter give the product of three 1-D causal
    convolutions; the delta filter returns u; the sampled entry point
    matches the full one."""
    from scipy.signal import convolve
    r = _rng(69)
    B, C, Dd, Hs, Ws, Kd, Kh, Kw = 2, 2, 4, 8, 16, 3, 5, 16
    u = r.standard_normal((B, C, Dd, Hs, Ws))
    k = r.standard_normal((C, Kd, Kh, Kw))
    y = oracle.causal_conv3d(u, k)
    for b in range(B):
        for c in range(C):
            want = convolve(u[b, c], k[c], method="direct")[:Dd, :Hs, :Ws]
            assert np.allclose(y[b, c], want, rtol=1e-11, atol=1e-11), (b, c)
    flat = oracle.causal_conv3d(u[:, :, :1], k[:, :1])
    assert np.allclose(flat[:, :, 0], oracle.causal_conv2d(u[:, :, 0], k[:, 0]), rtol=1e-12, atol=1e-12)
    a1, a2, a3 = r.standard_normal(Dd), r.standard_normal(Hs), r.standard_normal(Ws)
    f1, f2, f3 = r.standard_normal(Kd), r.standard_normal(Kh), r.standard_normal(Kw)
    us = np.einsum("d,i,j->dij", a1, a2, a3)[None, None]
    ks = np.einsum("d,i,j->dij", f1, f2, f3)[None]
    sep = np.einsum("d,i,j->dij", np.convolve(a1, f1)[:Dd], np.convolve(a2, f2)[:Hs], np.convolve(a3, f3)[:Ws])
    assert np.allclose(oracle.causal_conv3d(us, ks)[0, 0], sep, rtol=1e-11, atol=1e-11)
    delta = np.zeros((C, Kd, Kh, Kw))
    delta[:, 0, 0, 0] = 1.0
    assert np.array_equal(oracle.causal_conv3d(u, delta), u)
    bi, ci, di = np.array([0, 1, 1]), np.array([1, 0, 1]), np.array([3, 0, 2])
    ii, jj = np.array([7, 0, 4]), np.array([15, 3, 0])
    pts = oracle.causal_conv3d_points(u, k, bi, ci, di, ii, jj)
    assert np.allclose(pts, y[bi, ci, di, ii, jj], rtol=1e-12, atol=1e-12)


def check_conv2d_offset():
    """Crop offsets: (0, 0) is the first-quadrant oracle; any offset is the
    window of scipy.signal.convolve2d's full linear convolution."""
    r = _rng(67)
    u = r.standard_normal((2, 2, 12, 10))
    k = r.standard_normal((2, 7, 10))
    assert np.array_equal(oracle.causal_conv2d_offset(u, k, 0, 0), oracle.causal_conv2d(u, k))
    for oy, ox in ((6, 5), (12, 10), (3, 0), (0, 8)):
        y = oracle.causal_conv2d_offset(u, k, oy, ox)
        for b in range(2):
            for c in range(2):
                full = scipy.signal.convolve2d(u[b, c], k[c], mode="full")
                want = np.zeros((12, 10))
                win = full[oy:oy + 12, ox:ox + 10]
                want[:win.shape[0], :win.shape[1]] = win
                assert np.allclose(y[b, c], want, rtol=1e-12, atol=1e-12), (oy, ox)


ALL_CHECKS = [
    check_golden_1d, check_golden_2d, check_fft_formula_1d, check_numpy_convolve_1d,
    check_dft_route_1d, check_delta_identities, check_linearity_commutativity,
    check_causality_shift, check_closed_forms, check_points_match_full_1d,
    check_conv2d_library, check_conv2d_separable_and_dft, check_points_match_full_2d,
    check_bwd_central_differences, check_bwd_numpy_correlate, check_bwd_delta_kernel, check_dynamic_kernels,
    check_ssm_kernel, check_freq_sparse, check_conv2d_offset, check_conv2d_dynamic, check_conv3d,
]
