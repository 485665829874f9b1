/*
 * fftconv_oracle.c -- plain, slow, obviously correct CPU oracle for the causal
 * long convolution.  TEST INFRASTRUCTURE ONLY: it is called by the tests, by
 * __graft_entry__.smoke() and by bench.py's CPU-baseline leg, never by the
 * product path.  It shares no code, header, table or constant with the CUDA
 * library under fft_long_convolution_causal_b200/.
 *
 * Everything is IEEE fp64, accumulated in natural index order, compiled
 * without fast-math or FMA contraction.  Inputs are whatever the GPU path saw
 * (bf16 or fp32 values widened exactly to fp64).
 *
 * What it computes (citations are page title + part of the page):
 *
 *  1-D causal long convolution.  "FlashFFTConv: Efficient Convolutions for
 *  Long Sequences with Tensor Cores" (abstract) computes exact convolutions
 *  y = u * k in O(N log N) through the FFT; "RubiConv -- Efficient
 *  Boundary-Respecting Convolutions" (Caracal abstract) makes the FFT route
 *  causal by asymmetric zero padding and truncation.  Together this is
 *      y[t] = irfft(rfft(u,2N) . rfft(k,2N))[t],   t < N,
 *  which, because the full linear convolution of two length-<=N sequences is
 *  shorter than 2N (no wrap-around), is exactly the direct causal sum
 *      y[t] = sum_{s=0}^{min(t,L-1)} k[s] u[t-s].
 *  The oracle evaluates that sum directly.  A per-channel skip term D[h]*u[t]
 *  is added when D is given.
 *
 *  Gated form y = v (.) ((u (.) w) * k): the conv input is x = u*w and the
 *  result is multiplied by v; D (if given) applies to x inside the gate.
 *
 *  2-D variant.  "Native Multi-Dimensional Subquadratic Operators via Input
 *  Dependent Long Convolutions" (abstract: HyenaND convolves with global
 *  multi-dimensional kernels, FFT route).  Zero-padded linear convolution,
 *  first-quadrant crop (the 2-D analogue of [:N]):
 *      y[i][j] = sum_{p<=i} sum_{q<=j} k[p][q] u[i-p][j-q].
 *
 *  Independent second route for tiny sizes: the FFT formula itself, with the
 *  FFT replaced by an explicit O(M^2) DFT (fp64 cos/sin) of length M = 2N
 *  (2-D: 2Hs x 2Ws), pointwise product, inverse DFT, crop.
 *
 * Parity pins: every function is checked by tests/test_oracle_pins.py
 * against the numpy/scipy library routines for the same definition, closed
 * forms, identities (delta kernels, linearity, commutativity, causality,
 * shift invariance) and hand-derived fixtures under tests/golden/.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* One output of the 1-D causal convolution of row (b,h) at time t. */
static double conv1d_point(int64_t N, int64_t L, const double* ur, const double* wr,
                           const double* vr, const double* kr, const double* Dh, int64_t t)
{
    double acc = 0.0;
    int64_t smax = t < L - 1 ? t : L - 1;
    for (int64_t s = 0; s <= smax; ++s) {
        double x = wr ? ur[t - s] * wr[t - s] : ur[t - s];
        acc += kr[s] * x;
    }
    if (Dh) {
        double x = wr ? ur[t] * wr[t] : ur[t];
        acc += (*Dh) * x;
    }
    if (vr) acc *= vr[t];
    (void)N;
    return acc;
}

/*
 * Full 1-D oracle.  u, w, v, y: [B][H][N] row-major; k: [H][L]; D: [H] or NULL;
 * w and v are both NULL (ungated) or both non-NULL (gated).  L <= N.
 */
void oracle_causal_conv1d(int64_t B, int64_t H, int64_t N, int64_t L,
                          const double* u, const double* w, const double* v,
                          const double* k, const double* D, double* y)
{
    int64_t rows = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t h = r % H;
        const double* ur = u + r * N;
        const double* wr = w ? w + r * N : NULL;
        const double* vr = v ? v + r * N : NULL;
        const double* kr = k + h * L;
        const double* Dh = D ? D + h : NULL;
        for (int64_t t = 0; t < N; ++t)
            y[r * N + t] = conv1d_point(N, L, ur, wr, vr, kr, Dh, t);
    }
}

/* Sampled 1-D oracle: out[i] = y[bi[i], hi[i], ti[i]]. */
void oracle_causal_conv1d_points(int64_t B, int64_t H, int64_t N, int64_t L,
                                 const double* u, const double* w, const double* v,
                                 const double* k, const double* D, int64_t n_pts,
                                 const int64_t* bi, const int64_t* hi, const int64_t* ti,
                                 double* out)
{
    (void)B;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < n_pts; ++i) {
        int64_t r = bi[i] * H + hi[i];
        const double* ur = u + r * N;
        const double* wr = w ? w + r * N : NULL;
        const double* vr = v ? v + r * N : NULL;
        out[i] = conv1d_point(N, L, ur, wr, vr, k + hi[i] * L, D ? D + hi[i] : NULL, ti[i]);
    }
}

/*
 * Gradients of the 1-D causal convolution (the backward pass that training
 * the learned long filters of "Simple Hardware-Efficient Long Convolutions
 * for Sequence Modeling" (abstract) and "FlashFFTConv" (abstract) needs),
 * written as the chain rule applied to the forward definition above, term
 * by term, for a loss whose gradient with respect to y is dy:
 *   x = u (.) w (gated) or u;      g = dy (.) v (gated) or dy
 *   s[t]  = sum_{j <= min(t, L-1)} k[j] x[t-j] + D x[t]        (pre-gate output)
 *   dx[t] = sum_{j <= min(L-1, N-1-t)} k[j] g[t+j] + D g[t]     (y[t+j] depends on x[t] via k[j])
 *   du = dx (.) w or dx;   dw = dx (.) u;   dv = dy (.) s
 *   dk[h][j] = sum_b sum_{t >= j} g[b,h,t] x[b,h,t-j],  j < L
 *   dD[h]    = sum_b sum_t g[b,h,t] x[b,h,t]
 * Shapes as oracle_causal_conv1d; dv, dw are written only when gated (w, v
 * non-NULL); dD only when D is non-NULL.  fp64, natural order.
 */
void oracle_causal_conv1d_bwd(int64_t B, int64_t H, int64_t N, int64_t L,
                              const double* u, const double* w, const double* v,
                              const double* k, const double* D, const double* dy,
                              double* du, double* dv, double* dw, double* dk, double* dD)
{
    int64_t rows = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t h = r % H;
        const double* kr = k + h * L;
        const double* ur = u + r * N;
        const double* dyr = dy + r * N;
        for (int64_t t = 0; t < N; ++t) {
            double acc = 0.0;
            int64_t jmax = (L - 1 < N - 1 - t) ? L - 1 : N - 1 - t;
            for (int64_t j = 0; j <= jmax; ++j) {
                double g = v ? dyr[t + j] * v[r * N + t + j] : dyr[t + j];
                acc += kr[j] * g;
            }
            if (D) {
                double g = v ? dyr[t] * v[r * N + t] : dyr[t];
                acc += D[h] * g;
            }
            if (w) {
                du[r * N + t] = acc * w[r * N + t];
                dw[r * N + t] = acc * ur[t];
                /* dv = dy . s, s the pre-gate output at t */
                double sacc = 0.0;
                int64_t jtop = (t < L - 1) ? t : L - 1;
                for (int64_t j = 0; j <= jtop; ++j) sacc += kr[j] * (ur[t - j] * w[r * N + t - j]);
                if (D) sacc += D[h] * (ur[t] * w[r * N + t]);
                dv[r * N + t] = dyr[t] * sacc;
            } else {
                du[r * N + t] = acc;
            }
        }
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t h = 0; h < H; ++h) {
        for (int64_t j = 0; j < L; ++j) {
            double acc = 0.0;
            for (int64_t b = 0; b < B; ++b) {
                int64_t r = b * H + h;
                for (int64_t t = j; t < N; ++t) {
                    double g = v ? dy[r * N + t] * v[r * N + t] : dy[r * N + t];
                    double x = w ? u[r * N + t - j] * w[r * N + t - j] : u[r * N + t - j];
                    acc += g * x;
                }
            }
            dk[h * L + j] = acc;
        }
        if (D) {
            double acc = 0.0;
            for (int64_t b = 0; b < B; ++b) {
                int64_t r = b * H + h;
                for (int64_t t = 0; t < N; ++t) {
                    double g = v ? dy[r * N + t] * v[r * N + t] : dy[r * N + t];
                    double x = w ? u[r * N + t] * w[r * N + t] : u[r * N + t];
                    acc += g * x;
                }
            }
            dD[h] = acc;
        }
    }
}

/*
 * Input-dependent kernels ("Native Multi-Dimensional Subquadratic Operators
 * via Input Dependent Long Convolutions", abstract: HyenaND convolves with
 * input-dependent kernels): every batch row has its own filter,
 *   y[b,h,t] = sum_{s <= min(t, L-1)} k[b,h,s] x[b,h,t-s] + D[h] x[b,h,t],
 * x and the gate as in oracle_causal_conv1d.  k: [B][H][L].
 */
void oracle_causal_conv1d_dynamic(int64_t B, int64_t H, int64_t N, int64_t L,
                                  const double* u, const double* w, const double* v,
                                  const double* k, const double* D, double* y)
{
    int64_t rows = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t h = r % H;
        const double* ur = u + r * N;
        const double* wr = w ? w + r * N : NULL;
        const double* vr = v ? v + r * N : NULL;
        const double* kr = k + r * L;
        const double* Dh = D ? D + h : NULL;
        for (int64_t t = 0; t < N; ++t)
            y[r * N + t] = conv1d_point(N, L, ur, wr, vr, kr, Dh, t);
    }
}

/*
 * Filters of a diagonal state-space model, the setting of "FlashConv"
 * (Mechanism: state-space sequence convolutions, with the state passed
 * between chunks past the on-chip length): each channel's filter is
 *   k[h][t] = Re( sum_j c[h][j] lam[h][j]^t ),  t < L,
 * with complex lam (|lam| < 1) and c (the input and output maps folded into
 * c).  lam^t = |lam|^t (cos t.arg(lam) + i sin t.arg(lam)), in fp64.
 * lam, c: [H][d] as separate real / imaginary arrays; k: [H][L].
 */
void oracle_ssm_kernel(int64_t H, int64_t d, int64_t L, const double* lam_re, const double* lam_im,
                       const double* c_re, const double* c_im, double* k)
{
#pragma omp parallel for schedule(static)
    for (int64_t h = 0; h < H; ++h) {
        for (int64_t t = 0; t < L; ++t) {
            double acc = 0.0;
            for (int64_t j = 0; j < d; ++j) {
                double lr = lam_re[h * d + j], li = lam_im[h * d + j];
                double mag = pow(sqrt(lr * lr + li * li), (double)t);
                double ang = (double)t * atan2(li, lr);
                double pr = mag * cos(ang), pi = mag * sin(ang);
                acc += c_re[h * d + j] * pr - c_im[h * d + j] * pi;
            }
            k[h * L + t] = acc;
        }
    }
}

/* One output of the 2-D causal convolution of image (b,c) at (i,j). */
static double conv2d_point(int64_t Ws, int64_t Kh, int64_t Kw, const double* ui,
                           const double* kc, int64_t i, int64_t j)
{
    double acc = 0.0;
    int64_t pmax = i < Kh - 1 ? i : Kh - 1;
    int64_t qmax = j < Kw - 1 ? j : Kw - 1;
    for (int64_t p = 0; p <= pmax; ++p)
        for (int64_t q = 0; q <= qmax; ++q)
            acc += kc[p * Kw + q] * ui[(i - p) * Ws + (j - q)];
    return acc;
}

/* Full 2-D oracle.  u, y: [B][C][Hs][Ws]; k: [C][Kh][Kw], Kh <= Hs, Kw <= Ws. */
void oracle_causal_conv2d(int64_t B, int64_t C, int64_t Hs, int64_t Ws, int64_t Kh, int64_t Kw,
                          const double* u, const double* k, double* y)
{
    int64_t imgs = B * C;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < imgs; ++r) {
        int64_t c = r % C;
        const double* ui = u + r * Hs * Ws;
        const double* kc = k + c * Kh * Kw;
        for (int64_t i = 0; i < Hs; ++i)
            for (int64_t j = 0; j < Ws; ++j)
                y[r * Hs * Ws + i * Ws + j] = conv2d_point(Ws, Kh, Kw, ui, kc, i, j);
    }
}

/*
 * 2-D with a crop offset: the window [oy, oy + Hs) x [ox, ox + Ws) of the full
 * (2Hs - 1) x (2Ws - 1) linear convolution instead of its first quadrant
 * (oy = Hs/2, ox = Ws/2 is the centred "same" reading of a kernel anchored at
 * its middle).  y[i][j] = sum_{p,q} k[p][q] u[i + oy - p][j + ox - q] over the
 * indices inside both arrays.  0 <= oy <= Hs, 0 <= ox <= Ws.
 */
void oracle_causal_conv2d_offset(int64_t B, int64_t C, int64_t Hs, int64_t Ws, int64_t Kh, int64_t Kw,
                                 int64_t oy, int64_t ox, const double* u, const double* k, double* y)
{
    int64_t imgs = B * C;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < imgs; ++r) {
        int64_t c = r % C;
        const double* ui = u + r * Hs * Ws;
        const double* kc = k + c * Kh * Kw;
        for (int64_t i = 0; i < Hs; ++i)
            for (int64_t j = 0; j < Ws; ++j) {
                int64_t fi = i + oy, fj = j + ox;
                double acc = 0.0;
                for (int64_t p = 0; p < Kh; ++p) {
                    int64_t a = fi - p;
                    if (a < 0 || a >= Hs) continue;
                    for (int64_t q = 0; q < Kw; ++q) {
                        int64_t bq = fj - q;
                        if (bq < 0 || bq >= Ws) continue;
                        acc += kc[p * Kw + q] * ui[a * Ws + bq];
                    }
                }
                y[r * Hs * Ws + i * Ws + j] = acc;
            }
    }
}

/* Sampled 2-D oracle: out[n] = y[bi[n], ci[n], ii[n], jj[n]]. */
void oracle_causal_conv2d_points(int64_t B, int64_t C, int64_t Hs, int64_t Ws, int64_t Kh,
                                 int64_t Kw, const double* u, const double* k, int64_t n_pts,
                                 const int64_t* bi, const int64_t* ci, const int64_t* ii,
                                 const int64_t* jj, double* out)
{
    (void)B;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < n_pts; ++n) {
        const double* ui = u + (bi[n] * C + ci[n]) * Hs * Ws;
        const double* kc = k + ci[n] * Kh * Kw;
        out[n] = conv2d_point(Ws, Kh, Kw, ui, kc, ii[n], jj[n]);
    }
}

/*
 * 3-D variant ("Native Multi-Dimensional Subquadratic Operators via Input
 * Dependent Long Convolutions", abstract: the long convolution on native N-D
 * geometry), the first-octant crop of the zero-padded linear convolution:
 *     y[b,c,d,i,j] = sum_{e<=d, p<=i, q<=j} k[c,e,p,q] u[b,c,d-e,i-p,j-q],
 * d < Dd, i < Hs, j < Ws; k is [C][Kd][Kh][Kw] (taps outside it are zero).
 */
static double conv3d_point(int64_t Hs, int64_t Ws, int64_t Kd, int64_t Kh, int64_t Kw, const double* u,
                           const double* k, int64_t d, int64_t i, int64_t j)
{
    double acc = 0.0;
    int64_t emax = d < Kd - 1 ? d : Kd - 1;
    int64_t hmax = i < Kh - 1 ? i : Kh - 1;
    int64_t wmax = j < Kw - 1 ? j : Kw - 1;
    for (int64_t e = 0; e <= emax; ++e)
        for (int64_t p = 0; p <= hmax; ++p)
            for (int64_t q = 0; q <= wmax; ++q)
                acc += k[(e * Kh + p) * Kw + q] * u[((d - e) * Hs + (i - p)) * Ws + (j - q)];
    return acc;
}

void oracle_causal_conv3d(int64_t B, int64_t C, int64_t Dd, int64_t Hs, int64_t Ws, int64_t Kd, int64_t Kh,
                          int64_t Kw, const double* u, const double* k, double* y)
{
    int64_t vol = Dd * Hs * Ws, vols = B * C;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < vols; ++r) {
        int64_t c = r % C;
        const double* ur = u + r * vol;
        const double* kc = k + c * Kd * Kh * Kw;
        for (int64_t d = 0; d < Dd; ++d)
            for (int64_t i = 0; i < Hs; ++i)
                for (int64_t j = 0; j < Ws; ++j)
                    y[r * vol + (d * Hs + i) * Ws + j] = conv3d_point(Hs, Ws, Kd, Kh, Kw, ur, kc, d, i, j);
    }
}

/* Sampled 3-D oracle: out[n] = y[bi[n], ci[n], di[n], ii[n], jj[n]]. */
void oracle_causal_conv3d_points(int64_t B, int64_t C, int64_t Dd, int64_t Hs, int64_t Ws, int64_t Kd,
                                 int64_t Kh, int64_t Kw, const double* u, const double* k, int64_t n_pts,
                                 const int64_t* bi, const int64_t* ci, const int64_t* di, const int64_t* ii,
                                 const int64_t* jj, double* out)
{
    (void)B;
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t n = 0; n < n_pts; ++n) {
        const double* ur = u + (bi[n] * C + ci[n]) * Dd * Hs * Ws;
        const double* kc = k + ci[n] * Kd * Kh * Kw;
        out[n] = conv3d_point(Hs, Ws, Kd, Kh, Kw, ur, kc, di[n], ii[n], jj[n]);
    }
}

/* exp(-2*pi*i*m/M) for an integer m reduced mod M first, so the angle is exact. */
static void unit_root(int64_t m, int64_t M, double* re, double* im)
{
    int64_t r = m % M;
    if (r < 0) r += M;
    double ang = 2.0 * M_PI * (double)r / (double)M;
    *re = cos(ang);
    *im = -sin(ang);
}

/*
 * Second route, tiny N only: y = Re(iDFT_M(DFT_M(pad(x)) . DFT_M(pad(k))))[:N]
 * with M = 2N and explicit O(M^2) sums.  x: [N], k: [L], y: [N].
 */
void oracle_dft_causal_conv1d(int64_t N, int64_t L, const double* x, const double* k, double* y)
{
    int64_t M = 2 * N;
    double* Xr = calloc((size_t)M, sizeof(double));
    double* Xi = calloc((size_t)M, sizeof(double));
    double* Kr = calloc((size_t)M, sizeof(double));
    double* Ki = calloc((size_t)M, sizeof(double));
    for (int64_t f = 0; f < M; ++f) {
        double xr = 0, xi = 0, kr = 0, ki = 0, c, s;
        for (int64_t n = 0; n < N; ++n) {
            unit_root(f * n, M, &c, &s);
            xr += x[n] * c;
            xi += x[n] * s;
            if (n < L) {
                kr += k[n] * c;
                ki += k[n] * s;
            }
        }
        Xr[f] = xr; Xi[f] = xi; Kr[f] = kr; Ki[f] = ki;
    }
    for (int64_t t = 0; t < N; ++t) {
        double acc = 0.0, c, s;
        for (int64_t f = 0; f < M; ++f) {
            double pr = Xr[f] * Kr[f] - Xi[f] * Ki[f];
            double pi = Xr[f] * Ki[f] + Xi[f] * Kr[f];
            unit_root(-f * t, M, &c, &s); /* exp(+2 pi i f t / M) */
            acc += pr * c - pi * s;
        }
        y[t] = acc / (double)M;
    }
    free(Xr); free(Xi); free(Kr); free(Ki);
}

/*
 * Second route for 2-D, tiny sizes only: DFT of size (2Hs) x (2Ws) of the
 * zero-padded image and kernel, pointwise product, inverse DFT, crop to
 * [0,Hs) x [0,Ws).  x: [Hs][Ws], k: [Kh][Kw], y: [Hs][Ws].
 */
void oracle_dft_causal_conv2d(int64_t Hs, int64_t Ws, int64_t Kh, int64_t Kw,
                              const double* x, const double* k, double* y)
{
    int64_t Mh = 2 * Hs, Mw = 2 * Ws, MM = Mh * Mw;
    double* Pr = calloc((size_t)MM, sizeof(double));
    double* Pi = calloc((size_t)MM, sizeof(double));
    for (int64_t fh = 0; fh < Mh; ++fh)
        for (int64_t fw = 0; fw < Mw; ++fw) {
            double xr = 0, xi = 0, kr = 0, ki = 0, c1, s1, c2, s2;
            for (int64_t a = 0; a < Hs; ++a) {
                unit_root(fh * a, Mh, &c1, &s1);
                for (int64_t b = 0; b < Ws; ++b) {
                    unit_root(fw * b, Mw, &c2, &s2);
                    double c = c1 * c2 - s1 * s2, s = c1 * s2 + s1 * c2;
                    xr += x[a * Ws + b] * c;
                    xi += x[a * Ws + b] * s;
                    if (a < Kh && b < Kw) {
                        kr += k[a * Kw + b] * c;
                        ki += k[a * Kw + b] * s;
                    }
                }
            }
            Pr[fh * Mw + fw] = xr * kr - xi * ki;
            Pi[fh * Mw + fw] = xr * ki + xi * kr;
        }
    for (int64_t i = 0; i < Hs; ++i)
        for (int64_t j = 0; j < Ws; ++j) {
            double acc = 0.0, c1, s1, c2, s2;
            for (int64_t fh = 0; fh < Mh; ++fh) {
                unit_root(-fh * i, Mh, &c1, &s1);
                for (int64_t fw = 0; fw < Mw; ++fw) {
                    unit_root(-fw * j, Mw, &c2, &s2);
                    double c = c1 * c2 - s1 * s2, s = c1 * s2 + s1 * c2;
                    acc += Pr[fh * Mw + fw] * c - Pi[fh * Mw + fw] * s;
                }
            }
            y[i * Ws + j] = acc / (double)MM;
        }
    free(Pr); free(Pi);
}
