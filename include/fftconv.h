/*
 * fftconv.h -- C ABI of the B200 causal FFT long-convolution library
 * (libfftconv_b200.so).  Plain pointers and sizes only; no C++ or torch types.
 *
 * The operation.  For each batch row b and channel h,
 *
 *     y[b,h,:] = irfft(rfft(x[b,h,:], 2N) . rfft(k[h,:], 2N))[:N] + D[h] x[b,h,:]
 *
 * with x = u (ungated) or x = u (.) w and the result multiplied by v (gated,
 * y = v (.) ((u (.) w) * k + D (u (.) w))).  This is the exact FFT convolution
 * of "FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor
 * Cores" (abstract: O(N log N) FFT convolution, FFT as a matrix decomposition
 * on matmul units, kernel fusion), made causal by zero-padding to 2N and
 * truncating to [:N] as in "RubiConv -- Efficient Boundary-Respecting
 * Convolutions" (Caracal abstract: asymmetric padding and truncation); the
 * fused FFT -> pointwise product -> inverse FFT on chip follows "FlashConv"
 * (Mechanism).  The 2-D variant is the zero-padded linear convolution
 * cropped to the first quadrant, the multi-dimensional FFT convolution of
 * "Native Multi-Dimensional Subquadratic Operators via Input Dependent Long
 * Convolutions" (abstract), with one fixed kernel per channel.
 *
 * Memory and ownership.  Every large buffer (u, v, w, k, D, y, the spectrum
 * khat and the workspace) is device memory owned by the caller.  A plan owns
 * only small constant tables (twiddle factors), allocated by the *_create
 * call and released by fftconv_plan_destroy.  All tensors are dense and
 * row-major with the last dimension fastest:
 *     u, v, w, y : [B][H][N]          (fp32 or bf16, per the plan's dtype)
 *     k          : [H][L], L <= N     (fp32)
 *     D          : [H]                (fp32) or NULL
 *     2-D u, y   : [B][C][Hs][Ws]     k : [C][Kh][Kw] (fp32), Kh <= Hs, Kw <= Ws
 * Device pointers must be 16-byte aligned.  khat is an opaque buffer of
 * fftconv_spectrum_bytes() bytes, valid only for the plan that wrote it.
 *
 * Errors.  Every call returns a status and never throws.  Argument errors are
 * detected on the host before anything is launched.  FFTCONV_ERR_CUDA reports
 * a launch error (cudaGetLastError); a fault inside a kernel surfaces at the
 * caller's next synchronisation, as for any CUDA call.
 *
 * Streams.  Work is enqueued on the given stream (a cudaStream_t passed as
 * void*, NULL = legacy default stream) and returns without synchronising.  A
 * plan may be used by several streams for fftconv_fwd at once provided each
 * call gets its own workspace; plan creation and destruction are not
 * thread-safe with respect to other calls on the same plan.
 *
 * Graph capture.  The forward calls (fftconv_fwd, fftconv2d_fwd(_offset),
 * fftconv2d_fwd_dynamic, fftconv3d_fwd, and the forward of partial and
 * state-passing plans) and fftconv_bwd enqueue only kernel launches on the
 * given stream, so they may be captured into a CUDA graph once the same kind
 * of call has run eagerly in the process (that first call sets the kernels'
 * shared-memory limits).  A replay reads and writes the buffers named at
 * capture.  Plan creation, fftconv_spectrum_sparsify and
 * fftconv_device_status synchronise and are not capturable.
 */
#ifndef FFTCONV_H
#define FFTCONV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FFTCONV_API __attribute__((visibility("default")))
#else
#define FFTCONV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct fftconv_plan_s* fftconv_plan_t;

typedef enum {
    FFTCONV_OK = 0,
    FFTCONV_ERR_INVALID_ARG = 1, /* NULL/misaligned pointer, bad size, L > N, gated without v or w */
    FFTCONV_ERR_UNSUPPORTED = 2, /* N (or Hs, Ws) not a power of two in the supported range      */
    FFTCONV_ERR_NOT_READY = 3,   /* fftconv_fwd before any fftconv_kernel_spectrum on this plan   */
    FFTCONV_ERR_OOM = 4,         /* the plan's small tables could not be allocated               */
    FFTCONV_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed                  */
    FFTCONV_ERR_TIMEOUT = 6      /* a bounded device-side wait gave up (fftconv_device_status)   */
} fftconv_status;

typedef enum {
    FFTCONV_F32 = 0,  /* u, v, w, y in fp32; arithmetic in fp32                              */
    FFTCONV_BF16 = 1  /* u, v, w, y in bf16; transforms on bf16 tensor cores, fp32 accumulate */
} fftconv_dtype;

/* Kernel family a plan may use (fftconv_plan_options.kernel).  Every choice
 * computes the same convolution and passes the same parity tests; the choice
 * exists for measurement and for callers that pin one implementation. */
typedef enum {
    FFTCONV_KERNEL_AUTO = 0,     /* the library's choice: the fastest measured kernel for the size  */
    FFTCONV_KERNEL_SIMT = 1,     /* fp32 SIMT transforms only (bf16 I/O is still accepted)          */
    FFTCONV_KERNEL_MMA_SYNC = 2, /* bf16 plans: warp-level mma.sync tensor-core kernels             */
    FFTCONV_KERNEL_TCGEN05 = 3   /* bf16 plans: tcgen05 kernels where one exists for the size, else */
                                 /* the AUTO choice                                                  */
} fftconv_kernel;

/* Plan options.  Zero-initialise, or call fftconv_plan_options_init, then set
 * the fields to change; a NULL options pointer means the defaults. */
typedef struct {
    int kernel;          /* fftconv_kernel; default FFTCONV_KERNEL_AUTO                           */
    size_t group_bytes;  /* multi-pass and 2-D paths: workspace per group of row pairs processed  */
                         /* per launch; 0 = the default (1 GiB).  Smaller groups need less       */
                         /* workspace and run more launches; a group always holds >= 1 pair.     */
} fftconv_plan_options;

/* Default probes of a bounded device wait (each probe sleeps up to about
 * 20 us, so the default gives up after roughly a second). */
#define FFTCONV_DEFAULT_WAIT_PROBES 65536u

/* Supported sizes: 1-D N a power of two, FFTCONV_MIN_N <= N <= FFTCONV_MAX_N;
 * 2-D Hs, Ws powers of two in [FFTCONV2D_MIN_SIDE, FFTCONV2D_MAX_SIDE]. */
#define FFTCONV_MIN_N 64
#define FFTCONV_MAX_N (1 << 20)
#define FFTCONV2D_MIN_SIDE 16
#define FFTCONV2D_MAX_SIDE 256

/* Fill *opts with the defaults. */
FFTCONV_API void fftconv_plan_options_init(fftconv_plan_options* opts);

/*
 * Create a 1-D plan for B batch rows, H channels, sequence length N, I/O type
 * dtype, gated (nonzero) or not.  Chooses the execution path: a single fused
 * kernel per (channel, pair of batch rows) when the transform of length 2N
 * fits on chip ("FlashConv", Mechanism: FFT, product and inverse fused on
 * chip), else the multi-pass path that stages partial transforms in the
 * caller's workspace (same block: chunking past the on-chip capacity).
 * Uploads the plan's twiddle tables (synchronously) on the current device,
 * which every later call on the plan must also have current.  On success
 * *plan receives the handle.  Same as fftconv_plan_create_ex with NULL
 * options.
 */
FFTCONV_API fftconv_status fftconv_plan_create(fftconv_plan_t* plan, int B, int H, int64_t N,
                                   fftconv_dtype dtype, int gated);

/* fftconv_plan_create with options (NULL = defaults).  FFTCONV_ERR_INVALID_ARG
 * for an unknown kernel choice. */
FFTCONV_API fftconv_status fftconv_plan_create_ex(fftconv_plan_t* plan, int B, int H, int64_t N,
                                                  fftconv_dtype dtype, int gated,
                                                  const fftconv_plan_options* opts);

/*
 * Create a 2-D plan: B images, C channels, Hs x Ws pixels, I/O type dtype.
 * The transform is (2Hs) x (2Ws) over the zero-padded image.
 */
FFTCONV_API fftconv_status fftconv2d_plan_create(fftconv_plan_t* plan, int B, int C, int Hs, int Ws,
                                     fftconv_dtype dtype);

/* fftconv2d_plan_create with options (NULL = defaults; FFTCONV_KERNEL_SIMT
 * keeps bf16 plans off the tensor cores, the other choices mean AUTO). */
FFTCONV_API fftconv_status fftconv2d_plan_create_ex(fftconv_plan_t* plan, int B, int C, int Hs, int Ws,
                                                    fftconv_dtype dtype, const fftconv_plan_options* opts);

/* Release a plan and its tables.  NULL is accepted.  Not valid while work
 * using the plan's tables is still pending on a stream. */
FFTCONV_API fftconv_status fftconv_plan_destroy(fftconv_plan_t plan);

/* Bytes the caller must provide for khat (the cached kernel spectrum). */
FFTCONV_API size_t fftconv_spectrum_bytes(fftconv_plan_t plan);

/* Bytes of device workspace fftconv_fwd / fftconv2d_fwd / the spectrum calls
 * need; 0 when the plan's path needs none (then workspace may be NULL). */
FFTCONV_API size_t fftconv_workspace_bytes(fftconv_plan_t plan);

/* Name of the execution path the plan chose: "fused" (fp32 on-chip),
 * "fused_tc" (bf16 on-chip, 2N <= 32768, warp-level mma.sync tensor cores),
 * "fused_umma" (the same factorisation on tcgen05 tensor cores, 2N = 4096,
 * or 8192 gated, with FFTCONV_KERNEL_TCGEN05), "fused_t2" (two-stage tcgen05
 * kernel, data held in tensor memory between the stages: the default for
 * ungated bf16 at 2N = 8192), "multipass", "2d", "2d_tc", "partial_chunked",
 * "ssm_chunked". */
FFTCONV_API const char* fftconv_plan_path(fftconv_plan_t plan);

/* Tensor-core floating-point operations (2 per multiply-add, as executed,
 * padding included) of one fftconv_fwd / fftconv2d_fwd call on this plan;
 * 0 for paths that run no tensor-core products.  Lets a caller report the
 * tensor-pipe fraction of a measured time. */
FFTCONV_API double fftconv_plan_mma_flops(fftconv_plan_t plan);

/* Probes each bounded device wait of this plan's kernels makes before it
 * gives up (default FFTCONV_DEFAULT_WAIT_PROBES; 0 = give up at the first
 * check).  A wait that gives up abandons its launch after draining the
 * products it has in flight, leaves y incomplete and sets the status word
 * that fftconv_device_status reports.  Takes effect from the next launch.
 * Plans whose kernels never wait accept and ignore it. */
FFTCONV_API fftconv_status fftconv_plan_set_wait_limit(fftconv_plan_t plan, uint32_t probes);

/*
 * Kernel spectrum: khat <- DFT_{2N}(k[h] zero-padded) / (2N) for every
 * channel, in the plan's internal order and precision.  k is [H][L] fp32 on
 * the device with 1 <= L <= N (taps past L are zero: a partial convolution,
 * "FlashFFTConv", abstract).  Computed once per filter set and reused by
 * every fftconv_fwd of the plan (the filter's FFT is the operand of the
 * pointwise spectral product, "FlashConv", Mechanism).
 */
FFTCONV_API fftconv_status fftconv_kernel_spectrum(fftconv_plan_t plan, const float* k, int64_t L,
                                       void* khat, void* workspace, void* stream);

/*
 * Forward: y = the causal convolution above ("FlashFFTConv", abstract: the
 * exact FFT convolution; "RubiConv -- Efficient Boundary-Respecting
 * Convolutions", Caracal abstract: causal by padding to 2N and truncating).
 * u is [B][H][N]; v and w are [B][H][N] for a gated plan and must be NULL
 * otherwise; khat is the output of fftconv_kernel_spectrum on this plan; D is
 * [H] fp32 or NULL (no skip term); y is [B][H][N] and must not alias any
 * input.  FFTCONV_ERR_INVALID_ARG also when the current device is not the
 * plan's.
 */
FFTCONV_API fftconv_status fftconv_fwd(fftconv_plan_t plan, const void* u, const void* v, const void* w,
                           const void* khat, const float* D, void* y, void* workspace,
                           void* stream);

/*
 * Forward with input-dependent filters: every batch row has its own filter,
 *     y[b,h,:] = (x[b,h,:] * k[b,h,:])[:N] + D[h] x[b,h,:]   (gated: times v),
 * the input-dependent long convolution of "Native Multi-Dimensional
 * Subquadratic Operators via Input Dependent Long Convolutions" (abstract).
 * k is [B][H][L] fp32 on the device, 1 <= L <= N, and is transformed inside
 * the same launch (no cached spectrum; fftconv_kernel_spectrum is not needed).
 * Other arguments as fftconv_fwd.  Runs an fp32 fused kernel for 2N <= 8192
 * on any 1-D plan of that size; FFTCONV_ERR_UNSUPPORTED for longer N.
 */
FFTCONV_API fftconv_status fftconv_fwd_dynamic(fftconv_plan_t plan, const void* u, const void* v, const void* w,
                                               const float* k, int64_t L, const float* D, void* y, void* stream);

/*
 * Frequency-sparse convolutions ("FlashFFTConv", abstract: frequency-sparse
 * convolutions, computed by skipping blocks of the matrix decomposition), on
 * multi-pass plans (2N >= 32768).  The transform splits 2N = G x (2N / G)
 * with frequency f = k1 + G k2; keep[k1] = 0 zeroes the spectrum (skip term
 * included) at every frequency of outer digit k1, and the kernels skip those
 * rows: pass 1 stores nothing for them, pass 2 skips CTAs whose rows are all
 * dropped, pass 3 reads zeros.  The result is
 *     y = Re(iDFT(DFT(pad x) . (DFT(pad k) + D) . m))[:N],  m[f] = keep[f mod G].
 * keep: host array of nblocks = fftconv_spectrum_blocks(plan) = G flags,
 * Hermitian-symmetric (keep[j] == keep[(G - j) mod G], else
 * FFTCONV_ERR_INVALID_ARG: the two packed rows would mix).  Zeroes the rows
 * of khat (the output of fftconv_kernel_spectrum on this plan) and records
 * the mask in the plan (a G-byte device array the plan owns); keep = NULL,
 * nblocks = 0 makes the plan dense again (recompute khat).  Synchronises the
 * stream.  FFTCONV_ERR_UNSUPPORTED for other plans.
 */
FFTCONV_API int fftconv_spectrum_blocks(fftconv_plan_t plan);
FFTCONV_API fftconv_status fftconv_spectrum_sparsify(fftconv_plan_t plan, void* khat, const uint8_t* keep,
                                                     int nblocks, void* stream);

/*
 * Partial convolutions: a filter of at most L_max taps, much shorter than the
 * rows ("FlashFFTConv", abstract: partial convolutions, computed by skipping
 * blocks of the matrix decomposition).  The row is cut into chunks of T (the
 * power of two >= max(L_max, 64), at most FFTCONV_PARTIAL_MAX_CHUNK, dividing
 * N); chunk c is the upper half of a 2T-point circular convolution over the
 * window [cT - T, cT + T), which equals y there exactly because the filter
 * is no longer than T.  Work and traffic scale with N log T and every chunk
 * runs on chip, whatever N.  Same calls as a 1-D plan: fftconv_kernel_spectrum
 * (1 <= L <= T taps; khat of fftconv_spectrum_bytes) and fftconv_fwd (gated
 * or not, D optional; no workspace).  Path name "partial_chunked".
 */
#define FFTCONV_PARTIAL_MAX_CHUNK 8192
FFTCONV_API fftconv_status fftconv_partial_plan_create(fftconv_plan_t* plan, int B, int H, int64_t N,
                                                       fftconv_dtype dtype, int gated, int64_t L_max);

/*
 * Filters of a diagonal state-space model, computed in chunks with the state
 * passed between them ("FlashConv", Mechanism: chunk convolutions past the
 * on-chip length with the state-space boundary state propagated between
 * chunks).  Channel h's filter is
 *     k[h][t] = Re( sum_{j < d} c[h][j] lam[h][j]^t ),   t < N,  |lam| < 1,
 * and the forward is the causal convolution of the header's first formula
 * with that k (ungated).  A row is split into chunks of T (a power of two in
 * [FFTCONV_SSM_MIN_CHUNK, FFTCONV_SSM_MAX_CHUNK] dividing N): each chunk is
 * convolved on chip with k[:T] (the fp32 fused kernel) and the contribution
 * of all earlier input, Re(sum_j c_j lam_j^t S_j), is added from the d
 * states S entering the chunk, which a scan carries from chunk to chunk.
 * The plan owns the chunk plan and a small table (lam, c, lam^(32 i));
 * khat (fftconv_spectrum_bytes) and the workspace (fftconv_workspace_bytes)
 * are the caller's.  Path name "ssm_chunked".
 */
#define FFTCONV_SSM_MAX_STATE 64
#define FFTCONV_SSM_MIN_CHUNK 64
#define FFTCONV_SSM_MAX_CHUNK 8192
FFTCONV_API fftconv_status fftconv_ssm_plan_create(fftconv_plan_t* plan, int B, int H, int64_t N,
                                                   fftconv_dtype dtype, int d_state, int64_t chunk);

/* Set the filters of a state-passing plan (the state-space filters of
 * "FlashConv", Mechanism, defined above): lam and c are [H][d] fp32 device
 * arrays (real and imaginary parts separately).  Materialises k[:T], writes
 * khat and keeps lam, c and their power table in the plan.  Then
 * fftconv_fwd(plan, u, NULL, NULL, khat, D, y, workspace, stream) runs the
 * chunked convolution. */
FFTCONV_API fftconv_status fftconv_ssm_spectrum(fftconv_plan_t plan, const float* lam_re, const float* lam_im,
                                                const float* c_re, const float* c_im, void* khat, void* workspace,
                                                void* stream);

/*
 * 2-D kernel spectrum: khat <- DFT_{2Hs x 2Ws}(k[c] zero-padded) / (4 Hs Ws)
 * ("Native Multi-Dimensional Subquadratic Operators via Input Dependent Long
 * Convolutions", abstract: global multi-dimensional kernels on the FFT path).
 * k is [C][Kh][Kw] fp32 with 1 <= Kh <= Hs, 1 <= Kw <= Ws.
 */
FFTCONV_API fftconv_status fftconv2d_kernel_spectrum(fftconv_plan_t plan, const float* k, int Kh, int Kw,
                                         void* khat, void* workspace, void* stream);

/*
 * 2-D forward: y[b,c,i,j] = sum_{p<=i, q<=j} k[c,p,q] u[b,c,i-p,j-q] for
 * 0 <= i < Hs, 0 <= j < Ws (the first-quadrant crop of the zero-padded
 * linear convolution, the 2-D analogue of [:N]; "Native Multi-Dimensional
 * Subquadratic Operators via Input Dependent Long Convolutions", abstract).
 * u, y: [B][C][Hs][Ws] of the plan's dtype.  FFTCONV_ERR_INVALID_ARG also
 * when the current device is not the plan's.
 */
FFTCONV_API fftconv_status fftconv2d_fwd(fftconv_plan_t plan, const void* u, const void* khat, void* y,
                             void* workspace, void* stream);

/*
 * 2-D forward with a crop offset: y[b,c,i,j] = full[i + oy][j + ox], the
 * window [oy, oy + Hs) x [ox, ox + Ws) of the full (2Hs - 1) x (2Ws - 1)
 * linear convolution full[r][s] = sum_{p,q} k[c,p,q] u[b,c,r-p,s-q] (indices
 * inside both arrays).  (0, 0) is fftconv2d_fwd's first-quadrant crop;
 * (Hs/2, Ws/2) the centred reading of a kernel anchored at its middle (the
 * zero-padded multi-dimensional convolution of "Native Multi-Dimensional
 * Subquadratic Operators via Input Dependent Long Convolutions", abstract,
 * does not say which window).  0 <= oy <= Hs,
 * 0 <= ox <= Ws, both multiples of 8 (else FFTCONV_ERR_INVALID_ARG).  The
 * transform of length 2Hs x 2Ws holds the full convolution without
 * wrap-around, so only the last inverse passes change: they keep rows
 * oy.. and columns ox.. instead of 0...
 */
FFTCONV_API fftconv_status fftconv2d_fwd_offset(fftconv_plan_t plan, const void* u, const void* khat, void* y,
                                                void* workspace, void* stream, int oy, int ox);

/*
 * 2-D forward with one filter per image (input-dependent kernels, "Native
 * Multi-Dimensional Subquadratic Operators via Input Dependent Long
 * Convolutions", abstract):
 *     y[b,c,i,j] = sum_{p<=i, q<=j} k[b,c,p,q] u[b,c,i-p,j-q]
 * (fftconv2d_fwd's crop).  Plans from fftconv2d_dynamic_plan_create (B, C,
 * Hs, Ws, dtype as fftconv2d_plan_create); k is [B][C][Kh][Kw] fp32 on the
 * device, 1 <= Kh <= Hs, 1 <= Kw <= Ws, transformed inside the call (no
 * cached spectrum: fftconv2d_kernel_spectrum is not needed).  The images run
 * as the channels of a single-image batch, so each transform carries one
 * image (half of fftconv2d_fwd's packing of two).  workspace: device,
 * fftconv_workspace_bytes(plan) bytes (the images' spectra, then the passes'
 * workspace), 16-byte aligned.  FFTCONV_ERR_INVALID_ARG for plans of any
 * other kind, or when the current device is not the plan's.
 */
FFTCONV_API fftconv_status fftconv2d_dynamic_plan_create(fftconv_plan_t* plan, int B, int C, int Hs, int Ws,
                                                         fftconv_dtype dtype);
FFTCONV_API fftconv_status fftconv2d_fwd_dynamic(fftconv_plan_t plan, const void* u, const float* k, int Kh, int Kw,
                                                 void* y, void* workspace, void* stream);

/*
 * 3-D causal convolution (N-D beyond 2-D; "Native Multi-Dimensional
 * Subquadratic Operators via Input Dependent Long Convolutions", abstract:
 * the long convolution on native N-D geometry): the first-octant crop of the
 * zero-padded linear convolution,
 *     y[b,c,d,i,j] = sum_{e<=d, p<=i, q<=j} k[c,e,p,q] u[b,c,d-e,i-p,j-q],
 * d < Dd, i < Hs, j < Ws, by a (2Dd) x (2Hs) x (2Ws) transform (fp32 SIMT).
 * Dd, Hs, Ws powers of two in [FFTCONV3D_MIN_SIDE, FFTCONV3D_MAX_SIDE]
 * (else FFTCONV_ERR_UNSUPPORTED).  u, y: [B][C][Dd][Hs][Ws] of the plan's
 * dtype; k: [C][Kd][Kh][Kw] fp32, 1 <= Kd <= Dd, 1 <= Kh <= Hs, 1 <= Kw <= Ws.
 * khat: fftconv_spectrum_bytes(plan) bytes, computed once by
 * fftconv3d_kernel_spectrum; workspace: fftconv_workspace_bytes(plan) bytes
 * (both calls need it).  All device pointers 16-byte aligned; y must not
 * alias u.  FFTCONV_ERR_NOT_READY before the spectrum; FFTCONV_ERR_INVALID_ARG
 * for other plans or when the current device is not the plan's.  Path name
 * "3d".
 */
#define FFTCONV3D_MIN_SIDE 16
#define FFTCONV3D_MAX_SIDE 256
FFTCONV_API fftconv_status fftconv3d_plan_create(fftconv_plan_t* plan, int B, int C, int Dd, int Hs, int Ws,
                                                 fftconv_dtype dtype);
FFTCONV_API fftconv_status fftconv3d_kernel_spectrum(fftconv_plan_t plan, const float* k, int Kd, int Kh, int Kw,
                                                     void* khat, void* workspace, void* stream);
FFTCONV_API fftconv_status fftconv3d_fwd(fftconv_plan_t plan, const void* u, const void* khat, void* y,
                                         void* workspace, void* stream);

/*
 * Conjugate spectrum: khat_conj <- conj(khat) in the plan's layout, the
 * spectrum of the correlation with k (the backward pass's filter, below; the
 * training of "Simple Hardware-Efficient Long Convolutions for Sequence
 * Modeling", abstract).  khat is
 * the output of fftconv_kernel_spectrum on this plan; khat_conj is a buffer of
 * fftconv_spectrum_bytes() bytes and may equal khat (in place).
 */
FFTCONV_API fftconv_status fftconv_spectrum_conjugate(fftconv_plan_t plan, const void* khat, void* khat_conj,
                                                      void* stream);

/* Bytes of device workspace fftconv_bwd needs (0: none). */
FFTCONV_API size_t fftconv_bwd_workspace_bytes(fftconv_plan_t plan);

/*
 * Backward pass: the gradients of the forward's y with respect to its inputs
 * for an upstream gradient dy ([B][H][N], the plan's dtype).  Training the
 * learned long filters of "Simple Hardware-Efficient Long Convolutions for
 * Sequence Modeling" (abstract) and of "FlashFFTConv" (abstract) needs them;
 * the pages give no formula, so these are the chain rule of the forward:
 *   g = dy (.) v (gated) or dy,  x = u (.) w (gated) or u
 *   du = dx (.) w (gated) or dx,  dx[t] = sum_j k[j] g[t+j] + D g[t]
 *   dw = dx (.) u,  dv = dy (.) (x * k + D x)          (gated plans only)
 *   dk[h][j] = sum_b sum_t g[b,h,t] x[b,h,t-j], j < L  (fp32 [H][L])
 *   dD[h] = sum_b sum_t g[b,h,t] x[b,h,t]              (fp32 [H])
 * dx runs through the plan's forward kernel with khat_conj (the output of
 * fftconv_spectrum_conjugate); dk and dD through an fp32 transform of the
 * pairs (N <= 8192: otherwise FFTCONV_ERR_UNSUPPORTED when dk or dD is
 * requested).  dk and dD may be NULL (not computed); dD requires D.  v, w, dv,
 * dw must be given for a gated plan and NULL otherwise.  Outputs must not
 * alias inputs.  workspace: fftconv_bwd_workspace_bytes() bytes.
 */
FFTCONV_API fftconv_status fftconv_bwd(fftconv_plan_t plan, const void* dy, const void* u, const void* v,
                                       const void* w, const void* khat, const void* khat_conj, const float* D,
                                       int64_t L, void* du, void* dv, void* dw, float* dk, float* dD,
                                       void* workspace, void* stream);

/*
 * Forward without a workspace argument: the same result as fftconv_fwd on a
 * multi-pass plan (2N > 16384), with the scratch taken from a device array
 * of FFTCONV_STATIC_WORKSPACE_BYTES built into the library instead of a
 * caller buffer.  No counterpart on the pages: it exists for callers that
 * cannot allocate device memory at the time they convolve (allocation is
 * forbidden there, or would synchronise the device, or all memory belongs to
 * someone else's pool).  It allocates nothing.
 *   - Arguments and layouts as fftconv_fwd, minus the workspace.
 *   - FFTCONV_ERR_UNSUPPORTED for a plan that is not multi-pass, or whose
 *     scratch for one pair of rows (8 bytes per point of the length-2N
 *     transform) is larger than the array; every N this library supports
 *     (up to 2^20, 16 MiB per pair) fits.
 *   - The array's device address is looked up on the first call on each
 *     device, with that device current; make that first call before any
 *     stream capture.
 *   - Every call uses the same array: calls whose GPU work overlaps (other
 *     streams, other threads) race on it and give wrong results; serialise
 *     them.  Nothing in the array needs to be cleared between calls.
 *   - The array occupies every GPU that loads the library until exit.
 */
#define FFTCONV_STATIC_WORKSPACE_BYTES ((size_t)16 << 20)
FFTCONV_API fftconv_status fftconv_fwd_static_workspace(fftconv_plan_t plan, const void* u, const void* v,
                                                        const void* w, const void* khat, const float* D,
                                                        void* y, void* stream);

/* Size in bytes of the device array fftconv_fwd_static_workspace uses. */
FFTCONV_API size_t fftconv_static_workspace_bytes(void);

/*
 * Device status of a plan: synchronises the stream, then reads and clears the
 * plan's device status word.  Kernels that wait on the tensor cores bound
 * every wait (fftconv_plan_set_wait_limit); a wait that gives up abandons
 * the launch once the products in flight have drained, leaves y incomplete
 * and sets the word.  Returns FFTCONV_OK, or FFTCONV_ERR_TIMEOUT once after
 * such a launch; FFTCONV_ERR_CUDA if the synchronisation or the read fails.
 * No counterpart on the pages.
 */
FFTCONV_API fftconv_status fftconv_device_status(fftconv_plan_t plan, void* stream);

/* Human-readable name of a status code (static string). */
FFTCONV_API const char* fftconv_status_string(fftconv_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
FFTCONV_API int fftconv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FFTCONV_H */
