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

/* Supported sizes: 1-D N a power of two, FFTCONV_MIN_N <= N <= FFTCONV_MAX_N;
 * 2-D Hs, Ws powers of two in [FFTCONV2D_MIN_SIDE, FFTCONV2D_MAX_SIDE]. */
#define FFTCONV_MIN_N 64
#define FFTCONV_MAX_N (1 << 20)
#define FFTCONV2D_MIN_SIDE 16
#define FFTCONV2D_MAX_SIDE 256

/*
 * Create a 1-D plan for B batch rows, H channels, sequence length N, I/O type
 * dtype, gated (nonzero) or not.  Chooses the execution path: a single fused
 * kernel per (channel, pair of batch rows) when the transform of length 2N
 * fits on chip, else the multi-pass path that stages partial transforms in
 * the caller's workspace.  Uploads the plan's twiddle tables (synchronously).
 * On success *plan receives the handle.
 */
FFTCONV_API fftconv_status fftconv_plan_create(fftconv_plan_t* plan, int B, int H, int64_t N,
                                   fftconv_dtype dtype, int gated);

/*
 * Create a 2-D plan: B images, C channels, Hs x Ws pixels, I/O type dtype.
 * The transform is (2Hs) x (2Ws) over the zero-padded image.
 */
FFTCONV_API fftconv_status fftconv2d_plan_create(fftconv_plan_t* plan, int B, int C, int Hs, int Ws,
                                     fftconv_dtype dtype);

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
 * "fused_umma" (the same on tcgen05 tensor cores, 2N = 4096 or 8192, chosen
 * when the environment variable FFTCONV_UMMA=1 is set at plan creation),
 * "multipass", "2d". */
FFTCONV_API const char* fftconv_plan_path(fftconv_plan_t plan);

/*
 * Kernel spectrum: khat <- DFT_{2N}(k[h] zero-padded) / (2N) for every
 * channel, in the plan's internal order and precision.  k is [H][L] fp32 on
 * the device with 1 <= L <= N (taps past L are zero: a partial convolution).
 * Computed once per filter set and reused by every fftconv_fwd of the plan.
 */
FFTCONV_API fftconv_status fftconv_kernel_spectrum(fftconv_plan_t plan, const float* k, int64_t L,
                                       void* khat, void* workspace, void* stream);

/*
 * Forward: y = the causal convolution above.  u is [B][H][N]; v and w are
 * [B][H][N] for a gated plan and must be NULL otherwise; khat is the output
 * of fftconv_kernel_spectrum on this plan; D is [H] fp32 or NULL (no skip
 * term); y is [B][H][N] and must not alias any input.
 */
FFTCONV_API fftconv_status fftconv_fwd(fftconv_plan_t plan, const void* u, const void* v, const void* w,
                           const void* khat, const float* D, void* y, void* workspace,
                           void* stream);

/*
 * 2-D kernel spectrum: khat <- DFT_{2Hs x 2Ws}(k[c] zero-padded) / (4 Hs Ws).
 * k is [C][Kh][Kw] fp32 with 1 <= Kh <= Hs, 1 <= Kw <= Ws.
 */
FFTCONV_API fftconv_status fftconv2d_kernel_spectrum(fftconv_plan_t plan, const float* k, int Kh, int Kw,
                                         void* khat, void* workspace, void* stream);

/*
 * 2-D forward: y[b,c,i,j] = sum_{p<=i, q<=j} k[c,p,q] u[b,c,i-p,j-q] for
 * 0 <= i < Hs, 0 <= j < Ws (the first-quadrant crop of the zero-padded
 * linear convolution).  u, y: [B][C][Hs][Ws] of the plan's dtype.
 */
FFTCONV_API fftconv_status fftconv2d_fwd(fftconv_plan_t plan, const void* u, const void* khat, void* y,
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
 * every wait; a wait that gives up (the hardware never signalled) abandons
 * the launch, leaves y incomplete and sets the word.  Returns FFTCONV_OK, or
 * FFTCONV_ERR_TIMEOUT once after such a launch; FFTCONV_ERR_CUDA if the
 * synchronisation or the read fails.  No counterpart on the pages.
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
