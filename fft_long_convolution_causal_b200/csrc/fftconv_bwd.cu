// fftconv_bwd.cu -- the backward pass of the 1-D causal convolution behind
// the C ABI: gradients du (dv, dw for the gated form), dk and dD for an
// upstream gradient dy.  Training the learned long filters of "Simple
// Hardware-Efficient Long Convolutions for Sequence Modeling" (abstract) and
// the models of "FlashFFTConv" (abstract) needs them.
//
// * Data gradient: dx[t] = sum_j k[j] g[t + j] + D g[t] (g = dy, or dy v) is
//   the correlation with k, whose 2N-point spectrum is conj(Khat): with the
//   same zero padding it has no wrap-around, so dx = fwd(g, conj(Khat), D)
//   exactly, through whichever forward kernel the plan runs.
// * Gated form: g = dy v and x = u w (elementwise, into the workspace);
//   dx = fwd(g, conj Khat, D) -> du = dx w, dw = dx u; s = fwd(x, Khat, D),
//   the pre-gate output -> dv = dy s.
// * Filter gradient: dk[j] = sum_b sum_t g x[t - j] = Re(iDFT(sum_pairs
//   conj(DFT zx) DFT zg))[j] for the packed pairs zx, zg (kgrad_pairs writes
//   each pair's cross spectrum, kgrad_finish sums and inverts), and dD = the
//   same at lag 0.
#include <cuda_bf16.h>
#include <stdint.h>

#include "fft_simt.cuh"
#include "fftconv.h"
#include "plan.h"

namespace fftc {

// flip the sign of the imaginary parts of a spectrum stored as 32-bit words:
// kind 0: fp32 complex (odd words); 1: bf16 pairs, odd words Im (fragment
// order); 2: bf16 pairs in 16-byte quads [h][g][j][k_p], quads j = 2, 3 Im
// (two-stage layout)
__global__ void conj_words(const uint32_t* __restrict__ in, uint32_t* __restrict__ out, size_t n, int kind) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        uint32_t x = in[i];
        if (kind == 0 && (i & 1)) x ^= 0x80000000u;
        if (kind == 1 && (i & 1)) x ^= 0x80008000u;
        if (kind == 2 && ((i >> 9) & 2)) x ^= 0x80008000u;
        out[i] = x;
    }
}

template <typename IO>
__device__ __forceinline__ float ld(const IO* p, size_t i) {
    return to_f(p[i]);
}

// g = dy v, x = u w
template <typename IO>
__global__ void gate_in(const IO* __restrict__ dy, const IO* __restrict__ v, const IO* __restrict__ u,
                        const IO* __restrict__ w, IO* __restrict__ g, IO* __restrict__ x, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        g[i] = from_f<IO>(ld(dy, i) * ld(v, i));
        x[i] = from_f<IO>(ld(u, i) * ld(w, i));
    }
}

// du holds dx and dv holds s on entry: dw = dx u, du = dx w, dv = dy s
template <typename IO>
__global__ void gate_out(const IO* __restrict__ dy, const IO* __restrict__ u, const IO* __restrict__ w,
                         IO* __restrict__ du, IO* __restrict__ dv, IO* __restrict__ dw, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const float dx = ld(du, i);
        dw[i] = from_f<IO>(dx * ld(u, i));
        du[i] = from_f<IO>(dx * ld(w, i));
        dv[i] = from_f<IO>(ld(dy, i) * ld(dv, i));
    }
}

bool kgrad_supported(int log2M);
cudaError_t launch_kgrad(const fftconv_plan_s& p, const void* u, const void* w, const void* dy, const void* v,
                         float2* acc, float* dk, float* dD, int64_t L, cudaStream_t s);

}  // namespace fftc

namespace {

bool aligned16b(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// workspace pieces: [plan forward workspace][kgrad accumulator][g][x]
struct BwdWs {
    size_t fwd, acc, gx, total;
};
BwdWs bwd_ws(const fftconv_plan_s& p) {
    BwdWs w;
    w.fwd = up256(p.workspace_bytes);
    // the filter gradient's cross spectra, one per (channel, pair)
    w.acc = fftc::kgrad_supported(p.log2M)
                ? up256((size_t)p.H * ((p.B + 1) / 2) * ((size_t)1 << p.log2M) * sizeof(float2))
                : 0;
    const size_t esz = p.dtype == FFTCONV_BF16 ? 2 : 4;
    w.gx = p.gated ? up256((size_t)p.B * p.H * p.N * esz) : 0;
    w.total = w.fwd + w.acc + 2 * w.gx;
    return w;
}

cudaError_t fwd_launch(const fftconv_plan_s& p, const void* u, const void* khat, const float* D, void* y, void* work,
                       cudaStream_t s) {
    if (p.t2) return fftc::launch_t2_fwd(p, u, khat, D, y, s);
    if (p.path == fftc::PATH_FUSED_TC)
        return p.umma ? fftc::launch_umma_fwd(p, u, nullptr, nullptr, khat, D, y, s)
                      : fftc::launch_tc_fwd(p, u, nullptr, nullptr, khat, D, y, s);
    if (p.path == fftc::PATH_FUSED) return fftc::launch_fused_fwd(p, u, nullptr, nullptr, (const float2*)khat, D, y, s);
    return fftc::launch_multipass_fwd(p, u, nullptr, nullptr, (const float2*)khat, D, y, (float2*)work, s);
}

int grid_for(size_t n) {
    size_t b = (n + 255) / 256;
    return (int)(b < 4096 ? (b ? b : 1) : 4096);
}

}  // namespace

extern "C" {

fftconv_status fftconv_spectrum_conjugate(fftconv_plan_t p, const void* khat, void* khat_conj, void* stream) {
    if (!p || p->kind != 1 || !khat || !khat_conj) return FFTCONV_ERR_INVALID_ARG;
    if (!aligned16b(khat) || !aligned16b(khat_conj)) return FFTCONV_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != p->device) {
        cudaGetLastError();
        return FFTCONV_ERR_INVALID_ARG;
    }
    const int kind = p->t2 ? 2 : (p->path == fftc::PATH_FUSED_TC ? 1 : 0);
    const size_t n = p->spectrum_bytes / 4;
    fftc::conj_words<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>((const uint32_t*)khat, (uint32_t*)khat_conj, n,
                                                                    kind);
    return cudaGetLastError() == cudaSuccess ? FFTCONV_OK : FFTCONV_ERR_CUDA;
}

size_t fftconv_bwd_workspace_bytes(fftconv_plan_t p) { return (p && p->kind == 1) ? bwd_ws(*p).total : 0; }

fftconv_status fftconv_bwd(fftconv_plan_t p, const void* dy, const void* u, const void* v, const void* w,
                           const void* khat, const void* khat_conj, const float* D, int64_t L, void* du, void* dv,
                           void* dw, float* dk, float* dD, void* work, void* stream) {
    if (!p || p->kind != 1 || !dy || !u || !khat || !khat_conj || !du) return FFTCONV_ERR_INVALID_ARG;
    if (p->gated ? (!v || !w || !dv || !dw) : (v || w || dv || dw)) return FFTCONV_ERR_INVALID_ARG;
    const void* ptrs[] = {dy, u, v, w, khat, khat_conj, D, du, dv, dw, dk, dD};
    for (const void* q : ptrs)
        if (q && !aligned16b(q)) return FFTCONV_ERR_INVALID_ARG;
    if ((dk || dD) && (L < 1 || L > p->N)) return FFTCONV_ERR_INVALID_ARG;
    if (dD && !D) return FFTCONV_ERR_INVALID_ARG;
    const void* outs[] = {du, dv, dw};
    for (const void* o : outs)
        if (o && (o == dy || o == u || o == v || o == w)) return FFTCONV_ERR_INVALID_ARG;
    const BwdWs ws = bwd_ws(*p);
    if (ws.total && (!work || !aligned16b(work))) return FFTCONV_ERR_INVALID_ARG;
    if ((dk || dD) && !fftc::kgrad_supported(p->log2M)) return FFTCONV_ERR_UNSUPPORTED;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != p->device) {
        cudaGetLastError();
        return FFTCONV_ERR_INVALID_ARG;
    }
    if (!p->spectrum_ready) return FFTCONV_ERR_NOT_READY;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* base = (uint8_t*)work;
    void* fwork = base;
    float2* acc = (float2*)(base + ws.fwd);
    void* gbuf = base + ws.fwd + ws.acc;
    void* xbuf = base + ws.fwd + ws.acc + ws.gx;
    // the forward kernels run ungated here (the gates are applied elementwise)
    fftconv_plan_s q = *p;
    q.gated = 0;
    cudaError_t e = cudaSuccess;
    const size_t n = (size_t)p->B * p->H * p->N;
    if (!p->gated) {
        e = fwd_launch(q, dy, khat_conj, D, du, fwork, s);
    } else {
        if (p->dtype == FFTCONV_BF16)
            fftc::gate_in<__nv_bfloat16><<<grid_for(n), 256, 0, s>>>(
                (const __nv_bfloat16*)dy, (const __nv_bfloat16*)v, (const __nv_bfloat16*)u, (const __nv_bfloat16*)w,
                (__nv_bfloat16*)gbuf, (__nv_bfloat16*)xbuf, n);
        else
            fftc::gate_in<float><<<grid_for(n), 256, 0, s>>>((const float*)dy, (const float*)v, (const float*)u,
                                                             (const float*)w, (float*)gbuf, (float*)xbuf, n);
        e = cudaGetLastError();
        if (e == cudaSuccess) e = fwd_launch(q, gbuf, khat_conj, D, du, fwork, s);  // dx
        if (e == cudaSuccess) e = fwd_launch(q, xbuf, khat, D, dv, fwork, s);       // s (pre-gate output)
        if (e == cudaSuccess) {
            if (p->dtype == FFTCONV_BF16)
                fftc::gate_out<__nv_bfloat16><<<grid_for(n), 256, 0, s>>>(
                    (const __nv_bfloat16*)dy, (const __nv_bfloat16*)u, (const __nv_bfloat16*)w, (__nv_bfloat16*)du,
                    (__nv_bfloat16*)dv, (__nv_bfloat16*)dw, n);
            else
                fftc::gate_out<float><<<grid_for(n), 256, 0, s>>>((const float*)dy, (const float*)u, (const float*)w,
                                                                  (float*)du, (float*)dv, (float*)dw, n);
            e = cudaGetLastError();
        }
    }
    if (e == cudaSuccess && (dk || dD)) e = fftc::launch_kgrad(*p, u, w, dy, v, acc, dk, dD, L, s);
    return e == cudaSuccess ? FFTCONV_OK : FFTCONV_ERR_CUDA;
}

}  // extern "C"
