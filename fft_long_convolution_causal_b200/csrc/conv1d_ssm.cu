// conv1d_ssm.cu -- causal long convolution with filters of a diagonal
// state-space model, computed in chunks with the state passed between them
// ("FlashConv", Mechanism: fused FFT convolution on chip; past the on-chip
// length, chunk convolutions with the state-space boundary state propagated
// between chunks).
//
// Filter of channel h: k[t] = Re(sum_j c_j lam_j^t) (|lam_j| < 1, d states).
// Split a row into chunks of T.  For chunk c and t < T,
//   y[cT + t] = sum_{s <= t} k[s] x[cT + t - s]            (intra: the fused FFT
//                                                            convolution with k[:T])
//             + Re(sum_j c_j lam_j^t S_j(c)) + D x[cT + t]
//   S_j(c)    = sum_{m < cT} lam_j^{cT - m} x[m]            (state entering chunk c)
//   S_j(c+1)  = lam_j^T S_j(c) + E_j(c),  E_j(c) = sum_{i < T} lam_j^{T - i} x[cT + i].
// Kernels: ssm_setup (k[:T] and the power table lam^{32 i}, fp64 then fp32),
// ssm_chunk_states (E), ssm_scan (S, fp64 across chunks), the fused forward
// on the rows viewed as [B][H x nchunks][T] with one spectrum per channel,
// ssm_correct (adds the inter-chunk term to y).  Every thread covers runs of
// 32 consecutive positions: a power from the table, then 31 fp32 products.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>

#include "fft_simt.cuh"
#include "fftconv.h"
#include "plan.h"

namespace fftc {
namespace ssm {

constexpr int kRun = 32;       // consecutive positions per thread
constexpr int kThreads = 256;
constexpr int kMaxState = 64;

// plan-owned block: lam [H][d], c [H][d], pw [H][d][T/32 + 1] (float2 each)
struct Views {
    float2* lam;
    float2* cc;
    float2* pw;
};
inline Views views(const fftconv_plan_s& p) {
    float2* base = (float2*)p.d_ssm;
    const size_t hd = (size_t)p.H * p.d_state;
    return {base, base + hd, base + 2 * hd};
}
inline size_t block_words(int H, int d, int64_t T) { return (size_t)H * d * (2 + (size_t)(T / kRun + 1)); }

__device__ __forceinline__ double2 cpow_d(double lr, double li, double e) {
    const double mag = pow(sqrt(lr * lr + li * li), e), ang = e * atan2(li, lr);
    return make_double2(mag * cos(ang), mag * sin(ang));
}

// one CTA per channel: copy lam and c, the power table, and k[h][:T] (fp64 sums)
__global__ void __launch_bounds__(kThreads)
ssm_setup(const float* __restrict__ lr, const float* __restrict__ li, const float* __restrict__ cr,
          const float* __restrict__ ci, int d, int T, float2* __restrict__ lam, float2* __restrict__ cc,
          float2* __restrict__ pw, float* __restrict__ k) {
    const int h = blockIdx.x, tid = threadIdx.x;
    const int nrun = T / kRun;
    for (int j = tid; j < d; j += kThreads) {
        lam[h * d + j] = make_float2(lr[h * d + j], li[h * d + j]);
        cc[h * d + j] = make_float2(cr[h * d + j], ci[h * d + j]);
    }
    for (int idx = tid; idx < d * (nrun + 1); idx += kThreads) {
        const int j = idx / (nrun + 1), i = idx % (nrun + 1);
        const double2 p = cpow_d(lr[h * d + j], li[h * d + j], (double)(kRun * i));
        pw[((size_t)h * d + j) * (nrun + 1) + i] = make_float2((float)p.x, (float)p.y);
    }
    for (int t = tid; t < T; t += kThreads) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) {
            const double2 p = cpow_d(lr[h * d + j], li[h * d + j], (double)t);
            acc += (double)cr[h * d + j] * p.x - (double)ci[h * d + j] * p.y;
        }
        k[(size_t)h * T + t] = (float)acc;
    }
}

template <typename IO>
__device__ __forceinline__ void load_run(const IO* __restrict__ x, float (&v)[kRun]) {
#pragma unroll
    for (int i = 0; i < kRun; ++i) v[i] = to_f(x[i]);
}

// E[b][h][c][j] = sum_{i < T} lam_j^{T - i} x[cT + i]; grid (nchunks, H, B)
template <typename IO>
__global__ void __launch_bounds__(kThreads)
ssm_chunk_states(const IO* __restrict__ u, const float2* __restrict__ lam, const float2* __restrict__ pw, int d,
                 int T, int nc, int H, float2* __restrict__ E) {
    __shared__ float2 part[kThreads / 32][kMaxState];
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nrun = T / kRun;
    const size_t row = ((size_t)b * H + h) * ((size_t)nc * T) + (size_t)c * T;
    float v[kRun];
    const bool active = tid < nrun;
    if (active) load_run(u + row + (size_t)kRun * tid, v);
    for (int j = 0; j < d; ++j) {
        float2 acc = make_float2(0.f, 0.f);
        if (active) {
            const float2 l = lam[h * d + j];
            // lam^{T - (32 tid + 31)} = lam^{32 (nrun - tid - 1)} lam
            float2 p = cmul(pw[((size_t)h * d + j) * (nrun + 1) + (nrun - tid - 1)], l);
#pragma unroll
            for (int i = kRun - 1; i >= 0; --i) {
                acc.x = fmaf(p.x, v[i], acc.x);
                acc.y = fmaf(p.y, v[i], acc.y);
                p = cmul(p, l);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
            acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
        }
        if (lane == 0) part[warp][j] = acc;
    }
    __syncthreads();
    for (int j = tid; j < d; j += kThreads) {
        float2 s = make_float2(0.f, 0.f);
        for (int w = 0; w < kThreads / 32; ++w) s = cadd(s, part[w][j]);
        E[(((size_t)b * H + h) * nc + c) * d + j] = s;
    }
}

// S[b][h][c][j]: the state entering chunk c, S(0) = 0, S(c+1) = lam^T S(c) + E(c), in fp64
__global__ void ssm_scan(const float2* __restrict__ lam, const float2* __restrict__ E, int d, int T, int nc, int H,
                         int B, float2* __restrict__ S) {
    const int idx = blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= B * H * d) return;
    const int j = idx % d, bh = idx / d, h = bh % H;
    const float2 l = lam[h * d + j];
    const double2 lT = cpow_d(l.x, l.y, (double)T);
    double sr = 0.0, si = 0.0;
    for (int c = 0; c < nc; ++c) {
        const size_t o = ((size_t)bh * nc + c) * d + j;
        S[o] = make_float2((float)sr, (float)si);
        const float2 e = E[o];
        const double nr = lT.x * sr - lT.y * si + (double)e.x;
        const double ni = lT.x * si + lT.y * sr + (double)e.y;
        sr = nr;
        si = ni;
    }
}

// y[cT + t] += Re(sum_j c_j lam_j^t S_j(c)) for chunks c >= 1; grid (nchunks - 1, H, B)
template <typename IO>
__global__ void __launch_bounds__(kThreads)
ssm_correct(IO* __restrict__ y, const float2* __restrict__ lam, const float2* __restrict__ cc,
            const float2* __restrict__ pw, const float2* __restrict__ S, int d, int T, int nc, int H) {
    __shared__ float2 a[kMaxState], ls[kMaxState];
    const int c = blockIdx.x + 1, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
    const int nrun = T / kRun;
    for (int j = tid; j < d; j += kThreads) {
        a[j] = cmul(cc[h * d + j], S[(((size_t)b * H + h) * nc + c) * d + j]);
        ls[j] = lam[h * d + j];
    }
    __syncthreads();
    if (tid >= nrun) return;
    float o[kRun];
#pragma unroll
    for (int i = 0; i < kRun; ++i) o[i] = 0.f;
    for (int j = 0; j < d; ++j) {
        const float2 aj = a[j], l = ls[j];
        float2 p = pw[((size_t)h * d + j) * (nrun + 1) + tid];  // lam^{32 tid}
#pragma unroll
        for (int i = 0; i < kRun; ++i) {
            o[i] = fmaf(aj.x, p.x, fmaf(-aj.y, p.y, o[i]));
            p = cmul(p, l);
        }
    }
    IO* __restrict__ yr = y + ((size_t)b * H + h) * ((size_t)nc * T) + (size_t)c * T + (size_t)kRun * tid;
#pragma unroll
    for (int i = 0; i < kRun; ++i) yr[i] = from_f<IO>(to_f(yr[i]) + o[i]);
}

}  // namespace ssm

size_t ssm_block_bytes(int H, int d, int64_t T) { return ssm::block_words(H, d, T) * sizeof(float2); }

// workspace: [k scratch H x T fp32][E][S] (B x H x nchunks x d float2 each)
size_t ssm_workspace_bytes(const fftconv_plan_s& p) {
    const size_t kb = ((size_t)p.H * p.T * sizeof(float) + 255) & ~size_t(255);
    const size_t st = (size_t)p.B * p.H * p.nchunks * p.d_state * sizeof(float2);
    return kb + 2 * ((st + 255) & ~size_t(255));
}

cudaError_t launch_ssm_setup(const fftconv_plan_s& p, const float* lr, const float* li, const float* cr,
                             const float* ci, void* khat, void* work, cudaStream_t s) {
    const ssm::Views v = ssm::views(p);
    float* k = (float*)work;
    ssm::ssm_setup<<<p.H, ssm::kThreads, 0, s>>>(lr, li, cr, ci, p.d_state, (int)p.T, v.lam, v.cc, v.pw, k);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // one spectrum per channel, of k[:T] zero-padded to 2T, in the layout of the
    // chunk plan's forward kernel
    fftconv_plan_s q = *p.chunk;
    q.H = p.H;
    if (q.t2) return launch_t2_spectrum(q, k, p.T, khat, s);
    return launch_fused_spectrum(q, k, p.T, (float2*)khat, s);
}

cudaError_t launch_ssm_fwd(const fftconv_plan_s& p, const void* u, const void* khat, const float* D, void* y,
                           void* work, cudaStream_t s) {
    const ssm::Views v = ssm::views(p);
    const size_t kb = ((size_t)p.H * p.T * sizeof(float) + 255) & ~size_t(255);
    const size_t st = (((size_t)p.B * p.H * p.nchunks * p.d_state * sizeof(float2)) + 255) & ~size_t(255);
    float2* E = (float2*)((uint8_t*)work + kb);
    float2* S = (float2*)((uint8_t*)work + kb + st);
    const int d = p.d_state, T = (int)p.T, nc = (int)p.nchunks;
    cudaError_t e = cudaSuccess;
    if (nc > 1) {
        const dim3 g(nc, p.H, p.B);
        if (p.dtype == FFTCONV_BF16)
            ssm::ssm_chunk_states<__nv_bfloat16><<<g, ssm::kThreads, 0, s>>>((const __nv_bfloat16*)u, v.lam, v.pw, d,
                                                                           T, nc, p.H, E);
        else
            ssm::ssm_chunk_states<float><<<g, ssm::kThreads, 0, s>>>((const float*)u, v.lam, v.pw, d, T, nc, p.H, E);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const int n = p.B * p.H * d;
        ssm::ssm_scan<<<(n + 127) / 128, 128, 0, s>>>(v.lam, E, d, T, nc, p.H, p.B, S);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // intra-chunk convolutions: rows [B][H x nc][T], one spectrum and D per channel
    // (bf16 chunks of 4096: the two-stage tensor-core kernel; else the fp32 fused kernel)
    e = p.chunk->t2 ? launch_t2_fwd(*p.chunk, u, khat, D, y, s)
                    : launch_fused_fwd(*p.chunk, u, nullptr, nullptr, (const float2*)khat, D, y, s);
    if (e != cudaSuccess || nc <= 1) return e;
    const dim3 g(nc - 1, p.H, p.B);
    if (p.dtype == FFTCONV_BF16)
        ssm::ssm_correct<__nv_bfloat16><<<g, ssm::kThreads, 0, s>>>((__nv_bfloat16*)y, v.lam, v.cc, v.pw, S, d, T, nc,
                                                                  p.H);
    else
        ssm::ssm_correct<float><<<g, ssm::kThreads, 0, s>>>((float*)y, v.lam, v.cc, v.pw, S, d, T, nc, p.H);
    return cudaGetLastError();
}

}  // namespace fftc
