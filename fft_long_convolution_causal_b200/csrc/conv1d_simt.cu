// conv1d_simt.cu -- fp32 SIMT kernels of the 1-D causal FFT convolution.
//
// Two batch rows b, b+1 of one channel h are packed as one complex sequence
// z = x_b + i x_{b+1}; because k is real, iDFT(DFT(z) . K) = (x_b * k) + i (x_{b+1} * k),
// so one complex transform of length M = 2N serves two rows.  The input is
// zero-padded to 2N and the output truncated to [:N] ("RubiConv -- Efficient
// Boundary-Respecting Convolutions", Caracal abstract: causal masking by
// asymmetric padding and truncation); FFT, pointwise product and inverse
// FFT are fused with no intermediate off-chip traffic ("FlashConv",
// Mechanism).  The skip term D x is folded into the pointwise product as the
// constant spectrum D/M of D.delta, so x is never re-read.
//
// Fused path (2N <= 16384): one CTA per (pair, channel) holds the whole
// transform in shared memory.
//
// Multi-pass path (2N > 16384): M = N1 x N2, n = N2 n1 + n2, k = k1 + N1 k2
// (the four-step / Monarch split of the DFT that "FlashFFTConv" (abstract)
// uses to map the FFT onto matrix units and to fuse long sequences):
//   pass 1: per column n2, DFT_N1 over n1 < N1/2 (the nonzero half), times
//           W_M^{n2 k1}, into the workspace as [k1][n2];
//   pass 2: per row k1, DFT_N2 over n2, times Khat[k1][k2] (+ D/M), inverse
//           DFT_N2, times W_M^{-n2 k1}, back into the workspace;
//   pass 3: per column n2, inverse DFT_N1, only n1 < N1/2 (n < N) kept.
// Pairs are processed in groups (the plan sizes them, up to 1 GiB of
// workspace) and the workspace is reused group after group.
#include <cuda_bf16.h>

#include "fft_simt.cuh"
#include "plan.h"
#include "tables.h"
#include "tc_common.cuh"

namespace fftc {

// Load x = u (or u*w) of the pair (row0, row1) at position n.
template <typename IO, bool GATED>
__device__ __forceinline__ float2 load_pair(const IO* __restrict__ u, const IO* __restrict__ w,
                                            size_t row0, size_t row1, bool has1, size_t n) {
    float a = to_f(u[row0 + n]);
    if (GATED) a *= to_f(w[row0 + n]);
    float b = 0.f;
    if (has1) {
        b = to_f(u[row1 + n]);
        if (GATED) b *= to_f(w[row1 + n]);
    }
    return make_float2(a, b);
}

// Store the pair (re -> row0, im -> row1) at position n, gated by v.
template <typename IO, bool GATED>
__device__ __forceinline__ void store_pair(IO* __restrict__ y, const IO* __restrict__ v, size_t row0,
                                           size_t row1, bool has1, size_t n, float2 z) {
    float a = z.x, b = z.y;
    if (GATED) a *= to_f(v[row0 + n]);
    y[row0 + n] = from_f<IO>(a);
    if (has1) {
        if (GATED) b *= to_f(v[row1 + n]);
        y[row1 + n] = from_f<IO>(b);
    }
}

template <class G>
constexpr int first_radix() { return 1 << G::Plan::log2r(0); }
template <class G>
constexpr int last_radix() { return 1 << G::Plan::log2r(G::Plan::kStages - 1); }

// ============================================================== fused path
template <int LOG2M>
using FusedG = Geometry<LOG2M, 1, false>;

template <int LOG2M, typename IO, bool GATED>
__global__ void __launch_bounds__(FusedG<LOG2M>::T)
fused_fwd_simt(const IO* __restrict__ u, const IO* __restrict__ v, const IO* __restrict__ w,
               const float2* __restrict__ khat, const float* __restrict__ D, IO* __restrict__ y,
               const float2* __restrict__ tw, int B, int H, int kdiv) {
    using G = FusedG<LOG2M>;
    using Lay = typename G::Lay;
    constexpr int M = G::L, N = M / 2, NS = G::Plan::kStages;
    static_assert(NS >= 2, "transform too short");
    constexpr int R0 = first_radix<G>(), RL = last_radix<G>();
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x, h = blockIdx.y;
    const int b0 = 2 * blockIdx.x;
    const bool has1 = b0 + 1 < B;
    const size_t row0 = ((size_t)b0 * H + h) * N;
    const size_t row1 = ((size_t)(b0 + 1) * H + h) * N;
    auto lds = [&](int i, int) { return smem[Lay::at(i, 0)]; };
    auto sts = [&](int i, int, float2 z) { smem[Lay::at(i, 0)] = z; };

    // forward DFT_M; stage 0 reads the nonzero half straight from global memory
    stage<G, 0, false, R0 / 2, R0, false>(
        tid, tw, [&](int n, int) { return load_pair<IO, GATED>(u, w, row0, row1, has1, n); }, sts);
    __syncthreads();
    smem_stages<G, 1, NS, false>(smem, tid, tw);

    // pointwise product with (Khat + D/M), fused into the first inverse stage;
    // kdiv consecutive row channels share one spectrum and skip weight (the
    // chunks of one channel in the chunked state-passing path; 1 otherwise)
    const int hk = h / kdiv;
    const float dm = D ? D[hk] * (1.0f / M) : 0.f;
    const float2* __restrict__ kh = khat + (size_t)hk * M;
    stage<G, 0, true, R0, R0, true>(
        tid, tw,
        [&](int i, int) {
            float2 kk = __ldg(&kh[i]);
            kk.x += dm;
            return cmul(smem[Lay::at(i, 0)], kk);
        },
        sts);
    __syncthreads();
    smem_stages<G, 1, NS - 1, true>(smem, tid, tw);
    // last inverse stage writes only n < N to global memory
    stage<G, NS - 1, true, RL, RL / 2, false>(
        tid, tw, lds, [&](int n, int, float2 z) { store_pair<IO, GATED>(y, v, row0, row1, has1, n, z); });
}

template <int LOG2M>
__global__ void __launch_bounds__(FusedG<LOG2M>::T)
fused_spectrum_simt(const float* __restrict__ k, int L, float2* __restrict__ khat,
                    const float2* __restrict__ tw) {
    using G = FusedG<LOG2M>;
    using Lay = typename G::Lay;
    constexpr int M = G::L, NS = G::Plan::kStages;
    constexpr int R0 = first_radix<G>(), RL = last_radix<G>();
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x, h = blockIdx.x;
    const float* __restrict__ kr = k + (size_t)h * L;
    auto lds = [&](int i, int) { return smem[Lay::at(i, 0)]; };
    auto sts = [&](int i, int, float2 z) { smem[Lay::at(i, 0)] = z; };
    stage<G, 0, false, R0 / 2, R0, false>(
        tid, tw, [&](int n, int) { return make_float2(n < L ? kr[n] : 0.f, 0.f); }, sts);
    __syncthreads();
    smem_stages<G, 1, NS - 1, false>(smem, tid, tw);
    float2* __restrict__ out = khat + (size_t)h * M;
    stage<G, NS - 1, false, RL, RL, false>(
        tid, tw, lds, [&](int i, int, float2 z) { out[i] = cscale(z, 1.0f / M); });
}

// The spectrum in the layout of the two-stage tensor-core kernel (2N = 8192 =
// 128 x 64, frequency k = k_p + 128 c): per channel, row k_p and column group
// g = c / 16, 16 words: 8 bf16 pairs of Re (c, c + 1) then 8 of -Im, scaled
// 1/M; stored as 16-byte quads [h][g][word / 4][k_p], so that consecutive rows
// k_p of one quad are adjacent.
__global__ void __launch_bounds__(FusedG<13>::T)
t2_spectrum_simt(const float* __restrict__ k, int L, uint16_t* __restrict__ khat, const float2* __restrict__ tw) {
    using G = FusedG<13>;
    using Lay = typename G::Lay;
    constexpr int M = G::L, NS = G::Plan::kStages;
    constexpr int R0 = first_radix<G>(), RL = last_radix<G>();
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x, h = blockIdx.x;
    const float* __restrict__ kr = k + (size_t)h * L;
    auto lds = [&](int i, int) { return smem[Lay::at(i, 0)]; };
    auto sts = [&](int i, int, float2 z) { smem[Lay::at(i, 0)] = z; };
    stage<G, 0, false, R0 / 2, R0, false>(
        tid, tw, [&](int n, int) { return make_float2(n < L ? kr[n] : 0.f, 0.f); }, sts);
    __syncthreads();
    smem_stages<G, 1, NS - 1, false>(smem, tid, tw);
    uint16_t* __restrict__ out = khat + (size_t)h * M * 2;
    stage<G, NS - 1, false, RL, RL, false>(tid, tw, lds, [&](int i, int, float2 z) {
        const int kp = i & 127, c = i >> 7;
        // 32-bit word index of word w (< 16) of group c / 16 of row kp
        auto word = [&](int w) { return ((size_t)((c >> 4) * 4 + (w >> 2)) * 128 + kp) * 4 + (w & 3); };
        const int w = (c & 15) >> 1;
        const __nv_bfloat16 re = __float2bfloat16_rn(z.x * (1.0f / M)), nim = __float2bfloat16_rn(-z.y * (1.0f / M));
        out[2 * word(w) + (c & 1)] = *reinterpret_cast<const uint16_t*>(&re);
        out[2 * word(w + 8) + (c & 1)] = *reinterpret_cast<const uint16_t*>(&nim);
    });
}

// Filter gradient of the backward pass, in two launches spread over every
// (pair, channel).  For a pair of batch rows, Zx = DFT_M(pad(x_b + i x_b+1))
// and Zg = DFT_M(pad(g_b + i g_b+1)) (x = u or u w, g = dy or dy v);
// kgrad_pairs (one CTA per pair pp and channel h) writes the cross spectrum
// conj(Zx) Zg to part[h][pp][f]; kgrad_finish (one CTA per channel) sums
// the pairs' spectra in pair order into T.  The real part of the inverse of
// T is sum_b corr(g_b, x_b): the cross terms of the packed pair land in the
// imaginary part.  dk[h][j] = that at lags j < L, dD[h] = that at lag 0
// (when dD is given).
template <int LOG2M, typename IO, bool GATED>
__global__ void __launch_bounds__(FusedG<LOG2M>::T)
kgrad_pairs(const IO* __restrict__ u, const IO* __restrict__ w, const IO* __restrict__ dy, const IO* __restrict__ v,
            float2* __restrict__ part, const float2* __restrict__ tw, int B, int H) {
    using G = FusedG<LOG2M>;
    using Lay = typename G::Lay;
    constexpr int M = G::L, N = M / 2, NS = G::Plan::kStages, T = G::T, FPT = M / T;
    constexpr int R0 = first_radix<G>();
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x, pp = blockIdx.x, h = blockIdx.y;
    const int npp = (B + 1) / 2;
    auto sts = [&](int i, int, float2 z) { smem[Lay::at(i, 0)] = z; };
    const int b0 = 2 * pp;
    const bool has1 = b0 + 1 < B;
    const size_t row0 = ((size_t)b0 * H + h) * N;
    const size_t row1 = ((size_t)(b0 + 1) * H + h) * N;
    stage<G, 0, false, R0 / 2, R0, false>(
        tid, tw, [&](int n, int) { return load_pair<IO, GATED>(u, w, row0, row1, has1, n); }, sts);
    __syncthreads();
    smem_stages<G, 1, NS, false>(smem, tid, tw);
    float2 zx[FPT];
#pragma unroll
    for (int m = 0; m < FPT; ++m) zx[m] = smem[Lay::at(tid + T * m, 0)];
    __syncthreads();
    stage<G, 0, false, R0 / 2, R0, false>(
        tid, tw, [&](int n, int) { return load_pair<IO, GATED>(dy, v, row0, row1, has1, n); }, sts);
    __syncthreads();
    smem_stages<G, 1, NS, false>(smem, tid, tw);
    float2* __restrict__ out = part + ((size_t)h * npp + pp) * M;
#pragma unroll
    for (int m = 0; m < FPT; ++m) {
        const int f = tid + T * m;
        out[f] = cmulc(smem[Lay::at(f, 0)], zx[m]);  // Zg conj(Zx)
    }
}

template <int LOG2M>
__global__ void __launch_bounds__(FusedG<LOG2M>::T)
kgrad_finish(const float2* __restrict__ part, float* __restrict__ dk, float* __restrict__ dD,
             const float2* __restrict__ tw, int npp, int L) {
    using G = FusedG<LOG2M>;
    using Lay = typename G::Lay;
    constexpr int M = G::L, NS = G::Plan::kStages, T = G::T, FPT = M / T;
    constexpr int RL = last_radix<G>();
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x, h = blockIdx.x;
    auto lds = [&](int i, int) { return smem[Lay::at(i, 0)]; };
    const float2* __restrict__ in = part + (size_t)h * npp * M;
#pragma unroll
    for (int m = 0; m < FPT; ++m) {
        const int f = tid + T * m;
        float2 t = in[f];
        for (int pp = 1; pp < npp; ++pp) t = cadd(t, in[(size_t)pp * M + f]);
        smem[Lay::at(f, 0)] = t;
    }
    __syncthreads();
    smem_stages<G, 0, NS - 1, true>(smem, tid, tw);
    stage<G, NS - 1, true, RL, RL / 2, false>(tid, tw, lds, [&](int n, int, float2 z) {
        const float c = z.x * (1.0f / M);
        if (dk && n < L) dk[(size_t)h * L + n] = c;
        if (n == 0 && dD) dD[h] = c;
    });
}

// Input-dependent filters ("Native Multi-Dimensional Subquadratic Operators
// via Input Dependent Long Convolutions", abstract: input-dependent long
// convolutions), one CTA per (pair of batch rows, channel), 2N <= 8192: each
// row's filter k[b][h] is transformed in the same launch.  Row b is packed
// with its own filter, z = x_b + i k_b, so one transform gives both spectra
// (X = (Z[f] + conj Z[-f]) / 2, K = (Z[f] - conj Z[-f]) / 2i); the products
// P_b = X_b (K_b + D) of the two rows are packed again, W = P_b + i P_b+1
// (P is Hermitian, so W[-f] = conj P_b[f] + i conj P_b+1[f]), and one inverse
// transform gives both outputs.  Two transforms in shared memory.
template <int LOG2M, typename IO, bool GATED>
__global__ void __launch_bounds__(FusedG<LOG2M>::T)
fused_dyn_simt(const IO* __restrict__ u, const IO* __restrict__ v, const IO* __restrict__ w,
               const float* __restrict__ k, int L, const float* __restrict__ D, IO* __restrict__ y,
               const float2* __restrict__ tw, int B, int H) {
    using G = FusedG<LOG2M>;
    using Lay = typename G::Lay;
    constexpr int M = G::L, N = M / 2, NS = G::Plan::kStages;
    static_assert(NS >= 2, "transform too short");
    constexpr int R0 = first_radix<G>(), RL = last_radix<G>();
    extern __shared__ float2 smem[];
    float2* sa = smem;
    float2* sb = smem + Lay::kWords;
    const int tid = threadIdx.x, h = blockIdx.y;
    const int b0 = 2 * blockIdx.x;
    const bool has1 = b0 + 1 < B;
    const size_t row0 = ((size_t)b0 * H + h) * N;
    const size_t row1 = ((size_t)(b0 + 1) * H + h) * N;
    const float* __restrict__ k0 = k + ((size_t)b0 * H + h) * L;
    const float* __restrict__ k1 = k + ((size_t)(b0 + 1) * H + h) * L;
    // z_b = x_b + i k_b, zero-padded, for both rows
    stage<G, 0, false, R0 / 2, R0, false>(
        tid, tw,
        [&](int n, int) {
            const float2 xx = load_pair<IO, GATED>(u, w, row0, row1, false, n);
            return make_float2(xx.x, n < L ? k0[n] : 0.f);
        },
        [&](int i, int, float2 z) { sa[Lay::at(i, 0)] = z; });
    stage<G, 0, false, R0 / 2, R0, false>(
        tid, tw,
        [&](int n, int) {
            if (!has1) return make_float2(0.f, 0.f);
            const float2 xx = load_pair<IO, GATED>(u, w, row1, row1, false, n);
            return make_float2(xx.x, n < L ? k1[n] : 0.f);
        },
        [&](int i, int, float2 z) { sb[Lay::at(i, 0)] = z; });
    __syncthreads();
    smem_stages<G, 1, NS, false>(sa, tid, tw);
    smem_stages<G, 1, NS, false>(sb, tid, tw);
    // P = X (K + D) per row, packed W = P_b + i P_b+1 (scaled 1/M) into sa
    const float dd = D ? D[h] : 0.f;
    auto prod = [&](float2 zf, float2 zg) {
        const float2 X = make_float2(0.5f * (zf.x + zg.x), 0.5f * (zf.y - zg.y));
        const float2 K = make_float2(0.5f * (zf.y + zg.y) + dd, 0.5f * (zg.x - zf.x));
        return cmul(X, K);
    };
    for (int f = tid; f <= M / 2; f += G::T) {
        const int g = (M - f) & (M - 1);
        const float2 af = sa[Lay::at(f, 0)], ag = sa[Lay::at(g, 0)];
        const float2 bf = sb[Lay::at(f, 0)], bg = sb[Lay::at(g, 0)];
        const float2 p1 = prod(af, ag), p2 = prod(bf, bg);
        constexpr float s = 1.0f / M;
        sa[Lay::at(f, 0)] = make_float2((p1.x - p2.y) * s, (p1.y + p2.x) * s);
        if (g != f) sa[Lay::at(g, 0)] = make_float2((p1.x + p2.y) * s, (p2.x - p1.y) * s);
    }
    __syncthreads();
    smem_stages<G, 0, NS - 1, true>(sa, tid, tw);
    stage<G, NS - 1, true, RL, RL / 2, false>(
        tid, tw, [&](int i, int) { return sa[Lay::at(i, 0)]; },
        [&](int n, int, float2 z) { store_pair<IO, GATED>(y, v, row0, row1, has1, n, z); });
}

// Partial convolutions ("FlashFFTConv", abstract: partial convolutions, a
// filter shorter than the sequence, computed by skipping blocks of the
// decomposition): for L <= T the row is cut into chunks of T and chunk c is
// computed by overlap-save on a transform of 2T = M points over the window
// x[cT - T, cT + T) (zeros before the row start).  The circular convolution
// with the zero-padded k[:L] wraps only into outputs n < L - 1 of the window,
// so its upper half n in [T, 2T) is exactly y[cT, cT + T): the cost is
// O(N log T) on chip instead of O(N log N) through memory.  One CTA per (pair
// of batch rows, channel x chunk); every chunk of a channel shares its
// spectrum.
template <int LOG2M, typename IO, bool GATED>
__global__ void __launch_bounds__(FusedG<LOG2M>::T)
fused_part_simt(const IO* __restrict__ u, const IO* __restrict__ v, const IO* __restrict__ w,
                const float2* __restrict__ khat, const float* __restrict__ D, IO* __restrict__ y,
                const float2* __restrict__ tw, int B, int H, int nc) {
    using G = FusedG<LOG2M>;
    using Lay = typename G::Lay;
    constexpr int M = G::L, T = M / 2, NS = G::Plan::kStages;
    static_assert(NS >= 2, "transform too short");
    constexpr int R0 = first_radix<G>(), RL = last_radix<G>();
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x, h = blockIdx.y / nc, c = blockIdx.y % nc;
    const int b0 = 2 * blockIdx.x;
    const bool has1 = b0 + 1 < B;
    const size_t NR = (size_t)nc * T;  // row length
    const size_t row0 = ((size_t)b0 * H + h) * NR;
    const size_t row1 = ((size_t)(b0 + 1) * H + h) * NR;
    const int64_t start = (int64_t)c * T - T;
    auto lds = [&](int i, int) { return smem[Lay::at(i, 0)]; };
    auto sts = [&](int i, int, float2 z) { smem[Lay::at(i, 0)] = z; };
    stage<G, 0, false, R0, R0, false>(
        tid, tw,
        [&](int n, int) {
            const int64_t pos = start + n;
            return pos < 0 ? make_float2(0.f, 0.f) : load_pair<IO, GATED>(u, w, row0, row1, has1, (size_t)pos);
        },
        sts);
    __syncthreads();
    smem_stages<G, 1, NS, false>(smem, tid, tw);
    const float dm = D ? D[h] * (1.0f / M) : 0.f;
    const float2* __restrict__ kh = khat + (size_t)h * M;
    stage<G, 0, true, R0, R0, true>(
        tid, tw,
        [&](int i, int) {
            float2 kk = __ldg(&kh[i]);
            kk.x += dm;
            return cmul(smem[Lay::at(i, 0)], kk);
        },
        sts);
    __syncthreads();
    smem_stages<G, 1, NS - 1, true>(smem, tid, tw);
    stage<G, NS - 1, true, RL, RL, false>(tid, tw, lds, [&](int n, int, float2 z) {
        if (n >= T) store_pair<IO, GATED>(y, v, row0, row1, has1, (size_t)(start + n), z);
    });
}

template <int LOG2M>
static size_t fused_smem() { return FusedG<LOG2M>::Lay::kWords * sizeof(float2); }

template <class K>
static void ensure_smem(K kern, size_t bytes) {
    if (bytes > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int LOG2M, typename IO, bool GATED>
static cudaError_t fused_fwd_go(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                                const float2* khat, const float* D, void* y, cudaStream_t s) {
    auto kern = fused_fwd_simt<LOG2M, IO, GATED>;
    const size_t smem = fused_smem<LOG2M>();
    ensure_smem(kern, smem);
    dim3 grid((p.B + 1) / 2, p.H);
    kern<<<grid, FusedG<LOG2M>::T, smem, s>>>((const IO*)u, (const IO*)v, (const IO*)w, khat, D, (IO*)y,
                                               p.tw.wL, p.B, p.H, p.kdiv);
    return cudaGetLastError();
}

template <int LOG2M>
static cudaError_t fused_fwd_dtype(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                                   const float2* khat, const float* D, void* y, cudaStream_t s) {
    if (p.dtype == FFTCONV_F32)
        return p.gated ? fused_fwd_go<LOG2M, float, true>(p, u, v, w, khat, D, y, s)
                       : fused_fwd_go<LOG2M, float, false>(p, u, v, w, khat, D, y, s);
    return p.gated ? fused_fwd_go<LOG2M, __nv_bfloat16, true>(p, u, v, w, khat, D, y, s)
                   : fused_fwd_go<LOG2M, __nv_bfloat16, false>(p, u, v, w, khat, D, y, s);
}

template <int LOG2M>
static cudaError_t fused_spec_go(const fftconv_plan_s& p, const float* k, int64_t L, float2* khat,
                                 cudaStream_t s) {
    auto kern = fused_spectrum_simt<LOG2M>;
    const size_t smem = fused_smem<LOG2M>();
    ensure_smem(kern, smem);
    kern<<<p.H, FusedG<LOG2M>::T, smem, s>>>(k, (int)L, khat, p.tw.wL);
    return cudaGetLastError();
}

bool fused_tables(int log2M, std::vector<float2>& out, size_t* offL) {
    *offL = out.size();
    switch (log2M) {
#define FFTC_T(X) case X: append_stage_twiddles<FusedG<X>>(out); return true;
        FFTC_T(7) FFTC_T(8) FFTC_T(9) FFTC_T(10) FFTC_T(11) FFTC_T(12) FFTC_T(13) FFTC_T(14)
#undef FFTC_T
        default: return false;
    }
}

cudaError_t launch_fused_fwd(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                             const float2* khat, const float* D, void* y, cudaStream_t s) {
    switch (p.log2M) {
        case 7: return fused_fwd_dtype<7>(p, u, v, w, khat, D, y, s);
        case 8: return fused_fwd_dtype<8>(p, u, v, w, khat, D, y, s);
        case 9: return fused_fwd_dtype<9>(p, u, v, w, khat, D, y, s);
        case 10: return fused_fwd_dtype<10>(p, u, v, w, khat, D, y, s);
        case 11: return fused_fwd_dtype<11>(p, u, v, w, khat, D, y, s);
        case 12: return fused_fwd_dtype<12>(p, u, v, w, khat, D, y, s);
        case 13: return fused_fwd_dtype<13>(p, u, v, w, khat, D, y, s);
        case 14: return fused_fwd_dtype<14>(p, u, v, w, khat, D, y, s);
        default: return cudaErrorInvalidValue;
    }
}

// acc: [H][pairs per channel][M] fp32 complex (kgrad_workspace_elems)
template <int LOG2M, typename IO, bool GATED>
static cudaError_t kgrad_go(const fftconv_plan_s& p, const void* u, const void* w, const void* dy, const void* v,
                            float2* acc, float* dk, float* dD, int L, cudaStream_t s) {
    auto k1 = kgrad_pairs<LOG2M, IO, GATED>;
    auto k2 = kgrad_finish<LOG2M>;
    const size_t smem = fused_smem<LOG2M>();
    ensure_smem(k1, smem);
    ensure_smem(k2, smem);
    const int npp = (p.B + 1) / 2;
    k1<<<dim3(npp, p.H), FusedG<LOG2M>::T, smem, s>>>((const IO*)u, (const IO*)w, (const IO*)dy, (const IO*)v, acc,
                                                      p.tw.wL, p.B, p.H);
    k2<<<p.H, FusedG<LOG2M>::T, smem, s>>>(acc, dk, dD, p.tw.wL, npp, L);
    return cudaGetLastError();
}

template <int LOG2M>
static cudaError_t kgrad_dt(const fftconv_plan_s& p, const void* u, const void* w, const void* dy, const void* v,
                            float2* acc, float* dk, float* dD, int L, cudaStream_t s) {
    if (p.dtype == FFTCONV_BF16)
        return p.gated ? kgrad_go<LOG2M, __nv_bfloat16, true>(p, u, w, dy, v, acc, dk, dD, L, s)
                       : kgrad_go<LOG2M, __nv_bfloat16, false>(p, u, w, dy, v, acc, dk, dD, L, s);
    return p.gated ? kgrad_go<LOG2M, float, true>(p, u, w, dy, v, acc, dk, dD, L, s)
                   : kgrad_go<LOG2M, float, false>(p, u, w, dy, v, acc, dk, dD, L, s);
}

bool kgrad_supported(int log2M) { return log2M >= 7 && log2M <= 14; }

// frequency-sparse plans: zero the spectrum rows k1 (all k2) the mask drops;
// the multi-pass spectrum is [H][k1 N1][k2 N2]
__global__ void zero_spectrum_rows(float2* __restrict__ khat, const uint8_t* __restrict__ keep, int N1, int N2,
                                   size_t total) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const int k1 = (int)((i / N2) % N1);
        if (!keep[k1]) khat[i] = make_float2(0.f, 0.f);
    }
}

cudaError_t launch_zero_spectrum_rows(const fftconv_plan_s& p, void* khat, cudaStream_t s) {
    const size_t total = (size_t)p.H << p.log2M;
    const size_t blocks = (total + 255) / 256;
    zero_spectrum_rows<<<(unsigned)(blocks < 8192 ? blocks : 8192), 256, 0, s>>>(
        (float2*)khat, p.d_keep, 1 << p.log2N1, 1 << p.log2N2, total);
    return cudaGetLastError();
}

template <int LOG2M, typename IO, bool GATED>
static cudaError_t dyn_go(const fftconv_plan_s& p, const void* u, const void* v, const void* w, const float* k,
                          int L, const float* D, void* y, cudaStream_t s) {
    auto kern = fused_dyn_simt<LOG2M, IO, GATED>;
    const size_t smem = 2 * fused_smem<LOG2M>();
    ensure_smem(kern, smem);
    dim3 grid((p.B + 1) / 2, p.H);
    kern<<<grid, FusedG<LOG2M>::T, smem, s>>>((const IO*)u, (const IO*)v, (const IO*)w, k, L, D, (IO*)y, p.tw.wL,
                                               p.B, p.H);
    return cudaGetLastError();
}

template <int LOG2M>
static cudaError_t dyn_dt(const fftconv_plan_s& p, const void* u, const void* v, const void* w, const float* k,
                          int L, const float* D, void* y, cudaStream_t s) {
    if (p.dtype == FFTCONV_BF16)
        return p.gated ? dyn_go<LOG2M, __nv_bfloat16, true>(p, u, v, w, k, L, D, y, s)
                       : dyn_go<LOG2M, __nv_bfloat16, false>(p, u, v, w, k, L, D, y, s);
    return p.gated ? dyn_go<LOG2M, float, true>(p, u, v, w, k, L, D, y, s)
                   : dyn_go<LOG2M, float, false>(p, u, v, w, k, L, D, y, s);
}

bool dyn_supported(int log2M) { return log2M >= 7 && log2M <= 13; }

template <int LOG2M, typename IO, bool GATED>
static cudaError_t part_go(const fftconv_plan_s& p, const void* u, const void* v, const void* w, const float2* khat,
                           const float* D, void* y, cudaStream_t s) {
    auto kern = fused_part_simt<LOG2M, IO, GATED>;
    const size_t smem = fused_smem<LOG2M>();
    ensure_smem(kern, smem);
    dim3 grid((p.B + 1) / 2, (unsigned)(p.H * p.nchunks));
    kern<<<grid, FusedG<LOG2M>::T, smem, s>>>((const IO*)u, (const IO*)v, (const IO*)w, khat, D, (IO*)y,
                                               p.chunk->tw.wL, p.B, p.H, (int)p.nchunks);
    return cudaGetLastError();
}

template <int LOG2M>
static cudaError_t part_dt(const fftconv_plan_s& p, const void* u, const void* v, const void* w, const float2* khat,
                           const float* D, void* y, cudaStream_t s) {
    if (p.dtype == FFTCONV_BF16)
        return p.gated ? part_go<LOG2M, __nv_bfloat16, true>(p, u, v, w, khat, D, y, s)
                       : part_go<LOG2M, __nv_bfloat16, false>(p, u, v, w, khat, D, y, s);
    return p.gated ? part_go<LOG2M, float, true>(p, u, v, w, khat, D, y, s)
                   : part_go<LOG2M, float, false>(p, u, v, w, khat, D, y, s);
}

cudaError_t launch_partial_fwd(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                               const float2* khat, const float* D, void* y, cudaStream_t s) {
    switch (p.chunk->log2M) {
#define FFTC_P(X) case X: return part_dt<X>(p, u, v, w, khat, D, y, s);
        FFTC_P(7) FFTC_P(8) FFTC_P(9) FFTC_P(10) FFTC_P(11) FFTC_P(12) FFTC_P(13) FFTC_P(14)
#undef FFTC_P
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_dyn_fwd(const fftconv_plan_s& p, const void* u, const void* v, const void* w, const float* k,
                           int64_t L, const float* D, void* y, cudaStream_t s) {
    switch (p.log2M) {
#define FFTC_D(X) case X: return dyn_dt<X>(p, u, v, w, k, (int)L, D, y, s);
        FFTC_D(7) FFTC_D(8) FFTC_D(9) FFTC_D(10) FFTC_D(11) FFTC_D(12) FFTC_D(13)
#undef FFTC_D
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_kgrad(const fftconv_plan_s& p, const void* u, const void* w, const void* dy, const void* v,
                         float2* acc, float* dk, float* dD, int64_t L, cudaStream_t s) {
    switch (p.log2M) {
#define FFTC_K(X) case X: return kgrad_dt<X>(p, u, w, dy, v, acc, dk, dD, (int)L, s);
        FFTC_K(7) FFTC_K(8) FFTC_K(9) FFTC_K(10) FFTC_K(11) FFTC_K(12) FFTC_K(13) FFTC_K(14)
#undef FFTC_K
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_t2_spectrum(const fftconv_plan_s& p, const float* k, int64_t L, void* khat, cudaStream_t s) {
    if (p.log2M != 13) return cudaErrorInvalidValue;
    auto kern = t2_spectrum_simt;
    const size_t smem = fused_smem<13>();
    ensure_smem(kern, smem);
    kern<<<p.H, FusedG<13>::T, smem, s>>>(k, (int)L, (uint16_t*)khat, p.tw.wL);
    return cudaGetLastError();
}

cudaError_t launch_fused_spectrum(const fftconv_plan_s& p, const float* k, int64_t L, float2* khat,
                                  cudaStream_t s) {
    switch (p.log2M) {
        case 7: return fused_spec_go<7>(p, k, L, khat, s);
        case 8: return fused_spec_go<8>(p, k, L, khat, s);
        case 9: return fused_spec_go<9>(p, k, L, khat, s);
        case 10: return fused_spec_go<10>(p, k, L, khat, s);
        case 11: return fused_spec_go<11>(p, k, L, khat, s);
        case 12: return fused_spec_go<12>(p, k, L, khat, s);
        case 13: return fused_spec_go<13>(p, k, L, khat, s);
        case 14: return fused_spec_go<14>(p, k, L, khat, s);
        default: return cudaErrorInvalidValue;
    }
}

// ========================================================== multi-pass path
// Columns per CTA in the column passes: as many as one CTA's 16384 points
// allow, at most 32 (rows of 256 B of fp32 complex in the workspace, 128 B of
// fp32 input and output).
template <int LOG2N1>
constexpr int kColTile = (16384 >> LOG2N1) < 32 ? (16384 >> LOG2N1) : 32;

template <int LOG2N1>
using ColG = Geometry<LOG2N1, kColTile<LOG2N1>, true>;
// Rows per CTA in the row pass: enough that one CTA holds 4096 points (at
// most 16 rows), so short rows do not leave single-warp CTAs.
constexpr int row_batch(int log2n2) { return log2n2 >= 12 ? 1 : ((4096 >> log2n2) > 16 ? 16 : (4096 >> log2n2)); }

// One row per CTA (2^12 points and up): a pad slot every 16 values, so the
// first stage's writes (16 consecutive outputs per thread, stride 16 across
// the lanes) land in distinct bank pairs; several rows: every 32.
template <int LOG2N2>
using RowG = Geometry<LOG2N2, row_batch(LOG2N2), false, row_batch(LOG2N2) == 1 ? 4 : 5>;

// Outputs per exact twiddle lookup in the pass epilogues; in between the
// twiddle is advanced by one fp32 complex product (at most kTwRun - 1 chained
// products: relative error below 1e-6).
constexpr int kTwRun = 8;

// W_M^e from the two-level table, e reduced mod M.
__device__ __forceinline__ float2 twiddle_M(const float2* __restrict__ lo, const float2* __restrict__ hi,
                                            uint32_t e, int log2M, int log2S) {
    e &= (1u << log2M) - 1u;
    return cmul(__ldg(&lo[e & ((1u << log2S) - 1u)]), __ldg(&hi[e >> log2S]));
}

// Pass 1.  MODE 0: x from (u[,w]) rows of pair P = first + blockIdx.y;
//          MODE 1: real kernel taps k[h] (h = first + blockIdx.y), n < L.
template <int LOG2N1, int LOG2N2, typename IO, bool GATED, int MODE>
__global__ void __launch_bounds__(ColG<LOG2N1>::T)
mp_pass1(const IO* __restrict__ u, const IO* __restrict__ w, const float* __restrict__ k, int L,
         float2* __restrict__ work, const float2* __restrict__ twC, const float2* __restrict__ lo,
         const float2* __restrict__ hi, int log2S, int B, int H, int64_t first, const uint8_t* __restrict__ keep) {
    using G = ColG<LOG2N1>;
    using Lay = typename G::Lay;
    constexpr int N1 = 1 << LOG2N1, N2 = 1 << LOG2N2, LOG2M = LOG2N1 + LOG2N2;
    constexpr int64_t N = (int64_t)N1 * N2 / 2;
    constexpr int NS = G::Plan::kStages, R0 = first_radix<G>(), RL = last_radix<G>();
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x;
    const int64_t P = first + blockIdx.y;
    const int n2_0 = blockIdx.x * kColTile<LOG2N1>;
    auto lds = [&](int i, int c) { return smem[Lay::at(i, c)]; };
    auto sts = [&](int i, int c, float2 z) { smem[Lay::at(i, c)] = z; };
    if constexpr (MODE == 0) {
        const int h = (int)(P % H);
        const int b0 = (int)(P / H) * 2;
        const bool has1 = b0 + 1 < B;
        const size_t row0 = ((size_t)b0 * H + h) * N, row1 = ((size_t)(b0 + 1) * H + h) * N;
        stage<G, 0, false, R0 / 2, R0, false>(
            tid, twC,
            [&](int n1, int c) {
                return load_pair<IO, GATED>(u, w, row0, row1, has1, (size_t)n1 * N2 + n2_0 + c);
            },
            sts);
    } else {
        const float* __restrict__ kr = k + (size_t)P * L;
        stage<G, 0, false, R0 / 2, R0, false>(
            tid, twC,
            [&](int n1, int c) {
                const int64_t n = (int64_t)n1 * N2 + n2_0 + c;
                return make_float2(n < L ? kr[n] : 0.f, 0.f);
            },
            sts);
    }
    __syncthreads();
    smem_stages<G, 1, NS - 1, false>(smem, tid, twC);
    float2* __restrict__ out = work + (size_t)blockIdx.y * ((size_t)N1 * N2);
    // W_M^{n2 k1} along the thread's outputs k1 = j + r N1/RL: looked up every
    // kTwRun outputs, advanced by W_M^{n2 N1/RL} in between
    float2 tw = make_float2(1.f, 0.f), step = make_float2(1.f, 0.f);
    stage<G, NS - 1, false, RL, RL, false>(tid, twC, lds, [&](int k1, int c, float2 z, int r) {
        const uint32_t n2 = (uint32_t)(n2_0 + c);
        if (r == 0) step = twiddle_M(lo, hi, n2 * (uint32_t)(N1 / RL), LOG2M, log2S);
        tw = (r % kTwRun == 0) ? twiddle_M(lo, hi, n2 * (uint32_t)k1, LOG2M, log2S) : cmul(tw, step);
        // frequency-sparse plans: rows k1 whose spectrum is zeroed are never read again
        if (!keep || keep[k1]) out[(size_t)k1 * N2 + n2] = cmul(z, tw);
    });
}

// Pass 1, persistent (ungated forward): a CTA walks column tiles t =
// blockIdx.x, + gridDim.x, ... (consecutive tiles share a pair), staging the
// next tile's input rows (both images, rows n1 < N1/2, 32 columns) with
// cp.async into a second buffer while it transforms the current one.
template <int LOG2N1, int LOG2N2, typename IO>
constexpr size_t mp1p_raw_bytes() {
    return (size_t)2 * ((1 << LOG2N1) / 2) * kColTile<LOG2N1> * sizeof(IO);
}

template <int LOG2N1, int LOG2N2, typename IO>
__global__ void __launch_bounds__(ColG<LOG2N1>::T)
mp_pass1p(const IO* __restrict__ u, float2* __restrict__ work, const float2* __restrict__ twC,
          const float2* __restrict__ lo, const float2* __restrict__ hi, int log2S, int B, int H, int64_t first,
          int g, const uint8_t* __restrict__ keep) {
    using G = ColG<LOG2N1>;
    using Lay = typename G::Lay;
    constexpr int N1 = 1 << LOG2N1, N2 = 1 << LOG2N2, LOG2M = LOG2N1 + LOG2N2;
    constexpr int64_t N = (int64_t)N1 * N2 / 2;
    constexpr int CT = kColTile<LOG2N1>, TPP = N2 / CT;  // columns per tile, tiles per pair
    constexpr int NS = G::Plan::kStages, R0 = first_radix<G>(), RL = last_radix<G>();
    constexpr int CPR = CT * (int)sizeof(IO) / 16;      // 16-byte chunks per input row of a tile
    extern __shared__ float2 smem[];
    IO* raw = reinterpret_cast<IO*>(smem + Lay::kWords);  // [image 2][n1 < N1/2][CT]
    const uint32_t raw_s = tc::smem_u32(raw);
    const int tid = threadIdx.x;
    const int tiles = TPP * g;
    auto lds = [&](int i, int c) { return smem[Lay::at(i, c)]; };
    auto sts = [&](int i, int c, float2 z) { smem[Lay::at(i, c)] = z; };
    auto prefetch = [&](int t) {
        const int64_t P = first + t / TPP;
        const int n2_0 = (t % TPP) * CT;
        const int h = (int)(P % H), b0 = (int)(P / H) * 2;
        const bool has1 = b0 + 1 < B;
        for (int j = tid; j < 2 * (N1 / 2) * CPR; j += G::T) {
            const int im = j / ((N1 / 2) * CPR), rem = j % ((N1 / 2) * CPR), n1 = rem / CPR, ch = rem % CPR;
            const bool ok = im == 0 || has1;
            const size_t row = ((size_t)(b0 + (ok ? im : 0)) * H + h) * N;
            const IO* src = u + row + (size_t)n1 * N2 + n2_0 + ch * (16 / (int)sizeof(IO));
            tc::cp_async16(raw_s + (uint32_t)j * 16u, src, ok ? 16 : 0);
        }
        tc::cp_async_commit();
    };
    int t = blockIdx.x;
    if (t < tiles) prefetch(t);
    for (; t < tiles; t += gridDim.x) {
        tc::cp_async_wait_all();
        __syncthreads();  // the tile's input is in; the previous tile's transform is written out
        const int64_t P = first + t / TPP;
        const int n2_0 = (t % TPP) * CT;
        stage<G, 0, false, R0 / 2, R0, false>(
            tid, twC,
            [&](int n1, int c) {
                return make_float2(to_f(raw[(size_t)n1 * CT + c]), to_f(raw[(size_t)(N1 / 2 + n1) * CT + c]));
            },
            sts);
        __syncthreads();  // the input buffer is free: stage the next tile's
        if (t + (int)gridDim.x < tiles) prefetch(t + gridDim.x);
        smem_stages<G, 1, NS - 1, false>(smem, tid, twC);
        float2* __restrict__ out = work + (size_t)(t / TPP) * ((size_t)N1 * N2);
        float2 tw = make_float2(1.f, 0.f), step = make_float2(1.f, 0.f);
        stage<G, NS - 1, false, RL, RL, false>(tid, twC, lds, [&](int k1, int c, float2 z, int r) {
            const uint32_t n2 = (uint32_t)(n2_0 + c);
            if (r == 0) step = twiddle_M(lo, hi, n2 * (uint32_t)(N1 / RL), LOG2M, log2S);
            tw = (r % kTwRun == 0) ? twiddle_M(lo, hi, n2 * (uint32_t)k1, LOG2M, log2S) : cmul(tw, step);
            if (!keep || keep[k1]) out[(size_t)k1 * N2 + n2] = cmul(z, tw);
        });
        (void)P;
    }
    tc::cp_async_wait_all();
}

// Pass 2.  MODE 0: forward row DFT, product with Khat (+D/M), inverse, conj
// twiddle, in place.  MODE 1: forward row DFT only, Khat[k1][k2] = X / M.
// Three CTAs of up to 256 threads per SM (at most 85 registers; no spills).
template <int LOG2N1, int LOG2N2, int MODE>
__global__ void __launch_bounds__(RowG<LOG2N2>::T, RowG<LOG2N2>::T <= 256 ? 3 : 1)
mp_pass2(float2* __restrict__ work, const float2* __restrict__ khat, float2* __restrict__ khat_out,
         const float* __restrict__ D, const float2* __restrict__ twR, const float2* __restrict__ lo,
         const float2* __restrict__ hi, int log2S, int H, int64_t first, const uint8_t* __restrict__ keep) {
    using G = RowG<LOG2N2>;
    using Lay = typename G::Lay;
    constexpr int N1 = 1 << LOG2N1, N2 = 1 << LOG2N2, LOG2M = LOG2N1 + LOG2N2;
    constexpr int M = N1 * N2;
    constexpr int NS = G::Plan::kStages, R0 = first_radix<G>(), RL = last_radix<G>();
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x;
    constexpr int RC = G::C;                    // rows k1 of this CTA: k1_0 .. k1_0 + RC - 1
    const int k1_0 = blockIdx.x * RC;
    const int64_t P = first + blockIdx.y;
    if (MODE == 0 && keep) {
        // frequency-sparse plans: a CTA whose rows all have a zeroed spectrum has no work
        bool any = false;
#pragma unroll
        for (int c = 0; c < RC; ++c) any |= keep[k1_0 + c] != 0;
        if (!any) return;
    }
    float2* __restrict__ rows = work + ((size_t)blockIdx.y * N1 + k1_0) * N2;
    auto lds = [&](int i, int c) { return smem[Lay::at(i, c)]; };
    auto sts = [&](int i, int c, float2 z) { smem[Lay::at(i, c)] = z; };
    stage<G, 0, false, R0, R0, false>(tid, twR, [&](int n2, int c) { return rows[(size_t)c * N2 + n2]; }, sts);
    __syncthreads();
    if constexpr (MODE == 1) {
        smem_stages<G, 1, NS - 1, false>(smem, tid, twR);
        float2* __restrict__ out = khat_out + ((size_t)P * N1 + k1_0) * N2;
        stage<G, NS - 1, false, RL, RL, false>(
            tid, twR, lds, [&](int k2, int c, float2 z) { out[(size_t)c * N2 + k2] = cscale(z, 1.0f / M); });
    } else {
        smem_stages<G, 1, NS, false>(smem, tid, twR);
        const int h = (int)(P % H);
        const float dm = D ? D[h] * (1.0f / M) : 0.f;
        const float2* __restrict__ kh = khat + ((size_t)h * N1 + k1_0) * N2;
        stage<G, 0, true, R0, R0, true>(
            tid, twR,
            [&](int k2, int c) {
                float2 kk = __ldg(&kh[(size_t)c * N2 + k2]);
                kk.x += dm;
                return cmul(smem[Lay::at(k2, c)], kk);
            },
            sts);
        __syncthreads();
        smem_stages<G, 1, NS - 1, true>(smem, tid, twR);
        // W_M^{n2 k1} along the thread's outputs n2 = j + r N2/RL (see pass 1)
        float2 tw = make_float2(1.f, 0.f), step = make_float2(1.f, 0.f);
        stage<G, NS - 1, true, RL, RL, false>(tid, twR, lds, [&](int n2, int c, float2 z, int r) {
            const uint32_t k1 = (uint32_t)(k1_0 + c);
            if (r == 0) step = twiddle_M(lo, hi, k1 * (uint32_t)(N2 / RL), LOG2M, log2S);
            tw = (r % kTwRun == 0) ? twiddle_M(lo, hi, (uint32_t)n2 * k1, LOG2M, log2S) : cmul(tw, step);
            rows[(size_t)c * N2 + n2] = cmulc(z, tw);
        });
    }
}

// Pass 3: inverse column DFT; outputs n1 < N1/2 (n < N) to y.
template <int LOG2N1, int LOG2N2, typename IO, bool GATED>
__global__ void __launch_bounds__(ColG<LOG2N1>::T)
mp_pass3(const float2* __restrict__ work, const IO* __restrict__ v, IO* __restrict__ y,
         const float2* __restrict__ twC, int B, int H, int64_t first, const uint8_t* __restrict__ keep) {
    using G = ColG<LOG2N1>;
    using Lay = typename G::Lay;
    constexpr int N1 = 1 << LOG2N1, N2 = 1 << LOG2N2;
    constexpr int64_t N = (int64_t)N1 * N2 / 2;
    constexpr int NS = G::Plan::kStages, R0 = first_radix<G>(), RL = last_radix<G>();
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x;
    const int64_t P = first + blockIdx.y;
    const int n2_0 = blockIdx.x * kColTile<LOG2N1>;
    const float2* __restrict__ in = work + (size_t)blockIdx.y * ((size_t)N1 * N2);
    auto lds = [&](int i, int c) { return smem[Lay::at(i, c)]; };
    auto sts = [&](int i, int c, float2 z) { smem[Lay::at(i, c)] = z; };
    stage<G, 0, true, R0, R0, false>(
        tid, twC,
        [&](int k1, int c) {
            return (!keep || keep[k1]) ? in[(size_t)k1 * N2 + n2_0 + c] : make_float2(0.f, 0.f);
        },
        sts);
    __syncthreads();
    smem_stages<G, 1, NS - 1, true>(smem, tid, twC);
    const int h = (int)(P % H);
    const int b0 = (int)(P / H) * 2;
    const bool has1 = b0 + 1 < B;
    const size_t row0 = ((size_t)b0 * H + h) * N, row1 = ((size_t)(b0 + 1) * H + h) * N;
    stage<G, NS - 1, true, RL, RL / 2, false>(tid, twC, lds, [&](int n1, int c, float2 z) {
        store_pair<IO, GATED>(y, v, row0, row1, has1, (size_t)n1 * N2 + n2_0 + c, z);
    });
}

template <int LOG2N1, int LOG2N2, typename IO, bool GATED>
static cudaError_t mp_fwd_go(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                             const float2* khat, const float* D, void* y, float2* work, cudaStream_t s) {
    constexpr int N2 = 1 << LOG2N2, N1 = 1 << LOG2N1;
    auto k1 = mp_pass1<LOG2N1, LOG2N2, IO, GATED, 0>;
    auto k2 = mp_pass2<LOG2N1, LOG2N2, 0>;
    auto k3 = mp_pass3<LOG2N1, LOG2N2, IO, GATED>;
    const size_t sc = ColG<LOG2N1>::Lay::kWords * sizeof(float2);
    const size_t sr = RowG<LOG2N2>::Lay::kWords * sizeof(float2);
    ensure_smem(k1, sc);
    ensure_smem(k2, sr);
    ensure_smem(k3, sc);
    // ungated: the persistent pass 1 that stages the next tile's input while it
    // transforms the current one (one CTA per SM)
    auto k1p = mp_pass1p<LOG2N1, LOG2N2, IO>;
    const size_t sp = sc + mp1p_raw_bytes<LOG2N1, LOG2N2, IO>();
    static int sms = 0;
    if (!GATED) {
        ensure_smem(k1p, sp);
        if (sms == 0) {
            int dev = 0;
            cudaGetDevice(&dev);
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (sms <= 0) sms = 1;
        }
    }
    for (int64_t first = 0; first < p.pairs; first += p.group) {
        const int g = (int)((p.pairs - first) < p.group ? (p.pairs - first) : p.group);
        if (!GATED) {
            const int tiles = (N2 / kColTile<LOG2N1>) * g;
            k1p<<<tiles < sms ? tiles : sms, ColG<LOG2N1>::T, sp, s>>>((const IO*)u, work, p.tw.wC, p.tw.wLo,
                                                                      p.tw.wHi, p.log2S, p.B, p.H, first, g,
                                                                      p.d_keep);
        } else {
            k1<<<dim3(N2 / kColTile<LOG2N1>, g), ColG<LOG2N1>::T, sc, s>>>((const IO*)u, (const IO*)w, nullptr, 0,
                                                                   work, p.tw.wC, p.tw.wLo, p.tw.wHi, p.log2S,
                                                                   p.B, p.H, first, p.d_keep);
        }
        k2<<<dim3(N1 / RowG<LOG2N2>::C, g), RowG<LOG2N2>::T, sr, s>>>(work, khat, nullptr, D, p.tw.wL, p.tw.wLo, p.tw.wHi,
                                                    p.log2S, p.H, first, p.d_keep);
        k3<<<dim3(N2 / kColTile<LOG2N1>, g), ColG<LOG2N1>::T, sc, s>>>(work, (const IO*)v, (IO*)y, p.tw.wC, p.B,
                                                               p.H, first, p.d_keep);
    }
    return cudaGetLastError();
}

template <int LOG2N1, int LOG2N2>
static cudaError_t mp_fwd_dtype(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                                const float2* khat, const float* D, void* y, float2* work, cudaStream_t s) {
    if (p.dtype == FFTCONV_F32)
        return p.gated ? mp_fwd_go<LOG2N1, LOG2N2, float, true>(p, u, v, w, khat, D, y, work, s)
                       : mp_fwd_go<LOG2N1, LOG2N2, float, false>(p, u, v, w, khat, D, y, work, s);
    return p.gated ? mp_fwd_go<LOG2N1, LOG2N2, __nv_bfloat16, true>(p, u, v, w, khat, D, y, work, s)
                   : mp_fwd_go<LOG2N1, LOG2N2, __nv_bfloat16, false>(p, u, v, w, khat, D, y, work, s);
}

template <int LOG2N1, int LOG2N2>
static cudaError_t mp_spec_go(const fftconv_plan_s& p, const float* k, int64_t L, float2* khat, float2* work,
                              cudaStream_t s) {
    constexpr int N2 = 1 << LOG2N2, N1 = 1 << LOG2N1;
    auto k1 = mp_pass1<LOG2N1, LOG2N2, float, false, 1>;
    auto k2 = mp_pass2<LOG2N1, LOG2N2, 1>;
    const size_t sc = ColG<LOG2N1>::Lay::kWords * sizeof(float2);
    const size_t sr = RowG<LOG2N2>::Lay::kWords * sizeof(float2);
    ensure_smem(k1, sc);
    ensure_smem(k2, sr);
    for (int64_t first = 0; first < p.H; first += p.group) {
        const int g = (int)((p.H - first) < p.group ? (p.H - first) : p.group);
        k1<<<dim3(N2 / kColTile<LOG2N1>, g), ColG<LOG2N1>::T, sc, s>>>(nullptr, nullptr, k, (int)L, work, p.tw.wC,
                                                               p.tw.wLo, p.tw.wHi, p.log2S, p.B, p.H, first,
                                                               nullptr);
        k2<<<dim3(N1 / RowG<LOG2N2>::C, g), RowG<LOG2N2>::T, sr, s>>>(work, nullptr, khat, nullptr, p.tw.wL, p.tw.wLo, p.tw.wHi,
                                                    p.log2S, p.H, first, nullptr);
    }
    return cudaGetLastError();
}

#define FFTC_MP_SWITCH(CALL)             \
    switch (p.log2M) {                   \
        case 15: return CALL(7, 8);      \
        case 16: return CALL(8, 8);      \
        case 17: return CALL(8, 9);      \
        case 18: return CALL(9, 9);      \
        case 19: return CALL(9, 10);     \
        case 20: return CALL(9, 11);     \
        case 21: return CALL(9, 12);     \
        default: return cudaErrorInvalidValue; \
    }

template <int LOG2N1, int LOG2N2>
static bool mp_tables_go(std::vector<float2>& out, size_t* offC, size_t* offR) {
    *offC = out.size();
    append_stage_twiddles<ColG<LOG2N1>>(out);
    *offR = out.size();
    append_stage_twiddles<RowG<LOG2N2>>(out);
    return true;
}

bool multipass_tables(int log2M, std::vector<float2>& out, size_t* offC, size_t* offR) {
    switch (log2M) {
        case 15: return mp_tables_go<7, 8>(out, offC, offR);
        case 16: return mp_tables_go<8, 8>(out, offC, offR);
        case 17: return mp_tables_go<8, 9>(out, offC, offR);
        case 18: return mp_tables_go<9, 9>(out, offC, offR);
        case 19: return mp_tables_go<9, 10>(out, offC, offR);
        case 20: return mp_tables_go<9, 11>(out, offC, offR);
        case 21: return mp_tables_go<9, 12>(out, offC, offR);
        default: return false;
    }
}

cudaError_t launch_multipass_fwd(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                                 const float2* khat, const float* D, void* y, float2* work, cudaStream_t s) {
#define FFTC_CALL(a, b) mp_fwd_dtype<a, b>(p, u, v, w, khat, D, y, work, s)
    FFTC_MP_SWITCH(FFTC_CALL)
#undef FFTC_CALL
}

cudaError_t launch_multipass_spectrum(const fftconv_plan_s& p, const float* k, int64_t L, float2* khat,
                                      float2* work, cudaStream_t s) {
#define FFTC_CALL(a, b) mp_spec_go<a, b>(p, k, L, khat, work, s)
    FFTC_MP_SWITCH(FFTC_CALL)
#undef FFTC_CALL
}

}  // namespace fftc
