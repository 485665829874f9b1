// conv2d_simt.cu -- fp32 SIMT kernels of the 2-D causal FFT convolution.
//
// y[b,c] = crop_{[0,Hs) x [0,Ws)}( iDFT2( DFT2(pad(u[b,c])) . Khat[c] ) ), the
// zero-padded linear convolution of each image with its channel's kernel,
// first-quadrant crop -- the multi-dimensional FFT convolution of "Native
// Multi-Dimensional Subquadratic Operators via Input Dependent Long
// Convolutions" (abstract), with one fixed kernel per channel.  Two images
// b, b+1 of the same channel share one complex transform (real + imaginary).
// The transform is (2Hs) x (2Ws):
//   pass 1: row DFT_{2Ws} of the Hs nonzero rows (only j < Ws nonzero) -> work[i][kx]
//   pass 2: per 16-column tile: column DFT_{2Hs} over the Hs nonzero rows,
//           times Khat[c][ky][kx], inverse column DFT keeping rows i < Hs -> work
//   pass 3: inverse row DFT_{2Ws} of the Hs rows, keeping j < Ws -> y.
#include <type_traits>

#include "fft_simt.cuh"
#include "plan.h"
#include "tables.h"

namespace fftc {

constexpr int kTile2d = 16;  // columns per CTA in pass 2

// Rows per CTA in the row passes: as many as fit 8192 complex values.
template <int LOG2LR>
constexpr int rows_per_cta(int Hs) {
    return ((8192 >> LOG2LR) < Hs) ? (8192 >> LOG2LR) : Hs;
}

template <int LOG2LR, int RB>
using Row2G = Geometry<LOG2LR, RB, false>;
template <int LOG2LC>
using Col2G = Geometry<LOG2LC, kTile2d, true>;

template <class K>
static void ensure_smem2(K kern, size_t bytes) {
    if (bytes > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Pass 1. MODE 0: images of pair P; MODE 1: kernel k[c] (real), Kh x Kw taps.
template <int LOG2LR, int RB, typename IO, int MODE>
__global__ void __launch_bounds__(Row2G<LOG2LR, RB>::T)
c2_pass1(const IO* __restrict__ u, const float* __restrict__ k, int Kh, int Kw, float2* __restrict__ work,
         const float2* __restrict__ twR, int B, int C, int Hs, int64_t first) {
    using G = Row2G<LOG2LR, RB>;
    using Lay = typename G::Lay;
    constexpr int LR = 1 << LOG2LR, Ws = LR / 2;
    constexpr int NS = G::Plan::kStages;
    constexpr int R0 = 1 << G::Plan::log2r(0), RL = 1 << G::Plan::log2r(NS - 1);
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x;
    const int64_t P = first + blockIdx.y;
    const int i0 = blockIdx.x * RB;  // first image row of this CTA
    auto lds = [&](int i, int c) { return smem[Lay::at(i, c)]; };
    auto sts = [&](int i, int c, float2 z) { smem[Lay::at(i, c)] = z; };
    if constexpr (MODE == 0) {
        // pairs are channel-major (P = ch * npp + pp): a channel's pairs run together
        const int npp = (B + 1) / 2;
        const int ch = (int)(P / npp), b0 = (int)(P % npp) * 2;
        const bool has1 = b0 + 1 < B;
        const size_t img0 = ((size_t)b0 * C + ch) * Hs * Ws, img1 = ((size_t)(b0 + 1) * C + ch) * Hs * Ws;
        stage<G, 0, false, R0 / 2, R0, false>(
            tid, twR,
            [&](int j, int r) {
                const size_t off = (size_t)(i0 + r) * Ws + j;
                return make_float2(to_f(u[img0 + off]), has1 ? to_f(u[img1 + off]) : 0.f);
            },
            sts);
    } else {
        const float* __restrict__ kc = k + (size_t)P * Kh * Kw;
        stage<G, 0, false, R0 / 2, R0, false>(
            tid, twR,
            [&](int j, int r) {
                const int i = i0 + r;
                return make_float2((i < Kh && j < Kw) ? kc[(size_t)i * Kw + j] : 0.f, 0.f);
            },
            sts);
    }
    __syncthreads();
    smem_stages<G, 1, NS - 1, false>(smem, tid, twR);
    float2* __restrict__ out = work + (size_t)blockIdx.y * Hs * LR;
    stage<G, NS - 1, false, RL, RL, false>(tid, twR, lds, [&](int kx, int r, float2 z) {
        out[(size_t)(i0 + r) * LR + kx] = z;
    });
}

// Pass 2. MODE 0: column DFT, product, inverse column DFT (rows < Hs kept).
//         MODE 1: column DFT only; Khat[c][ky][kx] = X / (LC LR).
// KB: the spectrum is stored as packed bf16 (re, im) words (bf16 plans), else fp32 complex.
// KTC (MODE 1, bf16, 2 Hs = 512): stored in the order the tensor-core column
// pass reads -- per channel, column kx and parity of ky, per lane the packed
// (re pair, im pair) of the four A-fragment registers of the [c][d] tile,
// ky = parity + 2 (c + 16 d).
template <int LOG2LC, int LOG2LR, int MODE, bool KB, bool KTC = false>
__global__ void __launch_bounds__(Col2G<LOG2LC>::T)
c2_pass2(float2* __restrict__ work, const void* __restrict__ khat, void* __restrict__ khat_out,
         const float2* __restrict__ twC, int npp, int64_t first, int oy) {
    using G = Col2G<LOG2LC>;
    using Lay = typename G::Lay;
    constexpr int LC = 1 << LOG2LC, LR = 1 << LOG2LR, Hs = LC / 2;
    constexpr int NS = G::Plan::kStages;
    constexpr int R0 = 1 << G::Plan::log2r(0), RL = 1 << G::Plan::log2r(NS - 1);
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x;
    const int64_t P = first + blockIdx.y;
    const int kx0 = blockIdx.x * kTile2d;
    float2* __restrict__ img = work + (size_t)blockIdx.y * Hs * LR;
    auto lds = [&](int i, int c) { return smem[Lay::at(i, c)]; };
    auto sts = [&](int i, int c, float2 z) { smem[Lay::at(i, c)] = z; };
    stage<G, 0, false, R0 / 2, R0, false>(
        tid, twC, [&](int i, int c) { return img[(size_t)i * LR + kx0 + c]; }, sts);
    __syncthreads();
    if constexpr (MODE == 1) {
        smem_stages<G, 1, NS - 1, false>(smem, tid, twC);
        const size_t base = (size_t)P * LC * LR;
        constexpr float scale = 1.0f / ((float)LC * (float)LR);
        stage<G, NS - 1, false, RL, RL, false>(tid, twC, lds, [&](int ky, int c, float2 z) {
            const size_t o = base + (size_t)ky * LR + kx0 + c;
            z = cscale(z, scale);
            if constexpr (KTC) {
                static_assert(LC == 512 && KB, "fragment order: bf16, 512-point columns");
                const int kq = ky >> 1, cc = kq & 15, d = kq >> 4;
                const int ln = 4 * (cc & 7) + ((d >> 1) & 3), reg = (cc >> 3) + 2 * (d >> 3);
                const size_t word = (((size_t)P * LR + kx0 + c) * 2 + (ky & 1)) * 256 + ln * 8 + 2 * reg;
                uint16_t* h = static_cast<uint16_t*>(khat_out);
                h[word * 2 + (d & 1)] = __bfloat16_as_ushort(__float2bfloat16_rn(z.x));
                h[(word + 1) * 2 + (d & 1)] = __bfloat16_as_ushort(__float2bfloat16_rn(z.y));
            } else if (KB)
                static_cast<uint32_t*>(khat_out)[o] =
                    (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(z.x)) |
                    ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(z.y)) << 16);
            else
                static_cast<float2*>(khat_out)[o] = z;
        });
    } else {
        smem_stages<G, 1, NS, false>(smem, tid, twC);
        const size_t kbase = (size_t)(P / npp) * LC * LR;
        stage<G, 0, true, R0, R0, true>(
            tid, twC,
            [&](int ky, int c) {
                const size_t o = kbase + (size_t)ky * LR + kx0 + c;
                float2 kk;
                if (KB) {
                    const uint32_t wv = __ldg(static_cast<const uint32_t*>(khat) + o);
                    kk = make_float2(__uint_as_float(wv << 16), __uint_as_float(wv & 0xffff0000u));
                } else {
                    kk = __ldg(static_cast<const float2*>(khat) + o);
                }
                return cmul(smem[Lay::at(ky, c)], kk);
            },
            sts);
        __syncthreads();
        smem_stages<G, 1, NS - 1, true>(smem, tid, twC);
        // rows oy .. oy + Hs - 1 of the inverse (the crop window; 0 .. Hs - 1 by default)
        stage<G, NS - 1, true, RL, RL, false>(tid, twC, lds, [&](int i, int c, float2 z) {
            if (i >= oy && i < oy + Hs) img[(size_t)(i - oy) * LR + kx0 + c] = z;
        });
    }
}

// Pass 3: inverse row DFT, keep j < Ws, store the pair of images.
template <int LOG2LR, int RB, typename IO>
__global__ void __launch_bounds__(Row2G<LOG2LR, RB>::T)
c2_pass3(const float2* __restrict__ work, IO* __restrict__ y, const float2* __restrict__ twR, int B, int C,
         int Hs, int64_t first, int ox) {
    using G = Row2G<LOG2LR, RB>;
    using Lay = typename G::Lay;
    constexpr int LR = 1 << LOG2LR, Ws = LR / 2;
    constexpr int NS = G::Plan::kStages;
    constexpr int R0 = 1 << G::Plan::log2r(0), RL = 1 << G::Plan::log2r(NS - 1);
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x;
    const int64_t P = first + blockIdx.y;
    const int i0 = blockIdx.x * RB;
    const float2* __restrict__ in = work + (size_t)blockIdx.y * Hs * LR;
    auto lds = [&](int i, int c) { return smem[Lay::at(i, c)]; };
    auto sts = [&](int i, int c, float2 z) { smem[Lay::at(i, c)] = z; };
    stage<G, 0, true, R0, R0, false>(
        tid, twR, [&](int kx, int r) { return in[(size_t)(i0 + r) * LR + kx]; }, sts);
    __syncthreads();
    smem_stages<G, 1, NS - 1, true>(smem, tid, twR);
    const int npp = (B + 1) / 2;
    const int ch = (int)(P / npp), b0 = (int)(P % npp) * 2;
    const bool has1 = b0 + 1 < B;
    const size_t img0 = ((size_t)b0 * C + ch) * Hs * Ws, img1 = ((size_t)(b0 + 1) * C + ch) * Hs * Ws;
    // columns ox .. ox + Ws - 1 of the inverse (the crop window; 0 .. Ws - 1 by default)
    stage<G, NS - 1, true, RL, RL, false>(tid, twR, lds, [&](int j, int r, float2 z) {
        if (j < ox || j >= ox + Ws) return;
        const size_t off = (size_t)(i0 + r) * Ws + (j - ox);
        y[img0 + off] = from_f<IO>(z.x);
        if (has1) y[img1 + off] = from_f<IO>(z.y);
    });
}

template <int LOG2LC, int LOG2LR, typename IO>
static cudaError_t c2_fwd_go(const fftconv_plan_s& p, const void* u, const float2* khat, void* y, float2* work,
                             cudaStream_t s, int oy, int ox) {
    constexpr int Hs = (1 << LOG2LC) / 2;
    constexpr int RB = rows_per_cta<LOG2LR>(Hs);
    constexpr int LR = 1 << LOG2LR;
    auto k1 = c2_pass1<LOG2LR, RB, IO, 0>;
    auto k2 = c2_pass2<LOG2LC, LOG2LR, 0, std::is_same<IO, __nv_bfloat16>::value>;
    auto k3 = c2_pass3<LOG2LR, RB, IO>;
    const size_t sr = Row2G<LOG2LR, RB>::Lay::kWords * sizeof(float2);
    const size_t sc = Col2G<LOG2LC>::Lay::kWords * sizeof(float2);
    ensure_smem2(k1, sr);
    ensure_smem2(k2, sc);
    ensure_smem2(k3, sr);
    for (int64_t first = 0; first < p.pairs; first += p.group) {
        const int g = (int)((p.pairs - first) < p.group ? (p.pairs - first) : p.group);
        const bool tc_rows = c2tc_rows_supported(p);
        if (tc_rows) {
            const cudaError_t e = launch_c2tc_rows_fwd(p, u, work, g, first, s);
            if (e != cudaSuccess) return e;
        } else {
            k1<<<dim3(Hs / RB, g), Row2G<LOG2LR, RB>::T, sr, s>>>((const IO*)u, nullptr, 0, 0, work, p.tw.wL, p.B,
                                                                 p.H, Hs, first);
        }
        if (p.tc2d) {
            const cudaError_t e = launch_c2tc_cols(p, work, khat, g, first, s, oy);
            if (e != cudaSuccess) return e;
        } else {
            k2<<<dim3(LR / kTile2d, g), Col2G<LOG2LC>::T, sc, s>>>(work, khat, nullptr, p.tw.wC, (p.B + 1) / 2,
                                                                    first, oy);
        }
        if (tc_rows) {
            const cudaError_t e = launch_c2tc_rows_inv(p, work, y, g, first, s, ox);
            if (e != cudaSuccess) return e;
        } else {
            k3<<<dim3(Hs / RB, g), Row2G<LOG2LR, RB>::T, sr, s>>>(work, (IO*)y, p.tw.wL, p.B, p.H, Hs, first, ox);
        }
    }
    return cudaGetLastError();
}

template <int LOG2LC, int LOG2LR, bool KB, bool KTC = false>
static cudaError_t c2_spec_go(const fftconv_plan_s& p, const float* k, int Kh, int Kw, void* khat, float2* work,
                              cudaStream_t s) {
    if constexpr (KB && !KTC && LOG2LC == 9) {
        if (p.tc2d) return c2_spec_go<LOG2LC, LOG2LR, true, true>(p, k, Kh, Kw, khat, work, s);
    }
    constexpr int Hs = (1 << LOG2LC) / 2;
    constexpr int RB = rows_per_cta<LOG2LR>(Hs);
    constexpr int LR = 1 << LOG2LR;
    auto k1 = c2_pass1<LOG2LR, RB, float, 1>;
    auto k2 = c2_pass2<LOG2LC, LOG2LR, 1, KB, KTC>;
    const size_t sr = Row2G<LOG2LR, RB>::Lay::kWords * sizeof(float2);
    const size_t sc = Col2G<LOG2LC>::Lay::kWords * sizeof(float2);
    ensure_smem2(k1, sr);
    ensure_smem2(k2, sc);
    for (int64_t first = 0; first < p.H; first += p.group) {
        const int g = (int)((p.H - first) < p.group ? (p.H - first) : p.group);
        k1<<<dim3(Hs / RB, g), Row2G<LOG2LR, RB>::T, sr, s>>>(nullptr, k, Kh, Kw, work, p.tw.wL, p.B, p.H, Hs,
                                                             first);
        k2<<<dim3(LR / kTile2d, g), Col2G<LOG2LC>::T, sc, s>>>(work, nullptr, khat, p.tw.wC, 1, first, 0);
    }
    return cudaGetLastError();
}

static int ilog2_host(int x) {
    int r = 0;
    while ((1 << r) < x) ++r;
    return r;
}

template <int LOG2LC>
static cudaError_t c2_fwd_w(const fftconv_plan_s& p, const void* u, const float2* khat, void* y, float2* work,
                            cudaStream_t s, int oy, int ox) {
    const bool bf = p.dtype == FFTCONV_BF16;
    switch (ilog2_host(p.Ws)) {
#define FFTC_C(LW) \
    case LW: return bf ? c2_fwd_go<LOG2LC, LW + 1, __nv_bfloat16>(p, u, khat, y, work, s, oy, ox) \
                       : c2_fwd_go<LOG2LC, LW + 1, float>(p, u, khat, y, work, s, oy, ox);
        FFTC_C(4) FFTC_C(5) FFTC_C(6) FFTC_C(7) FFTC_C(8)
#undef FFTC_C
        default: return cudaErrorInvalidValue;
    }
}

template <int LOG2LC>
static cudaError_t c2_spec_w(const fftconv_plan_s& p, const float* k, int Kh, int Kw, float2* khat, float2* work,
                             cudaStream_t s) {
    switch (ilog2_host(p.Ws)) {
#define FFTC_C(LW) \
    case LW: return p.dtype == FFTCONV_BF16 ? c2_spec_go<LOG2LC, LW + 1, true>(p, k, Kh, Kw, khat, work, s) \
                                            : c2_spec_go<LOG2LC, LW + 1, false>(p, k, Kh, Kw, khat, work, s);
        FFTC_C(4) FFTC_C(5) FFTC_C(6) FFTC_C(7) FFTC_C(8)
#undef FFTC_C
        default: return cudaErrorInvalidValue;
    }
}

template <int LOG2LC, int LOG2LR>
static bool c2_tables_go(std::vector<float2>& out, size_t* offR, size_t* offC) {
    constexpr int RB = rows_per_cta<LOG2LR>((1 << LOG2LC) / 2);
    *offR = out.size();
    append_stage_twiddles<Row2G<LOG2LR, RB>>(out);
    *offC = out.size();
    append_stage_twiddles<Col2G<LOG2LC>>(out);
    return true;
}

template <int LOG2LC>
static bool c2_tables_w(int Ws, std::vector<float2>& out, size_t* offR, size_t* offC) {
    switch (ilog2_host(Ws)) {
#define FFTC_C(LW) case LW: return c2_tables_go<LOG2LC, LW + 1>(out, offR, offC);
        FFTC_C(4) FFTC_C(5) FFTC_C(6) FFTC_C(7) FFTC_C(8)
#undef FFTC_C
        default: return false;
    }
}

bool conv2d_tables(int Hs, int Ws, std::vector<float2>& out, size_t* offR, size_t* offC) {
    switch (ilog2_host(Hs)) {
        case 4: return c2_tables_w<5>(Ws, out, offR, offC);
        case 5: return c2_tables_w<6>(Ws, out, offR, offC);
        case 6: return c2_tables_w<7>(Ws, out, offR, offC);
        case 7: return c2_tables_w<8>(Ws, out, offR, offC);
        case 8: return c2_tables_w<9>(Ws, out, offR, offC);
        default: return false;
    }
}

cudaError_t launch_conv2d_fwd(const fftconv_plan_s& p, const void* u, const float2* khat, void* y, float2* work,
                              cudaStream_t s, int oy, int ox) {
    switch (ilog2_host(p.Hs)) {
        case 4: return c2_fwd_w<5>(p, u, khat, y, work, s, oy, ox);
        case 5: return c2_fwd_w<6>(p, u, khat, y, work, s, oy, ox);
        case 6: return c2_fwd_w<7>(p, u, khat, y, work, s, oy, ox);
        case 7: return c2_fwd_w<8>(p, u, khat, y, work, s, oy, ox);
        case 8: return c2_fwd_w<9>(p, u, khat, y, work, s, oy, ox);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_conv2d_spectrum(const fftconv_plan_s& p, const float* k, int Kh, int Kw, float2* khat,
                                   float2* work, cudaStream_t s) {
    switch (ilog2_host(p.Hs)) {
        case 4: return c2_spec_w<5>(p, k, Kh, Kw, khat, work, s);
        case 5: return c2_spec_w<6>(p, k, Kh, Kw, khat, work, s);
        case 6: return c2_spec_w<7>(p, k, Kh, Kw, khat, work, s);
        case 7: return c2_spec_w<8>(p, k, Kh, Kw, khat, work, s);
        case 8: return c2_spec_w<9>(p, k, Kh, Kw, khat, work, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fftc
