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

// ====================================================================== 3-D
// The 3-D causal convolution ("Native Multi-Dimensional Subquadratic
// Operators via Input Dependent Long Convolutions", abstract: the long
// convolution on native N-D geometry), first-octant crop of the zero-padded
// linear convolution, over (2 Dd) x (2 Hs) x (2 Ws) points.  Every depth
// slice of a volume is an image of a 2-D plan with C Dd channels (channel
// c Dd + d), so the 2-D row and column passes serve unchanged:
//   1. rows of every slice pair (c2_pass1)            -> W2 [slice pair][Hs][LR]
//   2. columns, forward only (c2_pass2 MODE 1)         -> W3 [slice pair][LC][LR] = X2 / (LC LR)
//   3. depth: DFT over d (Dd nonzero of LD = 2 Dd), product with K3, inverse,
//      d < Dd kept, in place in W3 (c3_depth MODE 0)
//   4. columns, inverse only, rows i < Hs kept (c3_colinv) -> W2
//   5. rows, inverse, crop, store (c2_pass3)
// The spectrum K3 = DFT3(pad k) / LD is built the same way (steps 1, 2 on the
// filter slices, then c3_depth MODE 1); with step 2's 1 / (LC LR) the product
// carries the whole 1 / (LD LC LR) of the inverse.

// Inverse column DFT of full column spectra: spec[g][ky][kx] (LC x LR) -> rows
// i < Hs of work[g] (Hs x LR).
template <int LOG2LC, int LOG2LR>
__global__ void __launch_bounds__(Col2G<LOG2LC>::T)
c3_colinv(const float2* __restrict__ spec, float2* __restrict__ work, const float2* __restrict__ twC) {
    using G = Col2G<LOG2LC>;
    using Lay = typename G::Lay;
    constexpr int LC = 1 << LOG2LC, LR = 1 << LOG2LR, Hs = LC / 2;
    constexpr int NS = G::Plan::kStages;
    constexpr int R0 = 1 << G::Plan::log2r(0), RL = 1 << G::Plan::log2r(NS - 1);
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x;
    const int kx0 = blockIdx.x * kTile2d;
    const float2* __restrict__ in = spec + (size_t)blockIdx.y * LC * LR;
    float2* __restrict__ img = work + (size_t)blockIdx.y * Hs * LR;
    auto lds = [&](int i, int c) { return smem[Lay::at(i, c)]; };
    auto sts = [&](int i, int c, float2 z) { smem[Lay::at(i, c)] = z; };
    stage<G, 0, true, R0, R0, false>(
        tid, twC, [&](int ky, int c) { return in[(size_t)ky * LR + kx0 + c]; }, sts);
    __syncthreads();
    smem_stages<G, 1, NS - 1, true>(smem, tid, twC);
    stage<G, NS - 1, true, RL, RL / 2, false>(tid, twC, lds, [&](int i, int c, float2 z) {
        img[(size_t)i * LR + kx0 + c] = z;
    });
}

// Depth pass over the slices of one volume ("set": channel c_rel of the
// group, pair bp), 16 plane positions f0 .. f0 + 15 per CTA: slice d of the
// set at work + c_rel cstride + bp plane + d dstride; the first nz of the LD
// depth points are nonzero (the rest is the padding).
//   MODE 0: forward DFT over d, product with K3[c][kd][f], inverse, d < LD/2 kept, in place;
//   MODE 1: forward DFT over d times scale -> khat_out[c][kd][f].
template <int LOG2LD, int MODE>
__global__ void __launch_bounds__(Col2G<LOG2LD>::T)
c3_depth(float2* __restrict__ work, const float2* __restrict__ khat3, float2* __restrict__ khat_out,
         const float2* __restrict__ twD, int nz, int64_t plane, int64_t dstride, int64_t cstride, int npp,
         int64_t first_c, float scale) {
    using G = Col2G<LOG2LD>;
    using Lay = typename G::Lay;
    constexpr int LD = 1 << LOG2LD;
    constexpr int NS = G::Plan::kStages;
    constexpr int R0 = 1 << G::Plan::log2r(0), RL = 1 << G::Plan::log2r(NS - 1);
    extern __shared__ float2 smem[];
    const int tid = threadIdx.x;
    const int c_rel = blockIdx.y / npp, bp = blockIdx.y % npp;
    float2* __restrict__ base = work + (size_t)c_rel * cstride + (size_t)bp * plane;
    const size_t f0 = (size_t)blockIdx.x * kTile2d;
    auto lds = [&](int i, int c) { return smem[Lay::at(i, c)]; };
    auto sts = [&](int i, int c, float2 z) { smem[Lay::at(i, c)] = z; };
    stage<G, 0, false, R0 / 2, R0, false>(
        tid, twD,
        [&](int d, int c) { return d < nz ? base[(size_t)d * dstride + f0 + c] : make_float2(0.f, 0.f); }, sts);
    __syncthreads();
    if constexpr (MODE == 1) {
        smem_stages<G, 1, NS - 1, false>(smem, tid, twD);
        float2* __restrict__ out = khat_out + (size_t)(first_c + c_rel) * LD * plane;
        stage<G, NS - 1, false, RL, RL, false>(tid, twD, lds, [&](int kd, int c, float2 z) {
            out[(size_t)kd * plane + f0 + c] = cscale(z, scale);
        });
    } else {
        smem_stages<G, 1, NS, false>(smem, tid, twD);
        const float2* __restrict__ kh = khat3 + (size_t)(first_c + c_rel) * LD * plane;
        stage<G, 0, true, R0, R0, true>(
            tid, twD,
            [&](int kd, int c) { return cmul(smem[Lay::at(kd, c)], __ldg(&kh[(size_t)kd * plane + f0 + c])); },
            sts);
        __syncthreads();
        smem_stages<G, 1, NS - 1, true>(smem, tid, twD);
        stage<G, NS - 1, true, RL, RL / 2, false>(tid, twD, lds, [&](int d, int c, float2 z) {
            base[(size_t)d * dstride + f0 + c] = z;
        });
    }
}

template <int LOG2LD, int MODE>
static cudaError_t c3_depth_go(const fftconv_plan_s& p, float2* work, const float2* khat3, float2* khat_out,
                               int nz, int64_t plane, int64_t dstride, int64_t cstride, int npp, int64_t first_c,
                               int sets, float scale, cudaStream_t s) {
    auto kern = c3_depth<LOG2LD, MODE>;
    const size_t sm = Col2G<LOG2LD>::Lay::kWords * sizeof(float2);
    ensure_smem2(kern, sm);
    kern<<<dim3((unsigned)(plane / kTile2d), sets), Col2G<LOG2LD>::T, sm, s>>>(
        work, khat3, khat_out, p.tw3.wD, nz, plane, dstride, cstride, npp, first_c, scale);
    return cudaGetLastError();
}

template <int MODE>
static cudaError_t c3_depth_sw(const fftconv_plan_s& p, float2* work, const float2* khat3, float2* khat_out, int nz,
                               int64_t plane, int64_t dstride, int64_t cstride, int npp, int64_t first_c, int sets,
                               float scale, cudaStream_t s) {
    switch (ilog2_host(p.Dd)) {
#define FFTC_D(LD)                                                                                                \
    case LD: return c3_depth_go<LD + 1, MODE>(p, work, khat3, khat_out, nz, plane, dstride, cstride, npp, first_c, \
                                              sets, scale, s);
        FFTC_D(4) FFTC_D(5) FFTC_D(6) FFTC_D(7) FFTC_D(8)
#undef FFTC_D
        default: return cudaErrorInvalidValue;
    }
}

// the workspace of a group of gc channels: W2 then W3 (whole slice pairs)
static void c3_split(const fftconv_plan_s& p, float2* work, float2** w2, float2** w3) {
    const size_t LR = 2 * (size_t)p.Ws, LC = 2 * (size_t)p.Hs;
    const size_t slices = (size_t)p.group * p.Dd * ((p.B + 1) / 2);
    *w2 = work;
    *w3 = work + slices * p.Hs * LR;
    (void)LC;
}

template <int LOG2LC, int LOG2LR, typename IO>
static cudaError_t c3_fwd_go(const fftconv_plan_s& p, const void* u, const float2* khat3, void* y, float2* work,
                             cudaStream_t s) {
    constexpr int Hs = (1 << LOG2LC) / 2;
    constexpr int RB = rows_per_cta<LOG2LR>(Hs);
    constexpr int LR = 1 << LOG2LR, LC = 1 << LOG2LC;
    auto k1 = c2_pass1<LOG2LR, RB, IO, 0>;
    auto k2 = c2_pass2<LOG2LC, LOG2LR, 1, false>;
    auto k4 = c3_colinv<LOG2LC, LOG2LR>;
    auto k5 = c2_pass3<LOG2LR, RB, IO>;
    const size_t sr = Row2G<LOG2LR, RB>::Lay::kWords * sizeof(float2);
    const size_t sc = Col2G<LOG2LC>::Lay::kWords * sizeof(float2);
    ensure_smem2(k1, sr);
    ensure_smem2(k2, sc);
    ensure_smem2(k4, sc);
    ensure_smem2(k5, sr);
    const int npp = (p.B + 1) / 2;
    const int Cs = p.H * p.Dd;  // channels of the slice view
    const int64_t plane = (int64_t)LC * LR;
    float2 *w2, *w3;
    c3_split(p, work, &w2, &w3);
    for (int64_t c0 = 0; c0 < p.H; c0 += p.group) {
        const int gc = (int)((p.H - c0) < p.group ? (p.H - c0) : p.group);
        const int g = gc * p.Dd * npp;            // slice pairs of the group
        const int64_t first = c0 * p.Dd * npp;    // their first index in the slice view
        k1<<<dim3(Hs / RB, g), Row2G<LOG2LR, RB>::T, sr, s>>>((const IO*)u, nullptr, 0, 0, w2, p.tw.wL, p.B, Cs, Hs,
                                                             first);
        k2<<<dim3(LR / kTile2d, g), Col2G<LOG2LC>::T, sc, s>>>(w2, nullptr, w3, p.tw.wC, 1, 0, 0);
        cudaError_t e = c3_depth_sw<0>(p, w3, khat3, nullptr, p.Dd, plane, (int64_t)npp * plane,
                                       (int64_t)p.Dd * npp * plane, npp, c0, gc * npp, 1.0f, s);
        if (e != cudaSuccess) return e;
        k4<<<dim3(LR / kTile2d, g), Col2G<LOG2LC>::T, sc, s>>>(w3, w2, p.tw.wC);
        k5<<<dim3(Hs / RB, g), Row2G<LOG2LR, RB>::T, sr, s>>>(w2, (IO*)y, p.tw.wL, p.B, Cs, Hs, first, 0);
    }
    return cudaGetLastError();
}

template <int LOG2LC, int LOG2LR>
static cudaError_t c3_spec_go(const fftconv_plan_s& p, const float* k, int Kd, int Kh, int Kw, float2* khat3,
                              float2* work, cudaStream_t s) {
    constexpr int Hs = (1 << LOG2LC) / 2;
    constexpr int RB = rows_per_cta<LOG2LR>(Hs);
    constexpr int LR = 1 << LOG2LR, LC = 1 << LOG2LC;
    auto k1 = c2_pass1<LOG2LR, RB, float, 1>;
    auto k2 = c2_pass2<LOG2LC, LOG2LR, 1, false>;
    const size_t sr = Row2G<LOG2LR, RB>::Lay::kWords * sizeof(float2);
    const size_t sc = Col2G<LOG2LC>::Lay::kWords * sizeof(float2);
    ensure_smem2(k1, sr);
    ensure_smem2(k2, sc);
    const int64_t plane = (int64_t)LC * LR;
    const int LD = 2 * p.Dd;
    float2 *w2, *w3;
    c3_split(p, work, &w2, &w3);
    for (int64_t c0 = 0; c0 < p.H; c0 += p.group) {
        const int gc = (int)((p.H - c0) < p.group ? (p.H - c0) : p.group);
        const int g = gc * Kd;  // filter slices of the group, as images [C Kd][Kh][Kw]
        k1<<<dim3(Hs / RB, g), Row2G<LOG2LR, RB>::T, sr, s>>>(nullptr, k, Kh, Kw, w2, p.tw.wL, 1, p.H * Kd, Hs,
                                                             c0 * Kd);
        k2<<<dim3(LR / kTile2d, g), Col2G<LOG2LC>::T, sc, s>>>(w2, nullptr, w3, p.tw.wC, 1, 0, 0);
        cudaError_t e = c3_depth_sw<1>(p, w3, nullptr, khat3, Kd, plane, plane, (int64_t)Kd * plane, 1, c0, gc,
                                       (float)plane / (float)LD, s);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

template <int LOG2LC>
static cudaError_t c3_fwd_w(const fftconv_plan_s& p, const void* u, const float2* khat3, void* y, float2* work,
                            cudaStream_t s) {
    const bool bf = p.dtype == FFTCONV_BF16;
    switch (ilog2_host(p.Ws)) {
#define FFTC_C(LW) \
    case LW: return bf ? c3_fwd_go<LOG2LC, LW + 1, __nv_bfloat16>(p, u, khat3, y, work, s) \
                       : c3_fwd_go<LOG2LC, LW + 1, float>(p, u, khat3, y, work, s);
        FFTC_C(4) FFTC_C(5) FFTC_C(6) FFTC_C(7) FFTC_C(8)
#undef FFTC_C
        default: return cudaErrorInvalidValue;
    }
}

template <int LOG2LC>
static cudaError_t c3_spec_w(const fftconv_plan_s& p, const float* k, int Kd, int Kh, int Kw, float2* khat3,
                             float2* work, cudaStream_t s) {
    switch (ilog2_host(p.Ws)) {
#define FFTC_C(LW) case LW: return c3_spec_go<LOG2LC, LW + 1>(p, k, Kd, Kh, Kw, khat3, work, s);
        FFTC_C(4) FFTC_C(5) FFTC_C(6) FFTC_C(7) FFTC_C(8)
#undef FFTC_C
        default: return cudaErrorInvalidValue;
    }
}

template <int LOG2LD>
static bool c3_depth_tables_go(std::vector<float2>& out, size_t* offD) {
    *offD = out.size();
    append_stage_twiddles<Col2G<LOG2LD>>(out);
    return true;
}

bool conv3d_depth_tables(int Dd, std::vector<float2>& out, size_t* offD) {
    switch (ilog2_host(Dd)) {
        case 4: return c3_depth_tables_go<5>(out, offD);
        case 5: return c3_depth_tables_go<6>(out, offD);
        case 6: return c3_depth_tables_go<7>(out, offD);
        case 7: return c3_depth_tables_go<8>(out, offD);
        case 8: return c3_depth_tables_go<9>(out, offD);
        default: return false;
    }
}

cudaError_t launch_conv3d_fwd(const fftconv_plan_s& p, const void* u, const float2* khat3, void* y, float2* work,
                              cudaStream_t s) {
    switch (ilog2_host(p.Hs)) {
        case 4: return c3_fwd_w<5>(p, u, khat3, y, work, s);
        case 5: return c3_fwd_w<6>(p, u, khat3, y, work, s);
        case 6: return c3_fwd_w<7>(p, u, khat3, y, work, s);
        case 7: return c3_fwd_w<8>(p, u, khat3, y, work, s);
        case 8: return c3_fwd_w<9>(p, u, khat3, y, work, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_conv3d_spectrum(const fftconv_plan_s& p, const float* k, int Kd, int Kh, int Kw, float2* khat3,
                                   float2* work, cudaStream_t s) {
    switch (ilog2_host(p.Hs)) {
        case 4: return c3_spec_w<5>(p, k, Kd, Kh, Kw, khat3, work, s);
        case 5: return c3_spec_w<6>(p, k, Kd, Kh, Kw, khat3, work, s);
        case 6: return c3_spec_w<7>(p, k, Kd, Kh, Kw, khat3, work, s);
        case 7: return c3_spec_w<8>(p, k, Kd, Kh, Kw, khat3, work, s);
        case 8: return c3_spec_w<9>(p, k, Kd, Kh, Kw, khat3, work, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fftc
