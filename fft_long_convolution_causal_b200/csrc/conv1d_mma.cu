// conv1d_mma.cu -- fused bf16 tensor-core kernel of the 1-D causal FFT convolution.
//
// The DFT of length M = 2N is computed as a Monarch (four-step) product of
// small dense DFT matrices on the tensor cores, the matrix decomposition that
// "FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor Cores"
// (abstract) uses to run the FFT on matrix-multiply units, fused with the
// pointwise product and the inverse in one kernel as in "FlashConv"
// (Mechanism: FFT, pointwise product and inverse FFT on chip; block FFT as
// matrix multiplications).  Two batch rows b, b+1 of channel h travel as one
// complex sequence z = x_b + i x_{b+1}; x is zero-padded to M and y truncated
// to [:N] ("RubiConv -- Efficient Boundary-Respecting Convolutions", Caracal
// abstract).
//
// Index split, M = P * 256:   n = 256 p + q,  k = k_p + P (c + 16 d),  q = 16 a + b.
//   step 1 (outer): for each q, DFT_P over p < P/2 (the nonzero half), times
//                   W_M^{q k_p}  -> S[k_p][q]
//   step 3 (inner, one warp per row k_p): 256-point DFT as 16 x 16:
//                   over a -> c, times W_256^{b c}, transpose, over b -> d;
//                   times Khat[k] (+ D/M); inverse in reverse order; times
//                   W_M^{-q k_p}                                 -> S[k_p][q]
//   step 1' (outer inverse): for each q, inverse DFT_P over k_p, only p < P/2.
// Every DFT stage is a complex product of a bf16 tile (data, the A operand
// of mma.sync m16n8k16) with a bf16 DFT matrix (the B operand), accumulated
// in fp32: Yr = Xr Fr - Xi Fi, Yi = Xr Fi + Xi Fr.  Accumulator fragments are
// reused directly as the next A fragments; the 16 x 16 transpose between the
// inner stages is done in registers (movmatrix).  S lives in shared memory as
// two bf16 planes (re, im), rows k_p of 256 q, 16-byte chunks XOR-swizzled so
// that both the row-wise (step 3) and the column-wise (steps 1, 1')
// ldmatrix / stmatrix accesses are free of bank conflicts.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <vector>

#include "fft_simt.cuh"
#include "plan.h"
#include "tables.h"
#include "tc_common.cuh"
#include "umma.cuh"

namespace fftc {
namespace tc {
// Step 3 on RN rows k_p at once: the rows are independent, so the compiler
// interleaves their dependency chains (MMA -> convert -> twiddle -> MMA).
// kc0/kc1: the rows' Khat words, tw: their W_M^{-q k_p} twiddles.
template <int RN, bool IP>
__device__ __forceinline__ void inner_rows(uint32_t sre, uint32_t sim, const int (&kp)[RN], int lane,
                                           const uint2 (&f16)[3][2], const uint2 (&w256)[4],
                                           const uint32_t (&w256n)[4], const uint4 (&kc0)[RN],
                                           const uint4 (&kc1)[RN], const uint2 (&tw)[RN][4], __nv_bfloat162 dm2) {
    const int m8 = lane >> 3, r8 = lane & 7;
    const uint32_t a = r8 + 8 * (m8 >> 1), chunk = 2 * a + (m8 & 1);
    uint32_t xr[RN][4], xi[RN][4];
#pragma unroll
    for (int r = 0; r < RN; ++r) {
        ldsm_x4_t(xr[r], plane_addr(sre, kp[r], chunk));
        ldsm_x4_t(xi[r], plane_addr(sim, kp[r], chunk));
    }
    // stage i: [b][a] x F16 -> [b][c]; twiddle W_256^{b c}; transpose -> [c][b]
    float acr[RN][2][4], aci[RN][2][4];
#pragma unroll
    for (int r = 0; r < RN; ++r) cmma2z(acr[r], aci[r], xr[r], xi[r], f16[0], f16[1], f16[2]);
#pragma unroll
    for (int r = 0; r < RN; ++r) {
        uint32_t tr[4], ti[4];
        pack_tile<IP>(tr, acr[r]);
        pack_tile<IP>(ti, aci[r]);
#pragma unroll
        for (int i = 0; i < 4; ++i) twiddle2n<true>(tr[i], ti[i], w256[i], w256n[i]);
        transpose_tile(xr[r], tr);
        transpose_tile(xi[r], ti);
    }
    // stage ii: [c][b] x F16 -> [c][d] (spectrum at k = k_p + P (c + 16 d))
#pragma unroll
    for (int r = 0; r < RN; ++r) cmma2z(acr[r], aci[r], xr[r], xi[r], f16[0], f16[1], f16[2]);
    // pointwise product with (Khat + D/M) on packed pairs; Khat regs hold (re pair, im pair)
#pragma unroll
    for (int r = 0; r < RN; ++r) {
        pack_tile<IP>(xr[r], acr[r]);
        pack_tile<IP>(xi[r], aci[r]);
        const uint32_t kre[4] = {kc0[r].x, kc0[r].z, kc1[r].x, kc1[r].z};
        const uint32_t kim[4] = {kc0[r].y, kc0[r].w, kc1[r].y, kc1[r].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 zr = as_b2(xr[r][i]), zi = as_b2(xi[r][i]);
            const __nv_bfloat162 kr = __hadd2(as_b2(kre[i]), dm2), ki = as_b2(kim[i]);
            xr[r][i] = as_u(__hfma2(zr, kr, __hneg2(__hmul2(zi, ki))));
            xi[r][i] = as_u(__hfma2(zr, ki, __hmul2(zi, kr)));
        }
    }
    // inverse stage ii: [c][d] x conj(F16) -> [c][b]; conj parts (Re, Im, -Im) = (f16[0], f16[2], f16[1])
#pragma unroll
    for (int r = 0; r < RN; ++r) cmma2z(acr[r], aci[r], xr[r], xi[r], f16[0], f16[2], f16[1]);
    // transpose [c][b] -> [b][c], conj twiddle W_256^{-b c}
#pragma unroll
    for (int r = 0; r < RN; ++r) {
        uint32_t gr[4], gi[4];
        pack_tile<IP>(gr, acr[r]);
        pack_tile<IP>(gi, aci[r]);
        transpose_tile(xr[r], gr);
        transpose_tile(xi[r], gi);
#pragma unroll
        for (int i = 0; i < 4; ++i) twiddle2n<false>(xr[r][i], xi[r][i], w256[i], w256n[i]);
    }
    // inverse stage i: [b][c] x conj(F16) -> [b][a]
#pragma unroll
    for (int r = 0; r < RN; ++r) cmma2z(acr[r], aci[r], xr[r], xi[r], f16[0], f16[2], f16[1]);
    // conj twiddle W_M^{-q k_p} (q = 16 a + b), back to row k_p
#pragma unroll
    for (int r = 0; r < RN; ++r) {
        uint32_t qr[4], qi[4];
        pack_tile<IP>(qr, acr[r]);
        pack_tile<IP>(qi, aci[r]);
#pragma unroll
        for (int i = 0; i < 4; ++i) twiddle2<false>(qr[i], qi[i], tw[r][i]);
        // registers 0 (b 0-7, a 0-7), 1 (b 8-15, a 0-7), 2 (b 0-7, a 8-15), 3 (b 8-15, a 8-15)
        stsm_x4_t(plane_addr(sre, kp[r], chunk), qr[0], qr[1], qr[2], qr[3]);
        stsm_x4_t(plane_addr(sim, kp[r], chunk), qi[0], qi[1], qi[2], qi[3]);
    }
}

// Step 1: for each 16-q tile, the outer DFT over the P/2 nonzero p (rows of
// the staging planes x, times w when gated), times W_M^{q k_p}, stored
// transposed into S[k_p][q].  Shared by the forward kernel and the spectrum
// kernel of the largest transforms.
template <int P, int NW, bool GATED, bool PRE1, bool IP, bool RS, int F1, int F2>
__device__ __forceinline__ void outer_step1(uint32_t xre, uint32_t xim, uint32_t wre, uint32_t wim, uint32_t sre,
                                            uint32_t sim, int lane, int warp, const uint2 (&fp)[F1][F2][3],
                                            const TcTables& tb, uint32_t rsm) {
    using S = TcShape<P>;
    constexpr bool TW_PREFETCH = S::NT1 <= 4;  // small tables: fetch the next tile's twiddles early
    const int m8 = lane >> 3, r8 = lane & 7;
    uint2 twn[TW_PREFETCH ? S::NT1 : 1][2];
    if (TW_PREFETCH && warp < 16) {
#pragma unroll
        for (int j = 0; j < S::NT1; ++j)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                twn[TW_PREFETCH ? j : 0][hh] = __ldg(&tb.tw1[((warp * S::NT1 + j) * 2 + hh) * 32 + lane]);
    }
    for (int qt = warp; qt < 16; qt += NW) {
        uint2 twc[TW_PREFETCH ? S::NT1 : 1][2];
        uint2 tq0, tq1;  // otherwise: the next n-tile's twiddles, one tile ahead
        if (!TW_PREFETCH) {
            tq0 = __ldg(&tb.tw1[((qt * S::NT1) * 2 + 0) * 32 + lane]);
            tq1 = __ldg(&tb.tw1[((qt * S::NT1) * 2 + 1) * 32 + lane]);
        }
        if (TW_PREFETCH) {
#pragma unroll
            for (int j = 0; j < S::NT1; ++j) {
                twc[TW_PREFETCH ? j : 0][0] = twn[TW_PREFETCH ? j : 0][0];
                twc[TW_PREFETCH ? j : 0][1] = twn[TW_PREFETCH ? j : 0][1];
            }
            if (qt + NW < 16) {
#pragma unroll
                for (int j = 0; j < S::NT1; ++j)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                        twn[TW_PREFETCH ? j : 0][hh] =
                            __ldg(&tb.tw1[(((qt + NW) * S::NT1 + j) * 2 + hh) * 32 + lane]);
            }
        }
        uint32_t ar[S::KS1][4], ai[S::KS1][4];
#pragma unroll
        for (int ks = 0; ks < S::KS1; ++ks) {
            // A[q][p] from rows p, chunks 2 qt (+1).  Rows p >= P/2 are the
            // zero padding: those lanes point at row 0 (a select -- ldmatrix
            // must run warp-converged) and their registers are zeroed.
            const uint32_t prow0 = 16 * ks + r8 + 8 * (m8 >> 1), chunk = 2 * qt + (m8 & 1);
            const uint32_t prow = prow0 < (uint32_t)(P / 2) ? prow0 : 0u;
            ldsm_x4_t(ar[ks], plane_addr(xre, prow, chunk));
            ldsm_x4_t(ai[ks], plane_addr(xim, prow, chunk));
            if (GATED) {
                uint32_t gr[4], gi[4];
                ldsm_x4_t(gr, plane_addr(wre, prow, chunk));
                ldsm_x4_t(gi, plane_addr(wim, prow, chunk));
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    ar[ks][r] = as_u(__hmul2(as_b2(ar[ks][r]), as_b2(gr[r])));
                    ai[ks][r] = as_u(__hmul2(as_b2(ai[ks][r]), as_b2(gi[r])));
                }
            }
            if (16 * ks + 8 >= P / 2) ar[ks][2] = ar[ks][3] = ai[ks][2] = ai[ks][3] = 0u;
        }
        // every A fragment of this tile is in registers before any store below,
        // so S may alias the staging rows of this tile's columns
#pragma unroll
        for (int j = 0; j < S::NT1; ++j) {
            uint2 tw0, tw1;
            if (TW_PREFETCH) {
                tw0 = twc[TW_PREFETCH ? j : 0][0];
                tw1 = twc[TW_PREFETCH ? j : 0][1];
            } else {
                tw0 = tq0;
                tw1 = tq1;
                if (j + 1 < S::NT1) {
                    tq0 = __ldg(&tb.tw1[((qt * S::NT1 + j + 1) * 2 + 0) * 32 + lane]);
                    tq1 = __ldg(&tb.tw1[((qt * S::NT1 + j + 1) * 2 + 1) * 32 + lane]);
                }
            }
            float yr[4], yi[4];
#pragma unroll
            for (int ks = 0; ks < S::KS1; ++ks) {
                uint2 b0, b1, b2;
                if (PRE1) {
                    b0 = fp[PRE1 ? ks : 0][PRE1 ? j : 0][0];
                    b1 = fp[PRE1 ? ks : 0][PRE1 ? j : 0][1];
                    b2 = fp[PRE1 ? ks : 0][PRE1 ? j : 0][2];
                } else if (RS) {
                    // B[k = p][n = k_p] from the shared matrix rows k_p = 8 j + (0..7):
                    // matrices (cos, p lo), (cos, p hi), (-sin, p lo), (-sin, p hi)
                    uint32_t r[4];
                    ldsm_x4(r, rsm + (uint32_t)((lane >> 4) * (P * P)) +
                                   wr_off<P>(8 * j + (lane & 7), 2 * ks + ((lane >> 3) & 1)));
                    b0 = make_uint2(r[0], r[1]);
                    b1 = make_uint2(r[2], r[3]);
                    b2 = make_uint2(r[2] ^ 0x80008000u, r[3] ^ 0x80008000u);
                } else {
                    const uint2* fb = tb.fp + ((size_t)(ks * S::NT1 + j) * 3) * 32 + lane;
                    b0 = __ldg(fb);
                    b1 = __ldg(fb + 32);
                    b2 = __ldg(fb + 64);
                }
                if (ks == 0) cmma_k<true>(yr, yi, ar[ks], ai[ks], b0, b1, b2);
                else cmma_k<false>(yr, yi, ar[ks], ai[ks], b0, b1, b2);
            }
            // rows q = 16 qt + g (+8), cols k_p = 8 j + 2t (+1)
            uint32_t pr[2] = {pack2<IP>(yr[0], yr[1]), pack2<IP>(yr[2], yr[3])};
            uint32_t pi[2] = {pack2<IP>(yi[0], yi[1]), pack2<IP>(yi[2], yi[3])};
            twiddle2<true>(pr[0], pi[0], tw0);
            twiddle2<true>(pr[1], pi[1], tw1);
            // store transposed: rows k_p = 8 j + r, chunk 2 qt + hh
            const uint32_t krow = 8 * j + r8, chunk = 2 * qt + (m8 & 1);
            stsm_x4_t(plane_addr((m8 >> 1) ? sim : sre, krow, chunk), pr[0], pr[1], pi[0], pi[1]);
        }
    }
}

// Step 1 for P = 128 on tcgen05: for each 128-row tile t of q, the complex
// product D[q][k_p] = X[q][p] W_128^{p k_p} over the 64 nonzero p as real
// products with W = C + i F (C = cos, F = -sin: the two stored planes):
// D_re = X_re C - X_im F (the negate-B bit), D_im = X_re F + X_im C; A = the staging planes
// (MN-major), B = the outer DFT matrix (K-major), fp32 accumulators in TMEM
// columns 256 t + 128 part.  Then every warp reads its quarter of the lanes
// (tile warp / 4 % 2, column half warp / 8) in the mma.sync accumulator
// layout, multiplies by W_M^{q k_p} on packed pairs and stores transposed
// into S[k_p][q], as the mma.sync step 1 does.  Returns false when the wait
// for the products gave up.
template <int NW, bool IP>
__device__ __forceinline__ bool outer_step1_umma(uint32_t xre, uint32_t xim, uint32_t rsm, uint32_t sre, uint32_t sim,
                                                 uint32_t tmem, uint32_t mbar, uint32_t phase, int tid, int lane,
                                                 int warp, const TcTables& tb, uint32_t wait_limit) {
    constexpr int P = 128;
    static_assert(NW == 16, "one warp per (tile, lane quarter, column half)");
    if (tid == 0) {
        um::fence_after();
        const uint32_t id = um::idesc_bf16(128, 128) | (1u << 15);  // A MN-major
#pragma unroll
        for (int t = 0; t < 2; ++t) {
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
#pragma unroll
                    for (int xi = 0; xi < 2; ++xi) {
                        // (part, x plane) -> B plane and sign: re: (re, C) (im, -F); im: (re, F) (im, C)
                        const int bplane = (part ^ xi) & 1;
                        const uint32_t neg = (part == 0 && xi == 1) ? (1u << 14) : 0u;
                        const uint32_t a = (xi ? xim : xre) + (uint32_t)(16 * t * 1024 + 2 * ks * 128);
                        const uint32_t b = rsm + (uint32_t)(bplane * P * P + 2 * ks * 128);
                        const uint64_t ad = (uint64_t)((a >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) |
                                            ((uint64_t)(1024u >> 4) << 32) | (1ull << 46);
                        const uint64_t bd = (uint64_t)((b >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) |
                                            ((uint64_t)(1024u >> 4) << 32) | (1ull << 46);
                        asm volatile(
                            "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
                            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
                                tmem + (uint32_t)(256 * t + 128 * part)),
                            "l"(ad), "l"(bd), "r"(id | neg), "r"((uint32_t)(ks | xi)));
                    }
            um::mma_commit(mbar + 8u * t);  // each tile's products on their own barrier
        }
    }
    const int t = (warp >> 2) & 1, qr = warp & 3, ch = warp >> 3;
    const int m8 = lane >> 3, r8 = lane & 7;
    // twiddles W_M^{q k_p} of the 4 blocks of iteration it (rg = it / 2, jh = it % 2), fetched one iteration ahead
    uint2 tw[4][2];
    auto fetch_tw = [&](int it) {
        const int qt = 8 * t + 2 * qr + (it >> 1);
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
            const int j = 8 * ch + 4 * (it & 1) + jb;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) tw[jb][hh] = __ldg(&tb.tw1[((qt * 16 + j) * 2 + hh) * 32 + lane]);
        }
    };
    fetch_tw(0);
    const bool ok = um::mbar_wait(mbar + 8u * t, phase, wait_limit);
    um::fence_after();
#pragma unroll 1
    for (int it = 0; it < 4; ++it) {
        const int rg = it >> 1, jh = it & 1;
        const int qt = 8 * t + 2 * qr + rg;  // 16-row tile of q
        const uint32_t lrow = (uint32_t)(32 * qr + 16 * rg) << 16;
        uint32_t dr[16], di[16];
        const uint32_t col = (uint32_t)(256 * t + 64 * ch + 32 * jh);
        um::ld16x256<4>(tmem + lrow + col, dr);
        um::ld16x256<4>(tmem + lrow + col + 128, di);
        uint2 twc[4][2];
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
            twc[jb][0] = tw[jb][0];
            twc[jb][1] = tw[jb][1];
        }
        if (it + 1 < 4) fetch_tw(it + 1);
        um::wait_ld<16>(dr);
        um::wait_ld<16>(di);
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
            const int j = 8 * ch + 4 * jh + jb;  // 8-column block of k_p
            const float* yr = reinterpret_cast<const float*>(&dr[4 * jb]);
            const float* yi = reinterpret_cast<const float*>(&di[4 * jb]);
            uint32_t pr[2] = {pack2<IP>(yr[0], yr[1]), pack2<IP>(yr[2], yr[3])};
            uint32_t pi[2] = {pack2<IP>(yi[0], yi[1]), pack2<IP>(yi[2], yi[3])};
            twiddle2<true>(pr[0], pi[0], twc[jb][0]);
            twiddle2<true>(pr[1], pi[1], twc[jb][1]);
            const uint32_t krow = 8 * j + r8, chunk = 2 * qt + (m8 & 1);
            stsm_x4_t(plane_addr((m8 >> 1) ? sim : sre, krow, chunk), pr[0], pr[1], pi[0], pi[1]);
        }
    }
    um::fence_before();
    return ok;
}

// Persistent: each CTA walks work items (pair pp of channel h) with stride
// gridDim.x; items of one channel are consecutive so concurrent CTAs share
// Khat[h] in L2.  The next item's input is fetched with cp.async into the
// staging planes while the current item runs its inner transforms.
template <int P, int NW, bool GATED>
__global__ void __launch_bounds__(NW * 32, P <= 32 ? 3 : (P <= 64 ? 2 : 1))
fused_fwd_tc(const __nv_bfloat16* __restrict__ u, const __nv_bfloat16* __restrict__ v,
             const __nv_bfloat16* __restrict__ w, const uint4* __restrict__ khat, const float* __restrict__ D,
             __nv_bfloat16* __restrict__ y, TcTables tb, int* __restrict__ err, int B, int H,
             uint32_t wait_limit) {
    using S = TcShape<P>;
    using SM = TcSmem<P, GATED>;
    static_assert(P >= 16 && P <= 128, "outer factor");
    static_assert((P / NW) % 2 == 0, "step 3 takes rows in pairs");
    // bf16 packing by the conversion instruction at every size (the integer form measured
    // 3.7% slower at 2N = 32768 once step 1 ran on tcgen05, and slower at 2N = 8192)
    constexpr bool IP = false;
    constexpr int NT = NW * 32;
    constexpr int CH = S::N / 8;                          // 16-byte chunks per row of u
    constexpr bool PRE1 = S::NT1 * S::KS1 <= 4;           // keep step-1 B fragments in registers
    constexpr bool PRE3 = S::NT3 * S::KS3 <= 4;           // keep step-1' B fragments in registers
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m8 = lane >> 3, r8 = lane & 7;
    const int npp = (B + 1) / 2;
    const int items = npp * H;
    const uint32_t sre = smem_u32(smem), sim = sre + S::kPlaneBytes;
    const uint32_t xre0 = sre + SM::kS;  // staging buffer 0 (buffer 1 follows when kNBuf = 2, ungated only)
    // w planes: separate, or S rows P/2 .. P-1 (plane_addr(w, p) == plane_addr(S, p + P/2))
    const uint32_t wre = SM::kWInS ? sre + (P / 2) * 512u : xre0 + SM::kX;
    const uint32_t wim = SM::kWInS ? sim + (P / 2) * 512u : xre0 + SM::kX + SM::kX / 2;

    // cp.async the input rows of one item into staging buffer buf: which = 1 (u), 2 (w), 3 (both)
    auto stage_input = [&](int item, int which, int buf) {
        const uint32_t xre = xre0 + buf * SM::kX, xim = xre + SM::kX / 2;
        const int hh = item / npp, b0 = 2 * (item % npp);
        const bool has1 = b0 + 1 < B;
        const size_t r0 = ((size_t)b0 * H + hh) * S::N;
        const size_t r1 = has1 ? ((size_t)(b0 + 1) * H + hh) * S::N : r0;
        for (int i = tid; i < 2 * CH; i += NT) {
            const int plane = i / CH;
            uint32_t p, chunk;
            if (SM::kUM1) {
                // a warp takes rows p0 .. p0 + 7 x chunks c0 .. c0 + 3: 64-byte global
                // runs, and 8 distinct bank groups in the canonical layout
                const int rem = i % CH;
                chunk = (rem >> 8) * 4 + ((rem & 31) >> 3);
                p = ((rem >> 5) & 7) * 8 + (rem & 7);
            } else {
                const int n0 = (i % CH) * 8;
                p = n0 >> 8;
                chunk = (n0 & 255) >> 3;
            }
            const int bytes = (plane == 0 || has1) ? 16 : 0;  // zero-fill the missing row
            const size_t off = (plane ? r1 : r0) + 256 * p + 8 * chunk;
            if (which & 1)
                cp_async16(SM::kUM1 ? (plane ? xim : xre) + xcan_off(p, chunk) : plane_addr(plane ? xim : xre, p, chunk),
                           u + off, bytes);
            if (GATED && (which & 2)) cp_async16(plane_addr(plane ? wim : wre, p, chunk), w + off, bytes);
        }
        cp_async_commit();
    };

    // constants for the whole kernel: inner DFT_16 fragments, W_256 twiddles
    uint2 f16[3][2], w256[4];
#pragma unroll
    for (int part = 0; part < 3; ++part)
#pragma unroll
        for (int j = 0; j < 2; ++j) f16[part][j] = __ldg(&tb.f16[(j * 3 + part) * 32 + lane]);
#pragma unroll
    for (int i = 0; i < 4; ++i) w256[i] = __ldg(&tb.w256[i * 32 + lane]);
    uint32_t w256n[4];  // the negated sines
#pragma unroll
    for (int i = 0; i < 4; ++i) w256n[i] = as_u(__hneg2(as_b2(w256[i].y)));
    uint2 fp[PRE1 ? S::KS1 : 1][PRE1 ? S::NT1 : 1][3];
    if (PRE1) {
#pragma unroll
        for (int ks = 0; ks < S::KS1; ++ks)
#pragma unroll
            for (int j = 0; j < S::NT1; ++j)
#pragma unroll
                for (int part = 0; part < 3; ++part)
                    fp[PRE1 ? ks : 0][PRE1 ? j : 0][part] =
                        __ldg(&tb.fp[((ks * S::NT1 + j) * 3 + part) * 32 + lane]);
    }
    uint2 fpi[PRE3 ? S::KS3 : 1][PRE3 ? S::NT3 : 1][3];
    if (PRE3) {
#pragma unroll
        for (int ks = 0; ks < S::KS3; ++ks)
#pragma unroll
            for (int j = 0; j < S::NT3; ++j)
#pragma unroll
                for (int part = 0; part < 3; ++part)
                    fpi[PRE3 ? ks : 0][PRE3 ? j : 0][part] =
                        __ldg(&tb.fpi[((ks * S::NT3 + j) * 3 + part) * 32 + lane]);
    }

    const uint32_t rsm = sre + SM::kROff;  // the outer DFT matrix (P >= 64)
    if constexpr (SM::kRS) {
        constexpr int RCH = P * P / 8;  // 16-byte chunks of both planes (P rows of P bytes each)
        for (int i = tid; i < RCH; i += NT) {
            const int plane = i / (RCH / 2), rem = i % (RCH / 2), r = rem / (P / 16), c = rem % (P / 16);
            cp_async16(rsm + (uint32_t)(plane * (P * P)) + wr_off<P>(r, c), tb.wr + i, 16);
        }
        cp_async_commit();
    }
    // P = 128: TMEM for the tcgen05 step 1 and its mbarriers.  The CTA takes all 512
    // columns; the allocation cannot wait on another CTA, because this kernel's
    // 224 KiB of shared memory leaves no room on the SM for a second CTA of it or
    // of the other TMEM user (the tcgen05 kernel of 2N <= 8192, 40-80 KiB each)
    __shared__ uint32_t s_tmem;
    __shared__ __align__(8) uint64_t s_mbar[3];  // tile 0, tile 1, drain
    uint32_t tmem = 0, mphase = 0;
    const uint32_t mbar = smem_u32(&s_mbar[0]);
    if constexpr (SM::kUM1) {
        if (warp == 0) {
            um::tmem_alloc(smem_u32(&s_tmem), 512);
            um::tmem_relinquish();
        }
        if (tid == 0) {
            um::mbar_init(mbar, 1);
            um::mbar_init(mbar + 8u, 1);
            um::mbar_init(mbar + 16u, 1);
        }
        um::fence_before();
        __syncthreads();
        um::fence_after();
        tmem = s_tmem;
    }
    if ((int)blockIdx.x < items) stage_input(blockIdx.x, 3, 0);

    bool dead = false;  // a bounded wait of this CTA gave up (P = 128 only)
    int k = 0;  // items done by this CTA
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++k) {
        const int h = item / npp, b0 = 2 * (item % npp);
        const bool has1 = b0 + 1 < B;
        const size_t row0 = ((size_t)b0 * H + h) * S::N;
        const size_t row1 = ((size_t)(b0 + 1) * H + h) * S::N;
        const int buf = SM::kNBuf == 2 ? (k & 1) : 0;
        if (SM::kNBuf == 2 && item + (int)gridDim.x < items) {
            // the other buffer was last read by the previous item's step 1 (a barrier ago)
            stage_input(item + gridDim.x, 3, buf ^ 1);
            asm volatile("cp.async.wait_group 1;\n" ::: "memory");
        } else {
            cp_async_wait_all();
        }
        __syncthreads();
        const uint32_t xre = xre0 + buf * SM::kX, xim = xre + SM::kX / 2;

        // ---- step 1: outer DFT over p for 16 q at a time; times W_M^{q k_p}
        if constexpr (SM::kUM1) {
            if constexpr (GATED) {
                // x = u w in place in the staging planes (w sits in S rows P/2 .. P-1)
                for (int i = tid; i < 2 * (P / 2) * 32; i += NT) {
                    // consecutive threads on consecutive 16-byte chunks of the canonical planes
                    const int plane = i / ((P / 2) * 32), rem = i % ((P / 2) * 32), c = rem / (P / 2), p = rem % (P / 2);
                    const uint32_t ua = (plane ? xim : xre) + xcan_off(p, c);
                    const uint32_t wa = plane_addr(plane ? wim : wre, p, c);
                    uint4 a, g;
                    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w)
                                 : "r"(ua));
                    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                                 : "=r"(g.x), "=r"(g.y), "=r"(g.z), "=r"(g.w)
                                 : "r"(wa));
                    a.x = as_u(__hmul2(as_b2(a.x), as_b2(g.x)));
                    a.y = as_u(__hmul2(as_b2(a.y), as_b2(g.y)));
                    a.z = as_u(__hmul2(as_b2(a.z), as_b2(g.z)));
                    a.w = as_u(__hmul2(as_b2(a.w), as_b2(g.w)));
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(ua), "r"(a.x), "r"(a.y), "r"(a.z),
                                 "r"(a.w)
                                 : "memory");
                }
            }
            um::fence_proxy_async();  // the staged (and gated) x is read by the tensor core
            __syncthreads();
            const bool ok =
                outer_step1_umma<NW, IP>(xre, xim, rsm, sre, sim, tmem, mbar, mphase, tid, lane, warp, tb, wait_limit);
            mphase ^= 1u;
            // a wait that gave up abandons the launch: the whole CTA leaves the item loop
            // (its S holds garbage) and drains the products before freeing TMEM below
            if (__syncthreads_or(!ok)) {
                dead = true;
                break;
            }
        } else {
            outer_step1<P, NW, GATED, PRE1, IP, SM::kRS>(xre, xim, wre, wim, sre, sim, lane, warp, fp, tb, rsm);
            __syncthreads();
        }
        // the staging planes are free: fetch the next item while this one runs
        if (SM::kNBuf == 1 && item + (int)gridDim.x < items) stage_input(item + gridDim.x, SM::kWInS ? 1 : 3, 0);

        // ---- step 3: inner 256-point DFT, product with Khat, inverse; two rows k_p per iteration
        {
            constexpr int RN = 2;
            static_assert((P / NW) % RN == 0, "rows per warp must split into pairs");
            const float dmf = D ? D[h] * (1.0f / S::M) : 0.f;
            const __nv_bfloat162 dm2 = __floats2bfloat162_rn(dmf, dmf);
            const uint4* __restrict__ kh = khat + (size_t)h * P * 64;  // 32 lanes x 2 uint4 per row
            // two sets of the rows' Khat words and twiddles, filled alternately one
            // iteration ahead (a ping-pong instead of copying the prefetched set)
            uint4 ka0[RN], ka1[RN], kb0[RN], kb1[RN];
            uint2 ta[RN][4], tq[RN][4];
            auto fetch = [&](int kp0, uint4(&k0)[RN], uint4(&k1)[RN], uint2(&t)[RN][4]) {
#pragma unroll
                for (int r = 0; r < RN; ++r) {
                    const int kp = kp0 + r * NW;
                    k0[r] = __ldg(&kh[(size_t)kp * 64 + lane * 2]);
                    k1[r] = __ldg(&kh[(size_t)kp * 64 + lane * 2 + 1]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) t[r][i] = __ldg(&tb.tw3[((size_t)kp * 4 + i) * 32 + lane]);
                }
            };
            static_assert((P / NW) % (2 * RN) == 0, "row pairs per warp come in twos");
            fetch(warp, ka0, ka1, ta);
            for (int kp0 = warp; kp0 < P; kp0 += 2 * RN * NW) {
                const int kq = kp0 + RN * NW;
                fetch(kq, kb0, kb1, tq);
                const int kps[RN] = {kp0, kp0 + NW};
                inner_rows<RN, IP>(sre, sim, kps, lane, f16, w256, w256n, ka0, ka1, ta, dm2);
                if (kq + RN * NW < P) fetch(kq + RN * NW, ka0, ka1, ta);
                const int kqs[RN] = {kq, kq + NW};
                inner_rows<RN, IP>(sre, sim, kqs, lane, f16, w256, w256n, kb0, kb1, tq, dm2);
            }
        }
        __syncthreads();

        // ---- step 1': inverse outer DFT over k_p, outputs p < P/2, into rows p
        for (int qt = warp; qt < 16; qt += NW) {
            uint32_t ar[S::KS3][4], ai[S::KS3][4];
#pragma unroll
            for (int ks = 0; ks < S::KS3; ++ks) {
                const uint32_t krow = 16 * ks + r8 + 8 * (m8 >> 1), chunk = 2 * qt + (m8 & 1);
                ldsm_x4_t(ar[ks], plane_addr(sre, krow, chunk));
                ldsm_x4_t(ai[ks], plane_addr(sim, krow, chunk));
            }
#pragma unroll
            for (int j = 0; j < S::NT3; ++j) {
                float yr[4], yi[4];
#pragma unroll
                for (int ks = 0; ks < S::KS3; ++ks) {
                    uint2 b0, b1, b2;
                    if (PRE3) {
                        b0 = fpi[PRE3 ? ks : 0][PRE3 ? j : 0][0];
                        b1 = fpi[PRE3 ? ks : 0][PRE3 ? j : 0][1];
                        b2 = fpi[PRE3 ? ks : 0][PRE3 ? j : 0][2];
                    } else if (SM::kRS) {
                        // B[k = k_p][n = p] = conj(W_P^{k_p p}): the shared matrix transposed,
                        // rows k_p = 16 ks + (0..15), chunk j (p = 8 j + 0..7)
                        uint32_t r[4];
                        ldsm_x4_t(r, rsm + (uint32_t)((lane >> 4) * (P * P)) +
                                         wr_off<P>(16 * ks + 8 * ((lane >> 3) & 1) + (lane & 7), j));
                        b0 = make_uint2(r[0], r[1]);                                    // cos
                        b1 = make_uint2(r[2] ^ 0x80008000u, r[3] ^ 0x80008000u);        // +sin
                        b2 = make_uint2(r[2], r[3]);                                    // -sin
                    } else {
                        const uint2* fb = tb.fpi + ((size_t)(ks * S::NT3 + j) * 3) * 32 + lane;
                        b0 = __ldg(fb);
                        b1 = __ldg(fb + 32);
                        b2 = __ldg(fb + 64);
                    }
                    if (ks == 0) cmma_k<true>(yr, yi, ar[ks], ai[ks], b0, b1, b2);
                    else cmma_k<false>(yr, yi, ar[ks], ai[ks], b0, b1, b2);
                }
                const uint32_t prow = 8 * j + r8, chunk = 2 * qt + (m8 & 1);
                stsm_x4_t(plane_addr((m8 >> 1) ? sim : sre, prow, chunk), pack2<IP>(yr[0], yr[1]), pack2<IP>(yr[2], yr[3]),
                          pack2<IP>(yi[0], yi[1]), pack2<IP>(yi[2], yi[3]));
            }
        }
        __syncthreads();

        // S rows P/2 .. P-1 are free again: fetch the next item's w into them
        if (GATED && SM::kWInS && item + (int)gridDim.x < items) stage_input(item + gridDim.x, 2, 0);

        // ---- store y (gate by v), coalesced 16-byte chunks of rows b and b+1
        if constexpr (!GATED) {
            // unrolled: every chunk's shared-memory read and global store issue back to back
            constexpr int ITER = 2 * CH / NT;
            static_assert(ITER * NT == 2 * CH, "store loop");
#pragma unroll
            for (int e = 0; e < ITER; ++e) {
                const int i = tid + e * NT;
                const int plane = i / CH, n0 = (i % CH) * 8;
                if (plane == 1 && !has1) continue;
                const uint32_t p = n0 >> 8, chunk = (n0 & 255) >> 3;
                uint4 val;
                asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                             : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                             : "r"(plane_addr(plane ? sim : sre, p, chunk)));
                *reinterpret_cast<uint4*>(y + (plane ? row1 : row0) + n0) = val;
            }
        } else if constexpr (SM::kRS) {
            // gated, 2N >= 16384: every gate load of the pair is issued before the
            // first product, so their latencies overlap instead of adding up chunk
            // by chunk (measured 5% faster at 2N = 32768 than groups of four,
            // despite a few spilled bytes)
            constexpr int ITER = 2 * CH / NT;
            static_assert(ITER * NT == 2 * CH, "store loop");
            uint4 vv[ITER];
#pragma unroll
            for (int e = 0; e < ITER; ++e) {
                const int i = tid + e * NT;
                const int plane = i / CH, n0 = (i % CH) * 8;
                if (plane == 1 && !has1) continue;
                vv[e] = __ldg(reinterpret_cast<const uint4*>(v + (plane ? row1 : row0) + n0));
            }
#pragma unroll
            for (int e = 0; e < ITER; ++e) {
                const int i = tid + e * NT;
                const int plane = i / CH, n0 = (i % CH) * 8;
                if (plane == 1 && !has1) continue;
                const uint32_t p = n0 >> 8, chunk = (n0 & 255) >> 3;
                uint4 val;
                asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                             : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                             : "r"(plane_addr(plane ? sim : sre, p, chunk)));
                val.x = as_u(__hmul2(as_b2(val.x), as_b2(vv[e].x)));
                val.y = as_u(__hmul2(as_b2(val.y), as_b2(vv[e].y)));
                val.z = as_u(__hmul2(as_b2(val.z), as_b2(vv[e].z)));
                val.w = as_u(__hmul2(as_b2(val.w), as_b2(vv[e].w)));
                *reinterpret_cast<uint4*>(y + (plane ? row1 : row0) + n0) = val;
            }
        } else {
            // gated, smaller transforms: chunk by chunk (their register budget is
            // taken by the step-3 state; hoisting the gate loads spills there)
            for (int i = tid; i < 2 * CH; i += NT) {
                const int plane = i / CH, n0 = (i % CH) * 8;
                if (plane == 1 && !has1) continue;
                const uint32_t p = n0 >> 8, chunk = (n0 & 255) >> 3;
                uint4 val;
                asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                             : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                             : "r"(plane_addr(plane ? sim : sre, p, chunk)));
                const size_t off = (plane ? row1 : row0) + n0;
                const uint4 vv = __ldg(reinterpret_cast<const uint4*>(v + off));
                val.x = as_u(__hmul2(as_b2(val.x), as_b2(vv.x)));
                val.y = as_u(__hmul2(as_b2(val.y), as_b2(vv.y)));
                val.z = as_u(__hmul2(as_b2(val.z), as_b2(vv.z)));
                val.w = as_u(__hmul2(as_b2(val.w), as_b2(vv.w)));
                *reinterpret_cast<uint4*>(y + off) = val;
            }
        }
        // the next iteration's wait + barrier orders these reads before S is rewritten
    }
    cp_async_wait_all();
    if constexpr (SM::kUM1) {
        // drain: the issuing thread commits once more and waits (bounded, default
        // limit) until every product it issued is complete; TMEM is freed only then
        __shared__ int s_drained;
        if (tid == 0) {
            um::mma_commit(mbar + 16u);
            s_drained = um::mbar_wait(mbar + 16u, 0u) ? 1 : 0;
            if (dead || !s_drained) atomicExch(err, 1);
        }
        um::fence_before();
        __syncthreads();
        if (warp == 0 && s_drained) {
            um::fence_after();
            um::tmem_dealloc(tmem, 512);
        }
    }
}

// Spectrum on the tensor cores, for transforms too long for one CTA's SIMT
// transform: k[h] (rounded to bf16) goes through step 1 and the forward half
// of step 3 exactly as x does in the forward kernel, and the [c][d]
// accumulators, scaled by 1/M, are written in the fragment order the forward
// kernel reads (per row k_p and lane: re pair, im pair of registers 0..3).
template <int P, int NW>
__global__ void __launch_bounds__(NW * 32, 1)
tc_spectrum_mma(const float* __restrict__ k, int L, uint4* __restrict__ khat, TcTables tb) {
    using S = TcShape<P>;
    constexpr int NT = NW * 32;
    constexpr bool PRE1 = S::NT1 * S::KS1 <= 4;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m8 = lane >> 3, r8 = lane & 7;
    const int h = blockIdx.x;
    const uint32_t sre = smem_u32(smem), sim = sre + S::kPlaneBytes;
    const uint32_t xre = sre + 2 * S::kPlaneBytes, xim = xre + S::kPlaneBytes / 2;
    uint2 f16[3][2], w256[4];
#pragma unroll
    for (int part = 0; part < 3; ++part)
#pragma unroll
        for (int j = 0; j < 2; ++j) f16[part][j] = __ldg(&tb.f16[(j * 3 + part) * 32 + lane]);
#pragma unroll
    for (int i = 0; i < 4; ++i) w256[i] = __ldg(&tb.w256[i * 32 + lane]);
    uint32_t w256n[4];  // the negated sines
#pragma unroll
    for (int i = 0; i < 4; ++i) w256n[i] = as_u(__hneg2(as_b2(w256[i].y)));
    uint2 fp[PRE1 ? S::KS1 : 1][PRE1 ? S::NT1 : 1][3];
    if (PRE1) {
#pragma unroll
        for (int ks = 0; ks < S::KS1; ++ks)
#pragma unroll
            for (int j = 0; j < S::NT1; ++j)
#pragma unroll
                for (int part = 0; part < 3; ++part)
                    fp[PRE1 ? ks : 0][PRE1 ? j : 0][part] =
                        __ldg(&tb.fp[((ks * S::NT1 + j) * 3 + part) * 32 + lane]);
    }
    // stage k[h] (taps n < L, zero after) as the real plane, zero imaginary plane
    const float* __restrict__ kr = k + (size_t)h * L;
    for (int i = tid; i < S::N / 8; i += NT) {
        const int n0 = i * 8;
        float t[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t[e] = (n0 + e < L) ? kr[n0 + e] : 0.f;
        const uint32_t p = n0 >> 8, chunk = (n0 & 255) >> 3;
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(plane_addr(xre, p, chunk)),
                     "r"(pack2(t[0], t[1])), "r"(pack2(t[2], t[3])), "r"(pack2(t[4], t[5])), "r"(pack2(t[6], t[7]))
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(plane_addr(xim, p, chunk)), "r"(0u), "r"(0u),
                     "r"(0u), "r"(0u)
                     : "memory");
    }
    __syncthreads();
    outer_step1<P, NW, false, PRE1, true, false>(xre, xim, 0u, 0u, sre, sim, lane, warp, fp, tb, 0u);
    __syncthreads();
    const uint32_t a = r8 + 8 * (m8 >> 1), chunk = 2 * a + (m8 & 1);
    const float inv_m = 1.0f / (float)S::M;
    for (int kp = warp; kp < P; kp += NW) {
        uint32_t xr[4], xi[4];
        ldsm_x4_t(xr, plane_addr(sre, kp, chunk));
        ldsm_x4_t(xi, plane_addr(sim, kp, chunk));
        float acr[2][4], aci[2][4];
        cmma2z(acr, aci, xr, xi, f16[0], f16[1], f16[2]);
        uint32_t tr[4], ti[4];
        pack_tile(tr, acr);
        pack_tile(ti, aci);
#pragma unroll
        for (int i = 0; i < 4; ++i) twiddle2<true>(tr[i], ti[i], w256[i]);
        transpose_tile(xr, tr);
        transpose_tile(xi, ti);
        float vr[2][4], vi[2][4];
        cmma2z(vr, vi, xr, xi, f16[0], f16[1], f16[2]);
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                vr[j][e] *= inv_m;
                vi[j][e] *= inv_m;
            }
        uint32_t zr[4], zi[4];
        pack_tile(zr, vr);
        pack_tile(zi, vi);
        uint4* out = khat + ((size_t)h * P + kp) * 64 + lane * 2;
        out[0] = make_uint4(zr[0], zi[0], zr[1], zi[1]);
        out[1] = make_uint4(zr[2], zi[2], zr[3], zi[3]);
    }
}

// Spectrum in the kernel's fragment order: the SIMT transform of k[h]
// (natural order, fp32, in shared memory), then per row k_p and lane 8 words:
// for A-fragment register i of the [c][d] tile (c = g + 8 (i & 1),
// d = 2t + 8 (i >> 1) + {0, 1}), the packed bf16 pair of real parts and the
// packed pair of imaginary parts of Khat[k_p + P (c + 16 d)] = X / M.
template <int LOG2M>
__global__ void __launch_bounds__(Geometry<LOG2M, 1, false>::T)
tc_spectrum(const float* __restrict__ k, int L, uint32_t* __restrict__ khat, const float2* __restrict__ tw) {
    using G = Geometry<LOG2M, 1, false>;
    using Lay = typename G::Lay;
    constexpr int M = G::L, NS = G::Plan::kStages, P = M / 256;
    constexpr int R0 = 1 << G::Plan::log2r(0);
    extern __shared__ float2 smem2[];
    const int tid = threadIdx.x, h = blockIdx.x;
    const float* __restrict__ kr = k + (size_t)h * L;
    stage<G, 0, false, R0 / 2, R0, false>(
        tid, tw, [&](int n, int) { return make_float2(n < L ? kr[n] : 0.f, 0.f); },
        [&](int i, int, float2 z) { smem2[Lay::at(i, 0)] = z; });
    __syncthreads();
    smem_stages<G, 1, NS, false>(smem2, tid, tw);
    uint32_t* out = khat + (size_t)h * M;
    for (int o = tid; o < M; o += G::T) {
        const int kp = o / 256, rem = o % 256, lane = rem / 8, wd = rem % 8;
        const int i = wd >> 1, part = wd & 1, g = lane >> 2, t = lane & 3;
        const int c = g + 8 * (i & 1), d0 = 2 * t + 8 * (i >> 1);
        const float2 z0 = cscale(smem2[Lay::at(kp + P * (c + 16 * d0), 0)], 1.0f / M);
        const float2 z1 = cscale(smem2[Lay::at(kp + P * (c + 16 * (d0 + 1)), 0)], 1.0f / M);
        const float lo = part ? z0.y : z0.x, hi = part ? z1.y : z1.x;
        out[o] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
                 ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
    }
}

}  // namespace tc

// ================================================================== host side
namespace {

uint16_t bf16_bits(double x) {
    const float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}
uint32_t pack_host(double lo, double hi) { return (uint32_t)bf16_bits(lo) | ((uint32_t)bf16_bits(hi) << 16); }

void push_u2(std::vector<float2>& out, uint32_t x, uint32_t y) {
    float2 f;
    memcpy(&f.x, &x, 4);
    memcpy(&f.y, &y, 4);
    out.push_back(f);
}

// cos and sin of 2 pi e / L, e reduced mod L, in fp64
void cs(int64_t e, int64_t L, double* c, double* s) {
    int64_t r = e % L;
    if (r < 0) r += L;
    const double a = 2.0 * M_PI * (double)r / (double)L;
    *c = cos(a);
    *s = sin(a);
}

// B fragments of a complex K x N matrix G given by value(k, n) -> (re, im):
// [ks][ntile][part (Re, Im, -Im)][lane] with b0b1 = (k = 2t, 2t+1), b2b3 = (k = 2t+8, 2t+9), n = g.
template <class F>
void push_bfrags(std::vector<float2>& out, int ksteps, int ntiles, F value) {
    for (int ks = 0; ks < ksteps; ++ks)
        for (int j = 0; j < ntiles; ++j)
            for (int part = 0; part < 3; ++part)
                for (int lane = 0; lane < 32; ++lane) {
                    const int g = lane >> 2, t = lane & 3, n = 8 * j + g;
                    double v[4];
                    const int ks4[4] = {2 * t, 2 * t + 1, 2 * t + 8, 2 * t + 9};
                    for (int q = 0; q < 4; ++q) {
                        double re, im;
                        value(16 * ks + ks4[q], n, &re, &im);
                        v[q] = part == 0 ? re : (part == 1 ? im : -im);
                    }
                    push_u2(out, pack_host(v[0], v[1]), pack_host(v[2], v[3]));
                }
}

}  // namespace

bool tc_supported(int log2M) { return log2M >= 12 && log2M <= 15; }

bool tc_tables(int log2M, std::vector<float2>& out, size_t off[7]) {
    if (!tc_supported(log2M)) return false;
    const int64_t M = int64_t(1) << log2M;
    const int P = (int)(M / 256);
    const int NT1 = P / 8, KS1 = (P / 2 + 15) / 16, NT3 = (P / 2 + 7) / 8, KS3 = P / 16;
    // f16: DFT_16, B[k][n] = W_16^{k n}
    off[0] = out.size();
    push_bfrags(out, 1, 2, [](int k, int n, double* re, double* im) {
        double c, s;
        cs((int64_t)k * n, 16, &c, &s);
        *re = c;
        *im = -s;
    });
    // w256: (cos, sin) pairs of W_256^{b c}; reg i: b = g + 8 (i & 1), c = 2t + 8 (i >> 1) + {0, 1}
    off[1] = out.size();
    for (int i = 0; i < 4; ++i)
        for (int lane = 0; lane < 32; ++lane) {
            const int g = lane >> 2, t = lane & 3, b = g + 8 * (i & 1), c0 = 2 * t + 8 * (i >> 1);
            double ca, sa, cb, sb;
            cs((int64_t)b * c0, 256, &ca, &sa);
            cs((int64_t)b * (c0 + 1), 256, &cb, &sb);
            push_u2(out, pack_host(ca, cb), pack_host(sa, sb));
        }
    // fp: outer forward, B[k = p][n = k_p] = W_P^{p k_p} for p < P/2, else 0
    off[2] = out.size();
    push_bfrags(out, KS1, NT1, [P](int k, int n, double* re, double* im) {
        if (k >= P / 2) {
            *re = *im = 0.0;
            return;
        }
        double c, s;
        cs((int64_t)k * n, P, &c, &s);
        *re = c;
        *im = -s;
    });
    // fpi: outer inverse, B[k = k_p][n = p] = conj(W_P^{k_p p}) for p < P/2, else 0
    off[3] = out.size();
    push_bfrags(out, KS3, NT3, [P](int k, int n, double* re, double* im) {
        if (n >= P / 2) {
            *re = *im = 0.0;
            return;
        }
        double c, s;
        cs((int64_t)k * n, P, &c, &s);
        *re = c;
        *im = s;
    });
    // tw1: (cos, sin) of W_M^{q k_p}, [qt][j][hh][lane]: q = 16 qt + g + 8 hh, k_p = 8 j + 2 t + {0, 1}
    off[4] = out.size();
    for (int qt = 0; qt < 16; ++qt)
        for (int j = 0; j < NT1; ++j)
            for (int hh = 0; hh < 2; ++hh)
                for (int lane = 0; lane < 32; ++lane) {
                    const int g = lane >> 2, t = lane & 3;
                    const int64_t q = 16 * qt + g + 8 * hh, k0 = 8 * j + 2 * t;
                    double ca, sa, cb, sb;
                    cs(q * k0, M, &ca, &sa);
                    cs(q * (k0 + 1), M, &cb, &sb);
                    push_u2(out, pack_host(ca, cb), pack_host(sa, sb));
                }
    // tw3: (cos, sin) of W_M^{q k_p}, [k_p][reg][lane]: b = g + 8 (i & 1), a = 2t + 8 (i >> 1) + {0, 1}
    off[5] = out.size();
    for (int kp = 0; kp < P; ++kp)
        for (int i = 0; i < 4; ++i)
            for (int lane = 0; lane < 32; ++lane) {
                const int g = lane >> 2, t = lane & 3, b = g + 8 * (i & 1), a0 = 2 * t + 8 * (i >> 1);
                double ca, sa, cb, sb;
                cs((int64_t)(16 * a0 + b) * kp, M, &ca, &sa);
                cs((int64_t)(16 * (a0 + 1) + b) * kp, M, &cb, &sb);
                push_u2(out, pack_host(ca, cb), pack_host(sa, sb));
            }
    // wr (P >= 64): W_P^{k_p p} for k_p < P, p < P/2 as two bf16 planes, cos and -sin,
    // rows k_p of P/2 values; 16-byte aligned (the kernels copy it to shared memory)
    if (out.size() & 1) out.push_back(make_float2(0.f, 0.f));
    off[6] = out.size();
    if (P >= 64)
        for (int plane = 0; plane < 2; ++plane)
            for (int kp = 0; kp < P; ++kp)
                for (int p0 = 0; p0 < P / 2; p0 += 4) {
                    double v[4];
                    for (int i = 0; i < 4; ++i) {
                        double c, sn;
                        cs((int64_t)kp * (p0 + i), P, &c, &sn);
                        v[i] = plane ? -sn : c;
                    }
                    push_u2(out, pack_host(v[0], v[1]), pack_host(v[2], v[3]));
                }
    return true;
}

template <int P, bool GATED>
static cudaError_t tc_fwd_go(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                             const void* khat, const float* D, void* y, cudaStream_t s) {
    constexpr int NW = P >= 128 ? 16 : 4;  // the largest transform runs one CTA per SM
    auto kern = tc::fused_fwd_tc<P, NW, GATED>;
    const size_t smem = tc::TcSmem<P, GATED>::kBytes;
    // persistent grid: as many CTAs as are resident at once (computed once)
    static int resident = 0;
    if (resident == 0) {
        if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        int per_sm = 0, sms = 0, dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NW * 32, smem);
        resident = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 1);
    }
    const int items = ((p.B + 1) / 2) * p.H;
    dim3 grid(items < resident ? items : resident);
    kern<<<grid, NW * 32, smem, s>>>((const __nv_bfloat16*)u, (const __nv_bfloat16*)v, (const __nv_bfloat16*)w,
                                     (const uint4*)khat, D, (__nv_bfloat16*)y, p.tc, p.d_err, p.B, p.H,
                                     p.wait_limit);
    return cudaGetLastError();
}

template <int P>
static cudaError_t tc_fwd_g(const fftconv_plan_s& p, const void* u, const void* v, const void* w, const void* khat,
                            const float* D, void* y, cudaStream_t s) {
    return p.gated ? tc_fwd_go<P, true>(p, u, v, w, khat, D, y, s) : tc_fwd_go<P, false>(p, u, v, w, khat, D, y, s);
}

cudaError_t launch_tc_fwd(const fftconv_plan_s& p, const void* u, const void* v, const void* w, const void* khat,
                          const float* D, void* y, cudaStream_t s) {
    switch (p.log2M) {
        case 12: return tc_fwd_g<16>(p, u, v, w, khat, D, y, s);
        case 13: return tc_fwd_g<32>(p, u, v, w, khat, D, y, s);
        case 14: return tc_fwd_g<64>(p, u, v, w, khat, D, y, s);
        case 15: return tc_fwd_g<128>(p, u, v, w, khat, D, y, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int LOG2M>
static cudaError_t tc_spec_go(const fftconv_plan_s& p, const float* k, int64_t L, void* khat, cudaStream_t s) {
    using G = Geometry<LOG2M, 1, false>;
    auto kern = tc::tc_spectrum<LOG2M>;
    const size_t smem = G::Lay::kWords * sizeof(float2);
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<p.H, G::T, smem, s>>>(k, (int)L, (uint32_t*)khat, p.tw.wL);
    return cudaGetLastError();
}

cudaError_t launch_tc_spectrum(const fftconv_plan_s& p, const float* k, int64_t L, void* khat, cudaStream_t s) {
    switch (p.log2M) {
        case 12: return tc_spec_go<12>(p, k, L, khat, s);
        case 13: return tc_spec_go<13>(p, k, L, khat, s);
        case 14: return tc_spec_go<14>(p, k, L, khat, s);
        case 15: {
            constexpr int P = 128, NW = 16;
            auto kern = tc::tc_spectrum_mma<P, NW>;
            const size_t smem = 3 * tc::TcShape<P>::kPlaneBytes;
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            kern<<<p.H, NW * 32, smem, s>>>(k, (int)L, (uint4*)khat, p.tc);
            return cudaGetLastError();
        }
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fftc
