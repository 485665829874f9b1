// conv1d_umma.cu -- fused bf16 causal FFT convolution on the fifth-generation
// tensor cores (tcgen05): the same Monarch factorisation of the length-M = 2N
// DFT as the mma.sync kernel, with every DFT-matrix product issued as a
// tcgen05.mma whose A operand (the data) sits in tensor memory and whose B
// operand (the small DFT matrix) sits in shared memory, accumulating in fp32
// in tensor memory.  The method is the matrix-multiply formulation of the FFT
// convolution in "FlashFFTConv: Efficient Convolutions for Long Sequences with
// Tensor Cores" (abstract) fused into one kernel as in "FlashConv" (Mechanism),
// with the causal zero padding and truncation of "RubiConv -- Efficient
// Boundary-Respecting Convolutions" (Caracal abstract).
//
// Index split (M = P * 256):  n = 256 p + q,  q = 16 a + b,  k = k_p + P (c + 16 d).
//   S1  : rows q (two 128-row tiles), K = p < P/2, N = k_p (Re | Im)  -> x W_M^{q k_p} -> S[k_p][q]
//   step 3, tiles of 8 rows k_p x 16: rows b, K = a -> rows c (after x W_256^{b c} and a 16x16
//         register transpose), K = b -> x (Khat + D/M) -> the conjugate products in reverse
//         order -> x W_M^{-q k_p} -> S[k_p][q]
//   S1' : rows q, K = k_p, N = p < P/2 (Re | Im) -> y rows p (n = 256 p + q < N)
// Between products the warps read the fp32 accumulators (tcgen05.ld 16x256b,
// the mma.sync accumulator layout), round to bf16, apply twiddles on packed
// pairs, transpose with movmatrix where the contraction index changes, and
// store the next A tile (tcgen05.st).  Transfers between the outer and inner
// index go through the swizzled shared-memory planes S exactly as in the
// mma.sync kernel.  Complex products use two real MMAs per K step:
// [Yr | Yi] = Xr [Gr | Gi] + Xi [-Gi | Gr].
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <vector>

#include "plan.h"
#include "tc_common.cuh"
#include "umma.cuh"

namespace fftc {
namespace tc {

template <int P>
struct UShape {
    static constexpr int M = P * 256, N = M / 2;
    static constexpr int KS1 = (P / 2 + 15) / 16;        // S1 K steps over p < P/2
    static constexpr int N1 = 2 * P;                     // S1 accumulator columns (Re k_p | Im k_p)
    static constexpr int NT1 = P / 8;                    // 8-column k_p blocks
    static constexpr int KS3 = P / 16;                   // S1' K steps over k_p
    static constexpr int PH = P / 2;                     // S1' outputs p < P/2
    static constexpr int N3 = 2 * PH;                    // S1' accumulator columns (Re p | Im p)
    static constexpr int NT3 = PH / 8;
    static constexpr int T3 = P / 8;                     // step-3 tiles of 8 rows k_p
    static constexpr int kCols = P <= 32 ? 128 : 256;    // TMEM columns per CTA
    // S1: R1 tiles per MMA batch; A columns 16 KS1 per tile, then the accumulators
    static constexpr int kA1 = 16 * KS1;
    static constexpr int R1 = 2 * (kA1 + N1) <= 96 ? 2 : 1;
    static constexpr int kD1 = N1;                       // first S1 accumulator column (aligned to N1)
    // step 3: R3 tiles per batch, A (16 columns) then the accumulators (32 columns)
    static constexpr int R3 = (T3 < (kCols - 32) / 48) ? T3 : ((kCols - 32) / 48 >= 4 ? 4 : 2);
    static constexpr int kD3 = ((16 * R3 + 31) / 32) * 32;
    // S1': both 128-row tiles in one batch
    static constexpr int kA3 = 16 * KS3;
    static constexpr int kD3p = ((2 * kA3 + N3 - 1) / N3) * N3;
    // B images (bf16, K-major core-matrix layout), bytes
    static constexpr int kB1 = N1 * 32, kBF = 32 * 32, kB3 = N3 * 32;
    static constexpr int kOffB1 = 0;                     // [ks][2]
    static constexpr int kOffBF = kOffB1 + KS1 * 2 * kB1;  // fwd 1, fwd 2, inv 1, inv 2
    static constexpr int kOffB3 = kOffBF + 4 * kBF;        // [ks][2]
    static constexpr int kBBytes = kOffB3 + KS3 * 2 * kB3;
    static_assert(R1 * kA1 <= kD1 && kD1 + R1 * N1 <= kCols, "S1 columns");
    static_assert(kD3 + 32 * R3 <= kCols && T3 % R3 == 0, "step-3 columns");
    static_assert(kD3p + 2 * N3 <= kCols, "S1' columns");
};

template <int P, bool GATED>
struct USmem {
    static constexpr int kS = 2 * P * 512;                       // S planes (re, im), P rows of 256 q
    static constexpr int kX = P * 512;                           // staging planes of x (P/2 rows each)
    static constexpr int kW = GATED ? kX : 0;                    // staging planes of w
    static constexpr int kB = UShape<P>::kBBytes;
    static constexpr int kOffX = kS, kOffW = kS + kX, kOffB = kS + kX + kW;
    static constexpr int kBytes = kOffB + kB;
};

__device__ __forceinline__ uint32_t lane_off(int lane0) { return (uint32_t)lane0 << 16; }

template <int P, bool GATED>
__global__ void __launch_bounds__(128, (P <= 32 && !GATED) ? 3 : 2)
fused_fwd_umma(const __nv_bfloat16* __restrict__ u, const __nv_bfloat16* __restrict__ v,
               const __nv_bfloat16* __restrict__ w, const uint4* __restrict__ khat, const float* __restrict__ D,
               __nv_bfloat16* __restrict__ y, TcTables tb, const uint4* __restrict__ bimg, int* __restrict__ err,
               int B, int H) {
    using S = TcShape<P>;
    using U = UShape<P>;
    using SM = USmem<P, GATED>;
    constexpr int NT = 128;
    constexpr int CH = S::N / 8;  // 16-byte chunks per row of u
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint32_t s_tmem;
    __shared__ __align__(8) uint64_t s_mbar;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m8 = lane >> 3, r8 = lane & 7;
    const int npp = (B + 1) / 2;
    const int items = npp * H;
    const uint32_t sre = tc::smem_u32(smem), sim = sre + S::kPlaneBytes;
    const uint32_t xre = sre + SM::kOffX, xim = xre + SM::kX / 2;
    const uint32_t wre = sre + SM::kOffW, wim = wre + SM::kX / 2;
    const uint32_t bsm = sre + SM::kOffB;
    const uint32_t mbar = tc::smem_u32(&s_mbar);

    auto stage_input = [&](int item) {
        const int hh = item / npp, b0 = 2 * (item % npp);
        const bool has1 = b0 + 1 < B;
        const size_t r0 = ((size_t)b0 * H + hh) * S::N;
        const size_t r1 = has1 ? ((size_t)(b0 + 1) * H + hh) * S::N : r0;
        for (int i = tid; i < 2 * CH; i += NT) {
            const int plane = i / CH, n0 = (i % CH) * 8;
            const uint32_t p = n0 >> 8, chunk = (n0 & 255) >> 3;
            const int bytes = (plane == 0 || has1) ? 16 : 0;  // zero-fill the missing row
            const size_t off = (plane ? r1 : r0) + n0;
            cp_async16(plane_addr(plane ? xim : xre, p, chunk), u + off, bytes);
            if (GATED) cp_async16(plane_addr(plane ? wim : wre, p, chunk), w + off, bytes);
        }
        cp_async_commit();
    };

    // B images into shared memory, visible to the tensor core
    for (int i = tid; i < U::kBBytes / 16; i += NT) {
        const uint4 val = __ldg(&bimg[i]);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(bsm + 16u * i), "r"(val.x), "r"(val.y),
                     "r"(val.z), "r"(val.w)
                     : "memory");
    }
    um::fence_proxy_async();
    if (warp == 0) {
        um::tmem_alloc(tc::smem_u32(&s_tmem), U::kCols);
        um::tmem_relinquish();
    }
    if (tid == 0) um::mbar_init(mbar, 1);
    um::fence_before();
    __syncthreads();
    um::fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t tl = tmem + lane_off(32 * warp);  // this warp's TMEM lane quarter

    uint2 w256[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w256[i] = __ldg(&tb.w256[i * 32 + lane]);

    const uint32_t id1 = um::idesc_bf16(128, U::N1), id16 = um::idesc_bf16(128, 32), id3 = um::idesc_bf16(128, U::N3);
    uint32_t phase = 0;
    bool dead = false;
    // All threads: finish TMEM stores, then one thread issues the batch and commits.
    auto issue = [&](auto&& body) {
        um::wait_st();
        um::fence_before();
        __syncthreads();
        if (tid == 0) {
            um::fence_after();
            body();
            um::mma_commit(mbar);
        }
        // reconverge warp 0 before any of its lanes waits on the barrier the
        // issuing lane has yet to arm
        __syncwarp();
    };
    // All threads: wait for the batch (bounded); a timeout marks the CTA dead.
    auto await = [&]() {
        const bool ok = um::mbar_wait(mbar, phase);
        phase ^= 1u;
        um::fence_after();
        if (__syncthreads_or(!ok)) {
            dead = true;
            if (tid == 0) atomicExch(err, 1);
        }
    };

    if ((int)blockIdx.x < items) stage_input(blockIdx.x);

    for (int item = blockIdx.x; item < items && !dead; item += gridDim.x) {
        const int h = item / npp, b0 = 2 * (item % npp);
        const bool has1 = b0 + 1 < B;
        const size_t row0 = ((size_t)b0 * H + h) * S::N;
        const size_t row1 = ((size_t)(b0 + 1) * H + h) * S::N;
        cp_async_wait_all();
        __syncthreads();

        // ---------------- S1: outer DFT over p < P/2, rows q, R1 tiles of 128 q per batch
        for (int t0 = 0; t0 < 2 && !dead; t0 += U::R1) {
#pragma unroll
            for (int uu = 0; uu < U::R1; ++uu)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int qt = 8 * (t0 + uu) + 2 * warp + r;
#pragma unroll
                    for (int ks = 0; ks < U::KS1; ++ks) {
                        uint32_t ar[4], ai[4];
                        const uint32_t prow0 = 16 * ks + r8 + 8 * (m8 >> 1), chunk = 2 * qt + (m8 & 1);
                        const uint32_t prow = prow0 < (uint32_t)(P / 2) ? prow0 : 0u;
                        ldsm_x4_t(ar, plane_addr(xre, prow, chunk));
                        ldsm_x4_t(ai, plane_addr(xim, prow, chunk));
                        if (GATED) {
                            uint32_t gr[4], gi[4];
                            ldsm_x4_t(gr, plane_addr(wre, prow, chunk));
                            ldsm_x4_t(gi, plane_addr(wim, prow, chunk));
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                ar[e] = as_u(__hmul2(as_b2(ar[e]), as_b2(gr[e])));
                                ai[e] = as_u(__hmul2(as_b2(ai[e]), as_b2(gi[e])));
                            }
                        }
                        if (16 * ks + 8 >= P / 2) ar[2] = ar[3] = ai[2] = ai[3] = 0u;
                        um::st_afrag2(tl + lane_off(16 * r) + uu * U::kA1 + 16 * ks, ar, ai);
                    }
                }
            issue([&] {
#pragma unroll
                for (int uu = 0; uu < U::R1; ++uu) {
                    const uint32_t d = tmem + U::kD1 + uu * U::N1, a = tmem + uu * U::kA1;
#pragma unroll
                    for (int ks = 0; ks < U::KS1; ++ks) {
                        um::mma_ts(d, a + 16 * ks, um::sdesc_kmajor(bsm + U::kOffB1 + (2 * ks) * U::kB1), id1, ks > 0);
                        um::mma_ts(d, a + 16 * ks + 8, um::sdesc_kmajor(bsm + U::kOffB1 + (2 * ks + 1) * U::kB1), id1, 1);
                    }
                }
            });
            await();
            if (dead) break;
            // x W_M^{q k_p}, stored transposed into S[k_p][q]
#pragma unroll
            for (int uu = 0; uu < U::R1; ++uu)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int qt = 8 * (t0 + uu) + 2 * warp + r;
                    const uint32_t dl = tl + lane_off(16 * r) + U::kD1 + uu * U::N1;
#pragma unroll
                    for (int j = 0; j < U::NT1; ++j) {
                        uint32_t yr[4], yi[4];
                        um::ld16x256_x1(dl + 8 * j, yr);
                        um::ld16x256_x1(dl + P + 8 * j, yi);
                        const uint2 tw0 = __ldg(&tb.tw1[((qt * U::NT1 + j) * 2 + 0) * 32 + lane]);
                        const uint2 tw1 = __ldg(&tb.tw1[((qt * U::NT1 + j) * 2 + 1) * 32 + lane]);
                        um::wait_ld(yr);
                        um::wait_ld(yi);
                        uint32_t pr[2] = {pack2(__uint_as_float(yr[0]), __uint_as_float(yr[1])),
                                          pack2(__uint_as_float(yr[2]), __uint_as_float(yr[3]))};
                        uint32_t pi[2] = {pack2(__uint_as_float(yi[0]), __uint_as_float(yi[1])),
                                          pack2(__uint_as_float(yi[2]), __uint_as_float(yi[3]))};
                        twiddle2<true>(pr[0], pi[0], tw0);
                        twiddle2<true>(pr[1], pi[1], tw1);
                        const uint32_t krow = 8 * j + r8, chunk = 2 * qt + (m8 & 1);
                        stsm_x4_t(plane_addr((m8 >> 1) ? sim : sre, krow, chunk), pr[0], pr[1], pi[0], pi[1]);
                    }
                }
        }
        if (dead) break;
        __syncthreads();
        // the staging planes are free: fetch the next item while this one runs
        if (item + (int)gridDim.x < items) stage_input(item + gridDim.x);

        // ---------------- step 3: inner 256-point DFT, product with Khat, inverse
        {
            const float dmf = D ? D[h] * (1.0f / S::M) : 0.f;
            const __nv_bfloat162 dm2 = __floats2bfloat162_rn(dmf, dmf);
            const uint4* __restrict__ kh = khat + (size_t)h * P * 64;  // 32 lanes x 2 uint4 per row
            const uint32_t ia = r8 + 8 * (m8 >> 1), ichunk = 2 * ia + (m8 & 1);
            for (int T0 = 0; T0 < U::T3 && !dead; T0 += U::R3) {
                // stage-0 A tiles: rows b, K = a, from S rows k_p
#pragma unroll
                for (int uu = 0; uu < U::R3; ++uu)
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int kp = 8 * (T0 + uu) + 2 * warp + r;
                        uint32_t xr[4], xi[4];
                        ldsm_x4_t(xr, plane_addr(sre, kp, ichunk));
                        ldsm_x4_t(xi, plane_addr(sim, kp, ichunk));
                        um::st_afrag2(tl + lane_off(16 * r) + 16 * uu, xr, xi);
                    }
#pragma unroll 1
                for (int s = 0; s < 4 && !dead; ++s) {
                    const uint32_t bf1 = bsm + U::kOffBF + (s < 2 ? 0 : 2) * U::kBF;
                    issue([&] {
#pragma unroll
                        for (int uu = 0; uu < U::R3; ++uu) {
                            const uint32_t d = tmem + U::kD3 + 32 * uu, a = tmem + 16 * uu;
                            um::mma_ts(d, a, um::sdesc_kmajor(bf1), id16, 0);
                            um::mma_ts(d, a + 8, um::sdesc_kmajor(bf1 + U::kBF), id16, 1);
                        }
                    });
                    // fetch what this stage's epilogue needs while the products run
                    uint4 kc0[U::R3][2], kc1[U::R3][2];
                    uint2 tc3[U::R3][2][4];
                    if (s == 1) {
#pragma unroll
                        for (int uu = 0; uu < U::R3; ++uu)
#pragma unroll
                            for (int r = 0; r < 2; ++r) {
                                const int kp = 8 * (T0 + uu) + 2 * warp + r;
                                kc0[uu][r] = __ldg(&kh[(size_t)kp * 64 + lane * 2]);
                                kc1[uu][r] = __ldg(&kh[(size_t)kp * 64 + lane * 2 + 1]);
                            }
                    }
                    if (s == 3) {
#pragma unroll
                        for (int uu = 0; uu < U::R3; ++uu)
#pragma unroll
                            for (int r = 0; r < 2; ++r) {
                                const int kp = 8 * (T0 + uu) + 2 * warp + r;
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    tc3[uu][r][i] = __ldg(&tb.tw3[((size_t)kp * 4 + i) * 32 + lane]);
                            }
                    }
                    await();
                    if (dead) break;
#pragma unroll
                    for (int uu = 0; uu < U::R3; ++uu)
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            const uint32_t dl = tl + lane_off(16 * r) + U::kD3 + 32 * uu;
                            const uint32_t al = tl + lane_off(16 * r) + 16 * uu;
                            uint32_t acc[16];
                            um::ld16x256_x4(dl, acc);
                            um::wait_ld(acc);
                            float acr[2][4], aci[2][4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                acr[0][e] = __uint_as_float(acc[e]);
                                acr[1][e] = __uint_as_float(acc[4 + e]);
                                aci[0][e] = __uint_as_float(acc[8 + e]);
                                aci[1][e] = __uint_as_float(acc[12 + e]);
                            }
                            uint32_t xr[4], xi[4];
                            if (s == 0) {
                                // [b][c]: x W_256^{b c}, transpose -> [c][b]
                                uint32_t tr[4], ti[4];
                                pack_tile(tr, acr);
                                pack_tile(ti, aci);
#pragma unroll
                                for (int i = 0; i < 4; ++i) twiddle2<true>(tr[i], ti[i], w256[i]);
                                transpose_tile(xr, tr);
                                transpose_tile(xi, ti);
                                um::st_afrag2(al, xr, xi);
                            } else if (s == 1) {
                                // [c][d]: spectrum at k = k_p + P (c + 16 d); x (Khat + D/M)
                                pack_tile(xr, acr);
                                pack_tile(xi, aci);
                                const uint32_t kre[4] = {kc0[uu][r].x, kc0[uu][r].z, kc1[uu][r].x, kc1[uu][r].z};
                                const uint32_t kim[4] = {kc0[uu][r].y, kc0[uu][r].w, kc1[uu][r].y, kc1[uu][r].w};
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const __nv_bfloat162 zr = as_b2(xr[i]), zi = as_b2(xi[i]);
                                    const __nv_bfloat162 kr = __hadd2(as_b2(kre[i]), dm2), ki = as_b2(kim[i]);
                                    xr[i] = as_u(__hfma2(zr, kr, __hneg2(__hmul2(zi, ki))));
                                    xi[i] = as_u(__hfma2(zr, ki, __hmul2(zi, kr)));
                                }
                                um::st_afrag2(al, xr, xi);
                            } else if (s == 2) {
                                // [c][b]: transpose -> [b][c], x W_256^{-b c}
                                uint32_t gr[4], gi[4];
                                pack_tile(gr, acr);
                                pack_tile(gi, aci);
                                transpose_tile(xr, gr);
                                transpose_tile(xi, gi);
#pragma unroll
                                for (int i = 0; i < 4; ++i) twiddle2<false>(xr[i], xi[i], w256[i]);
                                um::st_afrag2(al, xr, xi);
                            } else {
                                // [b][a]: x W_M^{-q k_p}, back to S row k_p
                                const int kp = 8 * (T0 + uu) + 2 * warp + r;
                                pack_tile(xr, acr);
                                pack_tile(xi, aci);
#pragma unroll
                                for (int i = 0; i < 4; ++i) twiddle2<false>(xr[i], xi[i], tc3[uu][r][i]);
                                stsm_x4_t(plane_addr(sre, kp, ichunk), xr[0], xr[1], xr[2], xr[3]);
                                stsm_x4_t(plane_addr(sim, kp, ichunk), xi[0], xi[1], xi[2], xi[3]);
                            }
                        }
                }
            }
        }
        if (dead) break;
        __syncthreads();

        // ---------------- S1': inverse outer DFT over k_p, outputs p < P/2 into S rows p
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int qt = 8 * t + 2 * warp + r;
#pragma unroll
                for (int ks = 0; ks < U::KS3; ++ks) {
                    uint32_t ar[4], ai[4];
                    const uint32_t krow = 16 * ks + r8 + 8 * (m8 >> 1), chunk = 2 * qt + (m8 & 1);
                    ldsm_x4_t(ar, plane_addr(sre, krow, chunk));
                    ldsm_x4_t(ai, plane_addr(sim, krow, chunk));
                    um::st_afrag2(tl + lane_off(16 * r) + t * U::kA3 + 16 * ks, ar, ai);
                }
            }
        issue([&] {
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const uint32_t d = tmem + U::kD3p + t * U::N3, a = tmem + t * U::kA3;
#pragma unroll
                for (int ks = 0; ks < U::KS3; ++ks) {
                    um::mma_ts(d, a + 16 * ks, um::sdesc_kmajor(bsm + U::kOffB3 + (2 * ks) * U::kB3), id3, ks > 0);
                    um::mma_ts(d, a + 16 * ks + 8, um::sdesc_kmajor(bsm + U::kOffB3 + (2 * ks + 1) * U::kB3), id3, 1);
                }
            }
        });
        await();
        if (dead) break;
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int qt = 8 * t + 2 * warp + r;
                const uint32_t dl = tl + lane_off(16 * r) + U::kD3p + t * U::N3;
#pragma unroll
                for (int j = 0; j < U::NT3; ++j) {
                    uint32_t yr[4], yi[4];
                    um::ld16x256_x1(dl + 8 * j, yr);
                    um::ld16x256_x1(dl + U::PH + 8 * j, yi);
                    um::wait_ld(yr);
                    um::wait_ld(yi);
                    const uint32_t prow = 8 * j + r8, chunk = 2 * qt + (m8 & 1);
                    stsm_x4_t(plane_addr((m8 >> 1) ? sim : sre, prow, chunk),
                              pack2(__uint_as_float(yr[0]), __uint_as_float(yr[1])),
                              pack2(__uint_as_float(yr[2]), __uint_as_float(yr[3])),
                              pack2(__uint_as_float(yi[0]), __uint_as_float(yi[1])),
                              pack2(__uint_as_float(yi[2]), __uint_as_float(yi[3])));
                }
            }
        __syncthreads();

        // ---------------- store y (gate by v), coalesced 16-byte chunks of rows b and b+1
        for (int i = tid; i < 2 * CH; i += NT) {
            const int plane = i / CH, n0 = (i % CH) * 8;
            if (plane == 1 && !has1) continue;
            const uint32_t p = n0 >> 8, chunk = (n0 & 255) >> 3;
            uint4 val;
            asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                         : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                         : "r"(plane_addr(plane ? sim : sre, p, chunk)));
            const size_t off = (plane ? row1 : row0) + n0;
            if (GATED) {
                const uint4 vv = __ldg(reinterpret_cast<const uint4*>(v + off));
                val.x = as_u(__hmul2(as_b2(val.x), as_b2(vv.x)));
                val.y = as_u(__hmul2(as_b2(val.y), as_b2(vv.y)));
                val.z = as_u(__hmul2(as_b2(val.z), as_b2(vv.z)));
                val.w = as_u(__hmul2(as_b2(val.w), as_b2(vv.w)));
            }
            *reinterpret_cast<uint4*>(y + off) = val;
        }
        // the next iteration's wait + barrier orders these reads before S is rewritten
    }
    cp_async_wait_all();
    // a timed-out batch may still be running (its phase is the one before
    // `phase`): wait for it, bounded, before freeing TMEM
    if (dead) um::mbar_wait(mbar, phase ^ 1u);
    um::fence_before();
    __syncthreads();
    if (warp == 0) {
        um::fence_after();
        um::tmem_dealloc(tmem, U::kCols);
    }
}

}  // namespace tc

// ================================================================== host side
namespace {

// bf16 bit pattern (a local type keeps the vector's instantiation internal)
struct Bits16 {
    uint16_t v;
};

uint16_t bf16_bits_u(double x) {
    const float f = (float)x;
    uint32_t b;
    memcpy(&b, &f, 4);
    b += 0x7fffu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

// cos and sin of 2 pi e / L, e reduced mod L, in fp64
void cs_u(int64_t e, int64_t L, double* c, double* s) {
    int64_t r = e % L;
    if (r < 0) r += L;
    const double a = 2.0 * M_PI * (double)r / (double)L;
    *c = cos(a);
    *s = sin(a);
}

// Append one B operand image (N rows x 16 K, bf16, K-major core-matrix layout,
// K in TMEM column order) for the K step ks of a complex matrix G(k, n):
// part 0 = [Gr | Gi] (n < NC: Re, else Im of column n - NC), part 1 = [-Gi | Gr].
template <class F>
void push_bimage(std::vector<Bits16>& out, int NC, int ks, int part, F g) {
    const int N = 2 * NC;
    std::vector<Bits16> img((size_t)N * 16, Bits16{0});
    for (int n = 0; n < N; ++n)
        for (int kappa = 0; kappa < 16; ++kappa) {
            const int k = 16 * ks + um::kperm(kappa);
            double re, im;
            g(k, n % NC, &re, &im);
            const double val = part == 0 ? (n < NC ? re : im) : (n < NC ? -im : re);
            img[um::kmajor_off(n, kappa) / 2].v = bf16_bits_u(val);
        }
    out.insert(out.end(), img.begin(), img.end());
}

}  // namespace

bool umma_supported(int log2M) { return log2M == 12 || log2M == 13; }

// The B images of one transform length, in the order the kernel stages them.
bool umma_bimages(int log2M, std::vector<float2>& out, size_t* off) {
    if (!umma_supported(log2M)) return false;
    const int P = (1 << log2M) / 256;
    const int KS1 = (P / 2 + 15) / 16, KS3 = P / 16, PH = P / 2;
    std::vector<Bits16> img;
    // S1: G(p, k_p) = W_P^{p k_p} for p < P/2, zero rows past it
    for (int ks = 0; ks < KS1; ++ks)
        for (int part = 0; part < 2; ++part)
            push_bimage(img, P, ks, part, [P](int p, int kp, double* re, double* im) {
                if (p >= P / 2) {
                    *re = *im = 0.0;
                    return;
                }
                double c, s;
                cs_u((int64_t)p * kp, P, &c, &s);
                *re = c;
                *im = -s;
            });
    // DFT_16 and its conjugate
    for (int inv = 0; inv < 2; ++inv)
        for (int part = 0; part < 2; ++part)
            push_bimage(img, 16, 0, part, [inv](int a, int c, double* re, double* im) {
                double co, si;
                cs_u((int64_t)a * c, 16, &co, &si);
                *re = co;
                *im = inv ? si : -si;
            });
    // S1': G(k_p, p) = conj(W_P^{k_p p}) for p < P/2
    for (int ks = 0; ks < KS3; ++ks)
        for (int part = 0; part < 2; ++part)
            push_bimage(img, PH, ks, part, [P](int kp, int p, double* re, double* im) {
                double c, s;
                cs_u((int64_t)kp * p, P, &c, &s);
                *re = c;
                *im = s;
            });
    // 16-byte aligned start in the float2 table
    if (out.size() % 2) out.push_back(make_float2(0.f, 0.f));
    *off = out.size();
    const size_t words = (img.size() + 3) / 4;  // float2 entries (4 bf16 each)
    img.resize(words * 4, Bits16{0});
    const size_t base = out.size();
    out.resize(base + words + (words % 2));
    memcpy(&out[base], img.data(), img.size() * sizeof(Bits16));
    return true;
}

template <int P, bool GATED>
static cudaError_t umma_fwd_go(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                               const void* khat, const float* D, void* y, cudaStream_t s) {
    auto kern = tc::fused_fwd_umma<P, GATED>;
    const size_t smem = tc::USmem<P, GATED>::kBytes;
    // persistent grid: as many CTAs as fit on the SMs at once, limited by
    // registers, shared memory and tensor memory (512 columns per SM)
    static int resident = 0;
    if (resident == 0) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        int sms = 0, dev = 0, regs_sm = 0, smem_sm = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        cudaFuncAttributes fa;
        int per_sm = 512 / tc::UShape<P>::kCols;
        if (cudaFuncGetAttributes(&fa, kern) == cudaSuccess) {
            const int regs = ((fa.numRegs + 7) / 8) * 8 * 128;
            const int by_regs = regs > 0 ? regs_sm / regs : 1;
            const int by_smem = smem_sm / (int)(smem + fa.sharedSizeBytes + 1024);
            per_sm = per_sm < by_regs ? per_sm : by_regs;
            per_sm = per_sm < by_smem ? per_sm : by_smem;
        }
        cudaGetLastError();
        resident = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 1);
    }
    const int items = ((p.B + 1) / 2) * p.H;
    dim3 grid(items < resident ? items : resident);
    kern<<<grid, 128, smem, s>>>((const __nv_bfloat16*)u, (const __nv_bfloat16*)v, (const __nv_bfloat16*)w,
                                 (const uint4*)khat, D, (__nv_bfloat16*)y, p.tc, (const uint4*)p.umma_b, p.d_err,
                                 p.B, p.H);
    return cudaGetLastError();
}

template <int P>
static cudaError_t umma_fwd_g(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                              const void* khat, const float* D, void* y, cudaStream_t s) {
    return p.gated ? umma_fwd_go<P, true>(p, u, v, w, khat, D, y, s)
                   : umma_fwd_go<P, false>(p, u, v, w, khat, D, y, s);
}

cudaError_t launch_umma_fwd(const fftconv_plan_s& p, const void* u, const void* v, const void* w, const void* khat,
                            const float* D, void* y, cudaStream_t s) {
    switch (p.log2M) {
        case 12: return umma_fwd_g<16>(p, u, v, w, khat, D, y, s);
        case 13: return umma_fwd_g<32>(p, u, v, w, khat, D, y, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fftc
