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

#include <type_traits>
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
    static constexpr int TS = T3 / 2;                    // step-3 tiles per slot (two slots)
    static constexpr int kCols = 256;                    // TMEM columns per CTA
    // S1: both 128-row tiles in one batch: A (16 KS1 columns each), then the accumulators
    static constexpr int kA1 = 16 * KS1;
    static constexpr int kD1 = ((2 * kA1 + N1 - 1) / N1) * N1;
    // step 3: slot s at column 128 s: A of tile u at 16 u, accumulator at 32 + 32 u
    // S1': both tiles in one batch
    static constexpr int kA3 = 16 * KS3;
    static constexpr int kD3p = ((2 * kA3 + N3 - 1) / N3) * N3;
    // B images (bf16, K-major core-matrix layout), bytes
    static constexpr int kB1 = N1 * 32, kBF = 32 * 32, kB3 = N3 * 32;
    static constexpr int kOffB1 = 0;                       // [ks][2]
    static constexpr int kOffBF = kOffB1 + KS1 * 2 * kB1;  // fwd 1, fwd 2, inv 1, inv 2
    static constexpr int kOffB3 = kOffBF + 4 * kBF;        // [ks][2]
    static constexpr int kBBytes = kOffB3 + KS3 * 2 * kB3;
    static_assert(kD1 + 2 * N1 <= kCols, "S1 columns");
    static_assert(TS >= 1 && 32 + 32 * TS <= 128 && 16 * TS <= 32, "step-3 columns");
    static_assert(kD3p + 2 * N3 <= kCols, "S1' columns");
};

template <int P, bool GATED>
struct USmem {
    static constexpr int kS = 2 * P * 512;                       // S planes (re, im), P rows of 256 q
    static constexpr int kX = P * 512;                           // staging planes of x (P/2 rows each)
    static constexpr int kW = GATED ? kX : 0;                    // staging planes of w
    static constexpr int kStage = kX + kW;                       // one staging buffer (two, alternating by item)
    static constexpr int kB = UShape<P>::kBBytes;
    static constexpr int kOffX = kS, kOffB = kS + 2 * kStage;
    static constexpr int kBytes = kOffB + kB;
};

__device__ __forceinline__ uint32_t lane_off(int lane0) { return (uint32_t)lane0 << 16; }

// warps 0-7 compute (warp w: TMEM lane quarter w % 4, row half w / 4 of every 16-row group), warp 8 issues the MMAs
constexpr int kUmmaCompute = 256;
constexpr int kUmmaThreads = kUmmaCompute + 32;

// Barriers in shared memory: afull[i] (8 arrivals: every compute warp has
// stored its A rows for batch slot i), dfull[i] (one arrival: the MMAs of the
// slot's batch are complete).  Slots 0 and 1 alternate in step 3; slot 2 is
// S1 and S1'.
struct UBars {
    uint64_t afull[3];
    uint64_t dfull[3];
    uint64_t drain;  // the issuer's last commit: every MMA it issued is complete
};

template <int P, bool GATED>
__global__ void __launch_bounds__(kUmmaThreads, 2)
fused_fwd_umma(const __nv_bfloat16* __restrict__ u, const __nv_bfloat16* __restrict__ v,
               const __nv_bfloat16* __restrict__ w, const uint4* __restrict__ khat, const float* __restrict__ D,
               __nv_bfloat16* __restrict__ y, TcTables tb, const uint4* __restrict__ bimg, int* __restrict__ err,
               int B, int H, uint32_t wait_limit) {
    using S = TcShape<P>;
    using U = UShape<P>;
    using SM = USmem<P, GATED>;
    constexpr int NT = kUmmaCompute;  // compute threads
    constexpr int CH = S::N / 8;  // 16-byte chunks per row of u
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint32_t s_tmem;
    __shared__ __align__(8) UBars s_bar;
    __shared__ int s_drained;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m8 = lane >> 3, r8 = lane & 7;
    const int npp = (B + 1) / 2;
    const int items = npp * H;
    const uint32_t sre = tc::smem_u32(smem), sim = sre + S::kPlaneBytes;
    const uint32_t xbase = sre + SM::kOffX;  // staging buffer of the item k-th in this CTA: xbase + (k & 1) kStage
    const uint32_t bsm = sre + SM::kOffB;
    const uint32_t afull = tc::smem_u32(&s_bar.afull[0]), dfull = tc::smem_u32(&s_bar.dfull[0]);

    // ---- set-up: B images into shared memory (visible to the tensor core), TMEM, barriers
    for (int i = tid; i < U::kBBytes / 16; i += kUmmaThreads) {
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
    if (tid == 0) {
#pragma unroll
        for (int i = 0; i < 3; ++i) {
            um::mbar_init(afull + 8 * i, kUmmaCompute / 32);
            um::mbar_init(dfull + 8 * i, 1);
        }
        um::mbar_init(tc::smem_u32(&s_bar.drain), 1);
    }
    um::fence_before();
    __syncthreads();
    um::fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == kUmmaCompute / 32) {
        // ================= MMA issuer: one lane walks the same batch sequence as the compute warps
        if (lane == 0) {
            const uint32_t id1 = um::idesc_bf16(128, U::N1), id16 = um::idesc_bf16(128, 32),
                           id3 = um::idesc_bf16(128, U::N3);
            uint32_t pa[3] = {0u, 0u, 0u};
            auto wait_a = [&](int i) {
                const bool ok = um::mbar_wait(afull + 8 * i, pa[i], wait_limit);
                pa[i] ^= 1u;
                um::fence_after();
                return ok;
            };
            bool ok = true;
            for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
                // S1: rows q, K = p < P/2, both tiles
                if (!(ok = wait_a(2))) break;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const uint32_t d = tmem + U::kD1 + t * U::N1, a = tmem + t * U::kA1;
#pragma unroll
                    for (int ks = 0; ks < U::KS1; ++ks) {
                        um::mma_ts(d, a + 16 * ks, um::sdesc_kmajor(bsm + U::kOffB1 + (2 * ks) * U::kB1), id1, ks > 0);
                        um::mma_ts(d, a + 16 * ks + 8, um::sdesc_kmajor(bsm + U::kOffB1 + (2 * ks + 1) * U::kB1), id1, 1);
                    }
                }
                um::mma_commit(dfull + 16);
                // step 3: four stages, the two slots alternating
#pragma unroll 1
                for (int st = 0; st < 4 && ok; ++st)
#pragma unroll
                    for (int sl = 0; sl < 2; ++sl) {
                        if (!(ok = wait_a(sl))) break;
                        const uint32_t bf = bsm + U::kOffBF + (st < 2 ? 0 : 2) * U::kBF;
#pragma unroll
                        for (int uu = 0; uu < U::TS; ++uu) {
                            const uint32_t d = tmem + 128 * sl + 32 + 32 * uu, a = tmem + 128 * sl + 16 * uu;
                            um::mma_ts(d, a, um::sdesc_kmajor(bf), id16, 0);
                            um::mma_ts(d, a + 8, um::sdesc_kmajor(bf + U::kBF), id16, 1);
                        }
                        um::mma_commit(dfull + 8 * sl);
                    }
                if (!ok) break;
                // S1': rows q, K = k_p, N = p < P/2, both tiles
                if (!(ok = wait_a(2))) break;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const uint32_t d = tmem + U::kD3p + t * U::N3, a = tmem + t * U::kA3;
#pragma unroll
                    for (int ks = 0; ks < U::KS3; ++ks) {
                        um::mma_ts(d, a + 16 * ks, um::sdesc_kmajor(bsm + U::kOffB3 + (2 * ks) * U::kB3), id3, ks > 0);
                        um::mma_ts(d, a + 16 * ks + 8, um::sdesc_kmajor(bsm + U::kOffB3 + (2 * ks + 1) * U::kB3), id3, 1);
                    }
                }
                um::mma_commit(dfull + 16);
            }
            // drain: one more commit, waited for with the default limit, so that no
            // product is in flight when TMEM is freed (after a give-up as well)
            um::mma_commit(tc::smem_u32(&s_bar.drain));
            s_drained = um::mbar_wait(tc::smem_u32(&s_bar.drain), 0u) ? 1 : 0;
            if (!ok || !s_drained) atomicExch(err, 1);
        }
    } else {
        // ================= compute warps: TMEM lanes 32 q + 16 r .. + 15 of every 128-lane tile
        const int q = warp & 3, r = warp >> 2;
        const uint32_t tl = tmem + lane_off(32 * q + 16 * r);
        uint2 w256[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) w256[i] = __ldg(&tb.w256[i * 32 + lane]);
        uint32_t pd[3] = {0u, 0u, 0u};
        bool dead = false;
        // this warp's A rows of slot i are in TMEM: tell the issuer
        auto signal = [&](int i) {
            um::wait_st();
            um::fence_before();
            __syncwarp();
            if (lane == 0) um::mbar_arrive(afull + 8 * i);
        };
        // wait for slot i's products (bounded); a timeout marks the CTA dead at the next named barrier
        auto wait_d = [&](int i) {
            const bool ok = um::mbar_wait(dfull + 8 * i, pd[i], wait_limit);
            pd[i] ^= 1u;
            um::fence_after();
            dead |= !ok;
        };
        auto stage_input = [&](int item, int buf) {
            const uint32_t xre = xbase + buf * SM::kStage, xim = xre + SM::kX / 2;
            const uint32_t wre = xre + SM::kX, wim = wre + SM::kX / 2;
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
        const uint32_t ia = r8 + 8 * (m8 >> 1), ichunk = 2 * ia + (m8 & 1);  // step-3 ldmatrix / stmatrix chunk

        if ((int)blockIdx.x < items) stage_input(blockIdx.x, 0);
        int k = 0;  // items done by this CTA
        for (int item = blockIdx.x; item < items; item += gridDim.x, ++k) {
            const int h = item / npp, b0 = 2 * (item % npp);
            const bool has1 = b0 + 1 < B;
            const size_t row0 = ((size_t)b0 * H + h) * S::N;
            const size_t row1 = ((size_t)(b0 + 1) * H + h) * S::N;
            // the next item's rows go to the other buffer (free: its last reader was the
            // previous item's S1, and the barrier below the previous S1 has passed)
            if (item + (int)gridDim.x < items) {
                stage_input(item + gridDim.x, (k + 1) & 1);
                asm volatile("cp.async.wait_group 1;\n" ::: "memory");
            } else {
                cp_async_wait_all();
            }
            if (um::bar_or(1, NT, dead)) break;
            const uint32_t xre = xbase + (k & 1) * SM::kStage, xim = xre + SM::kX / 2;
            const uint32_t wre = xre + SM::kX, wim = wre + SM::kX / 2;

            // ---------------- S1: A = x rows q of both tiles (K = p < P/2)
            uint2 tw[2][U::NT1][2];  // W_M^{q k_p} of this warp's rows, fetched ahead of use
#pragma unroll
            for (int t = 0; t < 2; ++t)
#pragma unroll
                for (int j = 0; j < U::NT1; ++j)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int qt = 8 * t + 2 * q + r;
                        tw[t][j][hh] = __ldg(&tb.tw1[((qt * U::NT1 + j) * 2 + hh) * 32 + lane]);
                    }
#pragma unroll
            for (int t = 0; t < 2; ++t)
                {
                    const int qt = 8 * t + 2 * q + r;
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
                        um::st_afrag2(tl + t * U::kA1 + 16 * ks, ar, ai);
                    }
                }
            signal(2);
            wait_d(2);
            // x W_M^{q k_p}, stored transposed into S[k_p][q]
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                uint32_t yv[8 * U::NT1];  // Re blocks then Im blocks
                {
                    const uint32_t dl = tl + U::kD1 + t * U::N1;
                    um::ld16x256<U::NT1>(dl, yv);
                    um::ld16x256<U::NT1>(dl + P, yv + 4 * U::NT1);
                }
                um::wait_ld<8 * U::NT1>(yv);
                {
                    const int qt = 8 * t + 2 * q + r;
#pragma unroll
                    for (int j = 0; j < U::NT1; ++j) {
                        const uint32_t* yr = yv + 4 * j;
                        const uint32_t* yi = yr + 4 * U::NT1;
                        uint32_t pr[2] = {pack2(__uint_as_float(yr[0]), __uint_as_float(yr[1])),
                                          pack2(__uint_as_float(yr[2]), __uint_as_float(yr[3]))};
                        uint32_t pi[2] = {pack2(__uint_as_float(yi[0]), __uint_as_float(yi[1])),
                                          pack2(__uint_as_float(yi[2]), __uint_as_float(yi[3]))};
                        twiddle2<true>(pr[0], pi[0], tw[t][j][0]);
                        twiddle2<true>(pr[1], pi[1], tw[t][j][1]);
                        const uint32_t krow = 8 * j + r8, chunk = 2 * qt + (m8 & 1);
                        stsm_x4_t(plane_addr((m8 >> 1) ? sim : sre, krow, chunk), pr[0], pr[1], pi[0], pi[1]);
                    }
                }
            }
            if (um::bar_or(1, NT, dead)) break;  // S complete

            // ---------------- step 3: inner 256-point DFT, product with Khat, inverse
            const float dmf = D ? D[h] * (1.0f / S::M) : 0.f;
            const __nv_bfloat162 dm2 = __floats2bfloat162_rn(dmf, dmf);
            const uint4* __restrict__ kh = khat + (size_t)h * P * 64;  // 32 lanes x 2 uint4 per row
            // stage-0 A tiles of both slots: rows b, K = a, from S rows k_p
#pragma unroll
            for (int sl = 0; sl < 2; ++sl) {
#pragma unroll
                for (int uu = 0; uu < U::TS; ++uu)
                    {
                        const int kp = 8 * (sl * U::TS + uu) + 2 * q + r;
                        uint32_t xr[4], xi[4];
                        ldsm_x4_t(xr, plane_addr(sre, kp, ichunk));
                        ldsm_x4_t(xi, plane_addr(sim, kp, ichunk));
                        um::st_afrag2(tl + 128 * sl + 16 * uu, xr, xi);
                    }
                signal(sl);
            }
            // spectrum words of this warp's rows (both slots), fetched two epilogues ahead of use
            uint4 kc0[2][U::TS], kc1[2][U::TS];
#pragma unroll
            for (int sl = 0; sl < 2; ++sl)
#pragma unroll
                for (int uu = 0; uu < U::TS; ++uu) {
                    const int kp = 8 * (sl * U::TS + uu) + 2 * q + r;
                    kc0[sl][uu] = __ldg(&kh[(size_t)kp * 64 + lane * 2]);
                    kc1[sl][uu] = __ldg(&kh[(size_t)kp * 64 + lane * 2 + 1]);
                }
            uint2 tc3[2][U::TS][4];  // W_M^{-q k_p}, fetched at the start of stage 2
            auto epilogue = [&](auto st_c, auto sl_c) {
                constexpr int ST = decltype(st_c)::value;
                constexpr int sl = decltype(sl_c)::value;
                if (ST == 2 && sl == 0) {
#pragma unroll
                    for (int s2 = 0; s2 < 2; ++s2)
#pragma unroll
                        for (int uu = 0; uu < U::TS; ++uu) {
                            const int kp = 8 * (s2 * U::TS + uu) + 2 * q + r;
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                tc3[s2][uu][i] = __ldg(&tb.tw3[((size_t)kp * 4 + i) * 32 + lane]);
                        }
                }
                wait_d(sl);
                uint32_t accs[U::TS * 16];
#pragma unroll
                for (int uu = 0; uu < U::TS; ++uu)
                        um::ld16x256<4>(tl + 128 * sl + 32 + 32 * uu, accs + uu * 16);
                um::wait_ld<U::TS * 16>(accs);
#pragma unroll
                for (int uu = 0; uu < U::TS; ++uu)
                    {
                        const uint32_t al = tl + 128 * sl + 16 * uu;
                        const uint32_t* acc = accs + uu * 16;
                        float acr[2][4], aci[2][4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            acr[0][e] = __uint_as_float(acc[e]);
                            acr[1][e] = __uint_as_float(acc[4 + e]);
                            aci[0][e] = __uint_as_float(acc[8 + e]);
                            aci[1][e] = __uint_as_float(acc[12 + e]);
                        }
                        uint32_t xr[4], xi[4];
                        if (ST == 0) {
                            // [b][c]: x W_256^{b c}, transpose -> [c][b]
                            uint32_t tr[4], ti[4];
                            pack_tile(tr, acr);
                            pack_tile(ti, aci);
#pragma unroll
                            for (int i = 0; i < 4; ++i) twiddle2<true>(tr[i], ti[i], w256[i]);
                            transpose_tile(xr, tr);
                            transpose_tile(xi, ti);
                            um::st_afrag2(al, xr, xi);
                        } else if (ST == 1) {
                            // [c][d]: spectrum at k = k_p + P (c + 16 d); x (Khat + D/M)
                            pack_tile(xr, acr);
                            pack_tile(xi, aci);
                            const uint32_t kre[4] = {kc0[sl][uu].x, kc0[sl][uu].z, kc1[sl][uu].x, kc1[sl][uu].z};
                            const uint32_t kim[4] = {kc0[sl][uu].y, kc0[sl][uu].w, kc1[sl][uu].y, kc1[sl][uu].w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const __nv_bfloat162 zr = as_b2(xr[i]), zi = as_b2(xi[i]);
                                const __nv_bfloat162 kr = __hadd2(as_b2(kre[i]), dm2), ki = as_b2(kim[i]);
                                xr[i] = as_u(__hfma2(zr, kr, __hneg2(__hmul2(zi, ki))));
                                xi[i] = as_u(__hfma2(zr, ki, __hmul2(zi, kr)));
                            }
                            um::st_afrag2(al, xr, xi);
                        } else if (ST == 2) {
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
                            const int kp = 8 * (sl * U::TS + uu) + 2 * q + r;
                            pack_tile(xr, acr);
                            pack_tile(xi, aci);
#pragma unroll
                            for (int i = 0; i < 4; ++i) twiddle2<false>(xr[i], xi[i], tc3[sl][uu][i]);
                            stsm_x4_t(plane_addr(sre, kp, ichunk), xr[0], xr[1], xr[2], xr[3]);
                            stsm_x4_t(plane_addr(sim, kp, ichunk), xi[0], xi[1], xi[2], xi[3]);
                        }
                    }
                if (ST < 3) signal(sl);
            };
            using I0 = std::integral_constant<int, 0>;
            using I1 = std::integral_constant<int, 1>;
            using I2 = std::integral_constant<int, 2>;
            using I3 = std::integral_constant<int, 3>;
            epilogue(I0{}, I0{});
            epilogue(I0{}, I1{});
            epilogue(I1{}, I0{});
            epilogue(I1{}, I1{});
            epilogue(I2{}, I0{});
            epilogue(I2{}, I1{});
            epilogue(I3{}, I0{});
            epilogue(I3{}, I1{});
            if (um::bar_or(1, NT, dead)) break;  // S complete

            // ---------------- S1': inverse outer DFT over k_p, outputs p < P/2 into S rows p
#pragma unroll
            for (int t = 0; t < 2; ++t)
                {
                    const int qt = 8 * t + 2 * q + r;
#pragma unroll
                    for (int ks = 0; ks < U::KS3; ++ks) {
                        uint32_t ar[4], ai[4];
                        const uint32_t krow = 16 * ks + r8 + 8 * (m8 >> 1), chunk = 2 * qt + (m8 & 1);
                        ldsm_x4_t(ar, plane_addr(sre, krow, chunk));
                        ldsm_x4_t(ai, plane_addr(sim, krow, chunk));
                        um::st_afrag2(tl + t * U::kA3 + 16 * ks, ar, ai);
                    }
                }
            signal(2);
            // every warp has read its S1' operands: S rows p may be rewritten below
            if (um::bar_or(1, NT, dead)) break;
            wait_d(2);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                uint32_t zv[8 * U::NT3];  // Re blocks then Im blocks
                {
                    const uint32_t dl = tl + U::kD3p + t * U::N3;
                    um::ld16x256<U::NT3>(dl, zv);
                    um::ld16x256<U::NT3>(dl + U::PH, zv + 4 * U::NT3);
                }
                um::wait_ld<8 * U::NT3>(zv);
                {
                    const int qt = 8 * t + 2 * q + r;
#pragma unroll
                    for (int j = 0; j < U::NT3; ++j) {
                        const uint32_t* yr = zv + 4 * j;
                        const uint32_t* yi = yr + 4 * U::NT3;
                        const uint32_t prow = 8 * j + r8, chunk = 2 * qt + (m8 & 1);
                        stsm_x4_t(plane_addr((m8 >> 1) ? sim : sre, prow, chunk),
                                  pack2(__uint_as_float(yr[0]), __uint_as_float(yr[1])),
                                  pack2(__uint_as_float(yr[2]), __uint_as_float(yr[3])),
                                  pack2(__uint_as_float(yi[0]), __uint_as_float(yi[1])),
                                  pack2(__uint_as_float(yi[2]), __uint_as_float(yi[3])));
                    }
                }
            }
            if (um::bar_or(1, NT, dead)) break;  // output rows complete

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
        if (dead && tid == 0) atomicExch(err, 1);
    }
    // every wait above is bounded, and the issuer has drained its products;
    // should even that drain give up, TMEM is left allocated rather than freed
    // under a running product (the status word is set)
    um::fence_before();
    __syncthreads();
    if (warp == 0 && s_drained) {
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
            const int regs = ((fa.numRegs + 7) / 8) * 8 * tc::kUmmaThreads;
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
    kern<<<grid, tc::kUmmaThreads, smem, s>>>((const __nv_bfloat16*)u, (const __nv_bfloat16*)v, (const __nv_bfloat16*)w,
                                 (const uint4*)khat, D, (__nv_bfloat16*)y, p.tc, (const uint4*)p.umma_b, p.d_err,
                                 p.B, p.H, p.wait_limit);
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
