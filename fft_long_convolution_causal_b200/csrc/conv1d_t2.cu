// conv1d_t2.cu -- fused bf16 causal FFT convolution for 2N = 8192 as a
// two-stage Monarch split on the fifth-generation tensor cores, with the data
// held in tensor memory between the stages.
//
// The method is the FFT convolution as matrix products of "FlashFFTConv:
// Efficient Convolutions for Long Sequences with Tensor Cores" (abstract),
// fused on chip as in "FlashConv" (Mechanism: FFT, pointwise spectral product
// and inverse without intermediate off-chip traffic; the FFT factored into
// block matrix multiplications), made causal by zero padding to 2N and
// truncation to [:N] ("RubiConv -- Efficient Boundary-Respecting
// Convolutions", Caracal abstract).
//
// Split: M = 8192 = P x Q, P = 128, Q = 64.  Input n = Q p + q (p < 64 holds
// the data, p >= 64 the zero padding), frequency k = k_p + P c.  Two batch
// rows b, b+1 of one channel are the real and imaginary parts z = x_b + i x_b+1.
//   A: Y[k_p][q]  = sum_{p < 64} W_128^{p k_p} z[p][q]          (smem x smem)
//      Y'         = Y W_M^{q k_p}                               (epilogue A)
//   B: X[k_p][c]  = sum_q Y'[k_p][q] W_64^{q c}                 (tmem x smem)
//      Z          = conj(X (Khat + D/M))                        (epilogue B)
//   C: V0[k_p][q] = sum_c Z[k_p][c] W_64^{c q} = conj(Z1)       (tmem x smem)
//      V          = V0 W_M^{q k_p} = conj(Z1 W_M^{-q k_p})      (epilogue C)
//   D: y[p][q]    = conj(sum_{k_p} W_128^{p k_p} V[k_p][q]), p < 64
// The inverse runs as the conjugate of a forward transform of the conjugate,
// so stage C reuses stage B's matrix and epilogue C stage A's twiddles.
// Stage D's A operand stacks the rows giving Re y (p) and Im y (64 + p) so
// that one 128-row product emits both output rows; stage A reads the upper
// blocks of the same shared-memory matrix as an MN-major operand (the outer
// DFT matrix is symmetric).
//
// Every TMEM lane is one row k_p (stages A-C), so each epilogue thread reads
// its row's accumulators, applies its twiddles or spectrum values in packed
// bf16 pairs and writes the next stage's A operand back into the same lane:
// no transposes and no shared-memory round trip between A, B and C.  The
// operand's columns run in groups of 16 (8 pairs of Re, then the 8 matching
// pairs of Im, for 16 consecutive q or c), so every group is rewritten in
// place in the columns that held its own real parts.
//
// Roles (576 threads, one CTA per SM, all 512 TMEM columns): two pipelines
// ("slots", 256 TMEM columns and their own shared memory each) working
// through alternate row pairs of the CTA, each with 8 epilogue warps (warp
// e of the slot: TMEM lanes 32 (e % 4) .., column half e / 4) and one warp
// whose first lane issues the slot's products and brings each pair's input
// rows in with one bulk tensor copy (TMA), issued once stage A has read the
// previous rows.  The two slots share the tensor core: one slot's product
// runs while the other slot's warps run an epilogue.  Every wait is bounded;
// a wait that gives up stops the CTA, each issuer drains its products before
// TMEM is freed, and the plan's status word is set.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <vector>

#include "plan.h"
#include "tc_common.cuh"
#include "umma.cuh"

namespace fftc {
namespace t2 {

constexpr int kP = 128, kQ = 64, kM = 8192, kN = 4096;

// shared memory (bytes)
constexpr uint32_t kOffGP = 0;            // outer DFT matrix, [m 128][k 256] K-major core matrices, 64 KiB
constexpr uint32_t kOffFQ = 65536;        // inner DFT matrix, [n 128][k 128] K-major, 32 KiB
constexpr uint32_t kOffX = 98304;         // input planes of slot s at + 16 KiB s: [p 64][n 128] MN-major
constexpr uint32_t kOffV = 131072;        // stage-D operand of slot s at + 32 KiB s: [k 256][n 64] MN-major
constexpr uint32_t kOffTW = 196608;       // twiddle pairs of W_M^{q k_p}: [q / 2][k_p 128] uint2, 32 KiB
constexpr uint32_t kSmemBytes = 229376;

// core-matrix strides of each operand (bytes)
constexpr uint32_t kGPm = 4096, kGPk = 128;   // GP: row group (8 m) / column group (8 k)
constexpr uint32_t kFQn = 2048, kFQk = 128;   // FQ: 8 n / 8 k
constexpr uint32_t kXp = 2048, kXn = 128;     // X: 8 p / 8 n
constexpr uint32_t kVk = 1024, kVn = 128;     // V: 8 k / 8 n

// roles: warps 8 s .. 8 s + 7 the epilogues of slot s, warp 16 + s its issuer
constexpr int kSlotWarps = 8, kIssuerWarp = 16, kThreads = 576;

struct SlotBars {
    uint64_t dA, dX, dD, afull, xfull;
};

__device__ __forceinline__ uint32_t lanes(int quarter) { return (uint32_t)(32 * quarter) << 16; }

// byte offset of element (row k, column n) of an MN-major operand with row
// group stride rk and column group stride cn (rows = K, 16-byte core rows of 8 n)
__device__ __forceinline__ uint32_t mn_off(int k, int n, uint32_t rk, uint32_t cn) {
    return (uint32_t)(k >> 3) * rk + (uint32_t)(n >> 3) * cn + (uint32_t)(k & 7) * 16u + (uint32_t)(n & 7) * 2u;
}

// a descriptor advanced by a compile-time byte offset (the start address field
// is the low 14 bits of address / 16; every operand ends below 256 KiB)
__device__ __forceinline__ uint64_t dadd(uint64_t d, uint32_t bytes) { return d + (uint64_t)(bytes >> 4); }

// the same value, opaque to the compiler: the descriptors of a stage are
// derived from it at issue time (one add each) instead of being hoisted out of
// the issue loop into dozens of live registers
__device__ __forceinline__ uint64_t opaque(uint64_t d) {
    uint64_t r;
    asm volatile("mov.b64 %0, %1;" : "=l"(r) : "l"(d));
    return r;
}

// The input rows of pair (h, b0) come in as one bulk tensor copy through a
// 5-D map of u whose dimensions, fastest first, are (q mod 8, p mod 8, q / 8,
// batch row b, 8 h + p / 8) with byte strides (2, 128, 16, 8192 H, 1024): the
// box (8, 8, 8, 2, 8) at (0, 0, 0, b0, 8 h) lands in X exactly in the
// MN-major core-matrix order of stage A's operand (p = 8 (p / 8) + p mod 8 is
// the K index, n = 64 (b - b0) + q the N index), and a row b = B past the end
// reads as zeros.
constexpr uint32_t kXBytes = 16384;

__global__ void __launch_bounds__(kThreads, 1)
fused_fwd_t2(const uint4* __restrict__ khat, const float* __restrict__ D,
             __nv_bfloat16* __restrict__ y, const uint4* __restrict__ mats, const uint2* __restrict__ twid,
             int* __restrict__ err, int B, int H, uint32_t wait_limit, int kdiv,
             const __grid_constant__ CUtensorMap xmap) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint32_t s_tmem;
    __shared__ __align__(8) SlotBars s_bar[2];
    __shared__ __align__(8) uint64_t s_drain[2];
    __shared__ int s_drained[2];
    __shared__ volatile int s_abort;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t sbase = tc::smem_u32(smem);
    const int npp = (B + 1) / 2;   // row pairs per channel
    const int pairs = npp * H;
    const int qstep = 2 * (int)gridDim.x;
    auto bar = [&](const uint64_t& b) { return tc::smem_u32(&b); };
    auto first_pair = [&](int slot) { return (int)blockIdx.x + slot * (int)gridDim.x; };

    // ---- set-up: barriers; the first input rows of both slots (bulk copies)
    // in flight while the constant matrices and twiddles come into shared
    // memory; TMEM
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            um::mbar_init(bar(s_bar[s].dA), 1);
            um::mbar_init(bar(s_bar[s].dX), 1);
            um::mbar_init(bar(s_bar[s].dD), 1);
            um::mbar_init(bar(s_bar[s].afull), kSlotWarps);
            um::mbar_init(bar(s_bar[s].xfull), 1);
        }
        for (int s = 0; s < 2; ++s) {
            um::mbar_init(bar(s_drain[s]), 1);
            s_drained[s] = 1;
        }
        s_abort = 0;
    }
    __syncthreads();
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            const int q = first_pair(s);
            if (q < pairs) {
                const uint32_t xb = bar(s_bar[s].xfull);
                um::mbar_arrive_expect_tx(xb, kXBytes);
                um::tma_load_5d(sbase + kOffX + kXBytes * (uint32_t)s, &xmap, 0, 0, 0, 2 * (q % npp), 8 * (q / npp),
                                xb);
            }
        }
    }
    for (int i = tid; i < (int)(kOffX / 16); i += kThreads) tc::cp_async16(sbase + 16u * i, mats + i, 16);
    for (int i = tid; i < 2048; i += kThreads)
        tc::cp_async16(sbase + kOffTW + 16u * i, reinterpret_cast<const uint4*>(twid) + i, 16);
    tc::cp_async_commit();
    tc::cp_async_wait_all();
    um::fence_proxy_async();
    if (warp == 0) {
        um::tmem_alloc(tc::smem_u32(&s_tmem), 512);
        um::tmem_relinquish();
    }
    um::fence_before();
    __syncthreads();
    um::fence_after();
    const uint32_t tmem = s_tmem;

    if (warp >= kIssuerWarp) {
        // ======================= products and input copies of slot warp - 16
        if (lane == 0) {
            const uint32_t idA128 = um::idesc_bf16(128, 128) | um::kAmn | um::kBmn;
            const uint32_t idA64 = um::idesc_bf16(128, 64) | um::kAmn | um::kBmn;
            const uint32_t idBC = um::idesc_bf16(128, 128);
            const uint32_t idD = um::idesc_bf16(128, 64) | um::kBmn;
            const uint64_t gpA0 = um::sdesc(sbase + kOffGP, kGPm, kGPk);   // MN-major view for stage A
            const uint64_t gpD0 = um::sdesc(sbase + kOffGP, kGPk, kGPm);   // K-major for stage D
            const uint64_t fq0 = um::sdesc(sbase + kOffFQ, kFQk, kFQn);
            const uint64_t xd0 = um::sdesc(sbase + kOffX, kXp, kXn);
            const uint64_t vd0 = um::sdesc(sbase + kOffV, kVk, kVn);
            // the input rows of pair q into slot s's X
            auto load_x = [&](int s, int q) {
                const uint32_t xb = bar(s_bar[s].xfull);
                um::mbar_arrive_expect_tx(xb, kXBytes);
                um::tma_load_5d(sbase + kOffX + kXBytes * (uint32_t)s, &xmap, 0, 0, 0, 2 * (q % npp), 8 * (q / npp), xb);
            };
            // A: Y = F_128 z (upper half of GP as an MN-major view) into Ra
            auto stage_a = [&](int s) {
                const uint32_t t = tmem + 256u * (uint32_t)s;
                const uint64_t xd = opaque(dadd(xd0, 16384u * (uint32_t)s)), gpA = opaque(gpA0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)  // cos view x [x_re | x_im]
                    um::mma_ss(t, dadd(gpA, ks * 2 * kGPm), dadd(xd, ks * 2 * kXp), idA128, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {  // sin view: + sin x_im -> Re, - sin x_re -> Im
                    const uint64_t a = dadd(gpA, 2048u + ks * 2 * kGPm);
                    um::mma_ss(t, a, dadd(xd, 1024u + ks * 2 * kXp), idA64, 1);
                    um::mma_ss(t + 64u, a, dadd(xd, ks * 2 * kXp), idA64 | um::kNegA, 1);
                }
                um::mma_commit(bar(s_bar[s].dA));
            };
            // B (Ra -> Rb) or C (Rb -> Ra): the epilogue's operand times F_64
            auto stage_bc = [&](int s, bool isC) {
                const uint32_t t = tmem + 256u * (uint32_t)s;
                const uint32_t src = t + (isC ? 128u : 0u), dst = t + (isC ? 0u : 128u);
                const uint64_t fq = opaque(fq0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) um::mma_ts(dst, src + 8u * ks, dadd(fq, ks * 2 * kFQk), idBC, ks > 0);
                um::mma_commit(bar(s_bar[s].dX));
            };
            // D: rows p (Re) and 64 + p (Im) of y, N = 64 q, into Rb
            auto stage_d = [&](int s) {
                const uint32_t t = tmem + 256u * (uint32_t)s;
                const uint64_t vd = opaque(dadd(vd0, 32768u * (uint32_t)s)), gpD = opaque(gpD0);
#pragma unroll
                for (int ks = 0; ks < 16; ++ks)
                    um::mma_ss(t + 128u, dadd(gpD, ks * 2 * kGPk), dadd(vd, ks * 2 * kVk), idD, ks > 0);
                um::mma_commit(bar(s_bar[s].dD));
            };
            // the slot's pairs in order: stage A once its input rows have landed (the
            // next pair's rows are copied in as soon as stage A has read these), then
            // stages B, C, D, each released by the epilogue warps' arrival
            const int s = warp - kIssuerWarp;
            uint32_t pa = 0u, px = 0u, pd = 0u;
            bool inflight = false, ok = true;
            auto wait = [&](uint32_t b, uint32_t& par) -> bool {
                const bool r = !s_abort && um::mbar_wait(b, par, wait_limit);
                par ^= 1u;
                if (!r) s_abort = 1;
                return r;
            };
            const SlotBars& sb = s_bar[s];
            int q = first_pair(s);
            inflight = q < pairs;  // the set-up issued this pair's copy
            for (; q < pairs && ok; q += qstep) {
                if (!(ok = wait(bar(sb.xfull), px))) break;
                inflight = false;
                stage_a(s);
                if (q + qstep < pairs) {
                    if (!(ok = wait(bar(sb.dA), pd))) break;
                    load_x(s, q + qstep);
                    inflight = true;
                }
                if (!(ok = wait(bar(sb.afull), pa))) break;
                um::fence_after();
                stage_bc(s, false);
                if (!(ok = wait(bar(sb.afull), pa))) break;
                um::fence_after();
                stage_bc(s, true);
                if (!(ok = wait(bar(sb.afull), pa))) break;
                um::fence_after();
                stage_d(s);
            }
            // a copy still in flight (after a wait gave up) lands before the CTA ends
            if (inflight && !um::mbar_wait(bar(sb.xfull), px)) s_abort = 1;
            // drain: every product issued is complete before TMEM is freed
            um::mma_commit(bar(s_drain[s]));
            s_drained[s] = um::mbar_wait(bar(s_drain[s]), 0u) ? 1 : 0;
            if (s_abort || !s_drained[s]) atomicExch(err, 1);
        }
        __syncwarp();
    } else {
        // ======================= epilogue warps of slot s: TMEM lanes 32 quarter .., column half hf
        const int slot = warp / kSlotWarps, e = warp % kSlotWarps;
        const int quarter = warp & 3, hf = e >> 2;
        const int r = 32 * quarter + lane;  // TMEM lane: k_p in stages A-C
        const uint32_t tl = tmem + 256u * (uint32_t)slot + lanes(quarter);
        const uint32_t vs = sbase + kOffV + 32768u * (uint32_t)slot;
        SlotBars& sb = s_bar[slot];
        uint32_t pdA = 0u, pdX = 0u, pdD = 0u;
        auto wait = [&](uint32_t b, uint32_t& par) -> bool {
            const bool ok = !s_abort && um::mbar_wait(b, par, wait_limit);
            par ^= 1u;
            if (!ok) s_abort = 1;
            return ok;
        };
        auto arrive = [&]() {
            um::fence_before();
            __syncwarp();
            if (lane == 0) um::mbar_arrive(bar(sb.afull));
        };
        // twiddle pairs (cos, sin) of W_M^{q k_p}, q = 16 g + 2 i, + 1
        auto fetch_tw = [&](int g, uint2 (&tw)[8]) {
            const uint32_t t = sbase + kOffTW + (uint32_t)(8 * g * 128 + r) * 8u;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];\n"
                             : "=r"(tw[i].x), "=r"(tw[i].y)
                             : "r"(t + (uint32_t)i * 1024u));
        };
        // column group g of Ra: Re (column 16 g) and Im (64 + 16 g)
        auto load1 = [&](int g, uint32_t (&re)[16], uint32_t (&im)[16]) {
            um::ld32x32_x16(tl + 16u * (uint32_t)g, re);
            um::ld32x32_x16(tl + 64u + 16u * (uint32_t)g, im);
            um::wait_ld<16>(re);
            um::wait_ld<16>(im);
        };
        // x W_M^{q k_p} for group g in packed pairs: o[0..7] Re pairs, o[8..15] Im pairs
        auto twiddle = [&](int g, const uint32_t (&re)[16], const uint32_t (&im)[16], uint32_t (&o)[16]) {
            uint2 tw[8];
            fetch_tw(g, tw);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                o[i] = tc::pack2(__uint_as_float(re[2 * i]), __uint_as_float(re[2 * i + 1]));
                o[8 + i] = tc::pack2(__uint_as_float(im[2 * i]), __uint_as_float(im[2 * i + 1]));
                tc::twiddle2<true>(o[i], o[8 + i], tw[i]);
            }
        };
        for (int q = first_pair(slot); q < pairs; q += qstep) {
            const int h = q / npp, b0 = 2 * (q % npp);
            // kdiv consecutive row channels share one spectrum and skip weight (the
            // chunks of one channel in the chunked state-passing path; 1 otherwise)
            const int hk = h / kdiv;
            // the skip weight, loaded here so that its latency passes before epilogue B
            const float dh = D ? __ldg(&D[hk]) : 0.f;
            // ---- epilogue A: -> A operand of stage B (Ra columns 0..63)
            if (!wait(bar(sb.dA), pdA)) break;
            um::fence_after();
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int g = 2 * hf + gg;
                uint32_t re[16], im[16], o[16];
                load1(g, re, im);
                twiddle(g, re, im, o);
                um::st32x32_x16(tl + 16u * (uint32_t)g, o);
            }
            um::wait_st();
            arrive();
            // spectrum words of (h, k_p) for the thread's two groups: 8 Re pairs and 8
            // negated-Im pairs each, stored [h][group][word / 4][k_p] so that the 32
            // lanes of a warp read 512 contiguous bytes
            uint4 kv[8];
            {
                const uint4* kp = khat + (size_t)(hk * 4 + 2 * hf) * 4 * kP + r;
#pragma unroll
                for (int i = 0; i < 8; ++i) kv[i] = __ldg(&kp[i * kP]);
            }
            // ---- epilogue B: Z = conj(X (Khat + D/M)) -> A operand of stage C (Rb columns 0..63)
            if (!wait(bar(sb.dX), pdX)) break;
            um::fence_after();
            {
                const float dmf = dh * (1.0f / kM);
                const __nv_bfloat162 dm2 = __floats2bfloat162_rn(dmf, dmf);
#pragma unroll
                for (int gg = 0; gg < 2; ++gg) {
                    const int g = 2 * hf + gg;
                    uint32_t re[16], im[16], o[16];
                    um::ld32x32_x16(tl + 128u + 16u * (uint32_t)g, re);
                    um::ld32x32_x16(tl + 192u + 16u * (uint32_t)g, im);
                    um::wait_ld<16>(re);
                    um::wait_ld<16>(im);
                    const uint32_t* kw = reinterpret_cast<const uint32_t*>(kv + 4 * gg);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const __nv_bfloat162 xr =
                            tc::as_b2(tc::pack2(__uint_as_float(re[2 * i]), __uint_as_float(re[2 * i + 1])));
                        const __nv_bfloat162 xi =
                            tc::as_b2(tc::pack2(__uint_as_float(im[2 * i]), __uint_as_float(im[2 * i + 1])));
                        const __nv_bfloat162 kr = __hadd2(tc::as_b2(kw[i]), dm2), kin = tc::as_b2(kw[8 + i]);
                        // Re Z = xr kr - xi ki;  -Im Z = -(xr ki + xi kr) = xr kin - xi kr
                        o[i] = tc::as_u(__hfma2(xr, kr, __hmul2(xi, kin)));
                        o[8 + i] = tc::as_u(__hfma2(xr, kin, __hneg2(__hmul2(xi, kr))));
                    }
                    um::st32x32_x16(tl + 128u + 16u * (uint32_t)g, o);
                }
            }
            um::wait_st();
            arrive();

            // ---- epilogue C: V = V0 W_M^{q k_p} -> stage-D operand: rows k_p (Re), 128 + k_p (Im)
            if (!wait(bar(sb.dX), pdX)) break;
            um::fence_after();
            {
#pragma unroll
                for (int gg = 0; gg < 2; ++gg) {
                    const int g = 2 * hf + gg;
                    uint32_t re[16], im[16], o[16];
                    load1(g, re, im);
                    twiddle(g, re, im, o);
#pragma unroll
                    for (int c8 = 0; c8 < 2; ++c8) {
                        const int n = 16 * g + 8 * c8;
                        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(vs + mn_off(r, n, kVk, kVn)),
                                     "r"(o[4 * c8]), "r"(o[4 * c8 + 1]), "r"(o[4 * c8 + 2]), "r"(o[4 * c8 + 3])
                                     : "memory");
                        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(vs + mn_off(128 + r, n, kVk, kVn)),
                                     "r"(o[8 + 4 * c8]), "r"(o[9 + 4 * c8]), "r"(o[10 + 4 * c8]), "r"(o[11 + 4 * c8])
                                     : "memory");
                    }
                }
            }
            um::fence_proxy_async();
            arrive();
            // ---- epilogue D: lane p (Re, row b0) or 64 + p (Im, row b0 + 1), q = 32 hf ..
            // 32 hf + 31.  The warp's 32 half-rows go through its own 2 KiB of the
            // slot's V (free once D is complete), 16-byte chunks rotated by row, and
            // out as 64-byte runs
            if (!wait(bar(sb.dD), pdD)) break;
            um::fence_after();
            {
                uint32_t v[32];
                um::ld32x32_x32(tl + 128u + 32u * (uint32_t)hf, v);
                um::wait_ld<32>(v);
                const int plane = quarter >> 1, p0 = 32 * (quarter & 1);
                const uint32_t wbase = vs + (uint32_t)e * 2048u;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t* vv = v + 8 * c;
                    const uint32_t w0 = tc::pack2(__uint_as_float(vv[0]), __uint_as_float(vv[1]));
                    const uint32_t w1 = tc::pack2(__uint_as_float(vv[2]), __uint_as_float(vv[3]));
                    const uint32_t w2 = tc::pack2(__uint_as_float(vv[4]), __uint_as_float(vv[5]));
                    const uint32_t w3 = tc::pack2(__uint_as_float(vv[6]), __uint_as_float(vv[7]));
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(
                                     wbase + (uint32_t)lane * 64u + 16u * (uint32_t)(c ^ ((lane >> 1) & 3))),
                                 "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                                 : "memory");
                }
                __syncwarp();
                const int b = b0 + plane;
                if (b < B) {
                    __nv_bfloat16* dst = y + ((size_t)b * H + h) * kN + (size_t)kQ * p0 + 32 * hf;
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int rr = 8 * m + (lane >> 2), c = lane & 3;
                        uint4 val;
                        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                                     : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                                     : "r"(wbase + (uint32_t)rr * 64u + 16u * (uint32_t)(c ^ ((rr >> 1) & 3))));
                        *reinterpret_cast<uint4*>(dst + (size_t)kQ * rr + 8 * c) = val;
                    }
                }
                __syncwarp();
            }
            // Rb and V are rewritten by the next pair's stage B and epilogue C only
            // after its epilogue A, which every warp of the slot reaches after these reads
        }
    }
    // every wait above is bounded and the issuer has drained its products; if
    // even the drain gave up, TMEM stays allocated rather than freed under a
    // running product (the status word is set)
    um::fence_before();
    __syncthreads();
    if (warp == 0 && s_drained[0] && s_drained[1]) {
        um::fence_after();
        um::tmem_dealloc(tmem, 512);
    }
    if (tid == 0 && s_abort) atomicExch(err, 1);
}

}  // namespace t2

// ================================================================== host side
namespace {

uint16_t bf16_bits_t2(double x) {
    const float f = (float)x;
    uint32_t b;
    memcpy(&b, &f, 4);
    b += 0x7fffu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

void cs_t2(int64_t e, int64_t L, double* c, double* s) {
    int64_t r = e % L;
    if (r < 0) r += L;
    const double a = 2.0 * M_PI * (double)r / (double)L;
    *c = cos(a);
    *s = sin(a);
}

// byte offset of (row m, column k) in a K-major core-matrix image
size_t kmaj(int m, int k, size_t sm, size_t sk) {
    return (size_t)(m / 8) * sm + (size_t)(k / 8) * sk + (size_t)(m % 8) * 16 + (size_t)(k % 8) * 2;
}

// 32-bit table word (a local type keeps the vector's instantiation internal)
struct Word32 {
    uint32_t v;
};

void put16(std::vector<uint8_t>& img, size_t off, double v) {
    const uint16_t b = bf16_bits_t2(v);
    memcpy(&img[off], &b, 2);
}

}  // namespace

bool t2_supported(int log2M, int gated) { return log2M == 13 && !gated; }

// Constant tables of the two-stage kernel, appended to the plan's table
// block: [0] the shared-memory image of GP and FQ (96 KiB, bf16), [1] the
// twiddle pairs (cos, sin) of W_M^{q k_p} per (q pair, k_p).
bool t2_tables(std::vector<float2>& out, size_t off[2]) {
    using namespace t2;
    std::vector<uint8_t> img(kOffX, 0);
    // GP: row p < 64 = [cos | sin](2 pi p k_p / 128); row 64 + p = [sin | -cos]
    for (int m = 0; m < 128; ++m)
        for (int k = 0; k < 256; ++k) {
            const int p = m & 63, kp = k & 127;
            double c, s;
            cs_t2((int64_t)p * kp, kP, &c, &s);
            const double v = m < 64 ? (k < 128 ? c : s) : (k < 128 ? s : -c);
            put16(img, kOffGP + kmaj(m, k, kGPm, kGPk), v);
        }
    // FQ: column kk = 2 col + t of the TMEM A operand is (part, j) with
    // col = 16 g + w: w < 8 -> Re, j = 16 g + 2 w + t; else Im, j = 16 g + 2 (w - 8) + t
    for (int n = 0; n < 128; ++n)
        for (int kk = 0; kk < 128; ++kk) {
            const int col = kk / 2, t = kk % 2, g = col / 16, w = col % 16;
            const bool im = w >= 8;
            const int j = 16 * g + 2 * (w % 8) + t, co = n % 64;
            double c, s;
            cs_t2((int64_t)j * co, kQ, &c, &s);
            const double v = !im ? (n < 64 ? c : -s) : (n < 64 ? s : c);
            put16(img, kOffFQ + kmaj(n, kk, kFQn, kFQk), v);
        }
    if (out.size() % 2) out.push_back(make_float2(0.f, 0.f));
    off[0] = out.size();
    size_t base = out.size();
    out.resize(base + img.size() / sizeof(float2));
    memcpy(&out[base], img.data(), img.size());
    // twiddles: [q0 / 2][k_p] -> (bf16x2 cos(q0, q0 + 1), bf16x2 sin(...)), q0 = 32 half + 2 i
    off[1] = out.size();
    std::vector<Word32> tw;
    for (int hf = 0; hf < 2; ++hf)
        for (int i = 0; i < 16; ++i)
            for (int kp = 0; kp < kP; ++kp) {
                double c0, s0, c1, s1;
                const int q0 = 32 * hf + 2 * i;
                cs_t2((int64_t)q0 * kp, kM, &c0, &s0);
                cs_t2((int64_t)(q0 + 1) * kp, kM, &c1, &s1);
                tw.push_back(Word32{(uint32_t)bf16_bits_t2(c0) | ((uint32_t)bf16_bits_t2(c1) << 16)});
                tw.push_back(Word32{(uint32_t)bf16_bits_t2(s0) | ((uint32_t)bf16_bits_t2(s1) << 16)});
            }
    base = out.size();
    out.resize(base + tw.size() / 2);
    memcpy(&out[base], tw.data(), tw.size() * 4);
    return true;
}

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once through the runtime.
EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static bool looked = false;
    if (!looked) {
        looked = true;
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)f;
        cudaGetLastError();
    }
    return fn;
}

}  // namespace

cudaError_t launch_t2_fwd(const fftconv_plan_s& p, const void* u, const void* khat, const float* D, void* y,
                          cudaStream_t s) {
    auto kern = t2::fused_fwd_t2;
    static int sms = 0;
    if (sms == 0) {
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)t2::kSmemBytes);
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaGetLastError();
        if (sms <= 0) sms = 1;
    }
    // the 5-D view of u that the kernel's bulk copies read (layout in the kernel's notes)
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap xmap;
    const cuuint64_t dims[5] = {8, 8, 8, (cuuint64_t)p.B, (cuuint64_t)8 * (cuuint64_t)p.H};
    const cuuint64_t strides[4] = {128, 16, (cuuint64_t)p.H * t2::kN * 2, 1024};
    const cuuint32_t box[5] = {8, 8, 8, 2, 8}, es[5] = {1, 1, 1, 1, 1};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(u), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const int pairs = ((p.B + 1) / 2) * p.H;  // each CTA walks its pairs alternately on its two slots
    dim3 grid(pairs < sms ? pairs : sms);
    kern<<<grid, t2::kThreads, t2::kSmemBytes, s>>>((const uint4*)khat, D, (__nv_bfloat16*)y, p.t2_mats, p.t2_twid,
                                                    p.d_err, p.B, p.H, p.wait_limit, p.kdiv, xmap);
    return cudaGetLastError();
}

}  // namespace fftc
