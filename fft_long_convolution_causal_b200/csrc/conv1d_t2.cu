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
// no transposes and no shared-memory round trip between A, B and C.
//
// Roles (320 threads, one CTA per SM, all 512 TMEM columns):
//   warps 0-7  epilogues (warp e: TMEM lanes 32 (e % 4) .., column half e / 4)
//   warp 8     issues every MMA (one lane) and commits to mbarriers
//   warp 9     stages the input rows with cp.async
// A unit is two row pairs of one channel (slot 0 and slot 1, 256 TMEM
// columns each); while the epilogue warps work on one slot the tensor core
// runs the other slot's product.  Every wait is bounded; a wait that gives
// up stops the CTA, the issuer drains its products before TMEM is freed, and
// the plan's status word is set.
#include <cuda_bf16.h>
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
constexpr uint32_t kOffV = 131072;        // stage-D operand of the unit, [k 256][n 128] MN-major, 64 KiB
constexpr uint32_t kSmemBytes = 196608;

// core-matrix strides of each operand (bytes)
constexpr uint32_t kGPm = 4096, kGPk = 128;   // GP: row group (8 m) / column group (8 k)
constexpr uint32_t kFQn = 2048, kFQk = 128;   // FQ: 8 n / 8 k
constexpr uint32_t kXp = 2048, kXn = 128;     // X: 8 p / 8 n
constexpr uint32_t kVk = 2048, kVn = 128;     // V: 8 k / 8 n

constexpr int kEpiWarps = 8, kIssuer = 8, kLoader = 9, kThreads = 320;

struct Bars {
    uint64_t xfull[2], xempty[2], dA[2], dX[2], afull[2], dD, drain;
};

__device__ __forceinline__ uint32_t lanes(int quarter) { return (uint32_t)(32 * quarter) << 16; }

// byte offset of element (row k, column n) of an MN-major operand with row
// group stride rk and column group stride cn (rows = K, 16-byte core rows of 8 n)
__device__ __forceinline__ uint32_t mn_off(int k, int n, uint32_t rk, uint32_t cn) {
    return (uint32_t)(k >> 3) * rk + (uint32_t)(n >> 3) * cn + (uint32_t)(k & 7) * 16u + (uint32_t)(n & 7) * 2u;
}

__global__ void __launch_bounds__(kThreads, 1)
fused_fwd_t2(const __nv_bfloat16* __restrict__ u, const uint4* __restrict__ khat, const float* __restrict__ D,
             __nv_bfloat16* __restrict__ y, const uint4* __restrict__ mats, const uint2* __restrict__ twid,
             int* __restrict__ err, int B, int H, uint32_t wait_limit) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint32_t s_tmem;
    __shared__ __align__(8) Bars s_bar;
    __shared__ int s_drained;
    __shared__ volatile int s_abort;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t sbase = tc::smem_u32(smem);
    const int npp = (B + 1) / 2;            // row pairs per channel
    const int nu = (npp + 1) / 2;           // units per channel
    const int units = nu * H;
    auto bar = [&](const uint64_t& b) { return tc::smem_u32(&b); };

    // ---- set-up: constant matrices into shared memory, barriers, TMEM
    for (int i = tid; i < (int)(kOffX / 16); i += kThreads) {
        const uint4 val = __ldg(&mats[i]);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(sbase + 16u * i), "r"(val.x), "r"(val.y),
                     "r"(val.z), "r"(val.w)
                     : "memory");
    }
    um::fence_proxy_async();
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            um::mbar_init(bar(s_bar.xfull[s]), 1);
            um::mbar_init(bar(s_bar.xempty[s]), 1);
            um::mbar_init(bar(s_bar.dA[s]), 1);
            um::mbar_init(bar(s_bar.dX[s]), 1);
            um::mbar_init(bar(s_bar.afull[s]), kEpiWarps);
        }
        um::mbar_init(bar(s_bar.dD), 1);
        um::mbar_init(bar(s_bar.drain), 1);
        s_abort = 0;
        s_drained = 1;
    }
    if (warp == 0) {
        um::tmem_alloc(tc::smem_u32(&s_tmem), 512);
        um::tmem_relinquish();
    }
    um::fence_before();
    __syncthreads();
    um::fence_after();
    const uint32_t tmem = s_tmem;

    // a bounded wait; on give-up the CTA stops (every role polls the flag)
    auto wait = [&](uint32_t b, uint32_t& parity) -> bool {
        const bool ok = !s_abort && um::mbar_wait(b, parity, wait_limit);
        parity ^= 1u;
        if (!ok) s_abort = 1;
        return ok;
    };

    if (warp == kIssuer) {
        // ======================= MMA issuer
        if (lane == 0) {
            const uint32_t idA128 = um::idesc_bf16(128, 128) | um::kAmn | um::kBmn;
            const uint32_t idA64 = um::idesc_bf16(128, 64) | um::kAmn | um::kBmn;
            const uint32_t idBC = um::idesc_bf16(128, 128);
            const uint32_t idD = um::idesc_bf16(128, 128) | um::kBmn;
            uint32_t px[2] = {0u, 0u}, pa[2] = {0u, 0u};
            auto stage_a = [&](int s) -> bool {
                if (!wait(bar(s_bar.xfull[s]), px[s])) return false;
                um::fence_after();
                const uint32_t d = tmem + 256u * s, xs = sbase + kOffX + 16384u * s;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {  // cos view x [x_re | x_im]
                    const uint64_t a = um::sdesc(sbase + kOffGP + ks * 2 * kGPm, kGPm, kGPk);
                    um::mma_ss(d, a, um::sdesc(xs + ks * 2 * kXp, kXp, kXn), idA128, ks > 0);
                }
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {  // sin view: + sin x_im -> Re, - sin x_re -> Im
                    const uint64_t a = um::sdesc(sbase + kOffGP + 2048u + ks * 2 * kGPm, kGPm, kGPk);
                    um::mma_ss(d, a, um::sdesc(xs + 1024u + ks * 2 * kXp, kXp, kXn), idA64, 1);
                    um::mma_ss(d + 64u, a, um::sdesc(xs + ks * 2 * kXp, kXp, kXn), idA64 | um::kNegA, 1);
                }
                um::mma_commit(bar(s_bar.dA[s]));
                um::mma_commit(bar(s_bar.xempty[s]));
                return true;
            };
            // B (src Ra -> dst Rb) or C (Rb -> Ra) of slot s
            auto stage_bc = [&](int s, bool isC) -> bool {
                if (!wait(bar(s_bar.afull[s]), pa[s])) return false;
                um::fence_after();
                const uint32_t base = tmem + 256u * s;
                const uint32_t src = base + (isC ? 128u : 0u), dst = base + (isC ? 0u : 128u);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    um::mma_ts(dst, src + 8u * ks, um::sdesc(sbase + kOffFQ + ks * 2 * kFQk, kFQk, kFQn), idBC, ks > 0);
                um::mma_commit(bar(s_bar.dX[s]));
                return true;
            };
            bool ok = true;
            int i = 0;
            for (int un = blockIdx.x; un < units && ok; un += gridDim.x, ++i) {
                const bool two = 2 * (un % nu) + 1 < npp;
                if (i == 0) {
                    ok = stage_a(0) && (!two || stage_a(1));
                    if (!ok) break;
                }
                ok = stage_bc(0, false) && (!two || stage_bc(1, false)) && stage_bc(0, true) &&
                     (!two || stage_bc(1, true));
                if (!ok) break;
                // D: both pairs of the unit side by side (N = 128), into slot 0's Rb
                ok = wait(bar(s_bar.afull[0]), pa[0]) && (!two || wait(bar(s_bar.afull[1]), pa[1]));
                if (!ok) break;
                um::fence_after();
#pragma unroll
                for (int ks = 0; ks < 16; ++ks)
                    um::mma_ss(tmem + 128u, um::sdesc(sbase + kOffGP + ks * 2 * kGPk, kGPk, kGPm),
                               um::sdesc(sbase + kOffV + ks * 2 * kVk, kVk, kVn), idD, ks > 0);
                um::mma_commit(bar(s_bar.dD));
                // the next unit's stage A (its rows are staged by now or soon)
                const int nx = un + gridDim.x;
                if (nx < units) {
                    const bool two2 = 2 * (nx % nu) + 1 < npp;
                    ok = stage_a(0) && (!two2 || stage_a(1));
                }
            }
            // drain: every product issued is complete before TMEM is freed
            um::mma_commit(bar(s_bar.drain));
            s_drained = um::mbar_wait(bar(s_bar.drain), 0u) ? 1 : 0;
            if (!ok || !s_drained) atomicExch(err, 1);
        }
        __syncwarp();
    } else if (warp == kLoader) {
        // ======================= input rows of a unit into the two slots' planes
        uint32_t pe[2] = {1u, 1u};  // a fresh barrier's previous phase counts as complete
        for (int un = blockIdx.x; un < units; un += gridDim.x) {
            const int h = un / nu, pp0 = 2 * (un % nu);
            const bool two = pp0 + 1 < npp;
            bool ok = true;
            for (int s = 0; s < (two ? 2 : 1) && ok; ++s) ok = wait(bar(s_bar.xempty[s]), pe[s]);
            if (!ok) break;
            for (int s = 0; s < (two ? 2 : 1); ++s) {
                const int b0 = 2 * (pp0 + s);
                const uint32_t xs = sbase + kOffX + 16384u * s;
#pragma unroll 4
                for (int it = 0; it < 32; ++it) {
                    // lane -> (p mod 8, 8-q chunk): 64-byte global runs, 8 bank groups per store
                    const int plane = it >> 4, pg = (it >> 1) & 7, qc = (lane >> 3) + 4 * (it & 1);
                    const int p = 8 * pg + (lane & 7);
                    const int b = b0 + plane;
                    const bool has = b < B;
                    const size_t off = ((size_t)(has ? b : b0) * H + h) * kN + (size_t)(kQ * p + 8 * qc);
                    tc::cp_async16(xs + mn_off(p, 64 * plane + 8 * qc, kXp, kXn), u + off, has ? 16 : 0);
                }
            }
            tc::cp_async_commit();
            tc::cp_async_wait_all();
            um::fence_proxy_async();
            __syncwarp();
            if (lane == 0)
                for (int s = 0; s < (two ? 2 : 1); ++s) um::mbar_arrive(bar(s_bar.xfull[s]));
        }
        tc::cp_async_wait_all();
    } else {
        // ======================= epilogue warps
        const int quarter = warp & 3, ch = warp >> 2;
        const int r = 32 * quarter + lane;  // TMEM lane: k_p in stages A-C
        const uint32_t tl = tmem + lanes(quarter);
        uint2 tw[16];  // (cos, sin) pairs of W_M^{q k_p}, q = 32 ch + 2 i, + 1
#pragma unroll
        for (int i = 0; i < 16; ++i) tw[i] = __ldg(&twid[(r * 2 + ch) * 16 + i]);
        uint32_t pdA[2] = {0u, 0u}, pdX[2] = {0u, 0u}, pdD = 0u;
        auto arrive = [&](int s) {
            um::fence_before();
            __syncwarp();
            if (lane == 0) um::mbar_arrive(bar(s_bar.afull[s]));
        };
        // read this thread's 32 Re and 32 Im accumulators of the half ch at column col
        auto load = [&](uint32_t col, uint32_t (&re)[32], uint32_t (&im)[32]) {
            um::ld32x32_x32(tl + col + 32u * ch, re);
            um::ld32x32_x32(tl + col + 64u + 32u * ch, im);
            um::wait_ld<32>(re);
            um::wait_ld<32>(im);
        };
        // the next stage's A operand, in this thread's own columns: Re pairs then Im pairs
        auto store_a = [&](uint32_t col, const uint32_t (&ar)[16], const uint32_t (&ai)[16]) {
            um::st32x32_x16(tl + col + 32u * ch, ar);
            um::st32x32_x16(tl + col + 32u * ch + 16u, ai);
            um::wait_st();
        };
        for (int un = blockIdx.x; un < units; un += gridDim.x) {
            const int h = un / nu, pp0 = 2 * (un % nu);
            const bool two = pp0 + 1 < npp;
            const int ns = two ? 2 : 1;
            bool ok = true;
            // spectrum words of (h, k_p, half): 16 Re pairs, 16 negated-Im pairs
            uint4 kv[8];
            const uint4* kp = khat + ((size_t)(h * kP + r) * 2 + ch) * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) kv[i] = __ldg(&kp[i]);
            const float dmf = D ? D[h] * (1.0f / kM) : 0.f;
            const __nv_bfloat162 dm2 = __floats2bfloat162_rn(dmf, dmf);
            // ---- epilogue A: x W_M^{q k_p} -> A operand of stage B (slot columns 0..63)
            for (int s = 0; s < ns && ok; ++s) {
                if (!(ok = wait(bar(s_bar.dA[s]), pdA[s]))) break;
                um::fence_after();
                uint32_t re[32], im[32], ar[16], ai[16];
                load(256u * s, re, im);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    ar[i] = tc::pack2(__uint_as_float(re[2 * i]), __uint_as_float(re[2 * i + 1]));
                    ai[i] = tc::pack2(__uint_as_float(im[2 * i]), __uint_as_float(im[2 * i + 1]));
                    tc::twiddle2<true>(ar[i], ai[i], tw[i]);
                }
                store_a(256u * s, ar, ai);
                arrive(s);
            }
            if (!ok) break;
            // ---- epilogue B: Z = conj(X (Khat + D/M)) -> A operand of stage C (columns 128..191)
            for (int s = 0; s < ns && ok; ++s) {
                if (!(ok = wait(bar(s_bar.dX[s]), pdX[s]))) break;
                um::fence_after();
                uint32_t re[32], im[32], ar[16], ai[16];
                load(256u * s + 128u, re, im);
                const uint32_t* kw = reinterpret_cast<const uint32_t*>(kv);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const __nv_bfloat162 xr = tc::as_b2(tc::pack2(__uint_as_float(re[2 * i]), __uint_as_float(re[2 * i + 1])));
                    const __nv_bfloat162 xi = tc::as_b2(tc::pack2(__uint_as_float(im[2 * i]), __uint_as_float(im[2 * i + 1])));
                    const __nv_bfloat162 kr = __hadd2(tc::as_b2(kw[i]), dm2), kin = tc::as_b2(kw[16 + i]);
                    // Re Z = xr kr - xi ki;  -Im Z = -(xr ki + xi kr) = xr kin - xi kr
                    ar[i] = tc::as_u(__hfma2(xr, kr, __hmul2(xi, kin)));
                    ai[i] = tc::as_u(__hfma2(xr, kin, __hneg2(__hmul2(xi, kr))));
                }
                store_a(256u * s + 128u, ar, ai);
                arrive(s);
            }
            if (!ok) break;
            // ---- epilogue C: V = V0 W_M^{q k_p} -> stage-D operand in shared memory
            for (int s = 0; s < ns && ok; ++s) {
                if (!(ok = wait(bar(s_bar.dX[s]), pdX[s]))) break;
                um::fence_after();
                uint32_t re[32], im[32], vr[16], vi[16];
                load(256u * s, re, im);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    vr[i] = tc::pack2(__uint_as_float(re[2 * i]), __uint_as_float(re[2 * i + 1]));
                    vi[i] = tc::pack2(__uint_as_float(im[2 * i]), __uint_as_float(im[2 * i + 1]));
                    tc::twiddle2<true>(vr[i], vi[i], tw[i]);
                }
                // rows k = k_p (Re) and 128 + k_p (Im), columns n = 64 s + q
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    const int n = 64 * s + 32 * ch + 8 * c8;
                    const uint32_t ar = sbase + kOffV + mn_off(r, n, kVk, kVn);
                    const uint32_t ai = sbase + kOffV + mn_off(128 + r, n, kVk, kVn);
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(ar), "r"(vr[4 * c8]),
                                 "r"(vr[4 * c8 + 1]), "r"(vr[4 * c8 + 2]), "r"(vr[4 * c8 + 3])
                                 : "memory");
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(ai), "r"(vi[4 * c8]),
                                 "r"(vi[4 * c8 + 1]), "r"(vi[4 * c8 + 2]), "r"(vi[4 * c8 + 3])
                                 : "memory");
                }
                um::fence_proxy_async();
                arrive(s);
            }
            if (!ok) break;
            // ---- epilogue D: rows p (Re, lanes 0..63) and 64 + p (Im) of pair ch, q = 0..63
            if (!(ok = wait(bar(s_bar.dD), pdD))) break;
            um::fence_after();
            {
                uint32_t v0[32], v1[32];
                um::ld32x32_x32(tl + 128u + 64u * ch, v0);
                um::ld32x32_x32(tl + 128u + 64u * ch + 32u, v1);
                um::wait_ld<32>(v0);
                um::wait_ld<32>(v1);
                const int b = 2 * (pp0 + ch) + (quarter >> 1);
                if (ch < ns && b < B) {
                    const int p = r & 63;
                    uint4* dst = reinterpret_cast<uint4*>(y + ((size_t)b * H + h) * kN + (size_t)kQ * p);
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        uint4 o;
                        o.x = tc::pack2(__uint_as_float(v0[8 * c8]), __uint_as_float(v0[8 * c8 + 1]));
                        o.y = tc::pack2(__uint_as_float(v0[8 * c8 + 2]), __uint_as_float(v0[8 * c8 + 3]));
                        o.z = tc::pack2(__uint_as_float(v0[8 * c8 + 4]), __uint_as_float(v0[8 * c8 + 5]));
                        o.w = tc::pack2(__uint_as_float(v0[8 * c8 + 6]), __uint_as_float(v0[8 * c8 + 7]));
                        dst[c8] = o;
                    }
#pragma unroll
                    for (int c8 = 0; c8 < 4; ++c8) {
                        uint4 o;
                        o.x = tc::pack2(__uint_as_float(v1[8 * c8]), __uint_as_float(v1[8 * c8 + 1]));
                        o.y = tc::pack2(__uint_as_float(v1[8 * c8 + 2]), __uint_as_float(v1[8 * c8 + 3]));
                        o.z = tc::pack2(__uint_as_float(v1[8 * c8 + 4]), __uint_as_float(v1[8 * c8 + 5]));
                        o.w = tc::pack2(__uint_as_float(v1[8 * c8 + 6]), __uint_as_float(v1[8 * c8 + 7]));
                        dst[4 + c8] = o;
                    }
                }
            }
            // Rb of slot 0 is rewritten by the next unit's stage B only after that
            // unit's epilogue A, which this warp reaches after these reads
            um::fence_before();
        }
    }
    // every wait above is bounded and the issuer has drained its products; if
    // even the drain gave up, TMEM stays allocated rather than freed under a
    // running product (the status word is set)
    um::fence_before();
    __syncthreads();
    if (warp == 0 && s_drained) {
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
// twiddle pairs (cos, sin) of W_M^{q k_p} per (k_p, half, q pair).
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
    // col = 32 hh + w: w < 16 -> Re, j = 32 hh + 2 w + t; else Im, j = 32 hh + 2 (w - 16) + t
    for (int n = 0; n < 128; ++n)
        for (int kk = 0; kk < 128; ++kk) {
            const int col = kk / 2, t = kk % 2, hh = col / 32, w = col % 32;
            const bool im = w >= 16;
            const int j = 32 * hh + 2 * (w % 16) + t, co = n % 64;
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
    // twiddles: [k_p][half][i] -> (bf16x2 cos(q0, q0 + 1), bf16x2 sin(...)), q0 = 32 half + 2 i
    off[1] = out.size();
    std::vector<Word32> tw;
    for (int kp = 0; kp < kP; ++kp)
        for (int hf = 0; hf < 2; ++hf)
            for (int i = 0; i < 16; ++i) {
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
    const int npp = (p.B + 1) / 2, units = ((npp + 1) / 2) * p.H;
    dim3 grid(units < sms ? units : sms);
    kern<<<grid, t2::kThreads, t2::kSmemBytes, s>>>((const __nv_bfloat16*)u, (const uint4*)khat, D,
                                                    (__nv_bfloat16*)y, p.t2_mats, p.t2_twid, p.d_err, p.B, p.H,
                                                    p.wait_limit);
    return cudaGetLastError();
}

}  // namespace fftc
