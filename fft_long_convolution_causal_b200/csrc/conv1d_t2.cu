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
// Roles (384 threads, one CTA per SM, all 512 TMEM columns): two
// independent pipelines ("slots", 256 TMEM columns and their own shared
// memory each), every slot with
//   4 epilogue warps (warp e: TMEM lanes 32 (e % 4) .., both column halves),
//   1 warp that issues its MMAs (one lane) and commits to its mbarriers,
//   1 warp that stages its input rows with cp.async,
// working through its own sequence of row pairs, so while one slot's warps
// run an epilogue the tensor core runs the other slot's product.  Every wait
// is bounded; a wait that gives up stops the CTA, each issuer drains its
// products before TMEM is freed, and the plan's status word is set.
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
constexpr uint32_t kOffV = 131072;        // stage-D operand of slot s at + 32 KiB s: [k 256][n 64] MN-major
constexpr uint32_t kOffTW = 196608;       // twiddle pairs of W_M^{q k_p}: [half 2][i 16][k_p 128] uint2, 32 KiB
constexpr uint32_t kSmemBytes = 229376;

// core-matrix strides of each operand (bytes)
constexpr uint32_t kGPm = 4096, kGPk = 128;   // GP: row group (8 m) / column group (8 k)
constexpr uint32_t kFQn = 2048, kFQk = 128;   // FQ: 8 n / 8 k
constexpr uint32_t kXp = 2048, kXn = 128;     // X: 8 p / 8 n
constexpr uint32_t kVk = 1024, kVn = 128;     // V: 8 k / 8 n

// roles: warps 4 s .. 4 s + 3 epilogues of slot s, warp 8 + s its MMA issuer,
// warp 10 + s its loader
constexpr int kGroupWarps = 4, kThreads = 384;

struct SlotBars {
    uint64_t xfull, xempty, dA, dX, dD, afull, drain;
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

__global__ void __launch_bounds__(kThreads, 1)
fused_fwd_t2(const __nv_bfloat16* __restrict__ u, const uint4* __restrict__ khat, const float* __restrict__ D,
             __nv_bfloat16* __restrict__ y, const uint4* __restrict__ mats, const uint2* __restrict__ twid,
             int* __restrict__ err, int B, int H, uint32_t wait_limit) {
    extern __shared__ __align__(1024) uint8_t smem[];
    __shared__ uint32_t s_tmem;
    __shared__ __align__(8) SlotBars s_bar[2];
    __shared__ int s_drained[2];
    __shared__ volatile int s_abort;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t sbase = tc::smem_u32(smem);
    const int npp = (B + 1) / 2;   // row pairs per channel
    const int pairs = npp * H;
    auto bar = [&](const uint64_t& b) { return tc::smem_u32(&b); };

    // ---- set-up: constant matrices into shared memory (all copies in flight at
    // once), barriers, TMEM
    for (int i = tid; i < (int)(kOffX / 16); i += kThreads) tc::cp_async16(sbase + 16u * i, mats + i, 16);
    for (int i = tid; i < 2048; i += kThreads)
        tc::cp_async16(sbase + kOffTW + 16u * i, reinterpret_cast<const uint4*>(twid) + i, 16);
    tc::cp_async_commit();
    tc::cp_async_wait_all();
    um::fence_proxy_async();
    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            um::mbar_init(bar(s_bar[s].xfull), 1);
            um::mbar_init(bar(s_bar[s].xempty), 1);
            um::mbar_init(bar(s_bar[s].dA), 1);
            um::mbar_init(bar(s_bar[s].dX), 1);
            um::mbar_init(bar(s_bar[s].dD), 1);
            um::mbar_init(bar(s_bar[s].afull), kGroupWarps);
            um::mbar_init(bar(s_bar[s].drain), 1);
            s_drained[s] = 1;
        }
        s_abort = 0;
    }
    if (warp == 0) {
        um::tmem_alloc(tc::smem_u32(&s_tmem), 512);
        um::tmem_relinquish();
    }
    um::fence_before();
    __syncthreads();
    um::fence_after();
    const uint32_t tmem = s_tmem;

    // a bounded wait on barrier b with the expected phase parity in *par; on
    // give-up the CTA stops (every role polls the flag)
    auto wait = [&](uint32_t b, uint32_t& par) -> bool {
        const bool ok = !s_abort && um::mbar_wait(b, par, wait_limit);
        par ^= 1u;
        if (!ok) s_abort = 1;
        return ok;
    };
    // the pairs of slot s: q = blockIdx.x + (2 i + s) gridDim.x
    const int slot = warp < 8 ? (warp >> 2) : (warp < 10 ? warp - 8 : warp - 10);
    const int q0 = blockIdx.x + slot * (int)gridDim.x, qstep = 2 * (int)gridDim.x;
    SlotBars& sb = s_bar[slot];
    const uint32_t tslot = tmem + 256u * (uint32_t)slot;           // Ra = + 0, Rb = + 128
    const uint32_t xs = sbase + kOffX + 16384u * (uint32_t)slot;
    const uint32_t vs = sbase + kOffV + 32768u * (uint32_t)slot;

    if (warp >= 8 && warp < 10) {
        // ======================= MMA issuer of slot s
        if (lane == 0) {
            const uint32_t idA128 = um::idesc_bf16(128, 128) | um::kAmn | um::kBmn;
            const uint32_t idA64 = um::idesc_bf16(128, 64) | um::kAmn | um::kBmn;
            const uint32_t idBC = um::idesc_bf16(128, 128);
            const uint32_t idD = um::idesc_bf16(128, 64) | um::kBmn;
            const uint64_t gpA = um::sdesc(sbase + kOffGP, kGPm, kGPk);   // MN-major view for stage A
            const uint64_t gpD = um::sdesc(sbase + kOffGP, kGPk, kGPm);   // K-major for stage D
            const uint64_t xd = um::sdesc(xs, kXp, kXn);
            const uint64_t fq = um::sdesc(sbase + kOffFQ, kFQk, kFQn);
            const uint64_t vd = um::sdesc(vs, kVk, kVn);
            uint32_t px = 0u, pa = 0u;
            auto stage_a = [&]() -> bool {
                if (!wait(bar(sb.xfull), px)) return false;
                um::fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)  // cos view x [x_re | x_im]
                    um::mma_ss(tslot, dadd(gpA, ks * 2 * kGPm), dadd(xd, ks * 2 * kXp), idA128, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {  // sin view: + sin x_im -> Re, - sin x_re -> Im
                    const uint64_t a = dadd(gpA, 2048u + ks * 2 * kGPm);
                    um::mma_ss(tslot, a, dadd(xd, 1024u + ks * 2 * kXp), idA64, 1);
                    um::mma_ss(tslot + 64u, a, dadd(xd, ks * 2 * kXp), idA64 | um::kNegA, 1);
                }
                um::mma_commit(bar(sb.dA));
                um::mma_commit(bar(sb.xempty));
                return true;
            };
            // B (Ra -> Rb) or C (Rb -> Ra), once the epilogue has written the operand
            auto stage_bc = [&](bool isC) -> bool {
                if (!wait(bar(sb.afull), pa)) return false;
                um::fence_after();
                const uint32_t src = tslot + (isC ? 128u : 0u), dst = tslot + (isC ? 0u : 128u);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) um::mma_ts(dst, src + 8u * ks, dadd(fq, ks * 2 * kFQk), idBC, ks > 0);
                um::mma_commit(bar(sb.dX));
                return true;
            };
            bool ok = true;
            for (int q = q0; q < pairs && ok; q += qstep) {
                if (q == q0 && !(ok = stage_a())) break;
                if (!(ok = stage_bc(false) && stage_bc(true))) break;
                // D once epilogue C has filled V: rows p (Re) and 64 + p (Im), N = 64 q, into Rb
                if (!(ok = wait(bar(sb.afull), pa))) break;
                um::fence_after();
#pragma unroll
                for (int ks = 0; ks < 16; ++ks)
                    um::mma_ss(tslot + 128u, dadd(gpD, ks * 2 * kGPk), dadd(vd, ks * 2 * kVk), idD, ks > 0);
                um::mma_commit(bar(sb.dD));
                // the next pair's stage A (Ra is free: epilogue C has read it)
                if (q + qstep < pairs && !(ok = stage_a())) break;
            }
            // drain: every product issued is complete before TMEM is freed
            um::mma_commit(bar(sb.drain));
            s_drained[slot] = um::mbar_wait(bar(sb.drain), 0u) ? 1 : 0;
            if (!ok || !s_drained[slot]) atomicExch(err, 1);
        }
        __syncwarp();
    } else if (warp >= 10) {
        // ======================= input rows of slot s's pairs
        uint32_t pe = 1u;  // a fresh barrier's previous phase counts as complete
        for (int q = q0; q < pairs; q += qstep) {
            if (!wait(bar(sb.xempty), pe)) break;
            const int h = q / npp, b0 = 2 * (q % npp);
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
            tc::cp_async_commit();
            tc::cp_async_wait_all();
            um::fence_proxy_async();
            __syncwarp();
            if (lane == 0) um::mbar_arrive(bar(sb.xfull));
        }
        tc::cp_async_wait_all();
    } else {
        // ======================= epilogue warps of slot s: TMEM lanes 32 quarter .., both column halves
        const int quarter = warp & 3;
        const int r = 32 * quarter + lane;  // TMEM lane: k_p in stages A-C
        const uint32_t tl = tslot + lanes(quarter);
        uint32_t pdA = 0u, pdX = 0u, pdD = 0u;
        auto arrive = [&]() {
            um::fence_before();
            __syncwarp();
            if (lane == 0) um::mbar_arrive(bar(sb.afull));
        };
        // this thread's 32 Re and 32 Im accumulators of column half hf at column col
        auto load = [&](uint32_t col, int hf, uint32_t (&re)[32], uint32_t (&im)[32]) {
            um::ld32x32_x32(tl + col + 32u * hf, re);
            um::ld32x32_x32(tl + col + 64u + 32u * hf, im);
            um::wait_ld<32>(re);
            um::wait_ld<32>(im);
        };
        // the next stage's A operand in the thread's own columns: Re pairs then Im pairs
        auto store_a = [&](uint32_t col, int hf, const uint32_t (&ar)[16], const uint32_t (&ai)[16]) {
            um::st32x32_x16(tl + col + 32u * hf, ar);
            um::st32x32_x16(tl + col + 32u * hf + 16u, ai);
        };
        // twiddles from shared memory: consecutive lanes read consecutive 8-byte words
        auto fetch_tw = [&](int hf, uint2 (&tw)[16]) {
            const uint32_t t = sbase + kOffTW + (uint32_t)((hf * 16) * 128 + r) * 8u;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];\n"
                             : "=r"(tw[i].x), "=r"(tw[i].y)
                             : "r"(t + (uint32_t)i * 1024u));
        };
        // epilogue A / C: x W_M^{q k_p} on packed pairs
        auto twiddle_half = [&](uint32_t col, int hf, uint32_t (&ar)[16], uint32_t (&ai)[16]) {
            uint2 tw[16];
            fetch_tw(hf, tw);
            uint32_t re[32], im[32];
            load(col, hf, re, im);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                ar[i] = tc::pack2(__uint_as_float(re[2 * i]), __uint_as_float(re[2 * i + 1]));
                ai[i] = tc::pack2(__uint_as_float(im[2 * i]), __uint_as_float(im[2 * i + 1]));
                tc::twiddle2<true>(ar[i], ai[i], tw[i]);
            }
        };
        for (int q = q0; q < pairs; q += qstep) {
            const int h = q / npp, b0 = 2 * (q % npp);
            bool ok = true;
            // spectrum words of (h, k_p): per half 16 Re pairs and 16 negated-Im pairs
            uint4 kv[16];
            {
                const uint4* kp = khat + (size_t)(h * kP + r) * 16;
#pragma unroll
                for (int i = 0; i < 16; ++i) kv[i] = __ldg(&kp[i]);
            }
            const float dmf = D ? __ldg(&D[h]) * (1.0f / kM) : 0.f;
            // ---- epilogue A: -> A operand of stage B (Ra columns 0..63)
            if (!(ok = wait(bar(sb.dA), pdA))) break;
            um::fence_after();
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t ar[16], ai[16];
                twiddle_half(0u, hf, ar, ai);
                store_a(0u, hf, ar, ai);
            }
            um::wait_st();
            arrive();
            // ---- epilogue B: Z = conj(X (Khat + D/M)) -> A operand of stage C (Rb columns 0..63)
            if (!(ok = wait(bar(sb.dX), pdX))) break;
            um::fence_after();
            {
                const __nv_bfloat162 dm2 = __floats2bfloat162_rn(dmf, dmf);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t re[32], im[32], ar[16], ai[16];
                    load(128u, hf, re, im);
                    const uint32_t* kw = reinterpret_cast<const uint32_t*>(kv + 8 * hf);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const __nv_bfloat162 xr =
                            tc::as_b2(tc::pack2(__uint_as_float(re[2 * i]), __uint_as_float(re[2 * i + 1])));
                        const __nv_bfloat162 xi =
                            tc::as_b2(tc::pack2(__uint_as_float(im[2 * i]), __uint_as_float(im[2 * i + 1])));
                        const __nv_bfloat162 kr = __hadd2(tc::as_b2(kw[i]), dm2), kin = tc::as_b2(kw[16 + i]);
                        // Re Z = xr kr - xi ki;  -Im Z = -(xr ki + xi kr) = xr kin - xi kr
                        ar[i] = tc::as_u(__hfma2(xr, kr, __hmul2(xi, kin)));
                        ai[i] = tc::as_u(__hfma2(xr, kin, __hneg2(__hmul2(xi, kr))));
                    }
                    store_a(128u, hf, ar, ai);
                }
            }
            um::wait_st();
            arrive();
            // ---- epilogue C: V = V0 W_M^{q k_p} -> stage-D operand: rows k_p (Re), 128 + k_p (Im)
            if (!(ok = wait(bar(sb.dX), pdX))) break;
            um::fence_after();
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t vr[16], vi[16];
                twiddle_half(0u, hf, vr, vi);
#pragma unroll
                for (int c8 = 0; c8 < 4; ++c8) {
                    const int n = 32 * hf + 8 * c8;
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(vs + mn_off(r, n, kVk, kVn)),
                                 "r"(vr[4 * c8]), "r"(vr[4 * c8 + 1]), "r"(vr[4 * c8 + 2]), "r"(vr[4 * c8 + 3])
                                 : "memory");
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(vs + mn_off(128 + r, n, kVk, kVn)),
                                 "r"(vi[4 * c8]), "r"(vi[4 * c8 + 1]), "r"(vi[4 * c8 + 2]), "r"(vi[4 * c8 + 3])
                                 : "memory");
                }
            }
            um::fence_proxy_async();
            arrive();
            // ---- epilogue D: lane p (Re, row b0) or 64 + p (Im, row b0 + 1), q = 0..63.  The
            // warp's 32 rows (contiguous in y) are staged in its own 4 KiB of the slot's V
            // (free once D is complete), 16-byte chunks swizzled by row, then written out
            // in whole 512-byte runs
            if (!(ok = wait(bar(sb.dD), pdD))) break;
            um::fence_after();
            {
                uint32_t v0[32], v1[32];
                um::ld32x32_x32(tl + 128u, v0);
                um::ld32x32_x32(tl + 160u, v1);
                um::wait_ld<32>(v0);
                um::wait_ld<32>(v1);
                const int plane = quarter >> 1, p0 = 32 * (quarter & 1);
                const uint32_t wbase = vs + (uint32_t)quarter * 4096u;
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    const uint32_t* vv = c8 < 4 ? v0 + 8 * c8 : v1 + 8 * (c8 - 4);
                    const uint32_t w0 = tc::pack2(__uint_as_float(vv[0]), __uint_as_float(vv[1]));
                    const uint32_t w1 = tc::pack2(__uint_as_float(vv[2]), __uint_as_float(vv[3]));
                    const uint32_t w2 = tc::pack2(__uint_as_float(vv[4]), __uint_as_float(vv[5]));
                    const uint32_t w3 = tc::pack2(__uint_as_float(vv[6]), __uint_as_float(vv[7]));
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(
                                     wbase + (uint32_t)lane * 128u + 16u * (uint32_t)(c8 ^ (lane & 7))),
                                 "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                                 : "memory");
                }
                __syncwarp();
                const int b = b0 + plane;
                if (b < B) {
                    __nv_bfloat16* dst = y + ((size_t)b * H + h) * kN + (size_t)kQ * p0;
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const int j = lane + 32 * m, rr = j >> 3, c = j & 7;
                        uint4 val;
                        asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                                     : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                                     : "r"(wbase + (uint32_t)rr * 128u + 16u * (uint32_t)(c ^ (rr & 7))));
                        *reinterpret_cast<uint4*>(dst + (size_t)kQ * rr + 8 * c) = val;
                    }
                }
                __syncwarp();
            }
            // Rb and V are rewritten by the next pair's stage B and epilogue C only
            // after its epilogue A, which every warp of the group reaches after these reads
        }
    }
    // every wait above is bounded and the issuers have drained their products;
    // if even a drain gave up, TMEM stays allocated rather than freed under a
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
    // twiddles: [half][i][k_p] -> (bf16x2 cos(q0, q0 + 1), bf16x2 sin(...)), q0 = 32 half + 2 i
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
    const int pairs = ((p.B + 1) / 2) * p.H;  // each CTA walks its pairs alternately on its two slots
    dim3 grid(pairs < sms ? pairs : sms);
    kern<<<grid, t2::kThreads, t2::kSmemBytes, s>>>((const __nv_bfloat16*)u, (const uint4*)khat, D,
                                                    (__nv_bfloat16*)y, p.t2_mats, p.t2_twid, p.d_err, p.B, p.H,
                                                    p.wait_limit);
    return cudaGetLastError();
}

}  // namespace fftc
