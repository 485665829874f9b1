// tc_common.cuh -- device helpers shared by the bf16 tensor-core kernels: PTX
// wrappers (mma.sync, ldmatrix / stmatrix, movmatrix), packed bf16 complex
// arithmetic, the swizzled shared-memory planes and fragment utilities.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "fft_simt.cuh"
#include "plan.h"

namespace fftc {
namespace tc {


// ------------------------------------------------------------ PTX wrappers
// Register-only operations (mma, movmatrix) are not volatile, so the compiler
// may interleave independent ones; shared-memory ones keep their order.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// d = A B (zero accumulator: C is the zero register, no moves to clear d)
__device__ __forceinline__ void mma16816z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void stsm_x4_t(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(r0),
                 "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}
__device__ __forceinline__ uint32_t movt(uint32_t x) {
    uint32_t y;
    asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
    return y;
}
// two fp32 -> packed bf16x2 (lo in the low half).  IP = false: the
// conversion instruction, round to nearest even.  IP = true: round to nearest
// (ties away from zero) with integer arithmetic -- adding half an ulp of bf16
// (0x8000) to the fp32 bit pattern carries into the kept upper 16 bits exactly
// when the dropped bits are at least half, and a byte permute takes the two
// upper halves.  The integer form runs on the ALU instead of the conversion
// unit; which is faster depends on the kernel's mix (measured per size).
// Inputs are finite and far below FLT_MAX, so the carry never overflows.
template <bool IP = false>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    uint32_t r;
    if (IP) {
        const uint32_t a = __float_as_uint(lo) + 0x8000u, b = __float_as_uint(hi) + 0x8000u;
        asm("prmt.b32 %0, %1, %2, 0x7632;\n" : "=r"(r) : "r"(a), "r"(b));
    } else {
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
    }
    return r;
}
__device__ __forceinline__ __nv_bfloat162 as_b2(uint32_t x) { return *reinterpret_cast<__nv_bfloat162*>(&x); }
__device__ __forceinline__ uint32_t as_u(__nv_bfloat162 x) { return *reinterpret_cast<uint32_t*>(&x); }
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Packed complex multiply on two adjacent elements: (re, im) pairs times
// (cos, sin) pairs.  FWD: z (c - i s);  otherwise z (c + i s).
template <bool FWD>
__device__ __forceinline__ void twiddle2(uint32_t& re, uint32_t& im, uint2 cs) {
    const __nv_bfloat162 r = as_b2(re), i = as_b2(im), c = as_b2(cs.x), s = as_b2(cs.y);
    if (FWD) {
        re = as_u(__hfma2(r, c, __hmul2(i, s)));
        im = as_u(__hfma2(i, c, __hneg2(__hmul2(r, s))));
    } else {
        re = as_u(__hfma2(r, c, __hneg2(__hmul2(i, s))));
        im = as_u(__hfma2(i, c, __hmul2(r, s)));
    }
}

// As twiddle2 with the negated sine ns = -s at hand: two products and two
// fused multiply-adds, no negation.
template <bool FWD>
__device__ __forceinline__ void twiddle2n(uint32_t& re, uint32_t& im, uint2 cs, uint32_t ns) {
    const __nv_bfloat162 r = as_b2(re), i = as_b2(im), c = as_b2(cs.x), s = as_b2(cs.y), n = as_b2(ns);
    if (FWD) {
        re = as_u(__hfma2(r, c, __hmul2(i, s)));
        im = as_u(__hfma2(i, c, __hmul2(r, n)));
    } else {
        re = as_u(__hfma2(r, c, __hmul2(i, n)));
        im = as_u(__hfma2(i, c, __hmul2(r, s)));
    }
}

// Complex product of one 16x16 A tile with the two n-tiles of a 16x16 B:
// the four products with Ar first, then the four with Ai, so each dependent
// accumulation is four MMAs behind the one it waits for.
__device__ __forceinline__ void cmma2(float (&yr)[2][4], float (&yi)[2][4], const uint32_t (&ar)[4],
                                      const uint32_t (&ai)[4], const uint2 (&br)[2], const uint2 (&bi)[2],
                                      const uint2 (&bni)[2]) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        mma16816(yr[j], ar, br[j].x, br[j].y);
        mma16816(yi[j], ar, bi[j].x, bi[j].y);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        mma16816(yr[j], ai, bni[j].x, bni[j].y);
        mma16816(yi[j], ai, br[j].x, br[j].y);
    }
}

// As cmma2, overwriting yr, yi (products start from zero).
__device__ __forceinline__ void cmma2z(float (&yr)[2][4], float (&yi)[2][4], const uint32_t (&ar)[4],
                                       const uint32_t (&ai)[4], const uint2 (&br)[2], const uint2 (&bi)[2],
                                       const uint2 (&bni)[2]) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        mma16816z(yr[j], ar, br[j].x, br[j].y);
        mma16816z(yi[j], ar, bi[j].x, bi[j].y);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        mma16816(yr[j], ai, bni[j].x, bni[j].y);
        mma16816(yi[j], ai, br[j].x, br[j].y);
    }
}

// Complex product on one 16 x 8 tile; FIRST: overwrite instead of accumulate.
template <bool FIRST>
__device__ __forceinline__ void cmma_k(float (&yr)[4], float (&yi)[4], const uint32_t (&ar)[4],
                                       const uint32_t (&ai)[4], uint2 br, uint2 bi, uint2 bni) {
    if (FIRST) {
        mma16816z(yr, ar, br.x, br.y);
        mma16816z(yi, ar, bi.x, bi.y);
    } else {
        mma16816(yr, ar, br.x, br.y);
        mma16816(yi, ar, bi.x, bi.y);
    }
    mma16816(yr, ai, bni.x, bni.y);
    mma16816(yi, ai, br.x, br.y);
}

// Complex tile product on one 16 x 8 output tile:
//   yr += Ar Br + Ai Bni,   yi += Ar Bi + Ai Br     (Bni = -Bi)
__device__ __forceinline__ void cmma(float (&yr)[4], float (&yi)[4], const uint32_t (&ar)[4],
                                     const uint32_t (&ai)[4], uint2 br, uint2 bi, uint2 bni) {
    mma16816(yr, ar, br.x, br.y);
    mma16816(yr, ai, bni.x, bni.y);
    mma16816(yi, ar, bi.x, bi.y);
    mma16816(yi, ai, br.x, br.y);
}

// ------------------------------------------------------------ smem layout
// Plane row = 256 bf16 = 32 chunks of 16 B.  Chunk c of row r is stored at
// chunk (c4 c0 ((c3 c2 c1) ^ r)) -- a bijection per row that makes 8 chunks
// {2a + cb : 8 consecutive a} of one row, and one chunk of 8 consecutive rows,
// land on 8 distinct 16-byte bank groups.
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {
    return (chunk & 16u) | ((chunk & 1u) << 3) | (((chunk >> 1) ^ row) & 7u);
}
__device__ __forceinline__ uint32_t plane_addr(uint32_t base, uint32_t row, uint32_t chunk) {
    return base + row * 512u + swz(row, chunk) * 16u;
}

using TcTables = TcTablePtrs;

template <int P>
struct TcShape {
    static constexpr int kLog2P = ilog2(P);
    static constexpr int M = P * 256;
    static constexpr int N = M / 2;
    static constexpr int NT1 = P / 8;                   // step-1 output n-tiles (k_p)
    static constexpr int KS1 = (P / 2 + 15) / 16;       // step-1 k-steps (p < P/2)
    static constexpr int NT3 = (P / 2 + 7) / 8;         // step-1' output n-tiles (p < P/2)
    static constexpr int KS3 = P / 16;                  // step-1' k-steps (k_p)
    static constexpr int kPlaneBytes = P * 512;         // one bf16 plane, P rows of 256
    static constexpr int kSmemPerPair = 2 * kPlaneBytes;
};

// ================================================================== kernel
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

template <int P, bool GATED>
struct TcSmem {
    static constexpr int kS = 2 * P * 512;      // S: re and im planes, P rows of 256 q
    static constexpr int kX = P * 512;          // x staging: re and im planes, P/2 rows
    // The gate input w has its own staging planes, except for the largest
    // transform, where it is staged in S's upper rows (free until step 1).
    static constexpr bool kWInS = P >= 128;
    // Ungated transforms up to 2N = 8192 keep two staging buffers, used by
    // alternate items, so the next item's rows are requested one item earlier.
    static constexpr int kNBuf = (!GATED && P <= 32) ? 2 : 1;
    // P >= 64: the outer DFT matrix (two bf16 planes of P x P/2), after the
    // staging buffers; its fragments are read with ldmatrix instead of from L2
    static constexpr bool kRS = P >= 64;
    static constexpr int kR = kRS ? 2 * P * P : 0;  // two planes of P rows x P bytes
    static constexpr int kROff = kS + kNBuf * kX * ((GATED && !kWInS) ? 2 : 1);
    static constexpr int kBytes = kROff + kR;
    // P = 128 (one CTA per SM): step 1 runs on tcgen05 from the staging planes
    // (canonical MN-major layout) and the outer DFT matrix, into 512 TMEM columns
    static constexpr bool kUM1 = P == 128;
};

// Byte offset of the 16-byte chunk c (8 values p) of row r (k_p) of one plane
// of the outer DFT matrix, in the canonical no-swizzle K-major core-matrix
// layout: core matrix (r / 8, c) of 8 rows x 16 bytes at (r / 8) (P / 16) 128
// + 128 c.  The 8 rows of an 8 x 8 ldmatrix block are one 128-byte core
// matrix (conflict-free), and the same bytes are the tcgen05 B operand
// (LBO 128 along p, SBO (P / 16) 128 along k_p).
template <int P>
__device__ __forceinline__ uint32_t wr_off(int r, int c) {
    return (uint32_t)((r >> 3) * (P / 16) * 128 + c * 128 + (r & 7) * 16);
}
// Byte offset of chunk c (8 values q) of row p of one staging plane of the
// P = 128 kernel, canonical MN-major for tcgen05 (A operand, M = q, K = p):
// core matrix (p / 8, c) at 1024 c + 128 (p / 8); LBO 128 along p, SBO 1024 along q.
__device__ __forceinline__ uint32_t xcan_off(int p, int c) {
    return (uint32_t)(c * 1024 + (p >> 3) * 128 + (p & 7) * 16);
}

// fp32 accumulators of two 16x8 tiles (n-tiles 0, 1) -> the four bf16x2
// registers of the 16x16 A fragment they form.
template <bool IP = false>
__device__ __forceinline__ void pack_tile(uint32_t (&o)[4], const float (&t)[2][4]) {
    o[0] = pack2<IP>(t[0][0], t[0][1]);
    o[1] = pack2<IP>(t[0][2], t[0][3]);
    o[2] = pack2<IP>(t[1][0], t[1][1]);
    o[3] = pack2<IP>(t[1][2], t[1][3]);
}
// 16x16 transpose of an A fragment: block (r, c) -> (c, r), each 8x8 block transposed.
__device__ __forceinline__ void transpose_tile(uint32_t (&o)[4], const uint32_t (&x)[4]) {
    o[0] = movt(x[0]);
    o[1] = movt(x[2]);
    o[2] = movt(x[1]);
    o[3] = movt(x[3]);
}

}  // namespace tc
}  // namespace fftc
