// conv2d_tc.cu -- the column pass of the 2-D causal FFT convolution on the
// bf16 tensor cores, for images of 256 rows (columns of 2 Hs = 512 points).
//
// After the row pass the workspace holds, per pair of images (real +
// imaginary part) and for every row i < 256 and column kx < 2 Ws, the row
// spectrum W[i][kx] (fp32 complex).  The column pass of "Native
// Multi-Dimensional Subquadratic Operators via Input Dependent Long
// Convolutions" (abstract: the multi-dimensional FFT convolution) is, per
// column, a 512-point DFT over the 256 nonzero rows, a product with the
// channel's spectrum column, and the inverse keeping rows i < 256.  With the
// upper half zero, the 512-point DFT splits into two 256-point DFTs (ky even:
// of x; ky odd: of x W_512^i), each the 16 x 16 Monarch product of
// "FlashFFTConv: Efficient Convolutions for Long Sequences with Tensor Cores"
// (abstract) on mma.sync: over a (i = 16 a + b), times W_256^{b c}, transpose,
// over b.  The inverse runs the conjugate products in reverse order and
// recombines the halves: z[i] = Z_even[i] + W_512^{-i} Z_odd[i].
// Per CTA: 16 consecutive columns of one pair; per warp: 4 columns, two
// units (even, odd) at a time.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <vector>

#include "plan.h"
#include "tables.h"
#include "tc_common.cuh"

namespace fftc {
namespace tc {

constexpr int kC2Cols = 16;  // columns per CTA

// Column pass.  work: [pair][256][LR] fp32 complex; khat: [channel][LR][2 (ky parity)][32 lanes][8 words]
// Output tile: row i, 16 columns of fp32 complex; column c of row i at
// position c ^ s(i), s(i) = (i & 7) | (((i >> 5) & 1) << 3), so the 32 lanes
// of one accumulator store (one column, rows g + 32 t + const) hit every
// position twice (two wavefronts, the minimum for 8-byte stores).
__device__ __forceinline__ int c2_outpos(int i, int c) { return i * kC2Cols + (c ^ ((i & 7) | (((i >> 5) & 1) << 3))); }

// bf16 workspace of the all-tensor-core 2-D path (256 x 256 images), per
// pair 512 KiB each:
//   rows -> columns  W1[kx 512][row tile 32][re, im][8 rows]
//   columns -> rows  W2[i 256][column tile 32][kx parity][re, im][8 k' = kx / 2]
// Every pass rounds to bf16 where it reads its operands, so storing bf16
// changes no result; each write is a whole 32- or 64-byte segment and each
// read a 16-byte copy into the reader's swizzled planes.
constexpr size_t kW1Bytes = 512 * 1024;

template <int LOG2LR, bool BW>
__global__ void __launch_bounds__(128, 4)
c2tc_cols(float2* __restrict__ work, const uint4* __restrict__ khat, C2TcTables tb, int npp, int64_t first, int oy) {
    constexpr int LR = 1 << LOG2LR, Hs = 256;
    __shared__ __align__(128) uint8_t smem[2 * kC2Cols * 512];  // re, im planes: row = column, 256 i
    __shared__ __align__(16) float2 otile[Hs * kC2Cols];        // results, rows i, before the coalesced store
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m8 = lane >> 3, r8 = lane & 7;
    const int64_t P = first + blockIdx.y;
    const int kx0 = blockIdx.x * kC2Cols;
    const int ch = (int)(P / npp);
    float2* __restrict__ img = work + (size_t)blockIdx.y * Hs * LR;
    const uint32_t pre = smem_u32(smem), pim = pre + kC2Cols * 512;

    uint8_t* __restrict__ w1 = reinterpret_cast<uint8_t*>(img);  // bf16 workspace (BW)
    if constexpr (BW) {
        // ---- W1 columns kx0 .. kx0 + 15 (1 KiB each) -> planes, 16-byte copies
        const uint8_t* src = w1 + (size_t)kx0 * 1024;
        for (int q = tid; q < kC2Cols * 64; q += 128) {
            const int col = q >> 6, tile = (q >> 1) & 31, pl = q & 1;
            cp_async16(plane_addr(pl ? pim : pre, col, tile), src + (size_t)q * 16, 16);
        }
        cp_async_commit();
    }
    // ---- fp32 workspace: tile of 256 rows x 16 columns -> bf16 planes (row = column, two rows i per 32-bit word)
#pragma unroll
    for (int it = 0; it < (BW ? 0 : (Hs / 2) * (kC2Cols / 2) / 128); ++it) {
        const int idx = tid + it * 128;
        const int i = 2 * (idx / (kC2Cols / 2)), c = 2 * (idx % (kC2Cols / 2));
        const float4 a = __ldcg(reinterpret_cast<const float4*>(img + (size_t)i * LR + kx0 + c));
        const float4 b = __ldcg(reinterpret_cast<const float4*>(img + (size_t)(i + 1) * LR + kx0 + c));
        const uint32_t o = (uint32_t)(i & 7) * 2u;
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(plane_addr(pre, c, i >> 3) + o), "r"(pack2(a.x, b.x)) : "memory");
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(plane_addr(pim, c, i >> 3) + o), "r"(pack2(a.y, b.y)) : "memory");
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(plane_addr(pre, c + 1, i >> 3) + o), "r"(pack2(a.z, b.z))
                     : "memory");
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(plane_addr(pim, c + 1, i >> 3) + o), "r"(pack2(a.w, b.w))
                     : "memory");
    }
    uint2 f16[3][2], w256[4], t512[4];
    float2 tz[2][4];  // W_512^{i} in accumulator order, fp32
#pragma unroll
    for (int part = 0; part < 3; ++part)
#pragma unroll
        for (int j = 0; j < 2; ++j) f16[part][j] = __ldg(&tb.f16[(j * 3 + part) * 32 + lane]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        w256[i] = __ldg(&tb.w256[i * 32 + lane]);
        t512[i] = __ldg(&tb.t512[i * 32 + lane]);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) tz[j][e] = __ldg(&tb.t512f[(j * 4 + e) * 32 + lane]);
    if (BW) cp_async_wait_all();
    __syncthreads();

    const uint32_t ia = r8 + 8 * (m8 >> 1), ichunk = 2 * ia + (m8 & 1);
    const uint4* __restrict__ kh = khat + ((size_t)ch * LR + kx0) * 2 * 64;
    // i = 16 a + b of accumulator element (j, e): a = 8 j + 2 t + (e & 1), b = g + 8 (e >> 1)
    const int g = lane >> 2, t = lane & 3;
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
        const int col = 4 * warp + cc;
        uint4 k0[2], k1[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            k0[u] = __ldg(&kh[((size_t)col * 2 + u) * 64 + lane * 2]);
            k1[u] = __ldg(&kh[((size_t)col * 2 + u) * 64 + lane * 2 + 1]);
        }
        uint32_t xr[2][4], xi[2][4];
        ldsm_x4_t(xr[0], plane_addr(pre, col, ichunk));
        ldsm_x4_t(xi[0], plane_addr(pim, col, ichunk));
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            xr[1][i] = xr[0][i];
            xi[1][i] = xi[0][i];
            twiddle2<true>(xr[1][i], xi[1][i], t512[i]);  // odd ky: x W_512^{i}
        }
        float acr[2][2][4], aci[2][2][4];
        // forward: [b][a] x F16 -> [b][c]; x W_256^{b c}; transpose -> [c][b]; x F16 -> [c][d]
#pragma unroll
        for (int u = 0; u < 2; ++u) cmma2z(acr[u], aci[u], xr[u], xi[u], f16[0], f16[1], f16[2]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            uint32_t tr[4], ti[4];
            pack_tile(tr, acr[u]);
            pack_tile(ti, aci[u]);
#pragma unroll
            for (int i = 0; i < 4; ++i) twiddle2<true>(tr[i], ti[i], w256[i]);
            transpose_tile(xr[u], tr);
            transpose_tile(xi[u], ti);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) cmma2z(acr[u], aci[u], xr[u], xi[u], f16[0], f16[1], f16[2]);
        // spectrum at ky = u + 2 (c + 16 d): product with Khat
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            pack_tile(xr[u], acr[u]);
            pack_tile(xi[u], aci[u]);
            const uint32_t kre[4] = {k0[u].x, k0[u].z, k1[u].x, k1[u].z};
            const uint32_t kim[4] = {k0[u].y, k0[u].w, k1[u].y, k1[u].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __nv_bfloat162 zr = as_b2(xr[u][i]), zi = as_b2(xi[u][i]);
                const __nv_bfloat162 kr = as_b2(kre[i]), ki = as_b2(kim[i]);
                xr[u][i] = as_u(__hfma2(zr, kr, __hneg2(__hmul2(zi, ki))));
                xi[u][i] = as_u(__hfma2(zr, ki, __hmul2(zi, kr)));
            }
        }
        // inverse: [c][d] x conj(F16) -> [c][b]; transpose -> [b][c]; x W_256^{-b c}; x conj(F16) -> [b][a]
#pragma unroll
        for (int u = 0; u < 2; ++u) cmma2z(acr[u], aci[u], xr[u], xi[u], f16[0], f16[2], f16[1]);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            uint32_t gr[4], gi[4];
            pack_tile(gr, acr[u]);
            pack_tile(gi, aci[u]);
            transpose_tile(xr[u], gr);
            transpose_tile(xi[u], gi);
#pragma unroll
            for (int i = 0; i < 4; ++i) twiddle2<false>(xr[u][i], xi[u][i], w256[i]);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) cmma2z(acr[u], aci[u], xr[u], xi[u], f16[0], f16[2], f16[1]);
        // z[i] = Z_even[i] + W_512^{-i} Z_odd[i] (fp32) into the output tile.  With a
        // crop offset oy the output row is i - oy, and for i < oy the row 256 + i of
        // the 512-point inverse: z[i + 256] = Z_even[i] - W_512^{-i} Z_odd[i]
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 w = tz[j][e];
                const int i = 16 * (8 * j + 2 * t + (e & 1)) + g + 8 * (e >> 1);
                const float sg = i < oy ? -1.f : 1.f;
                const float orr = sg * acr[1][j][e], oi = sg * aci[1][j][e];
                // W_512^{-i} = cos + i sin of 2 pi i / 512
                const float zr = acr[0][j][e] + fmaf(orr, w.x, -oi * w.y);
                const float zi = aci[0][j][e] + fmaf(oi, w.x, orr * w.y);
                otile[c2_outpos((i - oy) & (Hs - 1), col)] = make_float2(zr, zi);
            }
    }
    __syncthreads();
    if constexpr (BW) {
        // ---- W2 rows i: this tile's 64 bytes ([parity][re, im][8 k']); lane m of an
        // 8-lane group writes 8 bytes: segment m / 2 (parity, re/im), k' = 4 (m & 1) .. + 3.
        // A warp takes rows i0 + {0, 2, 4, 6}: their swizzles differ in bits 1 and 2,
        // so its 16 distinct tile reads fall in 16 distinct bank pairs.
        uint8_t* __restrict__ w2 = w1 + kW1Bytes + (size_t)(kx0 / kC2Cols) * 64;
#pragma unroll 4
        for (int it = 0; it < Hs / 16; ++it) {
            const int i = 16 * it + (warp & 1) + 8 * (warp >> 1) + 2 * (lane >> 3);
            const int m = lane & 7, seg = m >> 1, h = m & 1;
            const int parity = seg >> 1, im = seg & 1;
            float v[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const float2 z = otile[c2_outpos(i, 8 * h + 2 * jj + parity)];
                v[jj] = im ? z.y : z.x;
            }
            const uint2 o = make_uint2(pack2(v[0], v[1]), pack2(v[2], v[3]));
            *reinterpret_cast<uint2*>(w2 + (size_t)i * 2048 + seg * 16 + h * 8) = o;
        }
        return;
    }
    // ---- fp32 workspace: rows i < 256 of the 16 columns back, 128 bytes per row
#pragma unroll 4
    for (int it = 0; it < Hs * (kC2Cols / 2) / 128; ++it) {
        const int idx = tid + it * 128;
        const int i = idx / (kC2Cols / 2), c = 2 * (idx % (kC2Cols / 2));
        // columns c, c + 1 sit in adjacent positions (their order flips when s(i) is odd)
        const int p0 = c2_outpos(i, c);
        const float4 v = *reinterpret_cast<const float4*>(&otile[p0 & ~1]);
        const float4 o = (p0 & 1) ? make_float4(v.z, v.w, v.x, v.y) : v;
        __stcg(reinterpret_cast<float4*>(img + (size_t)i * LR + kx0 + c), o);
    }
}


// Row tile of the forward row pass: row r, LR = 512 columns of fp32 complex;
// column kx of row r at kx ^ ((kx >> 6) & 3), which spreads one accumulator
// store (kx = parity + 2 g + 64 t + const over the lanes) over every
// position twice; columns kx, kx + 1 (kx even) stay adjacent.
__device__ __forceinline__ int c2_rowpos(int r, int kx) { return r * 512 + (kx ^ ((kx >> 6) & 3)); }

// Forward row pass (images of 256 x 256): rows i of the pair's two images
// (real, imaginary part), 512-point DFT over j < 256 as two 256-point
// Monarch DFTs (kx even: of x; kx odd: of x W_512^j) -> W1 of the pair.
// Persistent: a CTA walks work items (8 rows of one pair; consecutive items
// share the pair) with stride gridDim.x, staging the next item's rows with
// cp.async into the other buffer while it transforms the current one.
constexpr int kC2RowsF = 8;  // rows per work item
__global__ void __launch_bounds__(128, 4)
c2tc_rows_fwd(const __nv_bfloat16* __restrict__ u, float2* __restrict__ work, C2TcTables tb, int B, int C,
              int64_t first, int items) {
    constexpr int Hs = 256, Ws = 256, LR = 512, RBLK = Hs / kC2RowsF;
    __shared__ __align__(128) uint8_t smem[2][2 * kC2RowsF * 512];  // two staging buffers: re, im planes, rows r
    __shared__ __align__(16) float2 otile[kC2RowsF * LR];           // row spectra before the W1 stores
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m8 = lane >> 3, r8 = lane & 7;
    const int npp = (B + 1) / 2;
    // rows i0 .. i0 + 7 of both images of the item's pair -> planes of buffer buf (16-byte chunks)
    auto stage = [&](int item, int buf) {
        const int64_t P = first + item / RBLK;
        const int i0 = (item % RBLK) * kC2RowsF;
        const int ch = (int)(P / npp), b0 = (int)(P % npp) * 2;
        const bool has1 = b0 + 1 < B;
        const size_t img0 = ((size_t)b0 * C + ch) * Hs * Ws, img1 = ((size_t)(b0 + 1) * C + ch) * Hs * Ws;
        const uint32_t pre = smem_u32(smem[buf]), pim = pre + kC2RowsF * 512;
        for (int idx = tid; idx < 2 * kC2RowsF * 32; idx += 128) {
            const int plane = idx / (kC2RowsF * 32), r = (idx / 32) % kC2RowsF, chunk = idx % 32;
            const int bytes = (plane == 0 || has1) ? 16 : 0;  // zero-fill the missing image
            const size_t off = (plane ? (has1 ? img1 : img0) : img0) + (size_t)(i0 + r) * Ws + chunk * 8;
            cp_async16(plane_addr(plane ? pim : pre, r, chunk), u + off, bytes);
        }
        cp_async_commit();
    };
    if ((int)blockIdx.x < items) stage(blockIdx.x, 0);
    uint2 f16[3][2], w256[4], t512[4];
#pragma unroll
    for (int part = 0; part < 3; ++part)
#pragma unroll
        for (int j = 0; j < 2; ++j) f16[part][j] = __ldg(&tb.f16[(j * 3 + part) * 32 + lane]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        w256[i] = __ldg(&tb.w256[i * 32 + lane]);
        t512[i] = __ldg(&tb.t512[i * 32 + lane]);
    }
    const uint32_t ia = r8 + 8 * (m8 >> 1), ichunk = 2 * ia + (m8 & 1);
    const int g = lane >> 2, t = lane & 3;
    int k = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++k) {
        const int buf = k & 1;
        if (item + (int)gridDim.x < items) {
            // the other buffer was last read by the previous item (two barriers ago)
            stage(item + gridDim.x, buf ^ 1);
            asm volatile("cp.async.wait_group 1;\n" ::: "memory");
        } else {
            cp_async_wait_all();
        }
        __syncthreads();
        const uint32_t pre = smem_u32(smem[buf]), pim = pre + kC2RowsF * 512;
#pragma unroll 1
        for (int rr = 0; rr < kC2RowsF / 4; ++rr) {
            const int r = 2 * warp + rr;
            uint32_t xr[2][4], xi[2][4];
            ldsm_x4_t(xr[0], plane_addr(pre, r, ichunk));
            ldsm_x4_t(xi[0], plane_addr(pim, r, ichunk));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xr[1][i] = xr[0][i];
                xi[1][i] = xi[0][i];
                twiddle2<true>(xr[1][i], xi[1][i], t512[i]);  // odd kx: x W_512^{j}
            }
            float acr[2][2][4], aci[2][2][4];
#pragma unroll
            for (int v = 0; v < 2; ++v) cmma2z(acr[v], aci[v], xr[v], xi[v], f16[0], f16[1], f16[2]);
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                uint32_t tr[4], ti[4];
                pack_tile(tr, acr[v]);
                pack_tile(ti, aci[v]);
#pragma unroll
                for (int i = 0; i < 4; ++i) twiddle2<true>(tr[i], ti[i], w256[i]);
                transpose_tile(xr[v], tr);
                transpose_tile(xi[v], ti);
            }
#pragma unroll
            for (int v = 0; v < 2; ++v) cmma2z(acr[v], aci[v], xr[v], xi[v], f16[0], f16[1], f16[2]);
            // accumulator (n, e) of unit v: c = g + 8 (e >> 1), d = 8 n + 2 t + (e & 1); kx = v + 2 (c + 16 d)
#pragma unroll
            for (int v = 0; v < 2; ++v)
#pragma unroll
                for (int n = 0; n < 2; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = g + 8 * (e >> 1), d = 8 * n + 2 * t + (e & 1);
                        otile[c2_rowpos(r, v + 2 * (c + 16 * d))] = make_float2(acr[v][n][e], aci[v][n][e]);
                    }
        }
        __syncthreads();
        // ---- W1[kx][row tile i0 / 8][re, im][8 rows]: 32 bytes per column kx
        static_assert(kC2RowsF == 8, "one row tile of W1 per item");
        uint8_t* __restrict__ w1 = reinterpret_cast<uint8_t*>(work + (size_t)(item / RBLK) * Hs * LR) +
                                   (size_t)(item % RBLK) * 32;
#pragma unroll
        for (int kx = tid; kx < LR; kx += 128) {
            float re[8], im[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const float2 z = otile[c2_rowpos(r, kx)];
                re[r] = z.x;
                im[r] = z.y;
            }
            uint4* dst = reinterpret_cast<uint4*>(w1 + (size_t)kx * 1024);
            dst[0] = make_uint4(pack2(re[0], re[1]), pack2(re[2], re[3]), pack2(re[4], re[5]), pack2(re[6], re[7]));
            dst[1] = make_uint4(pack2(im[0], im[1]), pack2(im[2], im[3]), pack2(im[4], im[5]), pack2(im[6], im[7]));
        }
        // the next item's wait + barrier orders these reads before otile is rewritten
    }
    cp_async_wait_all();
}

// Inverse row pass (images of 256 x 256): W2 of the pair -> 512-point
// inverse DFT over kx keeping j < 256, as two 256-point Monarch inverses
// (kx even, kx odd) recombined with W_512^{-j} -> y rows of both images.
// Persistent like the forward row pass: work items of 8 rows, the next
// item's W2 rows staged with cp.async into the other buffer.
constexpr int kC2RowsI = 8;  // rows per work item
__global__ void __launch_bounds__(128, 4)
c2tc_rows_inv(const float2* __restrict__ work, __nv_bfloat16* __restrict__ y, C2TcTables tb, int B, int C,
              int64_t first, int items, int ox) {
    constexpr int Hs = 256, Ws = 256, LR = 512, RBLK = Hs / kC2RowsI;
    // two staging buffers of planes (row r, 256 k'): [parity][re, im]; then y planes (row r, 256 j) [image]
    __shared__ __align__(128) uint8_t smem[2 * 4 * kC2RowsI * 512 + 2 * kC2RowsI * 512];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int m8 = lane >> 3, r8 = lane & 7;
    const int npp = (B + 1) / 2;
    const uint32_t base = smem_u32(smem);
    auto plane = [&](int buf, int par, int im) {
        return base + (uint32_t)((buf * 4 + 2 * par + im) * kC2RowsI * 512);
    };
    const uint32_t y0p = base + 8 * kC2RowsI * 512, y1p = y0p + kC2RowsI * 512;
    // W2 rows i0 .. i0 + 7 of the item's pair (2 KiB each: [column tile][parity][re, im][8 k']) -> buffer buf;
    // a warp copies 16 tiles of one (parity, re/im): 32 chunks over all 8 bank groups
    auto stage = [&](int item, int buf) {
        const uint8_t* __restrict__ w2 = reinterpret_cast<const uint8_t*>(work + (size_t)(item / RBLK) * Hs * LR) +
                                         kW1Bytes + (size_t)(item % RBLK) * kC2RowsI * 2048;
        const int tile = 16 * (warp & 1) + (lane >> 1), par = warp >> 1, pl = lane & 1;
        for (int r = 0; r < kC2RowsI; ++r)
            cp_async16(plane_addr(plane(buf, par, pl), r, tile), w2 + (size_t)r * 2048 + tile * 64 + par * 32 + pl * 16,
                       16);
        cp_async_commit();
    };
    if ((int)blockIdx.x < items) stage(blockIdx.x, 0);
    uint2 f16[3][2], w256[4];
    float2 tz[2][4];
#pragma unroll
    for (int part = 0; part < 3; ++part)
#pragma unroll
        for (int j = 0; j < 2; ++j) f16[part][j] = __ldg(&tb.f16[(j * 3 + part) * 32 + lane]);
#pragma unroll
    for (int i = 0; i < 4; ++i) w256[i] = __ldg(&tb.w256[i * 32 + lane]);
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) tz[j][e] = __ldg(&tb.t512f[(j * 4 + e) * 32 + lane]);
    const uint32_t ia = r8 + 8 * (m8 >> 1), ichunk = 2 * ia + (m8 & 1);
    int k = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++k) {
        const int buf = k & 1;
        if (item + (int)gridDim.x < items) {
            // the other buffer was last read by the previous item (two barriers ago)
            stage(item + gridDim.x, buf ^ 1);
            asm volatile("cp.async.wait_group 1;\n" ::: "memory");
        } else {
            cp_async_wait_all();
        }
        __syncthreads();
#pragma unroll 1
        for (int rr = 0; rr < kC2RowsI / 4; ++rr) {
            const int r = 2 * warp + rr;
            // A = [c][d], k' = c + 16 d, of the even and odd columns
            uint32_t xr[2][4], xi[2][4];
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                ldsm_x4_t(xr[v], plane_addr(plane(buf, v, 0), r, ichunk));
                ldsm_x4_t(xi[v], plane_addr(plane(buf, v, 1), r, ichunk));
            }
            float acr[2][2][4], aci[2][2][4];
            // [c][d] x conj(F16) -> [c][b]; transpose -> [b][c]; x W_256^{-b c}; x conj(F16) -> [b][a]
#pragma unroll
            for (int v = 0; v < 2; ++v) cmma2z(acr[v], aci[v], xr[v], xi[v], f16[0], f16[2], f16[1]);
#pragma unroll
            for (int v = 0; v < 2; ++v) {
                uint32_t gr[4], gi[4];
                pack_tile(gr, acr[v]);
                pack_tile(gi, aci[v]);
                transpose_tile(xr[v], gr);
                transpose_tile(xi[v], gi);
#pragma unroll
                for (int i = 0; i < 4; ++i) twiddle2<false>(xr[v][i], xi[v][i], w256[i]);
            }
#pragma unroll
            for (int v = 0; v < 2; ++v) cmma2z(acr[v], aci[v], xr[v], xi[v], f16[0], f16[2], f16[1]);
            // z[j] = Z_even[j] + W_512^{-j} Z_odd[j]: re -> image b0, im -> image b0 + 1;
            // with a crop offset ox, columns j < ox carry z[256 + j] (the minus sign)
            // and the store below rotates the columns by ox
            float zr[2][4], zi[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 w = tz[n][e];
                    const int jx = 16 * (8 * n + 2 * (lane & 3) + (e & 1)) + (lane >> 2) + 8 * (e >> 1);
                    const float sg = jx < ox ? -1.f : 1.f;
                    const float orr = sg * acr[1][n][e], oi = sg * aci[1][n][e];
                    zr[n][e] = acr[0][n][e] + fmaf(orr, w.x, -oi * w.y);
                    zi[n][e] = aci[0][n][e] + fmaf(oi, w.x, orr * w.y);
                }
            uint32_t pr[4], pi[4];
            pack_tile(pr, zr);
            pack_tile(pi, zi);
            stsm_x4_t(plane_addr(y0p, r, ichunk), pr[0], pr[1], pr[2], pr[3]);
            stsm_x4_t(plane_addr(y1p, r, ichunk), pi[0], pi[1], pi[2], pi[3]);
        }
        __syncthreads();
        // ---- y rows i0 .. i0 + 7 of both images, 16-byte chunks
        const int64_t P = first + item / RBLK;
        const int i0 = (item % RBLK) * kC2RowsI;
        const int ch = (int)(P / npp), b0 = (int)(P % npp) * 2;
        const bool has1 = b0 + 1 < B;
        const size_t img0 = ((size_t)b0 * C + ch) * Hs * Ws, img1 = ((size_t)(b0 + 1) * C + ch) * Hs * Ws;
        for (int idx = tid; idx < 2 * kC2RowsI * 32; idx += 128) {
            const int im = idx / (kC2RowsI * 32), r = (idx / 32) % kC2RowsI, chunk = idx % 32;
            if (im == 1 && !has1) continue;
            uint4 val;
            asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];\n"
                         : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                         : "r"(plane_addr(im ? y1p : y0p, r, chunk)));
            const int oc = (chunk - ox / 8) & (Ws / 8 - 1);  // ox is a multiple of 8
            *reinterpret_cast<uint4*>(y + (im ? img1 : img0) + (size_t)(i0 + r) * Ws + oc * 8) = val;
        }
        // the next item's wait + barrier orders these reads before the y planes are rewritten
    }
    cp_async_wait_all();
}

}  // namespace tc

// ================================================================== host side
namespace {

uint16_t bf16_bits_c2(double x) {
    const float f = (float)x;
    uint32_t b;
    memcpy(&b, &f, 4);
    b += 0x7fffu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}
uint32_t pack_c2(double lo, double hi) { return (uint32_t)bf16_bits_c2(lo) | ((uint32_t)bf16_bits_c2(hi) << 16); }
void cs_c2(int64_t e, int64_t L, double* c, double* s) {
    int64_t r = e % L;
    if (r < 0) r += L;
    const double a = 2.0 * M_PI * (double)r / (double)L;
    *c = cos(a);
    *s = sin(a);
}
void push_u2_c2(std::vector<float2>& out, uint32_t x, uint32_t y) {
    float2 f;
    memcpy(&f.x, &x, 4);
    memcpy(&f.y, &y, 4);
    out.push_back(f);
}

}  // namespace

bool c2tc_supported(int Hs, int Ws, int dtype) { return dtype == FFTCONV_BF16 && Hs == 256 && Ws >= 16; }
bool c2tc_rows_supported(const fftconv_plan_s& p) { return p.tc2d && p.Ws == 256; }

// Tables of the tensor-core column pass: DFT_16 fragments and W_256^{b c}
// (shared with the 1-D kernel's tables), W_512^{i} as packed bf16 pairs in
// A-fragment order and as fp32 in accumulator order.
bool c2tc_tables(std::vector<float2>& out, size_t off[4]) {
    size_t o1[7];
    if (!tc_tables(12, out, o1)) return false;
    off[0] = o1[0];
    off[1] = o1[1];
    // t512: A fragment [b][a], register r: b = g + 8 (r & 1), a = 2 t + 8 (r >> 1) + {0, 1}; (cos, sin) of W_512^{16 a + b}
    off[2] = out.size();
    for (int r = 0; r < 4; ++r)
        for (int lane = 0; lane < 32; ++lane) {
            const int g = lane >> 2, t = lane & 3, b = g + 8 * (r & 1), a0 = 2 * t + 8 * (r >> 1);
            double ca, sa, cb, sb;
            cs_c2(16 * a0 + b, 512, &ca, &sa);
            cs_c2(16 * (a0 + 1) + b, 512, &cb, &sb);
            push_u2_c2(out, pack_c2(ca, cb), pack_c2(sa, sb));
        }
    // t512f: accumulator (j, e): a = 8 j + 2 t + (e & 1), b = g + 8 (e >> 1); (cos, sin) of W_512^{16 a + b}, fp32
    off[3] = out.size();
    for (int j = 0; j < 2; ++j)
        for (int e = 0; e < 4; ++e)
            for (int lane = 0; lane < 32; ++lane) {
                const int g = lane >> 2, t = lane & 3;
                const int a = 8 * j + 2 * t + (e & 1), b = g + 8 * (e >> 1);
                double c, s;
                cs_c2(16 * a + b, 512, &c, &s);
                out.push_back(make_float2((float)c, (float)s));
            }
    return true;
}

template <int LOG2LR>
static cudaError_t c2tc_go(const fftconv_plan_s& p, float2* work, const void* khat, int g, int64_t first,
                           cudaStream_t s, int oy) {
    constexpr int LR = 1 << LOG2LR;
    if constexpr (LOG2LR == 9) {
        // all passes on the tensor cores: the bf16 workspace
        if (c2tc_rows_supported(p)) {
            tc::c2tc_cols<LOG2LR, true><<<dim3(LR / tc::kC2Cols, g), 128, 0, s>>>(work, (const uint4*)khat, p.c2tc,
                                                                                 (p.B + 1) / 2, first, oy);
            return cudaGetLastError();
        }
    }
    tc::c2tc_cols<LOG2LR, false><<<dim3(LR / tc::kC2Cols, g), 128, 0, s>>>(work, (const uint4*)khat, p.c2tc, (p.B + 1) / 2,
                                                                     first, oy);
    return cudaGetLastError();
}

cudaError_t launch_c2tc_rows_fwd(const fftconv_plan_s& p, const void* u, float2* work, int g, int64_t first,
                                 cudaStream_t s) {
    // persistent grid: as many CTAs as are resident at once (computed once)
    static int resident = 0;
    if (resident == 0) {
        int per_sm = 0, sms = 0, dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tc::c2tc_rows_fwd, 128, 0);
        resident = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 1);
    }
    const int items = (256 / tc::kC2RowsF) * g;
    tc::c2tc_rows_fwd<<<items < resident ? items : resident, 128, 0, s>>>((const __nv_bfloat16*)u, work, p.c2tc, p.B,
                                                                          p.H, first, items);
    return cudaGetLastError();
}

cudaError_t launch_c2tc_rows_inv(const fftconv_plan_s& p, const float2* work, void* y, int g, int64_t first,
                                 cudaStream_t s, int ox) {
    static int resident = 0;  // persistent grid, as for the forward row pass
    if (resident == 0) {
        int per_sm = 0, sms = 0, dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tc::c2tc_rows_inv, 128, 0);
        resident = (per_sm > 0 ? per_sm : 1) * (sms > 0 ? sms : 1);
    }
    const int items = (256 / tc::kC2RowsI) * g;
    tc::c2tc_rows_inv<<<items < resident ? items : resident, 128, 0, s>>>(work, (__nv_bfloat16*)y, p.c2tc, p.B, p.H,
                                                                          first, items, ox);
    return cudaGetLastError();
}

cudaError_t launch_c2tc_cols(const fftconv_plan_s& p, float2* work, const void* khat, int g, int64_t first,
                             cudaStream_t s, int oy) {
    switch (p.Ws) {
        case 16: return c2tc_go<5>(p, work, khat, g, first, s, oy);
        case 32: return c2tc_go<6>(p, work, khat, g, first, s, oy);
        case 64: return c2tc_go<7>(p, work, khat, g, first, s, oy);
        case 128: return c2tc_go<8>(p, work, khat, g, first, s, oy);
        case 256: return c2tc_go<9>(p, work, khat, g, first, s, oy);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace fftc
