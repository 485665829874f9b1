// fft_simt.cuh -- fp32 SIMT building blocks for the FFT convolution kernels.
//
// The FFT convolution of "FlashFFTConv: Efficient Convolutions for Long
// Sequences with Tensor Cores" (abstract) and "FlashConv" (Mechanism: FFT,
// pointwise product and inverse FFT fused on chip) is built here from:
//
//  * an in-register DFT of radix R <= 32 (decimation in frequency, compile-time
//    unit roots, special cases for 1, -1, +-i), natural order in and out;
//  * a batched Stockham autosort stage: L-point transforms of C independent
//    columns held in shared memory; each thread owns BPT butterflies of radix
//    R, reads R values at stride L/R, multiplies by W_{Ns R}^{r k}, applies
//    DFT_R and writes them to (j/Ns) Ns R + (j mod Ns) + r Ns, so that after
//    log_R(L) stages the spectrum is in natural order;
//  * a compile-time radix plan (one remainder stage, then radix-E stages,
//    with E = values per thread).
//
// Loads and stores are functors, so the first stage can read the zero-padded
// input straight from global memory (only the first half of each butterfly is
// nonzero) and the last inverse stage can write the truncated output straight
// to global memory (only the first half is kept).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

namespace fftc {

// ---------------------------------------------------------------- complex ops
__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cscale(float2 a, float s) { return make_float2(a.x * s, a.y * s); }
// a * b
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
// a * conj(b)
__device__ __forceinline__ float2 cmulc(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.y, b.x, -a.x * b.y));
}
template <bool INV>
__device__ __forceinline__ float2 cmul_dir(float2 a, float2 w) { return INV ? cmulc(a, w) : cmul(a, w); }

// ------------------------------------------------------- compile-time roots
// cos(2 pi m / 32) for m in [0, 8]; first-quadrant values of the 32nd roots.
__host__ __device__ constexpr double cos32_q(int m) {
    return m == 0 ? 1.0
         : m == 1 ? 0.98078528040323044912618223613424
         : m == 2 ? 0.92387953251128675612818318939679
         : m == 3 ? 0.83146961230254523707878837761791
         : m == 4 ? 0.70710678118654752440084436210485
         : m == 5 ? 0.55557023301960222474283081394853
         : m == 6 ? 0.38268343236508977172845998403040
         : m == 7 ? 0.19509032201612826784828486847702
         : 0.0;
}
// cos(2 pi m / 32) for any integer m, by quadrant symmetry.
__host__ __device__ constexpr double cos32(int m) {
    return ((m & 31) <= 8)  ? cos32_q(m & 31)
         : ((m & 31) <= 16) ? -cos32_q(16 - (m & 31))
         : ((m & 31) <= 24) ? -cos32_q((m & 31) - 16)
                            : cos32_q(32 - (m & 31));
}
// sin(2 pi m / 32) = cos(2 pi (m - 8) / 32)
__host__ __device__ constexpr double sin32(int m) { return cos32(m - 8); }

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x >> 1); }
__host__ __device__ constexpr int bitrev(int x, int bits) {
    return bits == 0 ? 0 : (((x & 1) << (bits - 1)) | bitrev(x >> 1, bits - 1));
}

// v * W_R^n (forward, W_R = exp(-2 pi i / R)) or v * W_R^-n (inverse); n is a
// compile-time constant after unrolling, so the branches fold away.
template <int R, bool INV>
__device__ __forceinline__ float2 rotate(float2 v, int n) {
    static_assert(R <= 32, "in-register radix limited to 32");
    const int m = (n * (32 / R)) & 31;
    if (m == 0) return v;
    if (m == 16) return make_float2(-v.x, -v.y);
    if (m == 8) return INV ? make_float2(-v.y, v.x) : make_float2(v.y, -v.x);
    if (m == 24) return INV ? make_float2(v.y, -v.x) : make_float2(-v.y, v.x);
    const float c = (float)cos32(m), s = (float)sin32(m);
    return INV ? make_float2(c * v.x - s * v.y, c * v.y + s * v.x)
               : make_float2(c * v.x + s * v.y, c * v.y - s * v.x);
}

// In-place decimation-in-frequency DFT; leaves X[bitrev(p)] at position p.
template <int R, bool INV>
__device__ __forceinline__ void dif_inplace(float2* v) {
    if constexpr (R > 1) {
        constexpr int H = R / 2;
#pragma unroll
        for (int n = 0; n < H; ++n) {
            const float2 a = v[n], b = v[n + H];
            v[n] = cadd(a, b);
            v[n + H] = rotate<R, INV>(csub(a, b), n);
        }
        dif_inplace<H, INV>(v);
        dif_inplace<H, INV>(v + H);
    }
}

// out[I] = in[bitrev(I)], unrolled at compile time so that every index is a
// constant and the arrays stay in registers.
template <int R, int I = 0>
__device__ __forceinline__ void permute_bitrev(float2* out, const float2* in) {
    if constexpr (I < R) {
        constexpr int J = bitrev(I, ilog2(R));
        out[I] = in[J];
        permute_bitrev<R, I + 1>(out, in);
    }
}

// v <- DFT_R(v) (INV: unnormalised inverse), natural order in and out.
template <int R, bool INV>
__device__ __forceinline__ void dft(float2* v) {
    dif_inplace<R, INV>(v);
    float2 t[R];
    permute_bitrev<R>(t, v);
#pragma unroll
    for (int i = 0; i < R; ++i) v[i] = t[i];
}

// --------------------------------------------------------------- I/O types
template <typename T> __device__ __forceinline__ float to_f(T v);
template <> __device__ __forceinline__ float to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// ------------------------------------------------------------ smem layout
// L-point transforms of C columns.  BF (batch-fast): element (i, c) at i*C + c;
// otherwise at c*L + i.  One pad slot per 2^PADSH complex values (default 32)
// breaks the bank conflicts of the strided Stockham writes.
template <int L, int C, bool BF, int PADSH = 5>
struct Layout {
    static constexpr int kWords = L * C + ((L * C) >> PADSH);  // float2 slots
    static __device__ __forceinline__ int at(int i, int c) {
        const int x = BF ? i * C + c : c * L + i;
        return x + (x >> PADSH);
    }
};

// ------------------------------------------------------------- radix plan
// L = 2^LOG2L points, E = 2^LOG2E values per thread per stage.  Stage 0 has
// radix 2^(LOG2L mod LOG2E) when that is nonzero; every other stage radix E.
template <int LOG2L, int LOG2E>
struct RadixPlan {
    static constexpr int kRem = LOG2L % LOG2E;
    static constexpr int kStages = LOG2L / LOG2E + (kRem ? 1 : 0);
    static constexpr int log2r(int s) { return (kRem && s == 0) ? kRem : LOG2E; }
    static constexpr int log2ns(int s) { return s == 0 ? 0 : (kRem ? kRem + (s - 1) * LOG2E : s * LOG2E); }
};

// Geometry of a batched transform: L points x C columns on T threads.
template <int LOG2L_, int C_, bool BF_, int PADSH_ = 5>
struct Geometry {
    static constexpr int LOG2L = LOG2L_;
    static constexpr int L = 1 << LOG2L_;
    static constexpr int C = C_;
    static constexpr bool BF = BF_;
    static constexpr int kTotal = L * C;
    static_assert(kTotal <= 16384, "batched transform too large for one CTA");
    // 16 values per thread, at least one warp, at most 512 threads (so the
    // register file is not capped at 64 per thread); 32 values at 16384 points.
    static constexpr int T = (kTotal / 16) < 32 ? 32 : ((kTotal / 16) > 512 ? 512 : (kTotal / 16));
    static constexpr int LOG2E = ilog2(kTotal / T);
    using Plan = RadixPlan<LOG2L, LOG2E>;
    using Lay = Layout<L, C, BF, PADSH_>;
};

// Twiddles of every stage of a geometry, one table: stage s holds
// W_{Ns R}^{r k} at offset(s) + r Ns + k for r < R, k < Ns.
template <class G>
struct StageTwiddles {
    static constexpr int offset(int s) {
        int o = 0;
        for (int i = 0; i < s; ++i) o += (1 << G::Plan::log2r(i)) << G::Plan::log2ns(i);
        return o;
    }
    static constexpr int total() { return offset(G::Plan::kStages); }
};

// Butterfly id -> (j, c).  Consecutive ids walk the fast axis of the layout.
template <class G, int R>
__device__ __forceinline__ void bfly_coords(int bid, int& j, int& c) {
    if (G::BF) { c = bid % G::C; j = bid / G::C; }
    else { j = bid % (G::L / R); c = bid / (G::L / R); }
}

// One Stockham stage.  load(i, c) -> float2 and store(i, c, float2) give the
// value of point i of column c before / after the stage.  Only the first IN_R
// of the R inputs are loaded (the rest are zero: the padding); only the first
// OUT_R outputs are stored (truncation).  SYNC: barrier between the loads and
// the stores (the stage reads and writes the same shared buffer).
template <class G, int S, bool INV, int IN_R, int OUT_R, bool SYNC, class LoadF, class StoreF>
__device__ __forceinline__ void stage(int tid, const float2* __restrict__ tw, LoadF load, StoreF store) {
    constexpr int LOG2R = G::Plan::log2r(S);
    constexpr int R = 1 << LOG2R;
    constexpr int LOG2NS = G::Plan::log2ns(S);
    constexpr int NS = 1 << LOG2NS;
    constexpr int NB = (G::L / R) * G::C;
    static_assert(NB % G::T == 0, "butterflies must divide evenly among threads");
    constexpr int BPT = NB / G::T;
    static_assert(IN_R <= R && OUT_R <= R, "bad partial stage");
    float2 v[BPT][R];
#pragma unroll
    for (int q = 0; q < BPT; ++q) {
        int j, c;
        bfly_coords<G, R>(tid + q * G::T, j, c);
#pragma unroll
        for (int r = 0; r < R; ++r)
            v[q][r] = (r < IN_R) ? load(j + r * (G::L / R), c) : make_float2(0.f, 0.f);
    }
    if (SYNC) __syncthreads();
#pragma unroll
    for (int q = 0; q < BPT; ++q) {
        int j, c;
        bfly_coords<G, R>(tid + q * G::T, j, c);
        const int k = j & (NS - 1);
        if (LOG2NS > 0) {
            // W_{Ns R}^{r k} from the stage's table, laid out [r][k] so that the
            // consecutive k of a warp read consecutive entries.  For R >= 16 only
            // the powers r = 1, 2, 4, 8 (16) are loaded; every other power is the
            // product of the loaded ones for the set bits of r (at most
            // log2(R) - 1 fp32 complex products, error ~1e-7), which moves the
            // stage from load throughput to FMA throughput.
            constexpr int OFF = StageTwiddles<G>::offset(S);
            if constexpr (R >= 16) {
                float2 wp[R];
#pragma unroll
                for (int r = 1; r < R; r <<= 1) wp[r] = __ldg(&tw[OFF + r * NS + k]);
#pragma unroll
                for (int r = 3; r < R; ++r)
                    if (r & (r - 1)) wp[r] = cmul(wp[r & (r - 1)], wp[r & -r]);
#pragma unroll
                for (int r = 1; r < IN_R; ++r) v[q][r] = cmul_dir<INV>(v[q][r], wp[r]);
            } else {
#pragma unroll
                for (int r = 1; r < IN_R; ++r) v[q][r] = cmul_dir<INV>(v[q][r], __ldg(&tw[OFF + r * NS + k]));
            }
        }
        dft<R, INV>(v[q]);
        const int base = ((j >> LOG2NS) << (LOG2NS + LOG2R)) + k;
#pragma unroll
        for (int r = 0; r < OUT_R; ++r) {
            // a store functor may also take r (a compile-time index after unrolling)
            if constexpr (std::is_invocable_v<StoreF, int, int, float2, int>)
                store(base + r * NS, c, v[q][r], r);
            else
                store(base + r * NS, c, v[q][r]);
        }
    }
}

// Run stages [S, END) of a plan entirely in shared memory (load and store
// through the layout), with a barrier after each.
template <class G, int S, int END, bool INV>
__device__ __forceinline__ void smem_stages(float2* s, int tid, const float2* __restrict__ tw) {
    if constexpr (S < END) {
        using Lay = typename G::Lay;
        stage<G, S, INV, (1 << G::Plan::log2r(S)), (1 << G::Plan::log2r(S)), true>(
            tid, tw, [&](int i, int c) { return s[Lay::at(i, c)]; },
            [&](int i, int c, float2 x) { s[Lay::at(i, c)] = x; });
        __syncthreads();
        smem_stages<G, S + 1, END, INV>(s, tid, tw);
    }
}

}  // namespace fftc
