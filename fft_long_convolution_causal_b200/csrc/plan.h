// plan.h -- internal plan object and kernel launchers (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <vector>

#include "fftconv.h"

namespace fftc {

enum Path { PATH_FUSED = 0, PATH_MULTIPASS = 1, PATH_2D = 2, PATH_FUSED_TC = 3, PATH_SSM = 4, PATH_PARTIAL = 5,
            PATH_3D = 6 };

// Twiddle tables of one plan (device pointers into one allocation).  wL / wC
// are per-stage tables of the row / column transforms (StageTwiddles layout);
// wLo / wHi the two-level table of W_M^e (e = e_hi 2^S + e_lo).
struct Tables {
    const float2* wL = nullptr;     // fused: length-M stages;  multipass: rows N2;  2-D: rows 2Ws
    const float2* wC = nullptr;     // multipass: columns N1;  2-D: columns 2Hs
    const float2* wLo = nullptr;    // multipass: W_M^e for e < 2^S
    const float2* wHi = nullptr;    // multipass: W_M^(e 2^S) for e < M / 2^S
};

// 3-D plans: the depth transform's stage table (2 Dd points).
struct Tables3 {
    const float2* wD = nullptr;
};

// Constant tables of the tensor-core path, in per-lane fragment order.
struct TcTablePtrs {
    const uint2* f16 = nullptr;   // [ntile 2][part 3][lane]        DFT_16 B fragments (Re, Im, -Im)
    const uint2* w256 = nullptr;  // [reg 4][lane]                  (cos, sin) pairs of W_256^{b c}
    const uint2* fp = nullptr;    // [kstep][ntile][part 3][lane]   outer DFT_P, p < P/2
    const uint2* fpi = nullptr;   // [kstep][ntile][part 3][lane]   outer inverse, conj(W_P^{k_p p}), p < P/2
    const uint2* tw1 = nullptr;   // [qt 16][ntile][half 2][lane]   (cos, sin) of W_M^{q k_p}
    const uint2* tw3 = nullptr;   // [k_p][reg 4][lane]             (cos, sin) of W_M^{q k_p}, q = 16 a + b
    const uint4* wr = nullptr;    // P >= 64: [plane 2][k_p][p < P/2] bf16 cos / -sin of W_P^{k_p p}
};

// Constant tables of the 2-D tensor-core column pass.
struct C2TcTables {
    const uint2* f16 = nullptr;     // DFT_16 B fragments (as TcTablePtrs::f16)
    const uint2* w256 = nullptr;    // W_256^{b c} pairs (as TcTablePtrs::w256)
    const uint2* t512 = nullptr;    // [reg 4][lane] (cos, sin) pairs of W_512^{i}, A-fragment order
    const float2* t512f = nullptr;  // [j 2][e 4][lane] (cos, sin) of W_512^{i}, accumulator order, fp32
};

}  // namespace fftc

struct fftconv_plan_s {
    int kind = 1;          // 1: 1-D, 2: 2-D, 3: state-space filters, chunked, 4: partial, chunked, 5: 3-D
    int path = 0;          // fftc::Path
    int B = 0, H = 0;      // 1-D batch, channels (2-D: B images, H = C channels)
    int64_t N = 0;         // 1-D sequence length
    int Hs = 0, Ws = 0;    // 2-D image size (3-D: the slices)
    int Dd = 0;            // 3-D depth
    int dtype = 0;         // fftconv_dtype
    int gated = 0;
    int log2M = 0;         // 1-D transform length 2N
    int log2N1 = 0;        // multipass: column transform length
    int log2N2 = 0;        // multipass: row transform length
    int log2S = 0;         // multipass: split of the two-level W_M table
    int group = 0;         // multipass / 2-D: pairs staged per group
    int64_t pairs = 0;     // (pairs of batch rows) x channels
    size_t spectrum_bytes = 0;
    size_t workspace_bytes = 0;
    void* d_tables = nullptr;
    fftc::Tables tw;
    fftc::Tables3 tw3;
    fftc::TcTablePtrs tc;
    bool umma = false;              // fused tensor-core path on tcgen05 (else mma.sync)
    bool t2 = false;                // two-stage tcgen05 kernel (2N = 8192)
    const uint4* t2_mats = nullptr; // its shared-memory matrix image
    const uint2* t2_twid = nullptr; // its twiddle pairs
    const void* umma_b = nullptr;   // tcgen05 path: B operand images of the DFT matrices
    int* d_err = nullptr;           // device status word: nonzero after a timed-out device wait
    bool tc2d = false;              // 2-D: column pass on the tensor cores (bf16, Hs = 256)
    // 2-D plans with one filter per image: the images run as channels of a
    // single-image batch (B = 1, C = B C of the caller), their spectra in the
    // head of the workspace
    bool dyn2d = false;
    int dynB = 0, dynC = 0;
    size_t dyn_spectrum_offset = 0;
    fftc::C2TcTables c2tc;
    bool spectrum_ready = false;
    int device = 0;
    int kernel = 0;                 // fftconv_kernel the caller asked for at creation
    uint32_t wait_limit = 1u << 16; // probes per bounded device wait (fftconv_plan_set_wait_limit)
    int kdiv = 1;                   // fused SIMT forward: row channels per spectrum channel
    // chunked state-passing plans (kind 3): the chunk plan and the filters' state-space model
    fftconv_plan_s* chunk = nullptr;  // fused plan of B x (H * nchunks) x T rows
    int d_state = 0;                  // states per channel
    int64_t T = 0, nchunks = 0;       // chunk length, chunks per row
    void* d_ssm = nullptr;            // plan-owned: lam, c, the power table (see conv1d_ssm.cu)
    bool ssm_ready = false;
    uint8_t* d_keep = nullptr;        // frequency-sparse multi-pass plans: keep flag per outer row k1
};

namespace fftc {

// Twiddle tables: each appends its geometry's stage tables to `out` and records
// their offsets (in float2 entries).  Returns false for an unsupported size.
bool fused_tables(int log2M, std::vector<float2>& out, size_t* offL);
bool multipass_tables(int log2M, std::vector<float2>& out, size_t* offC, size_t* offR);
bool conv2d_tables(int Hs, int Ws, std::vector<float2>& out, size_t* offR, size_t* offC);
bool conv3d_depth_tables(int Dd, std::vector<float2>& out, size_t* offD);
cudaError_t launch_conv3d_fwd(const fftconv_plan_s& p, const void* u, const float2* khat3, void* y, float2* work,
                              cudaStream_t s);
cudaError_t launch_conv3d_spectrum(const fftconv_plan_s& p, const float* k, int Kd, int Kh, int Kw, float2* khat3,
                                   float2* work, cudaStream_t s);

// 1-D bf16 two-stage tcgen05 path (2N = 8192, ungated): tables, spectrum
// (fp32 SIMT transform written in the kernel's bf16 layout), forward.
bool t2_supported(int log2M, int gated);
bool t2_tables(std::vector<float2>& out, size_t off[2]);
cudaError_t launch_t2_spectrum(const fftconv_plan_s& p, const float* k, int64_t L, void* khat, cudaStream_t s);
cudaError_t launch_t2_fwd(const fftconv_plan_s& p, const void* u, const void* khat, const float* D, void* y,
                          cudaStream_t s);

// Input-dependent filters, fused fp32 SIMT (2N <= 8192).
bool dyn_supported(int log2M);
cudaError_t launch_dyn_fwd(const fftconv_plan_s& p, const void* u, const void* v, const void* w, const float* k,
                           int64_t L, const float* D, void* y, cudaStream_t s);

// Chunked state passing for filters of a diagonal state-space model.
size_t ssm_block_bytes(int H, int d, int64_t T);
size_t ssm_workspace_bytes(const fftconv_plan_s& p);
cudaError_t launch_ssm_setup(const fftconv_plan_s& p, const float* lr, const float* li, const float* cr,
                             const float* ci, void* khat, void* work, cudaStream_t s);
cudaError_t launch_ssm_fwd(const fftconv_plan_s& p, const void* u, const void* khat, const float* D, void* y,
                           void* work, cudaStream_t s);

// Frequency-sparse multi-pass plans: zero the dropped spectrum rows.
cudaError_t launch_zero_spectrum_rows(const fftconv_plan_s& p, void* khat, cudaStream_t s);

// Partial convolutions (L <= T), overlap-save in chunks of T on the fused fp32 kernel.
cudaError_t launch_partial_fwd(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                               const float2* khat, const float* D, void* y, cudaStream_t s);

// Tensor-core flops of one forward call (0 for SIMT paths).
double plan_mma_flops(const fftconv_plan_s& p);

// 1-D bf16 tensor-core fused path (2N in {4096, 8192, 16384}).
bool tc_supported(int log2M);
bool tc_tables(int log2M, std::vector<float2>& out, size_t off[7]);
cudaError_t launch_tc_spectrum(const fftconv_plan_s& p, const float* k, int64_t L, void* khat, cudaStream_t s);
cudaError_t launch_tc_fwd(const fftconv_plan_s& p, const void* u, const void* v, const void* w, const void* khat,
                          const float* D, void* y, cudaStream_t s);

// 1-D bf16 fused path on tcgen05 (2N in {4096, 8192}); shares the spectrum
// layout and twiddle tables of the mma.sync path.
bool umma_supported(int log2M);
bool umma_bimages(int log2M, std::vector<float2>& out, size_t* off);
cudaError_t launch_umma_fwd(const fftconv_plan_s& p, const void* u, const void* v, const void* w, const void* khat,
                            const float* D, void* y, cudaStream_t s);

// 1-D fused path (one CTA per (pair of batch rows, channel)).
cudaError_t launch_fused_spectrum(const fftconv_plan_s& p, const float* k, int64_t L, float2* khat,
                                  cudaStream_t s);
cudaError_t launch_fused_fwd(const fftconv_plan_s& p, const void* u, const void* v, const void* w,
                             const float2* khat, const float* D, void* y, cudaStream_t s);

// 1-D multi-pass path (column DFT -> row DFT, product, inverse row DFT -> column iDFT).
cudaError_t launch_multipass_spectrum(const fftconv_plan_s& p, const float* k, int64_t L,
                                      float2* khat, float2* work, cudaStream_t s);
cudaError_t launch_multipass_fwd(const fftconv_plan_s& p, const void* u, const void* v,
                                 const void* w, const float2* khat, const float* D, void* y,
                                 float2* work, cudaStream_t s);

// 2-D column pass on the bf16 tensor cores (images of 256 rows); its spectrum
// is stored in per-lane fragment order.
bool c2tc_supported(int Hs, int Ws, int dtype);
bool c2tc_tables(std::vector<float2>& out, size_t off[4]);
cudaError_t launch_c2tc_cols(const fftconv_plan_s& p, float2* work, const void* khat, int g, int64_t first,
                             cudaStream_t s, int oy);
// the row passes too, for 256 x 256 images
bool c2tc_rows_supported(const fftconv_plan_s& p);
cudaError_t launch_c2tc_rows_fwd(const fftconv_plan_s& p, const void* u, float2* work, int g, int64_t first,
                                 cudaStream_t s);
cudaError_t launch_c2tc_rows_inv(const fftconv_plan_s& p, const float2* work, void* y, int g, int64_t first,
                                 cudaStream_t s, int ox);

// 2-D path (row DFT -> column DFT, product, inverse column DFT -> row iDFT).
cudaError_t launch_conv2d_spectrum(const fftconv_plan_s& p, const float* k, int Kh, int Kw,
                                   float2* khat, float2* work, cudaStream_t s);
cudaError_t launch_conv2d_fwd(const fftconv_plan_s& p, const void* u, const float2* khat, void* y,
                              float2* work, cudaStream_t s, int oy = 0, int ox = 0);

}  // namespace fftc
