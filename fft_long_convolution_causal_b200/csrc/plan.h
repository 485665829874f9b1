// plan.h -- internal plan object and kernel launchers (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "fftconv.h"

namespace fftc {

enum Path { PATH_FUSED = 0, PATH_MULTIPASS = 1, PATH_2D = 2 };

// Twiddle tables of one plan (device pointers into one allocation).  A table
// "W_L" holds exp(-2 pi i m / L) for m in [0, L), rounded from fp64.
struct Tables {
    const float2* wL = nullptr;     // fused: W_M;  multipass: W_N2 (rows);  2-D: W_{2Ws}
    const float2* wC = nullptr;     // multipass: W_N1 (columns);  2-D: W_{2Hs}
    const float2* wLo = nullptr;    // multipass: W_M^e for e < 2^S
    const float2* wHi = nullptr;    // multipass: W_M^(e 2^S) for e < M / 2^S
};

}  // namespace fftc

struct fftconv_plan_s {
    int kind = 1;          // 1: 1-D, 2: 2-D
    int path = 0;          // fftc::Path
    int B = 0, H = 0;      // 1-D batch, channels (2-D: B images, H = C channels)
    int64_t N = 0;         // 1-D sequence length
    int Hs = 0, Ws = 0;    // 2-D image size
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
    bool spectrum_ready = false;
    int device = 0;
};

namespace fftc {

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

// 2-D path (row DFT -> column DFT, product, inverse column DFT -> row iDFT).
cudaError_t launch_conv2d_spectrum(const fftconv_plan_s& p, const float* k, int Kh, int Kw,
                                   float2* khat, float2* work, cudaStream_t s);
cudaError_t launch_conv2d_fwd(const fftconv_plan_s& p, const void* u, const float2* khat, void* y,
                              float2* work, cudaStream_t s);

}  // namespace fftc
