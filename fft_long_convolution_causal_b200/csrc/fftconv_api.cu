// fftconv_api.cu -- the extern "C" boundary declared in include/fftconv.h:
// argument checks, path selection, twiddle tables, dispatch to the kernels.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <new>
#include <vector>

#include "fftconv.h"
#include "plan.h"

namespace {

// Largest transform the fused kernel holds in shared memory (complex fp32).
constexpr int kFusedMaxLog2M = 14;
// Workspace of one multi-pass / 2-D group: the pairs a pass covers per
// launch.  Measured on B200 (same box, both builds): fewer, larger launches
// beat groups sized to stay in L2 -- 1 GiB against 64 MiB is 14% faster at
// N = 2^20 and 17% faster on 256 x 256 images.  The plan option group_bytes
// overrides it (smaller workspaces; the tests use it to run several groups).
size_t group_bytes(const fftconv_plan_options& o) { return o.group_bytes ? o.group_bytes : size_t(1) << 30; }

fftconv_plan_options defaults() {
    fftconv_plan_options o;
    o.kernel = FFTCONV_KERNEL_AUTO;
    o.group_bytes = 0;
    return o;
}

bool valid_options(const fftconv_plan_options& o) {
    return o.kernel >= FFTCONV_KERNEL_AUTO && o.kernel <= FFTCONV_KERNEL_TCGEN05;
}

// The plan's device must be current for every call that launches on it.
bool on_plan_device(const fftconv_plan_s* p) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return dev == p->device;
}

bool is_pow2(int64_t x) { return x > 0 && (x & (x - 1)) == 0; }
int log2i(int64_t x) {
    int r = 0;
    while ((int64_t(1) << r) < x) ++r;
    return r;
}
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// exp(-2 pi i m / L), m in [0, count), computed in fp64 and rounded to fp32.
void fill_roots(std::vector<float2>& out, int64_t L, int64_t count, int64_t stride = 1) {
    for (int64_t m = 0; m < count; ++m) {
        const int64_t e = (m * stride) % L;
        const double a = 2.0 * M_PI * (double)e / (double)L;
        out.push_back(make_float2((float)cos(a), (float)-sin(a)));
    }
}

fftconv_status upload_tables(fftconv_plan_s* p, const std::vector<float2>& host) {
    void* d = nullptr;
    if (cudaMalloc(&d, host.size() * sizeof(float2)) != cudaSuccess) {
        cudaGetLastError();
        return FFTCONV_ERR_OOM;
    }
    if (cudaMemcpy(d, host.data(), host.size() * sizeof(float2), cudaMemcpyHostToDevice) != cudaSuccess) {
        cudaFree(d);
        cudaGetLastError();
        return FFTCONV_ERR_CUDA;
    }
    p->d_tables = d;
    return FFTCONV_OK;
}

// A zeroed 16-byte slot at the end of the tables for the device status word.
size_t append_status_word(std::vector<float2>& host) {
    if (host.size() % 2) host.push_back(make_float2(0.f, 0.f));
    const size_t off = host.size();
    host.push_back(make_float2(0.f, 0.f));
    host.push_back(make_float2(0.f, 0.f));
    return off;
}

fftconv_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return FFTCONV_OK;
    return FFTCONV_ERR_CUDA;
}

}  // namespace

namespace fftc {

// Tensor-core multiply-adds of one forward call, from each kernel's structure
// (every product as issued, K padding included), times 2.
double plan_mma_flops(const fftconv_plan_s& p) {
    double mac_pair = 0.0;
    if (p.path == PATH_FUSED_TC) {
        if (p.t2) {
            // two-stage kernel (2N = 128 x 64): four stages of 128 x 128 x 128 real
            // products per pair (stage A and the last inverse stage as 128 x 64 halves)
            mac_pair = 4.0 * 128 * 128 * 128;
        } else {
            // outer DFT_P over p < P/2 (K padded to 16), the 16 x 16 inner 256-point
            // DFT forward and inverse per row k_p, outer inverse to p < P/2; complex
            // products as four real ones
            const double P = (double)((int64_t(1) << p.log2M) / 256);
            const double kp1 = P / 2 < 16 ? 16 : P / 2;
            mac_pair = 4.0 * 256 * (P * kp1 + (P / 2) * P) + 65536.0 * P;
        }
    } else if (p.path == PATH_2D && p.tc2d) {
        // per 512-point line with 256 nonzero (or kept) points: two 256-point
        // 16 x 16 DFTs of 2 x 4 x 16^3 real multiply-adds each
        const double line = 2.0 * 2 * 4 * 4096;
        const double cols = 2.0 * p.Ws * 2 * line;  // forward and inverse per column
        const double rows = (p.Ws == 256) ? 2.0 * 256 * line : 0.0;
        mac_pair = cols + rows;
    }
    return 2.0 * mac_pair * (double)p.pairs;
}

}  // namespace fftc

extern "C" {

const char* fftconv_status_string(fftconv_status s) {
    switch (s) {
        case FFTCONV_OK: return "ok";
        case FFTCONV_ERR_INVALID_ARG: return "invalid argument";
        case FFTCONV_ERR_UNSUPPORTED: return "unsupported size";
        case FFTCONV_ERR_NOT_READY: return "kernel spectrum not computed for this plan";
        case FFTCONV_ERR_OOM: return "out of device memory";
        case FFTCONV_ERR_CUDA: return "CUDA error";
        case FFTCONV_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

int fftconv_version(void) { return 200; }

void fftconv_plan_options_init(fftconv_plan_options* opts) {
    if (opts) *opts = defaults();
}

fftconv_status fftconv_plan_create(fftconv_plan_t* out, int B, int H, int64_t N, fftconv_dtype dtype,
                                   int gated) {
    return fftconv_plan_create_ex(out, B, H, N, dtype, gated, nullptr);
}

fftconv_status fftconv_plan_create_ex(fftconv_plan_t* out, int B, int H, int64_t N, fftconv_dtype dtype,
                                      int gated, const fftconv_plan_options* opts) {
    if (!out) return FFTCONV_ERR_INVALID_ARG;
    *out = nullptr;
    const fftconv_plan_options o = opts ? *opts : defaults();
    if (!valid_options(o)) return FFTCONV_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || (dtype != FFTCONV_F32 && dtype != FFTCONV_BF16)) return FFTCONV_ERR_INVALID_ARG;
    if (!is_pow2(N) || N < FFTCONV_MIN_N || N > FFTCONV_MAX_N) return FFTCONV_ERR_UNSUPPORTED;
    fftconv_plan_s* p = new (std::nothrow) fftconv_plan_s();
    if (!p) return FFTCONV_ERR_OOM;
    p->kind = 1;
    p->B = B;
    p->H = H;
    p->N = N;
    p->dtype = dtype;
    p->gated = gated ? 1 : 0;
    p->log2M = log2i(2 * N);
    p->pairs = (int64_t)((B + 1) / 2) * H;
    p->kernel = o.kernel;
    cudaGetDevice(&p->device);
    std::vector<float2> host;
    const int64_t M = int64_t(1) << p->log2M;
    size_t offL = 0, offC = 0, offLo = 0, offHi = 0, offTc[7] = {0, 0, 0, 0, 0, 0, 0}, offU = 0, offT2[2] = {0, 0};
    const bool use_tc = dtype == FFTCONV_BF16 && fftc::tc_supported(p->log2M) && o.kernel != FFTCONV_KERNEL_SIMT;
    if (use_tc && (o.kernel == FFTCONV_KERNEL_AUTO || o.kernel == FFTCONV_KERNEL_TCGEN05) &&
        fftc::t2_supported(p->log2M, p->gated)) {
        // two-stage tcgen05 kernel, data in tensor memory between the stages (the
        // fastest measured at 2N = 8192: 72.4 us against 88.8-97 us for the
        // mma.sync kernel on the Hyena-style workload)
        p->path = fftc::PATH_FUSED_TC;
        p->t2 = true;
        fftc::fused_tables(p->log2M, host, &offL);  // stage tables of the SIMT spectrum transform
        fftc::t2_tables(host, offT2);
        p->spectrum_bytes = (size_t)H * M * sizeof(uint32_t);  // bf16 Re pairs and -Im pairs per row k_p
        p->workspace_bytes = 0;
    } else if (use_tc) {
        p->path = fftc::PATH_FUSED_TC;
        fftc::fused_tables(p->log2M, host, &offL);  // stage tables of the spectrum transform
        fftc::tc_tables(p->log2M, host, offTc);
        // the tcgen05 kernel of the same factorisation: on request only (the
        // mma.sync kernel measured faster at these sizes)
        if (fftc::umma_supported(p->log2M) && o.kernel == FFTCONV_KERNEL_TCGEN05) {
            p->umma = true;
            fftc::umma_bimages(p->log2M, host, &offU);
        }
        p->spectrum_bytes = (size_t)H * M * sizeof(uint32_t);  // bf16 (re, im) in fragment order
        p->workspace_bytes = 0;
    } else if (p->log2M <= kFusedMaxLog2M) {
        p->path = fftc::PATH_FUSED;
        fftc::fused_tables(p->log2M, host, &offL);
        p->spectrum_bytes = (size_t)H * M * sizeof(float2);
        p->workspace_bytes = 0;
    } else {
        p->path = fftc::PATH_MULTIPASS;
        p->log2N1 = p->log2M / 2 < 9 ? p->log2M / 2 : 9;  // columns of at most 512 points (32 per CTA)
        p->log2N2 = p->log2M - p->log2N1;
        p->log2S = (p->log2M + 1) / 2;
        const int64_t S = int64_t(1) << p->log2S;
        fftc::multipass_tables(p->log2M, host, &offC, &offL);
        offLo = host.size();
        fill_roots(host, M, S);                   // wLo: W_M^e, e < S
        offHi = host.size();
        fill_roots(host, M, M / S, S);            // wHi: W_M^(e S)
        const size_t per_pair = (size_t)M * sizeof(float2);
        int64_t g = (int64_t)(group_bytes(o) / per_pair);
        if (g < 1) g = 1;
        const int64_t most = p->pairs > H ? p->pairs : H;
        if (g > most) g = most;
        p->group = (int)g;
        p->spectrum_bytes = (size_t)H * M * sizeof(float2);
        p->workspace_bytes = (size_t)g * per_pair;
    }
    const size_t offErr = append_status_word(host);
    fftconv_status st = upload_tables(p, host);
    if (st != FFTCONV_OK) {
        delete p;
        return st;
    }
    const float2* base = (const float2*)p->d_tables;
    p->d_err = (int*)(base + offErr);
    if (p->umma) p->umma_b = base + offU;
    if (p->t2) {
        p->t2_mats = (const uint4*)(base + offT2[0]);
        p->t2_twid = (const uint2*)(base + offT2[1]);
    }
    p->tw.wL = base + offL;
    if (p->path == fftc::PATH_MULTIPASS) {
        p->tw.wC = base + offC;
        p->tw.wLo = base + offLo;
        p->tw.wHi = base + offHi;
    }
    if (p->path == fftc::PATH_FUSED_TC && !p->t2) {
        p->tc.f16 = (const uint2*)(base + offTc[0]);
        p->tc.w256 = (const uint2*)(base + offTc[1]);
        p->tc.fp = (const uint2*)(base + offTc[2]);
        p->tc.fpi = (const uint2*)(base + offTc[3]);
        p->tc.tw1 = (const uint2*)(base + offTc[4]);
        p->tc.tw3 = (const uint2*)(base + offTc[5]);
        p->tc.wr = (const uint4*)(base + offTc[6]);
    }
    *out = p;
    return FFTCONV_OK;
}

fftconv_status fftconv2d_plan_create(fftconv_plan_t* out, int B, int C, int Hs, int Ws, fftconv_dtype dtype) {
    return fftconv2d_plan_create_ex(out, B, C, Hs, Ws, dtype, nullptr);
}

fftconv_status fftconv2d_plan_create_ex(fftconv_plan_t* out, int B, int C, int Hs, int Ws, fftconv_dtype dtype,
                                        const fftconv_plan_options* opts) {
    if (!out) return FFTCONV_ERR_INVALID_ARG;
    *out = nullptr;
    const fftconv_plan_options o = opts ? *opts : defaults();
    if (!valid_options(o)) return FFTCONV_ERR_INVALID_ARG;
    if (B < 1 || C < 1 || (dtype != FFTCONV_F32 && dtype != FFTCONV_BF16)) return FFTCONV_ERR_INVALID_ARG;
    if (!is_pow2(Hs) || !is_pow2(Ws) || Hs < FFTCONV2D_MIN_SIDE || Ws < FFTCONV2D_MIN_SIDE ||
        Hs > FFTCONV2D_MAX_SIDE || Ws > FFTCONV2D_MAX_SIDE)
        return FFTCONV_ERR_UNSUPPORTED;
    fftconv_plan_s* p = new (std::nothrow) fftconv_plan_s();
    if (!p) return FFTCONV_ERR_OOM;
    p->kind = 2;
    p->path = fftc::PATH_2D;
    p->B = B;
    p->H = C;
    p->Hs = Hs;
    p->Ws = Ws;
    p->dtype = dtype;
    p->pairs = (int64_t)((B + 1) / 2) * C;
    p->kernel = o.kernel;
    cudaGetDevice(&p->device);
    const int64_t LR = 2 * (int64_t)Ws, LC = 2 * (int64_t)Hs;
    std::vector<float2> host;
    size_t offR = 0, offC = 0, offT[4] = {0, 0, 0, 0};
    fftc::conv2d_tables(Hs, Ws, host, &offR, &offC);
    if (fftc::c2tc_supported(Hs, Ws, dtype) && o.kernel != FFTCONV_KERNEL_SIMT) {
        p->tc2d = true;
        fftc::c2tc_tables(host, offT);
    }
    const size_t offErr = append_status_word(host);
    const size_t per_pair = (size_t)Hs * LR * sizeof(float2);
    int64_t g = (int64_t)(group_bytes(o) / per_pair);
    // whole channels per group: a channel's pairs then run together and share
    // the channel's spectrum in L2
    const int64_t npp = (B + 1) / 2;
    if (g >= npp) g -= g % npp;
    if (g < 1) g = 1;
    const int64_t most = p->pairs > C ? p->pairs : C;
    if (g > most) g = most;
    p->group = (int)g;
    // bf16 plans keep the spectrum as packed bf16 (re, im), fp32 plans as fp32 complex
    p->spectrum_bytes = (size_t)C * LC * LR * (dtype == FFTCONV_BF16 ? sizeof(uint32_t) : sizeof(float2));
    p->workspace_bytes = (size_t)g * per_pair;
    fftconv_status st = upload_tables(p, host);
    if (st != FFTCONV_OK) {
        delete p;
        return st;
    }
    p->tw.wL = (const float2*)p->d_tables + offR;
    p->tw.wC = (const float2*)p->d_tables + offC;
    p->d_err = (int*)((const float2*)p->d_tables + offErr);
    if (p->tc2d) {
        const float2* base = (const float2*)p->d_tables;
        p->c2tc.f16 = (const uint2*)(base + offT[0]);
        p->c2tc.w256 = (const uint2*)(base + offT[1]);
        p->c2tc.t512 = (const uint2*)(base + offT[2]);
        p->c2tc.t512f = base + offT[3];
    }
    *out = p;
    return FFTCONV_OK;
}

fftconv_status fftconv_plan_destroy(fftconv_plan_t p) {
    if (!p) return FFTCONV_OK;
    cudaError_t e = cudaSuccess;
    if (p->d_tables) e = cudaFree(p->d_tables);
    if (p->d_ssm && cudaFree(p->d_ssm) != cudaSuccess) e = cudaErrorUnknown;
    if (p->d_keep && cudaFree(p->d_keep) != cudaSuccess) e = cudaErrorUnknown;
    if (p->chunk && fftconv_plan_destroy(p->chunk) != FFTCONV_OK) e = cudaErrorUnknown;
    delete p;
    return e == cudaSuccess ? FFTCONV_OK : FFTCONV_ERR_CUDA;
}

fftconv_status fftconv_ssm_plan_create(fftconv_plan_t* out, int B, int H, int64_t N, fftconv_dtype dtype,
                                       int d_state, int64_t chunk) {
    if (!out) return FFTCONV_ERR_INVALID_ARG;
    *out = nullptr;
    if (B < 1 || H < 1 || (dtype != FFTCONV_F32 && dtype != FFTCONV_BF16)) return FFTCONV_ERR_INVALID_ARG;
    if (d_state < 1 || d_state > FFTCONV_SSM_MAX_STATE) return FFTCONV_ERR_INVALID_ARG;
    if (!is_pow2(chunk) || chunk < FFTCONV_SSM_MIN_CHUNK || chunk > FFTCONV_SSM_MAX_CHUNK) return FFTCONV_ERR_UNSUPPORTED;
    if (N < chunk || N % chunk != 0 || N / chunk > 65535) return FFTCONV_ERR_UNSUPPORTED;
    const int64_t nc = N / chunk;
    if ((int64_t)H * nc > 65535) return FFTCONV_ERR_UNSUPPORTED;
    // the chunk plan: bf16 chunks of 4096 (2T = 8192) on the two-stage tensor-core
    // kernel, every other chunk size on the fp32 fused kernel
    fftconv_plan_options o = defaults();
    const bool tc_chunks = dtype == FFTCONV_BF16 && chunk == 4096;
    o.kernel = tc_chunks ? FFTCONV_KERNEL_TCGEN05 : FFTCONV_KERNEL_SIMT;
    fftconv_plan_t ch = nullptr;
    fftconv_status st = fftconv_plan_create_ex(&ch, B, (int)(H * nc), chunk, dtype, 0, &o);
    if (st != FFTCONV_OK) return st;
    if (tc_chunks ? !ch->t2 : ch->path != fftc::PATH_FUSED) {
        fftconv_plan_destroy(ch);
        return FFTCONV_ERR_UNSUPPORTED;
    }
    ch->kdiv = (int)nc;
    fftconv_plan_s* p = new (std::nothrow) fftconv_plan_s();
    if (!p) {
        fftconv_plan_destroy(ch);
        return FFTCONV_ERR_OOM;
    }
    p->kind = 3;
    p->path = fftc::PATH_SSM;
    p->B = B;
    p->H = H;
    p->N = N;
    p->dtype = dtype;
    p->pairs = (int64_t)((B + 1) / 2) * H;
    p->chunk = ch;
    p->d_state = d_state;
    p->T = chunk;
    p->nchunks = nc;
    p->device = ch->device;
    p->d_err = ch->d_err;
    if (cudaMalloc(&p->d_ssm, fftc::ssm_block_bytes(H, d_state, chunk)) != cudaSuccess) {
        cudaGetLastError();
        p->d_ssm = nullptr;
        fftconv_plan_destroy(p);
        return FFTCONV_ERR_OOM;
    }
    p->spectrum_bytes = (size_t)H * 2 * chunk * sizeof(float2);
    p->workspace_bytes = fftc::ssm_workspace_bytes(*p);
    *out = p;
    return FFTCONV_OK;
}

int fftconv_spectrum_blocks(fftconv_plan_t p) {
    return (p && p->kind == 1 && p->path == fftc::PATH_MULTIPASS) ? (1 << p->log2N1) : 0;
}

fftconv_status fftconv_spectrum_sparsify(fftconv_plan_t p, void* khat, const uint8_t* keep, int nblocks,
                                         void* stream) {
    if (!p || !khat || !aligned16(khat)) return FFTCONV_ERR_INVALID_ARG;
    if (p->kind != 1 || p->path != fftc::PATH_MULTIPASS) return FFTCONV_ERR_UNSUPPORTED;
    if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (!keep) {  // dense again (the spectrum must be recomputed to undo the zeroing)
        if (nblocks != 0) return FFTCONV_ERR_INVALID_ARG;
        if (p->d_keep) {
            if (cudaStreamSynchronize(s) != cudaSuccess || cudaFree(p->d_keep) != cudaSuccess) {
                cudaGetLastError();
                return FFTCONV_ERR_CUDA;
            }
            p->d_keep = nullptr;
        }
        return FFTCONV_OK;
    }
    const int G = 1 << p->log2N1;
    if (nblocks != G) return FFTCONV_ERR_INVALID_ARG;
    for (int j = 0; j < G; ++j)  // Hermitian symmetry keeps the packed rows apart
        if ((keep[j] != 0) != (keep[(G - j) % G] != 0)) return FFTCONV_ERR_INVALID_ARG;
    if (!p->d_keep && cudaMalloc(&p->d_keep, (size_t)G) != cudaSuccess) {
        cudaGetLastError();
        p->d_keep = nullptr;
        return FFTCONV_ERR_OOM;
    }
    std::vector<uint8_t> flags(G);
    for (int j = 0; j < G; ++j) flags[j] = keep[j] ? 1 : 0;
    if (cudaMemcpyAsync(p->d_keep, flags.data(), (size_t)G, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return FFTCONV_ERR_CUDA;
    }
    return cuda_status(fftc::launch_zero_spectrum_rows(*p, khat, s));
}

fftconv_status fftconv_partial_plan_create(fftconv_plan_t* out, int B, int H, int64_t N, fftconv_dtype dtype,
                                           int gated, int64_t L_max) {
    if (!out) return FFTCONV_ERR_INVALID_ARG;
    *out = nullptr;
    if (B < 1 || H < 1 || L_max < 1 || (dtype != FFTCONV_F32 && dtype != FFTCONV_BF16)) return FFTCONV_ERR_INVALID_ARG;
    int64_t T = 64;
    while (T < L_max) T <<= 1;
    if (T > FFTCONV_PARTIAL_MAX_CHUNK || N < T || N % T != 0 || N / T > 65535) return FFTCONV_ERR_UNSUPPORTED;
    const int64_t nc = N / T;
    if ((int64_t)H * nc > 65535) return FFTCONV_ERR_UNSUPPORTED;
    fftconv_plan_options o = defaults();
    o.kernel = FFTCONV_KERNEL_SIMT;
    fftconv_plan_t ch = nullptr;  // the tables of the 2T-point transform
    fftconv_status st = fftconv_plan_create_ex(&ch, 1, H, T, dtype, 0, &o);
    if (st != FFTCONV_OK) return st;
    if (ch->path != fftc::PATH_FUSED) {
        fftconv_plan_destroy(ch);
        return FFTCONV_ERR_UNSUPPORTED;
    }
    fftconv_plan_s* p = new (std::nothrow) fftconv_plan_s();
    if (!p) {
        fftconv_plan_destroy(ch);
        return FFTCONV_ERR_OOM;
    }
    p->kind = 4;
    p->path = fftc::PATH_PARTIAL;
    p->B = B;
    p->H = H;
    p->N = N;
    p->dtype = dtype;
    p->gated = gated ? 1 : 0;
    p->pairs = (int64_t)((B + 1) / 2) * H;
    p->chunk = ch;
    p->T = T;
    p->nchunks = nc;
    p->device = ch->device;
    p->d_err = ch->d_err;
    p->spectrum_bytes = (size_t)H * 2 * T * sizeof(float2);
    p->workspace_bytes = 0;
    *out = p;
    return FFTCONV_OK;
}

fftconv_status fftconv_ssm_spectrum(fftconv_plan_t p, const float* lam_re, const float* lam_im, const float* c_re,
                                    const float* c_im, void* khat, void* work, void* stream) {
    if (!p || p->kind != 3 || !lam_re || !lam_im || !c_re || !c_im || !khat || !work) return FFTCONV_ERR_INVALID_ARG;
    if (!aligned16(khat) || !aligned16(work)) return FFTCONV_ERR_INVALID_ARG;
    if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
    const cudaError_t e = fftc::launch_ssm_setup(*p, lam_re, lam_im, c_re, c_im, khat, work, (cudaStream_t)stream);
    if (e == cudaSuccess) p->spectrum_ready = true;
    return cuda_status(e);
}

size_t fftconv_spectrum_bytes(fftconv_plan_t p) { return p ? p->spectrum_bytes : 0; }
size_t fftconv_workspace_bytes(fftconv_plan_t p) { return p ? p->workspace_bytes : 0; }

const char* fftconv_plan_path(fftconv_plan_t p) {
    if (!p) return "none";
    switch (p->path) {
        case fftc::PATH_FUSED: return "fused";
        case fftc::PATH_FUSED_TC: return p->t2 ? "fused_t2" : (p->umma ? "fused_umma" : "fused_tc");
        case fftc::PATH_MULTIPASS: return "multipass";
        case fftc::PATH_2D: return p->tc2d ? "2d_tc" : "2d";
        case fftc::PATH_SSM: return "ssm_chunked";
        case fftc::PATH_PARTIAL: return "partial_chunked";
        case fftc::PATH_3D: return "3d";
    }
    return "unknown";
}

fftconv_status fftconv_kernel_spectrum(fftconv_plan_t p, const float* k, int64_t L, void* khat, void* work,
                                       void* stream) {
    if (p && p->kind == 4) {
        // partial plans: the 2T-point spectrum of k[:L], L <= T
        if (!k || !khat || L < 1 || L > p->T || !aligned16(k) || !aligned16(khat)) return FFTCONV_ERR_INVALID_ARG;
        if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
        const cudaError_t e = fftc::launch_fused_spectrum(*p->chunk, k, L, (float2*)khat, (cudaStream_t)stream);
        if (e == cudaSuccess) p->spectrum_ready = true;
        return cuda_status(e);
    }
    if (!p || p->kind != 1 || !k || !khat || L < 1 || L > p->N) return FFTCONV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(khat)) return FFTCONV_ERR_INVALID_ARG;
    if (p->workspace_bytes && (!work || !aligned16(work))) return FFTCONV_ERR_INVALID_ARG;
    if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (p->t2)
        e = fftc::launch_t2_spectrum(*p, k, L, khat, s);
    else if (p->path == fftc::PATH_FUSED_TC)
        e = fftc::launch_tc_spectrum(*p, k, L, khat, s);
    else if (p->path == fftc::PATH_FUSED)
        e = fftc::launch_fused_spectrum(*p, k, L, (float2*)khat, s);
    else
        e = fftc::launch_multipass_spectrum(*p, k, L, (float2*)khat, (float2*)work, s);
    if (e == cudaSuccess) p->spectrum_ready = true;
    return cuda_status(e);
}

fftconv_status fftconv_fwd(fftconv_plan_t p, const void* u, const void* v, const void* w, const void* khat,
                           const float* D, void* y, void* work, void* stream) {
    if (!p || (p->kind != 1 && p->kind != 3 && p->kind != 4) || !u || !khat || !y) return FFTCONV_ERR_INVALID_ARG;
    if (p->gated ? (!v || !w) : (v || w)) return FFTCONV_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(khat) || !aligned16(y) || (v && !aligned16(v)) || (w && !aligned16(w)) ||
        (D && !aligned16(D)))
        return FFTCONV_ERR_INVALID_ARG;
    if (p->workspace_bytes && (!work || !aligned16(work))) return FFTCONV_ERR_INVALID_ARG;
    if (y == u || y == v || y == w) return FFTCONV_ERR_INVALID_ARG;
    if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
    if (!p->spectrum_ready) return FFTCONV_ERR_NOT_READY;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    if (p->kind == 3)
        e = fftc::launch_ssm_fwd(*p, u, khat, D, y, work, s);
    else if (p->kind == 4)
        e = fftc::launch_partial_fwd(*p, u, v, w, (const float2*)khat, D, y, s);
    else if (p->t2)
        e = fftc::launch_t2_fwd(*p, u, khat, D, y, s);
    else if (p->path == fftc::PATH_FUSED_TC)
        e = p->umma ? fftc::launch_umma_fwd(*p, u, v, w, khat, D, y, s) : fftc::launch_tc_fwd(*p, u, v, w, khat, D, y, s);
    else if (p->path == fftc::PATH_FUSED)
        e = fftc::launch_fused_fwd(*p, u, v, w, (const float2*)khat, D, y, s);
    else
        e = fftc::launch_multipass_fwd(*p, u, v, w, (const float2*)khat, D, y, (float2*)work, s);
    return cuda_status(e);
}

fftconv_status fftconv_fwd_dynamic(fftconv_plan_t p, const void* u, const void* v, const void* w, const float* k,
                                   int64_t L, const float* D, void* y, void* stream) {
    if (!p || p->kind != 1 || !u || !k || !y) return FFTCONV_ERR_INVALID_ARG;
    if (p->gated ? (!v || !w) : (v || w)) return FFTCONV_ERR_INVALID_ARG;
    if (L < 1 || L > p->N) return FFTCONV_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(k) || !aligned16(y) || (v && !aligned16(v)) || (w && !aligned16(w)) ||
        (D && !aligned16(D)))
        return FFTCONV_ERR_INVALID_ARG;
    if (y == u || y == v || y == w) return FFTCONV_ERR_INVALID_ARG;
    if (!fftc::dyn_supported(p->log2M) || p->path == fftc::PATH_MULTIPASS) return FFTCONV_ERR_UNSUPPORTED;
    if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
    return cuda_status(fftc::launch_dyn_fwd(*p, u, v, w, k, L, D, y, (cudaStream_t)stream));
}

fftconv_status fftconv2d_kernel_spectrum(fftconv_plan_t p, const float* k, int Kh, int Kw, void* khat, void* work,
                                         void* stream) {
    if (!p || p->kind != 2 || !k || !khat || !work) return FFTCONV_ERR_INVALID_ARG;
    if (Kh < 1 || Kw < 1 || Kh > p->Hs || Kw > p->Ws) return FFTCONV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(khat) || !aligned16(work)) return FFTCONV_ERR_INVALID_ARG;
    if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
    cudaError_t e = fftc::launch_conv2d_spectrum(*p, k, Kh, Kw, (float2*)khat, (float2*)work, (cudaStream_t)stream);
    if (e == cudaSuccess) p->spectrum_ready = true;
    return cuda_status(e);
}

fftconv_status fftconv2d_dynamic_plan_create(fftconv_plan_t* out, int B, int C, int Hs, int Ws,
                                             fftconv_dtype dtype) {
    if (!out) return FFTCONV_ERR_INVALID_ARG;
    *out = nullptr;
    if (B < 1 || C < 1 || (int64_t)B * C > (int64_t)1 << 30) return FFTCONV_ERR_INVALID_ARG;
    fftconv_plan_t p = nullptr;
    fftconv_status st = fftconv2d_plan_create_ex(&p, 1, B * C, Hs, Ws, dtype, nullptr);
    if (st != FFTCONV_OK) return st;
    p->dyn2d = true;
    p->dynB = B;
    p->dynC = C;
    // workspace: [the images' spectra][the passes' workspace]
    p->dyn_spectrum_offset = (p->spectrum_bytes + 255) & ~size_t(255);
    p->workspace_bytes += p->dyn_spectrum_offset;
    *out = p;
    return FFTCONV_OK;
}

fftconv_status fftconv2d_fwd_dynamic(fftconv_plan_t p, const void* u, const float* k, int Kh, int Kw, void* y,
                                     void* work, void* stream) {
    if (!p || p->kind != 2 || !p->dyn2d || !u || !k || !y || !work) return FFTCONV_ERR_INVALID_ARG;
    if (Kh < 1 || Kw < 1 || Kh > p->Hs || Kw > p->Ws) return FFTCONV_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(k) || !aligned16(y) || !aligned16(work)) return FFTCONV_ERR_INVALID_ARG;
    if (y == u) return FFTCONV_ERR_INVALID_ARG;
    if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    float2* khat = (float2*)work;
    float2* rest = (float2*)((uint8_t*)work + p->dyn_spectrum_offset);
    // every image's filter is a channel of the single-image batch: its spectrum, then the forward
    cudaError_t e = fftc::launch_conv2d_spectrum(*p, k, Kh, Kw, khat, rest, s);
    if (e == cudaSuccess) e = fftc::launch_conv2d_fwd(*p, u, khat, y, rest, s, 0, 0);
    return cuda_status(e);
}

fftconv_status fftconv3d_plan_create(fftconv_plan_t* out, int B, int C, int Dd, int Hs, int Ws, fftconv_dtype dtype) {
    if (!out) return FFTCONV_ERR_INVALID_ARG;
    *out = nullptr;
    if (B < 1 || C < 1 || (dtype != FFTCONV_F32 && dtype != FFTCONV_BF16)) return FFTCONV_ERR_INVALID_ARG;
    if ((int64_t)C * Dd > (int64_t)1 << 30) return FFTCONV_ERR_INVALID_ARG;
    auto side_ok = [](int x) { return is_pow2(x) && x >= FFTCONV3D_MIN_SIDE && x <= FFTCONV3D_MAX_SIDE; };
    if (!side_ok(Dd) || !side_ok(Hs) || !side_ok(Ws)) return FFTCONV_ERR_UNSUPPORTED;
    fftconv_plan_s* p = new (std::nothrow) fftconv_plan_s();
    if (!p) return FFTCONV_ERR_OOM;
    p->kind = 5;
    p->path = fftc::PATH_3D;
    p->B = B;
    p->H = C;
    p->Dd = Dd;
    p->Hs = Hs;
    p->Ws = Ws;
    p->dtype = dtype;
    p->pairs = (int64_t)((B + 1) / 2) * C;
    cudaGetDevice(&p->device);
    const int64_t LR = 2 * (int64_t)Ws, LC = 2 * (int64_t)Hs, LD = 2 * (int64_t)Dd;
    std::vector<float2> host;
    size_t offR = 0, offC = 0, offD = 0;
    fftc::conv2d_tables(Hs, Ws, host, &offR, &offC);
    fftc::conv3d_depth_tables(Dd, host, &offD);
    const size_t offErr = append_status_word(host);
    // workspace per channel: its slice pairs' row spectra (Hs x LR) and column spectra (LC x LR)
    const size_t per_channel = (size_t)Dd * ((B + 1) / 2) * (size_t)(Hs + LC) * LR * sizeof(float2);
    int64_t g = (int64_t)(group_bytes(defaults()) / per_channel);
    if (g < 1) g = 1;
    if (g > C) g = C;
    p->group = (int)g;
    p->spectrum_bytes = (size_t)C * LD * LC * LR * sizeof(float2);
    p->workspace_bytes = (size_t)g * per_channel;
    fftconv_status st = upload_tables(p, host);
    if (st != FFTCONV_OK) {
        delete p;
        return st;
    }
    const float2* base = (const float2*)p->d_tables;
    p->tw.wL = base + offR;
    p->tw.wC = base + offC;
    p->tw3.wD = base + offD;
    p->d_err = (int*)(base + offErr);
    *out = p;
    return FFTCONV_OK;
}

fftconv_status fftconv3d_kernel_spectrum(fftconv_plan_t p, const float* k, int Kd, int Kh, int Kw, void* khat,
                                         void* work, void* stream) {
    if (!p || p->kind != 5 || !k || !khat || !work) return FFTCONV_ERR_INVALID_ARG;
    if (Kd < 1 || Kh < 1 || Kw < 1 || Kd > p->Dd || Kh > p->Hs || Kw > p->Ws) return FFTCONV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(khat) || !aligned16(work)) return FFTCONV_ERR_INVALID_ARG;
    if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
    cudaError_t e =
        fftc::launch_conv3d_spectrum(*p, k, Kd, Kh, Kw, (float2*)khat, (float2*)work, (cudaStream_t)stream);
    if (e == cudaSuccess) p->spectrum_ready = true;
    return cuda_status(e);
}

fftconv_status fftconv3d_fwd(fftconv_plan_t p, const void* u, const void* khat, void* y, void* work, void* stream) {
    if (!p || p->kind != 5 || !u || !khat || !y || !work) return FFTCONV_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(khat) || !aligned16(y) || !aligned16(work)) return FFTCONV_ERR_INVALID_ARG;
    if (y == u) return FFTCONV_ERR_INVALID_ARG;
    if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
    if (!p->spectrum_ready) return FFTCONV_ERR_NOT_READY;
    return cuda_status(
        fftc::launch_conv3d_fwd(*p, u, (const float2*)khat, y, (float2*)work, (cudaStream_t)stream));
}

fftconv_status fftconv2d_fwd(fftconv_plan_t p, const void* u, const void* khat, void* y, void* work, void* stream) {
    return fftconv2d_fwd_offset(p, u, khat, y, work, stream, 0, 0);
}

fftconv_status fftconv2d_fwd_offset(fftconv_plan_t p, const void* u, const void* khat, void* y, void* work,
                                    void* stream, int oy, int ox) {
    if (!p || p->kind != 2 || !u || !khat || !y || !work) return FFTCONV_ERR_INVALID_ARG;
    if (oy < 0 || ox < 0 || oy > p->Hs || ox > p->Ws || (oy % 8) || (ox % 8)) return FFTCONV_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(khat) || !aligned16(y) || !aligned16(work)) return FFTCONV_ERR_INVALID_ARG;
    if (y == u) return FFTCONV_ERR_INVALID_ARG;
    if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
    if (!p->spectrum_ready) return FFTCONV_ERR_NOT_READY;
    return cuda_status(
        fftc::launch_conv2d_fwd(*p, u, (const float2*)khat, y, (float2*)work, (cudaStream_t)stream, oy, ox));
}

fftconv_status fftconv_plan_set_wait_limit(fftconv_plan_t p, uint32_t probes) {
    if (!p) return FFTCONV_ERR_INVALID_ARG;
    p->wait_limit = probes;
    if (p->chunk) p->chunk->wait_limit = probes;  // chunked plans launch their chunk plan's kernels
    return FFTCONV_OK;
}

double fftconv_plan_mma_flops(fftconv_plan_t p) { return p ? fftc::plan_mma_flops(*p) : 0.0; }

fftconv_status fftconv_device_status(fftconv_plan_t p, void* stream) {
    if (!p || !p->d_err) return FFTCONV_ERR_INVALID_ARG;
    if (!on_plan_device(p)) return FFTCONV_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return FFTCONV_ERR_CUDA;
    int word = 0;
    if (cudaMemcpy(&word, p->d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FFTCONV_ERR_CUDA;
    if (word == 0) return FFTCONV_OK;
    const int zero = 0;
    if (cudaMemcpy(p->d_err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return FFTCONV_ERR_CUDA;
    return FFTCONV_ERR_TIMEOUT;
}

}  // extern "C"
