// noalloc.cu -- multi-pass forward that needs no caller-provided workspace.
//
// Some callers cannot call cudaMalloc when they run the convolution: code that
// executes inside a region where device allocation is forbidden or would
// synchronise the device (a latency-critical loop, a host callback, a
// framework that owns every allocation through its own pool and hands out no
// scratch).  For them, fftconv_fwd_static_workspace runs the multi-pass path
// with its scratch held in a file-scope device array of a fixed size instead
// of a workspace argument.  It allocates nothing.
//
// The array lives in every GPU that loads this library until the process
// exits.  Its address is looked up once per device, on that device's first
// call, with the device current (cudaGetSymbolAddress); make that first call
// before any stream capture.  All calls share the one array: two calls whose
// work overlaps on the GPU (different streams, or different host threads)
// race on it and corrupt each other's results; serialise them.  The kernels
// overwrite every scratch element they read within the same call (pass 1
// writes what pass 2 reads, pass 2 writes what pass 3 reads), so nothing
// needs clearing between calls.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "fftconv.h"
#include "plan.h"

// the scratch array itself: file scope, internal linkage
static __device__ __align__(256) uint8_t g_static_scratch[FFTCONV_STATIC_WORKSPACE_BYTES];

namespace {

constexpr size_t kStaticScratchBytes = FFTCONV_STATIC_WORKSPACE_BYTES;

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up once).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

fftconv_status fftconv_fwd_static_workspace(fftconv_plan_t p, const void* u, const void* v, const void* w,
                                            const void* khat, const float* D, void* y, void* stream) {
    if (!p || p->kind != 1 || !u || !khat || !y) return FFTCONV_ERR_INVALID_ARG;
    if (p->path != fftc::PATH_MULTIPASS) return FFTCONV_ERR_UNSUPPORTED;
    if (p->gated ? (!v || !w) : (v || w)) return FFTCONV_ERR_INVALID_ARG;
    if (!aligned16(u) || !aligned16(khat) || !aligned16(y) || (v && !aligned16(v)) || (w && !aligned16(w)) ||
        (D && !aligned16(D)))
        return FFTCONV_ERR_INVALID_ARG;
    if (y == u || y == v || y == w) return FFTCONV_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return FFTCONV_ERR_CUDA;
    }
    if (dev != p->device) return FFTCONV_ERR_INVALID_ARG;  // the plan's tables live on its own device
    if (!p->spectrum_ready) return FFTCONV_ERR_NOT_READY;
    // one pair of rows needs a full transform of length 2N in fp32 complex
    const size_t per_pair = (size_t(1) << p->log2M) * sizeof(float2);
    if (per_pair > kStaticScratchBytes) return FFTCONV_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) {
        cudaGetLastError();
        return FFTCONV_ERR_CUDA;
    }
    // same kernels as fftconv_fwd; only the group of pairs staged at once is
    // sized to the static array (a stack copy of the plan, nothing allocated)
    fftconv_plan_s q = *p;
    int64_t g = (int64_t)(kStaticScratchBytes / per_pair);
    if (g > q.pairs) g = q.pairs;
    q.group = (int)g;
    const cudaError_t e = fftc::launch_multipass_fwd(q, u, v, w, (const float2*)khat, D, y, (float2*)scratch,
                                                     (cudaStream_t)stream);
    return e == cudaSuccess ? FFTCONV_OK : FFTCONV_ERR_CUDA;
}

size_t fftconv_static_workspace_bytes(void) { return kStaticScratchBytes; }

}  // extern "C"
