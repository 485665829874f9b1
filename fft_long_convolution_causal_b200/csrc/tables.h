// tables.h -- host construction of the per-stage twiddle tables (fp64 -> fp32).
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <vector>

namespace fftc {

// exp(-2 pi i m / L) computed in fp64 with m reduced mod L, rounded to fp32.
inline float2 host_root(int64_t m, int64_t L) {
    int64_t e = m % L;
    if (e < 0) e += L;
    const double a = 2.0 * M_PI * (double)e / (double)L;
    return make_float2((float)cos(a), (float)-sin(a));
}

// Append the stage twiddles of geometry G in the order StageTwiddles<G> reads them.
template <class G>
void append_stage_twiddles(std::vector<float2>& out) {
    for (int s = 0; s < G::Plan::kStages; ++s) {
        const int64_t R = int64_t(1) << G::Plan::log2r(s), NS = int64_t(1) << G::Plan::log2ns(s);
        for (int64_t r = 0; r < R; ++r)
            for (int64_t k = 0; k < NS; ++k) out.push_back(host_root(r * k, NS * R));
    }
}

}  // namespace fftc
