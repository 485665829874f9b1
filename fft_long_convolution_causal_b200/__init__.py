"""B200-native causal FFT long convolution.

y[b,h,:] = irfft(rfft(u[b,h,:], 2N) * rfft(k[h,:], 2N))[:N] + D[h] u[b,h,:],
its gated form y = v * ((u * w) conv k), and a 2-D zero-padded variant, computed
by hand-written sm_100a CUDA kernels behind the C ABI declared in
``include/fftconv.h``.  This package is the thin Python binding (argument
marshalling only) plus the seeded workload generator.

The CUDA library is loaded on first use; if it is missing the call raises.
"""
from . import workloads  # noqa: F401  (pure numpy, no arithmetic of the method)

_BINDING_NAMES = {
    "Plan", "Plan2D", "Plan2DDynamic", "Plan3D", "PartialPlan", "SSMPlan", "PlanOptions",
    "load_library", "library_path", "FFTConvError", "fftconv", "fftconv2d", "status_string",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
