// probe.cuh -- throughput probes for the roofline's compute denominators,
// measured in the same run as the kernels they rate: the MUFU exp2 rate (the
// prefill's binding unit: 22 transcendentals per token and channel, Axon-SSM
// page, "ZOH discretisation" and "Gating") and the float32 FMA rate.
//
// Every thread runs kProbeChains independent dependency chains for `iters`
// iterations, enough chains and warps to keep the unit busy; the results are
// summed into one float per thread so the work cannot be dropped.
#pragma once

#include "device_math.cuh"

namespace axon {

constexpr int kProbeChains = 8;

// kind 0: y = ex2.approx(y * c), one MUFU op (and one FMUL) per chain step;
// kind 1: y = fma(y, a, b), one FFMA per chain step.
template <int kKind>
__global__ void __launch_bounds__(256) peak_probe_kernel(float* out, long long iters) {
    float y[kProbeChains];
#pragma unroll
    for (int i = 0; i < kProbeChains; ++i) y[i] = 0.001f * (threadIdx.x + i);
    for (long long it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < kProbeChains; ++i) {
            if constexpr (kKind == 0) y[i] = ex2_approx(y[i] * -0.5f);
            else y[i] = fmaf(y[i], 0.999f, 0.001f);
        }
    }
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < kProbeChains; ++i) s += y[i];
    out[(size_t)blockIdx.x * blockDim.x + threadIdx.x] = s;
}

}  // namespace axon
