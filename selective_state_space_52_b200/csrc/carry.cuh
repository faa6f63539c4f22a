// carry.cuh -- the pieces of a sequence split across devices by time: per
// slice, the sum of its step sizes (its decay over the slice is
// exp(A * sum dt)), and the fold of the slices' summaries into the state that
// enters a slice.  The chunked associative scan of the SSD article (intra-block
// pass, inter-block carry), with devices as the blocks; the recurrence is the
// Axon-SSM page's, whose decay over a run of tokens is exp(A * sum dt).
#pragma once

#include "device_math.cuh"

namespace axon {

constexpr int kDtSumThreads = 128;
constexpr int kDtSumRun = 256;   // tokens per thread

// out[b, e] += sum over the thread's run of clip(softplus(dt_raw + dt_bias)).
// grid = (ceil(E / 128), ceil(L / 256), B); out zeroed by the caller first.
template <class Io>
__global__ void __launch_bounds__(kDtSumThreads) dt_sum_kernel(int L, int E, const void* dt_raw,
                                                             const float* dt_bias, float* out) {
    using T = typename Io::T;
    const int e = blockIdx.x * kDtSumThreads + threadIdx.x;
    if (e >= E) return;
    const int b = blockIdx.z;
    const int t0 = blockIdx.y * kDtSumRun;
    const int t1 = min(L, t0 + kDtSumRun);
    const T* d = static_cast<const T*>(dt_raw) + ((size_t)b * L) * E + e;
    const float bias = __ldg(dt_bias + e);
    float s = 0.0f;
    for (int t = t0; t < t1; ++t) s += dt_from_raw(Io::load(d + (size_t)t * E) + bias);
    atomicAdd(out + (size_t)b * E + e, s);
}

// h_in of slice r: h = h_end of slice 0 (computed from the true initial
// state), then for j = 1 .. r-1: h = exp(A * dtsum_j) * h + h_loc_j (slice j's
// end state from a zero state).  One thread per (b, e, n); h_loc (P,B,E,N),
// dtsum (P,B,E), out (B,E,N).
__global__ void __launch_bounds__(128) carry_fold_kernel(int r, int B, int E, const float* A_log,
                                                         const float* h_loc, const float* dtsum,
                                                         float* out) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t total = (size_t)B * E * kN;
    if (i >= total) return;
    const size_t be = i / kN;
    const int e = (int)(be % E);
    const int n = (int)(i % kN);
    const float A = -expf(__ldg(A_log + (size_t)e * kN + n));
    float h = h_loc[i];                                   // slice 0
    for (int j = 1; j < r; ++j)
        h = fmaf(expf(A * dtsum[(size_t)j * B * E + be]), h, h_loc[(size_t)j * total + i]);
    out[i] = h;
}

}  // namespace axon
