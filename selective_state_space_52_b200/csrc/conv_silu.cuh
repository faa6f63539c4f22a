// conv_silu.cuh -- the conv stage of the full layer on its own:
// u = SiLU(conv_b + sum_k conv_w[e,k] * x[t+k-(K-1)]), written in the io
// dtype.  It is the input of the projection to the SSM parameters (Axon-SSM
// page, "Selective mechanism": dt, B and C are projected from the conv
// output); the scan itself recomputes the same conv from x in registers.
#pragma once

#include "device_math.cuh"

namespace axon {

struct ConvParams {
    int B, L, E;
    const void* x;               // (B, L, E) io
    const float* conv_w;         // (E, K)
    const float* conv_b;         // (E)
    const void* conv_cache_in;   // (B, K-1, E) io, may be null (zeros)
    void* u;                     // (B, L, E) io
};

constexpr int kConvRun = 32;     // tokens per thread
constexpr int kConvThreads = 128;

// One thread: 8 consecutive channels (one 16-byte bf16 vector, two fp32
// vectors) of one batch row over kConvRun consecutive tokens; the K-1 previous
// inputs of each channel slide in registers.  grid = (ceil(E/8 / 128),
// ceil(L / kConvRun), B).  E is a multiple of 8.
template <class Io>
__global__ void __launch_bounds__(kConvThreads) conv_silu_kernel(ConvParams p) {
    using T = typename Io::T;
    const int g8 = blockIdx.x * kConvThreads + threadIdx.x;   // channel group
    if (g8 * 8 >= p.E) return;
    const int e0 = g8 * 8;
    const int b = blockIdx.z;
    const int t0 = blockIdx.y * kConvRun;
    const int t1 = min(p.L, t0 + kConvRun);
    const T* x = static_cast<const T*>(p.x);
    const T* cc = static_cast<const T*>(p.conv_cache_in);
    T* u = static_cast<T*>(p.u);

    float w[8][kK], cbias[8], win[8][kK - 1];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float4 wv = __ldg(reinterpret_cast<const float4*>(p.conv_w) + e0 + c);
        w[c][0] = wv.x; w[c][1] = wv.y; w[c][2] = wv.z; w[c][3] = wv.w;
        cbias[c] = __ldg(p.conv_b + e0 + c);
    }
    // the K-1 inputs before t0: x rows, or the cache (or zeros) before t = 0
#pragma unroll
    for (int j = 0; j < kK - 1; ++j) {
        const int t = t0 - (kK - 1) + j;
        const T* row = nullptr;
        if (t >= 0) row = x + ((size_t)b * p.L + t) * p.E + e0;
        else if (cc) row = cc + ((size_t)b * (kK - 1) + (kK - 1 + t)) * p.E + e0;
#pragma unroll
        for (int c = 0; c < 8; ++c) win[c][j] = row ? Io::load(row + c) : 0.0f;
    }
    for (int t = t0; t < t1; ++t) {
        const T* row = x + ((size_t)b * p.L + t) * p.E + e0;
        T* out = u + ((size_t)b * p.L + t) * p.E + e0;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float xt = Io::load(row + c);
            float xc = fmaf(w[c][0], win[c][0], cbias[c]);
            xc = fmaf(w[c][1], win[c][1], xc);
            xc = fmaf(w[c][2], win[c][2], xc);
            xc = fmaf(w[c][3], xt, xc);
            win[c][0] = win[c][1]; win[c][1] = win[c][2]; win[c][2] = xt;
            Io::store(out + c, silu(xc));
        }
    }
}

}  // namespace axon
