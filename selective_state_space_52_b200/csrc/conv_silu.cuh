// conv_silu.cuh -- the conv stage of the full layer on its own:
// u = SiLU(conv_b + sum_k conv_w[e,k] * x[t+k-(K-1)]), written in the io
// dtype.  It is the input of the projection to the SSM parameters (Axon-SSM
// page, "Selective mechanism": dt, B and C are projected from the conv
// output); the scan itself recomputes the same conv from x in registers.
#pragma once

#include "device_math.cuh"
#include "tc_ops.cuh"

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
constexpr int kConvCh = 4;       // channels per thread
constexpr int kConvThreads = 128;

// 4 consecutive io values <-> float32: one 8-byte vector at bf16, one
// 16-byte vector at fp32 (loads through the read-only path: x is never
// written by the kernel)
__device__ __forceinline__ void conv_ld4(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 q = __ldg(reinterpret_cast<const uint2*>(p));
    v[0] = __uint_as_float(q.x << 16);
    v[1] = __uint_as_float(q.x & 0xffff0000u);
    v[2] = __uint_as_float(q.y << 16);
    v[3] = __uint_as_float(q.y & 0xffff0000u);
}
__device__ __forceinline__ void conv_ld4(const float* p, float (&v)[4]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
__device__ __forceinline__ void conv_st4(__nv_bfloat16* p, const float (&v)[4]) {
    const __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<const uint32_t*>(&h0),
                                              *reinterpret_cast<const uint32_t*>(&h1));
}
__device__ __forceinline__ void conv_st4(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

// One thread: kConvCh consecutive channels of one batch row over kConvRun
// consecutive tokens, loaded and stored as whole vectors; the K-1 previous
// inputs of each channel slide in registers.  grid = (ceil(E/4 / 128),
// ceil(L / kConvRun), B).  E is a multiple of 8 and the rows 16-byte aligned.
// Four channels a thread rather than eight: about 60 registers instead of
// 104, twice the threads in flight to cover the loads' latency.  x and u
// never overlap (the layer's workspace holds them apart), so the loads of
// later tokens may run ahead of the stores of earlier ones: without that
// promise each token's load waited for the previous token's store, one
// memory latency per token.
template <class Io>
__global__ void __launch_bounds__(kConvThreads) conv_silu_kernel(ConvParams p) {
    using T = typename Io::T;
    grid_dep_launch();
    grid_dep_wait();
    const int g = blockIdx.x * kConvThreads + threadIdx.x;   // channel group
    if (g * kConvCh >= p.E) return;
    const int e0 = g * kConvCh;
    const int b = blockIdx.z;
    const int t0 = blockIdx.y * kConvRun;
    const int t1 = min(p.L, t0 + kConvRun);
    const T* __restrict__ x = static_cast<const T*>(p.x);
    const T* cc = static_cast<const T*>(p.conv_cache_in);
    T* __restrict__ u = static_cast<T*>(p.u);

    float w[kConvCh][kK], cbias[kConvCh], win[kK - 1][kConvCh];
#pragma unroll
    for (int c = 0; c < kConvCh; ++c) {
        const float4 wv = __ldg(reinterpret_cast<const float4*>(p.conv_w) + e0 + c);
        w[c][0] = wv.x; w[c][1] = wv.y; w[c][2] = wv.z; w[c][3] = wv.w;
        cbias[c] = __ldg(p.conv_b + e0 + c);
    }
    // the K-1 inputs before t0: x rows, or the cache (or zeros) before t = 0
#pragma unroll
    for (int j = 0; j < kK - 1; ++j) {
        const int t = t0 - (kK - 1) + j;
        if (t >= 0) conv_ld4(x + ((size_t)b * p.L + t) * p.E + e0, win[j]);
        else if (cc) conv_ld4(cc + ((size_t)b * (kK - 1) + (kK - 1 + t)) * p.E + e0, win[j]);
        else {
#pragma unroll
            for (int c = 0; c < kConvCh; ++c) win[j][c] = 0.0f;
        }
    }
    const T* __restrict__ row = x + ((size_t)b * p.L + t0) * p.E + e0;
    T* __restrict__ out = u + ((size_t)b * p.L + t0) * p.E + e0;
#pragma unroll 8
    for (int t = t0; t < t1; ++t, row += p.E, out += p.E) {
        float xt[kConvCh], o[kConvCh];
        conv_ld4(row, xt);
#pragma unroll
        for (int c = 0; c < kConvCh; ++c) {
            float xc = fmaf(w[c][0], win[0][c], cbias[c]);
            xc = fmaf(w[c][1], win[1][c], xc);
            xc = fmaf(w[c][2], win[2][c], xc);
            xc = fmaf(w[c][3], xt[c], xc);
            win[0][c] = win[1][c]; win[1][c] = win[2][c]; win[2][c] = xt[c];
            o[c] = silu(xc);
        }
        conv_st4(out, o);
    }
}

}  // namespace axon
