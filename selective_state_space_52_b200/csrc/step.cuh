// step.cuh -- cached single-token decode (Axon-SSM page, section
// "Autoregressive decoding"): per (b, e) read the K-1 cached inputs and the N
// float32 states, run one token of conv + SiLU + dt + recurrence + gate, write
// y, the shifted conv cache and the updated state in place.
//
// The step is bound by HBM traffic on the state read-modify-write (2 x 64 bytes
// per channel of the 148 bytes it moves at bf16).  Four lanes share a channel:
// each owns four consecutive states (one 16-byte vector), so a warp's state
// load/store is one contiguous 512-byte run, and the C contraction is finished
// with two butterfly shuffles.  The cheap per-channel prologue is recomputed
// by the four lanes instead of being broadcast.
#pragma once

#include "device_math.cuh"

namespace axon {

struct StepParams {
    int B, E;
    const void* x;
    const void* z;
    const void* dt_raw;
    const void* Bm;
    const void* Cm;
    const float* conv_w;
    const float* conv_b;
    const float* dt_bias;
    const float* A_log;
    const float* D;
    void* conv_cache;
    float* ssm_state;
    void* y;
};

// grid = ceil(B*E*4 / 256) blocks of 256 threads; thread -> (channel, quarter).
template <class Io>
__global__ void __launch_bounds__(256) step_kernel(StepParams p) {
    using T = typename Io::T;
    const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long nch = (long long)p.B * p.E;
    // Every lane stays to the end so that the full-warp shuffles below are
    // defined; lanes past the last channel compute channel 0 and store nothing.
    const bool valid = (gid >> 2) < nch;
    const long long ch = valid ? (gid >> 2) : 0;   // flattened (b, e)
    const int q = (int)(gid & 3);                  // states 4q .. 4q+3
    const int b = (int)(ch / p.E);
    const int e = (int)(ch - (long long)b * p.E);

    // conv window: oldest first, then this token
    T* cc = static_cast<T*>(p.conv_cache) + (size_t)b * (kK - 1) * p.E + e;
    const float c0 = Io::load_rw(cc);
    const float c1 = Io::load_rw(cc + p.E);
    const float c2 = Io::load_rw(cc + 2 * (size_t)p.E);
    const size_t io_off = (size_t)b * p.E + e;
    const float xt = Io::load(static_cast<const T*>(p.x) + io_off);
    const float zt = Io::load(static_cast<const T*>(p.z) + io_off);
    const float dr = Io::load(static_cast<const T*>(p.dt_raw) + io_off);

    const float4 w = __ldg(reinterpret_cast<const float4*>(p.conv_w) + e);
    float xc = fmaf(w.x, c0, __ldg(p.conv_b + e));
    xc = fmaf(w.y, c1, xc);
    xc = fmaf(w.z, c2, xc);
    xc = fmaf(w.w, xt, xc);
    const float u = silu(xc);
    const float dt = dt_from_raw(dr + __ldg(p.dt_bias + e));
    const float dtu = dt * u;

    // this lane's four states and their B, C, A entries
    float Bv[4], Cv[4], A2[4];
    {
        const float4 al = __ldg(reinterpret_cast<const float4*>(p.A_log + (size_t)e * kN) + q);
        A2[0] = -expf(al.x) * kLog2e; A2[1] = -expf(al.y) * kLog2e;
        A2[2] = -expf(al.z) * kLog2e; A2[3] = -expf(al.w) * kLog2e;
        const T* Bs = static_cast<const T*>(p.Bm) + (size_t)b * kN + 4 * q;
        const T* Cs = static_cast<const T*>(p.Cm) + (size_t)b * kN + 4 * q;
#pragma unroll
        for (int j = 0; j < 4; ++j) { Bv[j] = Io::load(Bs + j); Cv[j] = Io::load(Cs + j); }
    }
    float4* sp = reinterpret_cast<float4*>(p.ssm_state + ((size_t)b * p.E + e) * kN) + q;
    float4 hv = *sp;
    float h[4] = {hv.x, hv.y, hv.z, hv.w};
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float a = ex2_approx(dt * A2[j]);
        h[j] = fmaf(a, h[j], dtu * Bv[j]);
        acc = fmaf(Cv[j], h[j], acc);
    }
    if (valid) *sp = make_float4(h[0], h[1], h[2], h[3]);
    // sum over the four lanes of this channel (lanes 4c .. 4c+3 of the warp)
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (valid && q == 0) {
        const float yv = fmaf(__ldg(p.D + e), u, acc) * silu(zt);
        Io::store(static_cast<T*>(p.y) + io_off, yv);
        // shift the cache: drop the oldest input, append x_t (exact copies)
        Io::store(cc, c1);
        Io::store(cc + p.E, c2);
        Io::store(cc + 2 * (size_t)p.E, xt);
    }
}

}  // namespace axon
