// step.cuh -- cached single-token decode (Axon-SSM page, section
// "Autoregressive decoding"): per (b, e) read the K-1 cached inputs and the N
// float32 states, run one token of conv + SiLU + dt + recurrence + gate, write
// y, the shifted conv cache and the updated state in place.
//
// The step moves 148 bytes per channel at bf16, 128 of them the float32 state
// read and written back, and does 22 transcendentals per channel.  With the
// work spread thinly (one token), what limits it is the instructions issued
// per channel and the bytes each SM keeps in flight, so the kernel loads
// straight from global memory into registers, a round of four batch rows at a
// time, and keeps the per-row bookkeeping small.
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

constexpr int kStepThreads = 128;  // 32 channels x 4 lanes
constexpr int kStepChan = kStepThreads / 4;
constexpr int kStepMaxRows = 32;   // batch rows per block

// a raw io value as float (exact)
__device__ __forceinline__ float step_f(float v) { return v; }
__device__ __forceinline__ float step_f(__nv_bfloat16 v) { return __bfloat162float(v); }

// Four consecutive values of a B or C row (8 bytes at bf16, 16 at fp32), read
// through the non-coherent path: B and C are never written by the step.
template <class Io> struct StepQuad;
template <> struct StepQuad<IoBF16> {
    uint2 v;
    __device__ __forceinline__ void load(const void* row, int q) {
        v = __ldg(reinterpret_cast<const uint2*>(row) + q);
    }
    __device__ __forceinline__ void unpack(float (&r)[4]) const {
        r[0] = __uint_as_float(v.x << 16); r[1] = __uint_as_float(v.x & 0xffff0000u);
        r[2] = __uint_as_float(v.y << 16); r[3] = __uint_as_float(v.y & 0xffff0000u);
    }
};
template <> struct StepQuad<IoF32> {
    float4 v;
    __device__ __forceinline__ void load(const void* row, int q) {
        v = __ldg(reinterpret_cast<const float4*>(row) + q);
    }
    __device__ __forceinline__ void unpack(float (&r)[4]) const {
        r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
    }
};

// grid = (ceil(E / 32), ceil(B / rows)) blocks of 128 threads, rows <= 32.
// Lane (c, q) = thread 4c + q owns channel e0 + c and the state quadrant
// 4q .. 4q+3 (one 16-byte vector), so a warp's state traffic is one
// contiguous 512-byte run.  The block walks its rows in rounds of four:
//  - every lane loads the four rows' state vectors and B, C quadrants, and
//    the raw inputs (x, z, dt_raw, K-1 cached values) of round row q, all
//    issued before the first use, so they are in flight together;
//  - lane q runs the conv / SiLU / dt prologue and SiLU(z) of round row q; a
//    row's dt and input factor reach the other three lanes of the channel by
//    shuffles;
//  - each lane updates its quadrant of the four rows and stores the states;
//    the four per-quadrant partial C . h are summed by a two-step shuffle
//    reduce-scatter that leaves round row q's total on lane q, which writes
//    that row's y and shifted conv cache.
// State, cache and y are read and written by the same thread (plain loads:
// the state and cache are updated in place); lanes past E compute channel
// E-1 and store nothing.
template <class Io, bool kZoh>
__global__ void __launch_bounds__(kStepThreads) step_kernel(StepParams p, int rows) {
    using T = typename Io::T;
    constexpr int S = Io::kBytes;
    const int tid = threadIdx.x;
    const int q = tid & 3;
    const int e = blockIdx.x * kStepChan + (tid >> 2);
    const int b0 = blockIdx.y * rows;
    const int nb = min(rows, p.B - b0);
    const bool live = e < p.E;
    const int ec = live ? e : p.E - 1;
    const size_t E = (size_t)p.E;
    const size_t srow = E * kN;                       // floats between consecutive rows' states

    const float4 w = __ldg(reinterpret_cast<const float4*>(p.conv_w) + ec);
    const float cb = __ldg(p.conv_b + ec);
    const float db = __ldg(p.dt_bias + ec);
    const float Dv = __ldg(p.D + ec);
    float A2[4];
    {
        // exp(dt*A) = 2^(dt * A2) with A2 = A log2 e, A = -exp(A_log) = -2^(A_log log2 e)
        const float4 a4 = __ldg(reinterpret_cast<const float4*>(p.A_log + (size_t)ec * kN) + q);
        A2[0] = -ex2_approx(a4.x * kLog2e) * kLog2e;
        A2[1] = -ex2_approx(a4.y * kLog2e) * kLog2e;
        A2[2] = -ex2_approx(a4.z * kLog2e) * kLog2e;
        A2[3] = -ex2_approx(a4.w * kLog2e) * kLog2e;
    }
    const T* xg = static_cast<const T*>(p.x);
    const T* zg = static_cast<const T*>(p.z);
    const T* dg = static_cast<const T*>(p.dt_raw);
    T* cc = static_cast<T*>(p.conv_cache);
    T* yg = static_cast<T*>(p.y);
    const unsigned char* Bg = static_cast<const unsigned char*>(p.Bm);
    const unsigned char* Cg = static_cast<const unsigned char*>(p.Cm);

#pragma unroll 1
    for (int j0 = 0; j0 < nb; j0 += 4) {
        const int nr = min(4, nb - j0);               // rows of this round (block-uniform)
        // ---- loads of the round, all before the first use
        const size_t rq = (size_t)(b0 + j0 + min(q, nr - 1));   // this lane's prologue row
        const T xr = xg[rq * E + ec];                  // raw bits: also the cache's new last row
        const float z_t = Io::load(zg + rq * E + ec);
        const float d_t = Io::load(dg + rq * E + ec);
        T* ccq = cc + rq * (kK - 1) * E + ec;          // cache rows 0 .. K-2 of row rq
        const T c0 = ccq[0], c1 = ccq[E], c2 = ccq[2 * E];
        float* st = p.ssm_state + ((size_t)(b0 + j0) * E + ec) * kN + 4 * q;   // row j0's state vector
        const size_t bco = (size_t)(b0 + j0) * kN * S;                          // row j0's B / C row
        float4 hs[4];
        StepQuad<Io> Bq[4], Cq[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k < nr) {
                hs[k] = *reinterpret_cast<const float4*>(st + k * srow);
                Bq[k].load(Bg + bco + k * kN * S, q);
                Cq[k].load(Cg + bco + k * kN * S, q);
            }
        }
        // ---- prologue of row rq: conv over (cache 0, 1, 2, x_t), SiLU, dt, gate
        float xc = fmaf(w.x, step_f(c0), cb);
        xc = fmaf(w.y, step_f(c1), xc);
        xc = fmaf(w.z, step_f(c2), xc);
        xc = fmaf(w.w, step_f(xr), xc);
        const float uq = silu(xc);
        const float dtq = dt_from_raw(d_t + db);
        const float fq = kZoh ? uq : dtq * uq;        // input factor of Bbar u
        const float gzq = silu(z_t);
        // ---- the round's rows: quadrant update, state store, partial C . h
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k >= nr) break;                       // block-uniform
            const float dt = __shfl_sync(0xffffffffu, dtq, k, 4);
            const float f = __shfl_sync(0xffffffffu, fq, k, 4);
            float Bv[4], Cv[4];
            Bq[k].unpack(Bv);
            Cq[k].unpack(Cv);
            float h[4] = {hs[k].x, hs[k].y, hs[k].z, hs[k].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a = ex2_approx(dt * A2[i]);
                // first-order: (dt u) B;  ZOH: u ((exp(dt A) - 1) / A) B
                const float uin = kZoh ? f * zoh_bbar(dt, dt * A2[i] * kLn2, a, kLog2e / A2[i]) : f;
                h[i] = fmaf(a, h[i], uin * Bv[i]);
                acc[k] = fmaf(Cv[i], h[i], acc[k]);
            }
            if (live) *reinterpret_cast<float4*>(st + k * srow) = make_float4(h[0], h[1], h[2], h[3]);
        }
        // ---- reduce-scatter over the channel's four lanes: lanes with q & 2
        // keep rows 2, 3 (then q & 1 picks the odd row), so lane q ends with
        // the total of round row q
        const bool hi = (q & 2) != 0, lo = (q & 1) != 0;
        const float r0 = (hi ? acc[2] : acc[0]) + __shfl_xor_sync(0xffffffffu, hi ? acc[0] : acc[2], 2);
        const float r1 = (hi ? acc[3] : acc[1]) + __shfl_xor_sync(0xffffffffu, hi ? acc[1] : acc[3], 2);
        const float tot = (lo ? r1 : r0) + __shfl_xor_sync(0xffffffffu, lo ? r0 : r1, 1);
        if (live && q < nr) {
            Io::store(yg + rq * E + ec, fmaf(Dv, uq, tot) * gzq);
            // shifted cache: row i <- row i+1, the last <- x_t (raw bits)
            ccq[0] = c1;
            ccq[E] = c2;
            ccq[2 * E] = xr;
        }
    }
}

}  // namespace axon
