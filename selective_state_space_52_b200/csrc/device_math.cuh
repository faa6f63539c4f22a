// device_math.cuh -- float32 building blocks of the selective-scan layer core
// for sm_100a: the MUFU exp2/log2/reciprocal instructions, SiLU, the clipped
// softplus step size, and io-dtype loads/stores.
//
// Math follows the page "Axon-SSM: Selective State Space Model for Apple
// Silicon": SiLU gating (section "Gating"), dt = clip(softplus(dt_raw + b_dt),
// 1e-4, 100) (section "Selective mechanism"), abar = exp(dt*A) with
// A = -exp(A_log) (sections "ZOH discretisation", "Diagonal state matrix").
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace axon {

constexpr float kLog2e = 1.4426950408889634f;   // log2(e)
constexpr float kLn2 = 0.6931471805599453f;     // ln(2)
constexpr float kDtMin = 1e-4f;                 // epsilon of the dt clip
constexpr float kDtMax = 100.0f;                // dt_max of the dt clip
constexpr int kN = 16;                          // state size N
constexpr int kK = 4;                           // conv taps K

// Hardware (MUFU) approximations, issued directly as PTX instructions.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x for a pair of x <= 0 on the FMA pipe (packed float32 pairs), for
// kernels whose MUFU pipe is the busiest: Cody and Waite's reduction
// 2^x = 2^n 2^f, n = round(x), f = x - n in [-1/2, 1/2] (exact: adding
// 1.5 * 2^23 rounds to an integer, subtracting it back and then n from x are
// exact), 2^f by the degree-6 polynomial with constant term 1 (2^0 is exactly
// 1, a masked token's decay) minimising the largest relative error on
// [-1/2, 1/2] (Remez exchange; coefficients from
// selective_state_space_52_b200/exp2_poly_fit.py, rounded to float32; the
// float32 evaluation stays within 1.3 * 2^-24 relative), and 2^n added to the
// exponent field (n << 23: the low 9 bits of 1.5 * 2^23 are zero, so the
// sum's bit pattern shifted left by 23 is n << 23).  x is clamped at -126, so
// the result stays a normal float (2^-126 where MUFU's ftz form gives 0).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
    constexpr float kRound = 12582912.0f;            // 1.5 * 2^23
    const float2 xc = make_float2(fmaxf(x.x, -126.0f), fmaxf(x.y, -126.0f));
    const float2 j = __fadd2_rn(xc, make_float2(kRound, kRound));
    const float2 n = __fadd2_rn(j, make_float2(-kRound, -kRound));
    const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), xc);
    float2 p = make_float2(0x1.446c7ep-13f, 0x1.446c7ep-13f);
    p = __ffma2_rn(p, f, make_float2(0x1.5f88fep-10f, 0x1.5f88fep-10f));
    p = __ffma2_rn(p, f, make_float2(0x1.3b29e4p-7f, 0x1.3b29e4p-7f));
    p = __ffma2_rn(p, f, make_float2(0x1.c6ae2cp-5f, 0x1.c6ae2cp-5f));
    p = __ffma2_rn(p, f, make_float2(0x1.ebfbe0p-3f, 0x1.ebfbe0p-3f));
    p = __ffma2_rn(p, f, make_float2(0x1.62e432p-1f, 0x1.62e432p-1f));
    p = __ffma2_rn(p, f, make_float2(1.0f, 1.0f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(j.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(j.y) << 23)));
}

// SiLU(v) = v * sigmoid(v) = v / (1 + 2^(-v log2 e)).  For v -> -inf the
// exponential overflows to +inf and the reciprocal to 0, giving -0.
__device__ __forceinline__ float silu(float v) {
    return v * rcp_approx(1.0f + ex2_approx(-v * kLog2e));
}

// log(1 + e) for e in [0, 1].  Below 2^-6 the first four terms of the Taylor
// series e - e^2/2 + e^3/3 - e^4/4 are used (truncation below e^5/5, i.e. under
// 2^-26 relative); above it, log2(1 + e) * ln 2, where rounding 1 + e costs at
// most 2^-24 / log(1 + 2^-6) ~ 4e-6 relative.
__device__ __forceinline__ float log1p_unit(float e) {
    const float series = e * (1.0f - e * (0.5f - e * (0.33333334f - e * 0.25f)));
    const float viaLog = lg2_approx(1.0f + e) * kLn2;
    return e < 0.015625f ? series : viaLog;
}

// softplus(v) = max(v, 0) + log(1 + exp(-|v|)), overflow-free.
__device__ __forceinline__ float softplus(float v) {
    const float e = ex2_approx(-fabsf(v) * kLog2e);
    return fmaxf(v, 0.0f) + log1p_unit(e);
}

// dt = clip(softplus(v), 1e-4, 100), bounds inclusive.
__device__ __forceinline__ float dt_from_raw(float v) {
    return fminf(fmaxf(softplus(v), kDtMin), kDtMax);
}

// silu and dt_from_raw on a pair of values (two tokens), with the products,
// sums and polynomial on the paired float32 pipe (FMUL2 / FADD2 / FFMA2) and
// the roundings the scalar forms above compile to (the series as three FMAs),
// so a pair gives what two scalar calls give.
__device__ __forceinline__ float2 silu2(float2 v) {
    const float2 a = __fmul2_rn(v, make_float2(-kLog2e, -kLog2e));
    const float2 d = __fadd2_rn(make_float2(ex2_approx(a.x), ex2_approx(a.y)), make_float2(1.0f, 1.0f));
    return __fmul2_rn(v, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}
__device__ __forceinline__ float2 dt_from_raw2(float2 v) {
    const float2 a = __fmul2_rn(make_float2(fabsf(v.x), fabsf(v.y)), make_float2(-kLog2e, -kLog2e));
    const float2 e = make_float2(ex2_approx(a.x), ex2_approx(a.y));
    float2 r = __ffma2_rn(e, make_float2(-0.25f, -0.25f), make_float2(0.33333334f, 0.33333334f));
    r = __ffma2_rn(e, r, make_float2(-0.5f, -0.5f));
    r = __ffma2_rn(e, r, make_float2(1.0f, 1.0f));
    const float2 series = __fmul2_rn(e, r);
    const float2 onep = __fadd2_rn(e, make_float2(1.0f, 1.0f));
    const float2 via = __fmul2_rn(make_float2(lg2_approx(onep.x), lg2_approx(onep.y)), make_float2(kLn2, kLn2));
    const float2 l = make_float2(e.x < 0.015625f ? series.x : via.x, e.y < 0.015625f ? series.y : via.y);
    const float2 sp = __fadd2_rn(make_float2(fmaxf(v.x, 0.0f), fmaxf(v.y, 0.0f)), l);
    return make_float2(fminf(fmaxf(sp.x, kDtMin), kDtMax), fminf(fmaxf(sp.y, kDtMin), kDtMax));
}

// Exact zero-order-hold input factor (Axon-SSM page, "ZOH discretisation"):
// Bbar = (exp(dt A) - 1) / A * B.  With x = dt*A <= 0 and a = exp(x) already
// evaluated, this returns Bbar / B = dt * phi(x), phi(x) = expm1(x) / x:
//   |x| < 1/16: dt * (1 + x/2 + x^2/6 + x^3/24 + x^4/120)  (Taylor; the
//               truncation x^5/720 stays below 2e-9 relative), so the
//               cancellation in a - 1 for small |x| never enters;
//   otherwise:  (a - 1) * (1/A), where a - 1 <= -0.06 keeps its relative error
//               near that of a.
__device__ __forceinline__ float zoh_bbar(float dt, float x, float a, float invA) {
    const float series = dt * fmaf(x, fmaf(x, fmaf(x, fmaf(x, 1.0f / 120.0f, 1.0f / 24.0f), 1.0f / 6.0f), 0.5f), 1.0f);
    const float direct = (a - 1.0f) * invA;
    return fabsf(x) < 0.0625f ? series : direct;
}

// ---------------------------------------------------------------- io dtypes
struct IoF32 {
    using T = float;
    static constexpr int kBytes = 4;
    __device__ __forceinline__ static float load(const T* p) { return __ldg(p); }
    __device__ __forceinline__ static float load_rw(const T* p) { return *p; }
    __device__ __forceinline__ static void store(T* p, float v) { *p = v; }
    // one value / four consecutive values (16-byte aligned) from shared memory
    __device__ __forceinline__ static float sload(const void* p) { return *reinterpret_cast<const float*>(p); }
    __device__ __forceinline__ static void sload4(const void* p, float (&r)[4]) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        r[0] = v.x; r[1] = v.y; r[2] = v.z; r[3] = v.w;
    }
    // 16 consecutive values of a B/C row (64 bytes, 16-byte aligned).
    __device__ __forceinline__ static void load_row16(const T* p, float (&r)[kN]) {
        const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float4 v = __ldg(q + i);
            r[4 * i + 0] = v.x; r[4 * i + 1] = v.y; r[4 * i + 2] = v.z; r[4 * i + 3] = v.w;
        }
    }
};

struct IoBF16 {
    using T = __nv_bfloat16;
    static constexpr int kBytes = 2;
    __device__ __forceinline__ static float bits_to_f(uint32_t b16) {
        return __uint_as_float(b16 << 16);
    }
    __device__ __forceinline__ static float load(const T* p) {
        return bits_to_f(__ldg(reinterpret_cast<const unsigned short*>(p)));
    }
    __device__ __forceinline__ static float load_rw(const T* p) {
        return bits_to_f(*reinterpret_cast<const unsigned short*>(p));
    }
    __device__ __forceinline__ static void store(T* p, float v) { *p = __float2bfloat16_rn(v); }
    // one value / four consecutive values (8-byte aligned) from shared memory
    __device__ __forceinline__ static float sload(const void* p) {
        return bits_to_f(*reinterpret_cast<const unsigned short*>(p));
    }
    __device__ __forceinline__ static void sload4(const void* p, float (&r)[4]) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        r[0] = __uint_as_float(v.x << 16); r[1] = __uint_as_float(v.x & 0xffff0000u);
        r[2] = __uint_as_float(v.y << 16); r[3] = __uint_as_float(v.y & 0xffff0000u);
    }
    // 16 consecutive bf16 values of a B/C row (32 bytes, 16-byte aligned).
    __device__ __forceinline__ static void load_row16(const T* p, float (&r)[kN]) {
        const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint4 v = __ldg(q + i);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                r[8 * i + 2 * j + 0] = __uint_as_float(w[j] << 16);
                r[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
            }
        }
    }
};

}  // namespace axon
