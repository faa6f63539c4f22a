// step.cuh -- cached single-token decode (Axon-SSM page, section
// "Autoregressive decoding"): per (b, e) read the K-1 cached inputs and the N
// float32 states, run one token of conv + SiLU + dt + recurrence + gate, write
// y, the shifted conv cache and the updated state in place.
//
// The step is bound by HBM traffic on the state read-modify-write (2 x 64 bytes
// of the 148 bytes per channel it moves at bf16).  The state moves as 16-byte
// pieces, four lanes per channel, through per-lane asynchronous-copy rings, and
// every other input arrives through shared memory in one copy per block, so the
// HBM traffic of later rows overlaps the arithmetic of the current one.
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

__device__ __forceinline__ void step_cp_async16(void* smem_dst, const void* gmem_src, bool valid) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    const int n = valid ? 16 : 0;   // 0 source bytes: zero-fill
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem_src), "r"(n) : "memory");
}

constexpr int kStepThreads = 128;  // 32 channels x 4 lanes
constexpr int kStepChan = kStepThreads / 4;
constexpr int kStepStages = 4;     // state rows in flight per lane (shared-memory ring)
constexpr int kStepMaxRows = 32;   // batch rows per block

// grid = (ceil(E / 32), ceil(B / rows)) blocks of 128 threads, rows <= 32.
// Four lanes share a channel, each owning four consecutive states (one 16-byte
// vector), so a warp's state traffic is one contiguous 512-byte run.  A block
// owns 32 channels and walks `rows` batch rows:
//  - at the start it copies, for all its rows, the channels' x, z, dt_raw and
//    K-1 cache entries and the B_t, C_t rows into shared memory (one
//    cooperative cp.async group, one barrier);
//  - every lane streams its state pieces through a private kStepStages-deep
//    shared-memory ring with cp.async (a lane reads back only its own copies);
//  - A = -exp(A_log) is formed once per lane.
// The conv/SiLU/dt prologue of four consecutive rows is spread over the four
// lanes of a channel; C . h is finished with two shuffles.  y and the shifted
// conv caches of all the block's rows leave at the end as 16-byte pieces.
template <class Io, bool kZoh>
__global__ void __launch_bounds__(kStepThreads) step_kernel(StepParams p, int rows) {
    using T = typename Io::T;
    constexpr int S = Io::kBytes;
    constexpr int kSmall = 3 + (kK - 1);              // x, z, dt_raw, cache rows 0..K-2
    constexpr int kWin = kStepChan * S;               // bytes of a 32-channel window
    const int tid = threadIdx.x;
    const int q = tid & 3;                            // states 4q .. 4q+3
    const int c = tid >> 2;
    const int e0 = blockIdx.x * kStepChan;
    const int e = e0 + c;
    const int b0 = blockIdx.y * rows;
    const int nb = min(rows, p.B - b0);
    // Every lane stays to the end (the shuffles below need full warps); lanes
    // past E compute channel E-1 and store nothing.
    const bool live = e < p.E;
    const int ec = live ? e : p.E - 1;

    __shared__ __align__(16) unsigned char small[kStepMaxRows][kSmall][kWin];
    __shared__ __align__(16) unsigned char bcs[kStepMaxRows][2][kN * S];
    __shared__ __align__(16) unsigned char yst[kStepMaxRows][kWin];   // y of the block's rows
    __shared__ float4 ring[kStepStages][kStepThreads];

    {   // (1) every row's small inputs and B/C rows, 16-byte pieces
        constexpr int kPw = kWin / 16, kPb = kN * S / 16;
        constexpr int kPer = kSmall * kPw + 2 * kPb;   // pieces per row
        const size_t row_bytes = (size_t)p.E * S;
        for (int i = tid; i < nb * kPer; i += kStepThreads) {
            const int j = i / kPer, t = i - j * kPer, b = b0 + j;
            if (t < kSmall * kPw) {
                const int k = t / kPw, pc = t - k * kPw;
                const size_t col = (size_t)e0 * S + (size_t)pc * 16;
                const bool ok = col + 16 <= row_bytes;           // E*S is a multiple of 16
                const unsigned char* base;
                if (k < 3) base = static_cast<const unsigned char*>(k == 0 ? p.x : (k == 1 ? p.z : p.dt_raw)) + (size_t)b * row_bytes;
                else base = static_cast<const unsigned char*>(p.conv_cache) + ((size_t)b * (kK - 1) + (k - 3)) * row_bytes;
                step_cp_async16(&small[j][k][pc * 16], ok ? base + col : static_cast<const void*>(p.x), ok);
            } else {
                const int u = t - kSmall * kPw, w2 = u / kPb, pc = u - w2 * kPb;
                const unsigned char* base = static_cast<const unsigned char*>(w2 ? p.Cm : p.Bm) + (size_t)b * kN * S;
                step_cp_async16(&bcs[j][w2][pc * 16], base + pc * 16, true);
            }
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    }
    // (2) row j's state piece -> this lane's ring slot; rows are E*N floats apart
    const size_t srow = (size_t)p.E * kN;
    const float* sbase = p.ssm_state + ((size_t)b0 * p.E + ec) * kN + 4 * q;
    auto issue = [&](int j) { step_cp_async16(&ring[j % kStepStages][tid], sbase + (size_t)j * srow, true); };
#pragma unroll
    for (int j = 0; j < kStepStages - 1; ++j) {
        if (j < nb) issue(j);
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    }
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
    asm volatile("cp.async.wait_group %0;\n" ::"n"(kStepStages - 1) : "memory");   // (1) landed
    __syncthreads();

    const int co = (ec - e0) * S;                     // this channel's byte offset in a window
    // Rows go in rounds of four: lane q computes the conv / SiLU / dt prologue
    // and SiLU(z) of row j0+q only; each row's dt and dt*u reach the other
    // three lanes of the channel by shuffles, and the row's owner lane puts
    // its y in shared memory.
#pragma unroll 1
    for (int j0 = 0; j0 < nb; j0 += 4) {
        const int jq = min(j0 + q, nb - 1);
        float uq, dtq, dtuq, gzq;
        {
            const float x_t = Io::sload(&small[jq][0][co]);
            float xc = fmaf(w.x, Io::sload(&small[jq][3][co]), cb);
            xc = fmaf(w.y, Io::sload(&small[jq][4][co]), xc);
            xc = fmaf(w.z, Io::sload(&small[jq][5][co]), xc);
            xc = fmaf(w.w, x_t, xc);
            uq = silu(xc);
            dtq = dt_from_raw(Io::sload(&small[jq][2][co]) + db);
            dtuq = kZoh ? uq : dtq * uq;                  // input factor of Bbar u
            gzq = silu(Io::sload(&small[jq][1][co]));
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int j = j0 + k;
            if (j >= nb) break;                           // block-uniform
            const int b = b0 + j;
            if (j + kStepStages - 1 < nb) issue(j + kStepStages - 1);
            asm volatile("cp.async.commit_group;\n" ::: "memory");
            asm volatile("cp.async.wait_group %0;\n" ::"n"(kStepStages - 1) : "memory");   // row j landed
            const float dt = __shfl_sync(0xffffffffu, dtq, k, 4);
            const float dtu = __shfl_sync(0xffffffffu, dtuq, k, 4);
            float Bq[4], Cq[4];
            Io::sload4(&bcs[j][0][4 * q * S], Bq);
            Io::sload4(&bcs[j][1][4 * q * S], Cq);
            const float4 hq = ring[j % kStepStages][tid];
            float h[4] = {hq.x, hq.y, hq.z, hq.w};
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a = ex2_approx(dt * A2[i]);
                // first-order: (dt u) B;  ZOH: u ((exp(dt A) - 1) / A) B
                const float uin = kZoh ? dtu * zoh_bbar(dt, dt * A2[i] * kLn2, a, kLog2e / A2[i]) : dtu;
                h[i] = fmaf(a, h[i], uin * Bq[i]);
                acc = fmaf(Cq[i], h[i], acc);
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            if (live) *reinterpret_cast<float4*>(const_cast<float*>(sbase) + (size_t)j * srow) =
                          make_float4(h[0], h[1], h[2], h[3]);
            if (live && q == k) Io::store(reinterpret_cast<T*>(&yst[j][co]), fmaf(Dv, uq, acc) * gzq);
        }
    }
    // (3) y and the shifted conv caches of all rows, 16-byte pieces: cache row
    // i <- cache row i+1, the last <- x_t (exact copies of the raw bits; every
    // read of the old cache happened in (1), so in-place updates are safe)
    __syncthreads();
    {
        constexpr int kPw = kWin / 16;
        const size_t row_bytes = (size_t)p.E * S;
        for (int i = tid; i < nb * kK * kPw; i += kStepThreads) {
            const int j = i / (kK * kPw), t = i - j * (kK * kPw), k = t / kPw, pc = t - k * kPw;
            const size_t col = (size_t)e0 * S + (size_t)pc * 16;
            if (col + 16 > row_bytes) continue;          // E*S is a multiple of 16
            const int b = b0 + j;
            unsigned char* dst;
            const unsigned char* src;
            if (k == 0) {                                // y
                dst = static_cast<unsigned char*>(p.y) + (size_t)b * row_bytes + col;
                src = &yst[j][pc * 16];
            } else {                                     // cache row k-1
                dst = static_cast<unsigned char*>(p.conv_cache) + ((size_t)b * (kK - 1) + (k - 1)) * row_bytes + col;
                src = k < kK - 1 ? &small[j][3 + k][pc * 16] : &small[j][0][pc * 16];
            }
            *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
        }
    }
}

}  // namespace axon
