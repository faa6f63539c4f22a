// ssd.cuh -- the Mamba-2 (SSD) layer core, one scalar decay per head, as a
// chunked scan on the tensor cores (the SSD article: inside a chunk the
// recurrence is a masked matrix product on fast on-chip memory, between chunks
// a carried state; wiki page "Selective State Space Models (Mamba)", section
// "Mamba-2 block (SSD)": d_state 128, headdim 64).
//
// Per batch row b, head h, chunk of Q = 64 tokens starting at t0, with
// a_t = dt_t A_h and acum_i = sum_{k<=i} a_k inside the chunk:
//   G        = C B^T                                   (Q x Q, shared by all heads)
//   y_i      = exp(acum_i) C_i . S_in                  (the carried state)
//            + sum_{j<=i} G_ij exp(acum_i - acum_j) dt_j x_j  + D_h x_i
//   S_out    = exp(acum_{Q-1}) S_in + sum_j exp(acum_{Q-1} - acum_j) dt_j x_j B_j^T
// The three products run as bf16 m16n8k16 tensor-core MMAs with float32
// accumulation (mma.sync); the carried state stays float32 in registers, and
// its product with C uses it split in two bf16 parts (hi + lo, about 16
// significant bits), because C . S_in can cancel heavily for long-memory heads.
#pragma once

#include <cuda_bf16.h>

#include "device_math.cuh"
#include "scan_chunked.cuh"   // cp.async helpers

namespace axon {

constexpr int kSsdQ = 64;     // tokens per chunk
constexpr int kSsdP = 64;     // head dimension
constexpr int kSsdN = 128;    // state size
constexpr int kSsdPB = 16;    // head-dimension columns per CTA of the scan
constexpr int kSsdThreads = 128;

struct SsdParams {
    int B, L, H;
    const __nv_bfloat16* x;      // (B, L, H, P)
    const __nv_bfloat16* dt_raw; // (B, L, H)
    const float* dt_bias;        // (H)
    const float* A_log;          // (H)
    const __nv_bfloat16* Bm;     // (B, L, N)
    const __nv_bfloat16* Cm;     // (B, L, N)
    const float* D;              // (H)
    const float* h0;             // (B, H, P, N) or null
    __nv_bfloat16* y;            // (B, L, H, P)
    float* h_out;                // (B, H, P, N)
    float* G;                    // (B, nC, Q, Q) workspace
};

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t ld32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

// Stores the pair (v0, v1) as bf16 hi parts at hi and the rounding remainders
// v - hi as bf16 lo parts at lo.
__device__ __forceinline__ void store_split(__nv_bfloat16* hi, __nv_bfloat16* lo, float v0, float v1) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
    *reinterpret_cast<__nv_bfloat162*>(hi) = h;
    *reinterpret_cast<uint32_t*>(lo) = pack_bf16(v0 - __low2float(h), v1 - __high2float(h));
}

// Copies rows [t0, t0 + 64) of a (B, L, N) bf16 matrix into shared memory rows
// of `stride` elements (zeros past L).  All threads of the CTA take part.
__device__ __forceinline__ void ssd_load_rows(__nv_bfloat16* dst, int stride, const __nv_bfloat16* src, int b,
                                              int L, int t0) {
    constexpr int kPieces = kSsdN * 2 / 16;   // 16-byte pieces per row
    for (int w = threadIdx.x; w < kSsdQ * kPieces; w += kSsdThreads) {
        const int r = w / kPieces, pc = w % kPieces;
        const int t = t0 + r;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (t < L) v = *reinterpret_cast<const uint4*>(src + ((size_t)b * L + t) * kSsdN + pc * 8);
        *reinterpret_cast<uint4*>(dst + r * stride + pc * 8) = v;
    }
}

// G[b, c] = C_c B_c^T (float32).  grid = (nC, B), 128 threads: warp w owns
// rows 16w .. 16w+15 and all 64 columns.
__global__ void __launch_bounds__(kSsdThreads) ssd_gram_kernel(SsdParams p) {
    constexpr int kS = kSsdN + 8;            // padded row stride (bf16 elements)
    __shared__ __align__(16) __nv_bfloat16 Cs[kSsdQ * kS];
    __shared__ __align__(16) __nv_bfloat16 Bs[kSsdQ * kS];
    const int c = blockIdx.x, b = blockIdx.y;
    const int nC = gridDim.x;
    const int t0 = c * kSsdQ;
    ssd_load_rows(Cs, kS, p.Cm, b, p.L, t0);
    ssd_load_rows(Bs, kS, p.Bm, b, p.L, t0);
    __syncthreads();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int g = lane >> 2, tq = lane & 3;
    float acc[8][4] = {};
#pragma unroll
    for (int ks = 0; ks < kSsdN / 16; ++ks) {
        const int k0 = ks * 16 + 2 * tq;
        const __nv_bfloat16* r0 = Cs + (16 * w + g) * kS;
        const __nv_bfloat16* r1 = r0 + 8 * kS;
        const uint32_t a[4] = {ld32(r0 + k0), ld32(r1 + k0), ld32(r0 + k0 + 8), ld32(r1 + k0 + 8)};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const __nv_bfloat16* br = Bs + (8 * nt + g) * kS;     // B^T column j = B row j
            mma_16816(acc[nt], a, ld32(br + k0), ld32(br + k0 + 8));
        }
    }
    float* Gc = p.G + ((size_t)b * nC + c) * kSsdQ * kSsdQ;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        const int i = 16 * w + g, j = 8 * nt + 2 * tq;
        *reinterpret_cast<float2*>(Gc + i * kSsdQ + j) = make_float2(acc[nt][0], acc[nt][1]);
        *reinterpret_cast<float2*>(Gc + (i + 8) * kSsdQ + j) = make_float2(acc[nt][2], acc[nt][3]);
    }
}

// Dynamic shared-memory layout of the scan kernel (bytes).  Staged with
// cp.async: G (float rows), C rows (padded for fragment loads), raw B rows and
// raw x rows (16 head columns, both double-buffered: the next chunk's arrive
// while this one computes); built from them: w*B as [n][j] and x as [p][j]
// (stride 33 words: the pair stores that build them hit distinct banks).
struct SsdSmem {
    static constexpr int kGs = kSsdQ + 4;            // float row stride of G
    static constexpr int kCs = kSsdN + 8;            // bf16 row stride of C
    static constexpr int kWs = kSsdQ + 2;            // bf16 row stride of w*B^T and x^T
    static constexpr int kSs = kSsdN + 8;            // bf16 row stride of the carried state
    static constexpr int G = 0;
    static constexpr int C = G + kSsdQ * kGs * 4;
    static constexpr int BR = C + kSsdQ * kCs * 2;            // two buffers (this chunk, the next)
    static constexpr int XR = BR + 2 * kSsdQ * kSsdN * 2;     // two buffers
    static constexpr int WB = XR + 2 * kSsdQ * kSsdPB * 2;
    static constexpr int XT = WB + kSsdN * kWs * 2;
    static constexpr int SS = XT + kSsdPB * kWs * 2;          // hi part, then lo part
    static constexpr int ACUM = SS + 2 * kSsdPB * kSs * 2;    // cumulative decay, in log2 units
    static constexpr int DTV = ACUM + kSsdQ * 4;
    static constexpr int WV = DTV + kSsdQ * 4;                // w_j = exp(acum_last - acum_j) dt_j
    static constexpr int TOTAL = WV + kSsdQ * 4;
};

// grid = (H, P / 16, B), 128 threads; walks the chunks of one sequence in
// order for one head and 16 head-dimension columns, carrying the state
// (16 x 128, float32) in registers: warp w owns state columns 32w .. 32w+31
// and output rows 16w .. 16w+15 of every chunk.
__global__ void __launch_bounds__(kSsdThreads) ssd_scan_kernel(SsdParams p) {
    extern __shared__ __align__(16) unsigned char smem[];
    float* Gs = reinterpret_cast<float*>(smem + SsdSmem::G);
    __nv_bfloat16* Cs = reinterpret_cast<__nv_bfloat16*>(smem + SsdSmem::C);
    __nv_bfloat16* Br = reinterpret_cast<__nv_bfloat16*>(smem + SsdSmem::BR);    // [j][n]
    __nv_bfloat16* Xr = reinterpret_cast<__nv_bfloat16*>(smem + SsdSmem::XR);    // [j][p]
    __nv_bfloat16* WBt = reinterpret_cast<__nv_bfloat16*>(smem + SsdSmem::WB);   // [n][j]
    __nv_bfloat16* Xt = reinterpret_cast<__nv_bfloat16*>(smem + SsdSmem::XT);    // [p][j]
    __nv_bfloat16* Ss = reinterpret_cast<__nv_bfloat16*>(smem + SsdSmem::SS);    // [p][n], hi part
    __nv_bfloat16* Sl = Ss + kSsdPB * SsdSmem::kSs;                                // [p][n], lo part
    float* acum2 = reinterpret_cast<float*>(smem + SsdSmem::ACUM);
    float* dtv = reinterpret_cast<float*>(smem + SsdSmem::DTV);
    float* wv = reinterpret_cast<float*>(smem + SsdSmem::WV);

    const int h = blockIdx.x, pb = blockIdx.y * kSsdPB, b = blockIdx.z;
    const int H = p.H, L = p.L;
    const int nC = (L + kSsdQ - 1) / kSsdQ;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int g = lane >> 2, tq = lane & 3;
    const int tid = threadIdx.x;
    const float A2 = -expf(__ldg(p.A_log + h)) * kLog2e;     // exp(dt A) = 2^(dt A2)
    const float bias = __ldg(p.dt_bias + h);
    const float Dh = __ldg(p.D + h);

    // carried state: rows p = g, g+8 (of the CTA's 16), columns n = 32w + 8nt + 2tq (+1)
    float S[4][4];
    const float* h0 = p.h0 ? p.h0 + (((size_t)b * H + h) * kSsdP + pb) * kSsdN : nullptr;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const int n = 32 * w + 8 * nt + 2 * tq;
        S[nt][0] = h0 ? h0[g * kSsdN + n] : 0.f;
        S[nt][1] = h0 ? h0[g * kSsdN + n + 1] : 0.f;
        S[nt][2] = h0 ? h0[(g + 8) * kSsdN + n] : 0.f;
        S[nt][3] = h0 ? h0[(g + 8) * kSsdN + n + 1] : 0.f;
        store_split(Ss + g * SsdSmem::kSs + n, Sl + g * SsdSmem::kSs + n, S[nt][0], S[nt][1]);
        store_split(Ss + (g + 8) * SsdSmem::kSs + n, Sl + (g + 8) * SsdSmem::kSs + n, S[nt][2], S[nt][3]);
    }
    const bool has_h0 = p.h0 != nullptr;

    // ---- copies of chunk c: G and C (one buffer), raw B and x rows (buffer c % 2)
    auto copy_gc = [&](int c) {
        const int t0 = c * kSsdQ;
        const float* Gc = p.G + ((size_t)b * nC + c) * kSsdQ * kSsdQ;
        for (int v = tid; v < kSsdQ * (kSsdQ / 4); v += kSsdThreads) {
            const int i = v / (kSsdQ / 4), pc = v % (kSsdQ / 4);
            cp_async16(Gs + i * SsdSmem::kGs + 4 * pc, Gc + i * kSsdQ + 4 * pc, true);
        }
        for (int v = tid; v < kSsdQ * (kSsdN / 8); v += kSsdThreads) {
            const int r = v / (kSsdN / 8), pc = v % (kSsdN / 8);
            const int t = t0 + r;
            const bool ok = t < L;
            cp_async16(Cs + r * SsdSmem::kCs + 8 * pc, p.Cm + (ok ? ((size_t)b * L + t) * kSsdN + 8 * pc : 0), ok);
        }
    };
    auto copy_bx = [&](int c) {
        const int t0 = c * kSsdQ;
        __nv_bfloat16* br = Br + (c & 1) * kSsdQ * kSsdN;
        __nv_bfloat16* xr = Xr + (c & 1) * kSsdQ * kSsdPB;
        for (int v = tid; v < kSsdQ * (kSsdN / 8); v += kSsdThreads) {
            const int r = v / (kSsdN / 8), pc = v % (kSsdN / 8);
            const int t = t0 + r;
            const bool ok = t < L;
            cp_async16(br + r * kSsdN + 8 * pc, p.Bm + (ok ? ((size_t)b * L + t) * kSsdN + 8 * pc : 0), ok);
        }
        for (int v = tid; v < kSsdQ * (kSsdPB / 8); v += kSsdThreads) {
            const int j = v / (kSsdPB / 8), half = v % (kSsdPB / 8);
            const int t = t0 + j;
            const bool ok = t < L;
            cp_async16(xr + j * kSsdPB + 8 * half,
                       p.x + (ok ? (((size_t)b * L + t) * H + h) * kSsdP + pb + 8 * half : 0), ok);
        }
    };
    // warp 0: the raw dt of chunk c into registers (two tokens per lane)
    auto load_dt = [&](int c, float (&d)[2]) {
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int t = c * kSsdQ + 2 * lane + k;
            d[k] = t < L ? __bfloat162float(p.dt_raw[((size_t)b * L + t) * H + h]) : 0.f;
        }
    };

    float dtraw[2] = {0.f, 0.f};
    if (nC > 0) {
        copy_gc(0);
        copy_bx(0);
        cp_async_commit();
        if (w == 0) load_dt(0, dtraw);
    }
    for (int c = 0; c < nC; ++c) {
        const int t0 = c * kSsdQ;
        const __nv_bfloat16* br = Br + (c & 1) * kSsdQ * kSsdN;
        const __nv_bfloat16* xr = Xr + (c & 1) * kSsdQ * kSsdPB;
        if (w == 0) {
            // dt, the inclusive cumulative decay (log2 units) and w_j of this chunk
            float dt2[2], a2[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = t0 + 2 * lane + k;
                dt2[k] = t < L ? dt_from_raw(dtraw[k] + bias) : 0.f;
                a2[k] = dt2[k] * A2;
            }
            float sacc = a2[0] + a2[1];
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const float o = __shfl_up_sync(0xffffffffu, sacc, d);
                if (lane >= d) sacc += o;
            }
            const float alast = __shfl_sync(0xffffffffu, sacc, 31);
            const float c0 = sacc - a2[1], c1 = sacc;
            acum2[2 * lane] = c0;
            acum2[2 * lane + 1] = c1;
            dtv[2 * lane] = dt2[0];
            dtv[2 * lane + 1] = dt2[1];
            wv[2 * lane] = ex2_approx(alast - c0) * dt2[0];
            wv[2 * lane + 1] = ex2_approx(alast - c1) * dt2[1];
        }
        cp_async_wait_0();                     // this chunk's copies (this thread's share)
        __syncthreads();                       // ... everyone's; acum, dtv, wv written
        if (c + 1 < nC) {
            copy_bx(c + 1);                    // its buffers were last read before the previous barrier
            cp_async_commit();
            if (w == 0) load_dt(c + 1, dtraw);
        }
        // ---- x as [p][j] and w*B as [n][j], one bf16 pair (j, j+1) per store
        for (int v = tid; v < kSsdPB * (kSsdQ / 2); v += kSsdThreads) {
            const int pp = v % kSsdPB, jp = v / kSsdPB;
            *reinterpret_cast<uint32_t*>(Xt + pp * SsdSmem::kWs + 2 * jp) =
                pack_bf16(__bfloat162float(xr[(2 * jp) * kSsdPB + pp]), __bfloat162float(xr[(2 * jp + 1) * kSsdPB + pp]));
        }
        for (int v = tid; v < kSsdN * (kSsdQ / 2); v += kSsdThreads) {
            const int n = v % kSsdN, jp = v / kSsdN;
            *reinterpret_cast<uint32_t*>(WBt + n * SsdSmem::kWs + 2 * jp) =
                pack_bf16(wv[2 * jp] * __bfloat162float(br[(2 * jp) * kSsdN + n]),
                          wv[2 * jp + 1] * __bfloat162float(br[(2 * jp + 1) * kSsdN + n]));
        }
        __syncthreads();

        // ---- outputs of rows 16w .. 16w+15, columns pb .. pb+15
        float acc[2][4] = {};
        const int i0 = 16 * w + g, i1 = i0 + 8;
        const float ai0 = acum2[i0], ai1 = acum2[i1];
        if (c > 0 || has_h0) {
            // exp(acum_i) C_i . S_in: K = N, the state as hi + lo bf16 parts
#pragma unroll
            for (int ks = 0; ks < kSsdN / 16; ++ks) {
                const int k0 = ks * 16 + 2 * tq;
                const uint32_t a[4] = {ld32(Cs + i0 * SsdSmem::kCs + k0), ld32(Cs + i1 * SsdSmem::kCs + k0),
                                       ld32(Cs + i0 * SsdSmem::kCs + k0 + 8), ld32(Cs + i1 * SsdSmem::kCs + k0 + 8)};
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const __nv_bfloat16* sr = Ss + (8 * nt + g) * SsdSmem::kSs;
                    const __nv_bfloat16* lr = Sl + (8 * nt + g) * SsdSmem::kSs;
                    mma_16816(acc[nt], a, ld32(sr + k0), ld32(sr + k0 + 8));
                    mma_16816(acc[nt], a, ld32(lr + k0), ld32(lr + k0 + 8));
                }
            }
            const float e0 = ex2_approx(ai0), e1 = ex2_approx(ai1);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                acc[nt][0] *= e0; acc[nt][1] *= e0; acc[nt][2] *= e1; acc[nt][3] *= e1;
            }
        }
        // masked, decayed G times dt x: K = the chunk's tokens, only blocks on or below the diagonal
#pragma unroll
        for (int ks = 0; ks < kSsdQ / 16; ++ks) {
            if (ks > w) break;                 // j >= 16 ks > i for every row of this warp
            uint32_t a[4];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const int i = (q4 & 1) ? i1 : i0;
                const float ai = (q4 & 1) ? ai1 : ai0;
                const int j = ks * 16 + 2 * tq + ((q4 & 2) ? 8 : 0);
                const float m0 = j <= i ? Gs[i * SsdSmem::kGs + j] * ex2_approx(ai - acum2[j]) * dtv[j] : 0.f;
                const float m1 =
                    j + 1 <= i ? Gs[i * SsdSmem::kGs + j + 1] * ex2_approx(ai - acum2[j + 1]) * dtv[j + 1] : 0.f;
                a[q4] = pack_bf16(m0, m1);
            }
            const int k0 = ks * 16 + 2 * tq;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const __nv_bfloat16* xr = Xt + (8 * nt + g) * SsdSmem::kWs;
                mma_16816(acc[nt], a, ld32(xr + k0), ld32(xr + k0 + 8));
            }
        }
        // + D x, store rows inside the sequence
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int pc = 8 * nt + 2 * tq;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int i = r ? i1 : i0;
                const int t = t0 + i;
                if (t < L) {
                    const float x0 = __bfloat162float(xr[i * kSsdPB + pc]);
                    const float x1 = __bfloat162float(xr[i * kSsdPB + pc + 1]);
                    const float y0 = fmaf(Dh, x0, acc[nt][2 * r]), y1 = fmaf(Dh, x1, acc[nt][2 * r + 1]);
                    *reinterpret_cast<uint32_t*>(p.y + (((size_t)b * L + t) * H + h) * kSsdP + pb + pc) =
                        pack_bf16(y0, y1);
                }
            }
        }

        // ---- G and C of the next chunk, in flight during the state update
        const float el = ex2_approx(acum2[kSsdQ - 1]);
        __syncthreads();                       // every warp is done with G, C and this chunk's acum
        if (c + 1 < nC) {
            copy_gc(c + 1);
            cp_async_commit();
        }
        // ---- carried state: S = exp(acum_last) S + x^T (w B): K = the chunk's tokens
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int k = 0; k < 4; ++k) S[nt][k] *= el;
#pragma unroll
        for (int ks = 0; ks < kSsdQ / 16; ++ks) {
            const int k0 = ks * 16 + 2 * tq;
            const uint32_t a[4] = {ld32(Xt + g * SsdSmem::kWs + k0), ld32(Xt + (g + 8) * SsdSmem::kWs + k0),
                                   ld32(Xt + g * SsdSmem::kWs + k0 + 8), ld32(Xt + (g + 8) * SsdSmem::kWs + k0 + 8)};
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const __nv_bfloat16* wr = WBt + (32 * w + 8 * nt + g) * SsdSmem::kWs;
                mma_16816(S[nt], a, ld32(wr + k0), ld32(wr + k0 + 8));
            }
        }
        __syncthreads();                       // every warp has read the old carried state
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int n = 32 * w + 8 * nt + 2 * tq;
            store_split(Ss + g * SsdSmem::kSs + n, Sl + g * SsdSmem::kSs + n, S[nt][0], S[nt][1]);
            store_split(Ss + (g + 8) * SsdSmem::kSs + n, Sl + (g + 8) * SsdSmem::kSs + n, S[nt][2], S[nt][3]);
        }
    }
    // ---- final state
    float* ho = p.h_out + (((size_t)b * H + h) * kSsdP + pb) * kSsdN;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
        const int n = 32 * w + 8 * nt + 2 * tq;
        *reinterpret_cast<float2*>(ho + g * kSsdN + n) = make_float2(S[nt][0], S[nt][1]);
        *reinterpret_cast<float2*>(ho + (g + 8) * kSsdN + n) = make_float2(S[nt][2], S[nt][3]);
    }
}

}  // namespace axon
