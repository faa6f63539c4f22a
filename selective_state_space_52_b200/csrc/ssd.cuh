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
//
// Launches: ssd_chunk_prep_kernel (G per chunk; per chunk and head: acum,
// log2(dt_j) - acum_j and the state weights w_j), then the chunk walk.  To fill the GPU when B * H is small, the sequence is cut into
// segments of whole chunks, and the carried state crosses them as in the
// chunked associative scan of the SSD article: a first walk of every segment
// but the last from a zero state (state products only) gives its local end
// state and total decay; the full walk of segment k starts from the fold
// S_end(j) = exp(sum a over segment j) S_end(j-1) + S_loc(j) for j < k.
//
// The products run as bf16 m16n8k16 tensor-core MMAs (mma.sync) with float32
// accumulation; operands reach them by ldmatrix from padded shared tiles (x
// and B rows are read transposed, so no transposed copies are built).
// The carried state stays float32 in registers: warp w owns head columns
// 16w .. 16w+15 and all 128 state columns, and its accumulator layout is the
// B-operand layout of the C . S_in product, which therefore reads the state
// straight from registers, split in two bf16 parts (hi + lo, about 16
// significant bits) because C . S_in can cancel heavily for long-memory heads.
#pragma once

#include <cuda_bf16.h>

#include "device_math.cuh"
#include "scan_chunked.cuh"   // cp.async helpers

namespace axon {

constexpr int kSsdQ = 64;     // tokens per chunk
constexpr int kSsdP = 64;     // head dimension
constexpr int kSsdN = 128;    // state size
constexpr int kSsdThreads = 128;
constexpr int kSsdMaxSegs = 64;

struct SsdParams {
    int B, L, H;
    int nC;                      // chunks
    int segs, cps;               // segments of the sequence, chunks per segment
    int pcs, cpp;                // first walk: pieces per segment, chunks per piece
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
    float* prep;                 // (B, H, nC, 3, Q): acum (log2 units), log2(dt) - acum, w
    float* sloc;                 // ((segs - 1) pcs, B, H, P, N): local end states of the pieces
    float* sega;                 // ((segs - 1) pcs, B, H): total decay of a piece (log2 units)
    float* h0c;                  // (B, H, P, N): copy of h0 (h_out may overwrite h0) when segs > 1
};

// No side effects beyond its operands: not volatile, so the scheduler may
// interleave independent MMAs with the loads that feed later ones.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four 8x8 bf16 matrices from shared memory; lane l gives the address of row
// l % 8 of matrix l / 8.  ldsm_x4_t delivers them transposed.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], unsigned addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], unsigned addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ uint32_t ld32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }


// One launch for the two per-chunk preliminaries.  grid = (nC, B, 4 +
// ceil(H/4)), 128 threads; blockIdx.z < 4: rows 16z .. 16z+15 of the chunk's
// Gram matrix, else the per-head decays of heads 4 (z - 4) .. 4 (z - 4) + 3.
//
// Gram: G[b, c] = C_c B_c^T (float32); warp w owns columns 16w .. 16w+15 of
// the CTA's 16 rows.
//
// Decays, per head: dt_j, acum_j (log2 units: exp(acum) = 2^acum2),
// e_j = log2(dt_j) - acum2_j (so dt_j exp(acum_i - acum_j) = 2^(acum2_i + e_j),
// whose exponent never exceeds log2(dt_j) for j <= i), and the state weights
// w_j = dt_j 2^(acum2_{Q-1} - acum2_j).  Tokens past L get dt = 0, e = -inf.
// Warp -> head, lane -> 2 tokens.
constexpr int kGramBlocks = 4;
__global__ void __launch_bounds__(kSsdThreads) ssd_chunk_prep_kernel(SsdParams p) {
    constexpr int kS = kSsdN + 8;            // padded row stride (bf16 elements)
    constexpr int kRows = kSsdQ / kGramBlocks;
    __shared__ __align__(16) __nv_bfloat16 Cs[kRows * kS];
    __shared__ __align__(16) __nv_bfloat16 Bs[kSsdQ * kS];
    const int c = blockIdx.x, b = blockIdx.y;
    const int L = p.L, H = p.H, nC = p.nC;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int t0 = c * kSsdQ;
    if (blockIdx.z < kGramBlocks) {
        const int r0 = blockIdx.z * kRows;
        constexpr int kPieces = kSsdN * 2 / 16;   // 16-byte pieces per row
        for (int v = threadIdx.x; v < kSsdQ * kPieces; v += kSsdThreads) {
            const int r = v / kPieces, pc = v % kPieces;
            const bool ok = t0 + r < L;
            cp_async16(Bs + r * kS + pc * 8, p.Bm + (ok ? ((size_t)b * L + t0 + r) * kSsdN + pc * 8 : 0), ok);
        }
        for (int v = threadIdx.x; v < kRows * kPieces; v += kSsdThreads) {
            const int r = v / kPieces, pc = v % kPieces;
            const bool ok = t0 + r0 + r < L;
            cp_async16(Cs + r * kS + pc * 8, p.Cm + (ok ? ((size_t)b * L + t0 + r0 + r) * kSsdN + pc * 8 : 0), ok);
        }
        cp_async_commit();
        cp_async_wait_0();
        __syncthreads();
        const int g = lane >> 2, tq = lane & 3;
        float acc[2][4] = {};
#pragma unroll
        for (int ks = 0; ks < kSsdN / 16; ++ks) {
            const int k0 = ks * 16 + 2 * tq;
            const __nv_bfloat16* a0 = Cs + g * kS;
            const __nv_bfloat16* a1 = a0 + 8 * kS;
            const uint32_t a[4] = {ld32(a0 + k0), ld32(a1 + k0), ld32(a0 + k0 + 8), ld32(a1 + k0 + 8)};
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                const __nv_bfloat16* br = Bs + (16 * w + 8 * nt + g) * kS;     // B^T column j = B row j
                mma_16816(acc[nt], a, ld32(br + k0), ld32(br + k0 + 8));
            }
        }
        float* Gc = p.G + ((size_t)b * nC + c) * kSsdQ * kSsdQ;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int i = r0 + g, j = 16 * w + 8 * nt + 2 * tq;
            *reinterpret_cast<float2*>(Gc + i * kSsdQ + j) = make_float2(acc[nt][0], acc[nt][1]);
            *reinterpret_cast<float2*>(Gc + (i + 8) * kSsdQ + j) = make_float2(acc[nt][2], acc[nt][3]);
        }
        return;
    }
    const int h = (blockIdx.z - kGramBlocks) * 4 + w;
    if (h >= H) return;                        // whole warps
    const float A2 = -expf(__ldg(p.A_log + h)) * kLog2e;
    const float bias = __ldg(p.dt_bias + h);
    float dt[2], a2[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int t = t0 + 2 * lane + k;
        dt[k] = t < L ? dt_from_raw(__bfloat162float(p.dt_raw[((size_t)b * L + t) * H + h]) + bias) : 0.f;
        a2[k] = dt[k] * A2;
    }
    float s = a2[0] + a2[1];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, s, d);
        if (lane >= d) s += o;
    }
    const float alast = __shfl_sync(0xffffffffu, s, 31);
    const float c0 = s - a2[1], c1 = s;
    const int tl = t0 + 2 * lane;
    const float e0 = tl < L ? lg2_approx(dt[0]) - c0 : -INFINITY;
    const float e1 = tl + 1 < L ? lg2_approx(dt[1]) - c1 : -INFINITY;
    float* out = p.prep + (((size_t)b * H + h) * nC + c) * 3 * kSsdQ;
    *reinterpret_cast<float2*>(out + 2 * lane) = make_float2(c0, c1);
    *reinterpret_cast<float2*>(out + kSsdQ + 2 * lane) = make_float2(e0, e1);
    *reinterpret_cast<float2*>(out + 2 * kSsdQ + 2 * lane) =
        make_float2(dt[0] * ex2_approx(alast - c0), dt[1] * ex2_approx(alast - c1));
}

// Packed float pairs (one instruction for two lanes of arithmetic).
__device__ __forceinline__ unsigned long long f2_pack(float a, float b) {
    return (unsigned long long)__float_as_uint(a) | ((unsigned long long)__float_as_uint(b) << 32);
}
__device__ __forceinline__ float f2_lo(unsigned long long v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float f2_hi(unsigned long long v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ unsigned long long f2_sub(unsigned long long a, unsigned long long b) {
    unsigned long long d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// The pair (v0, v1) as bf16 pairs hi + lo: hi = the top 16 bits of each value
// (truncation), lo = the remainder v - hi (exact in float32), rounded to bf16;
// together about 16 significant bits.
__device__ __forceinline__ void split_bf16(float v0, float v1, uint32_t& hi, uint32_t& lo) {
    hi = __byte_perm(__float_as_uint(v0), __float_as_uint(v1), 0x7632);
    const unsigned long long v = f2_pack(v0, v1);
    const unsigned long long t = f2_pack(__uint_as_float(__float_as_uint(v0) & 0xffff0000u),
                                         __uint_as_float(__float_as_uint(v1) & 0xffff0000u));
    const unsigned long long r = f2_sub(v, t);
    lo = pack_bf16(f2_lo(r), f2_hi(r));
}

// Shared memory of the chunk walk (bytes).  Two stages of per-chunk rows (C,
// B, x of this head, the prep values), filled by cp.async one chunk ahead;
// the full walk adds G (float32) and the decayed, masked Gram matrix M (bf16).
// bf16 tiles have padded rows (128 columns: 272 bytes, 64 columns: 144
// bytes), so the eight rows of an ldmatrix phase fall in distinct banks and
// every fragment address is a per-lane base plus a constant.
constexpr int kRowCB = 272;   // bytes per row of the C and B tiles
constexpr int kRowX = 144;    // bytes per row of the x and M tiles
template <bool kFull> struct SsdSmem;
template <> struct SsdSmem<true> {
    static constexpr int CS = 0, BS = CS + 64 * kRowCB, XS = BS + 64 * kRowCB, PR = XS + 64 * kRowX;
    static constexpr int STAGE = PR + 3 * kSsdQ * 4;
    static constexpr int GS = 2 * STAGE, MS = GS + kSsdQ * kSsdQ * 4, TOTAL = MS + 64 * kRowX;
};
template <> struct SsdSmem<false> {
    static constexpr int CS = -1, BS = 0, XS = BS + 64 * kRowCB, PR = XS + 64 * kRowX;
    static constexpr int STAGE = PR + 3 * kSsdQ * 4;
    static constexpr int GS = -1, MS = -1, TOTAL = 2 * STAGE;
};

// The chunk walk of one (head h, run of chunks, batch row b), 128 threads.
// kFull = false, the first walk: grid = (H, (segs - 1) pcs, B), one piece of
// cpp chunks of a segment but the last, state products only, from h0 for the
// first piece and zeros otherwise, writing the piece's local end state and
// total decay.  kFull = true: grid = (H, segs, B), one segment, entering
// with the fold of the pieces before it; the outputs y and, for the last
// segment, the final state.
template <bool kFull>
__global__ void __launch_bounds__(kSsdThreads, kFull ? 2 : 3) ssd_chunk_scan_kernel(SsdParams p) {
    using Lay = SsdSmem<kFull>;
    constexpr int Q = kSsdQ, P = kSsdP, N = kSsdN;
    extern __shared__ __align__(16) unsigned char smem[];
    const unsigned sbase = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    const int h = blockIdx.x, seg = blockIdx.y, b = blockIdx.z;     // seg: segment, or piece of the first walk
    const int H = p.H, L = p.L, nC = p.nC;
    int c_begin, c_end;
    if constexpr (kFull) {
        c_begin = seg * p.cps;
        c_end = min(nC, c_begin + p.cps);
    } else {
        const int k = seg / p.pcs, m = seg - k * p.pcs;
        c_begin = k * p.cps + m * p.cpp;
        c_end = min(min(nC, (k + 1) * p.cps), c_begin + p.cpp);
    }
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, g = lane >> 2, tq = lane & 3;

    // ---- per-thread parts of the copy addresses: B/C rows r = tid/16 + 8k, 16-byte
    // piece tid%16; x rows r = tid/8 + 16k, piece tid%8; G rows as B/C
    const int rBC = tid >> 4, pBC = tid & 15, rX = tid >> 3, pX = tid & 7;
    const int sBC = rBC * kRowCB + pBC * 16, sX = rX * kRowX + pX * 16;
    const int sG = rBC * 256 + ((pBC ^ ((rBC & 1) << 2)) << 4);
    const size_t HP = (size_t)H * P;
    auto issue_stage = [&](int c, int s) {
        unsigned char* st = smem + s * Lay::STAGE;
        const int t0 = c * Q;
        const int left = L - t0;               // rows of this chunk inside the sequence
        const __nv_bfloat16* gB = p.Bm + ((size_t)b * L + t0 + rBC) * N + pBC * 8;
        const __nv_bfloat16* gC = p.Cm + ((size_t)b * L + t0 + rBC) * N + pBC * 8;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const bool ok = rBC + 8 * k < left;
            cp_async16(st + Lay::BS + sBC + k * 8 * kRowCB, ok ? gB + (size_t)k * 8 * N : p.Bm, ok);
            if constexpr (kFull) cp_async16(st + Lay::CS + sBC + k * 8 * kRowCB, ok ? gC + (size_t)k * 8 * N : p.Cm, ok);
        }
        const __nv_bfloat16* gX = p.x + (((size_t)b * L + t0 + rX) * H + h) * P + pX * 8;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const bool ok = rX + 16 * k < left;
            cp_async16(st + Lay::XS + sX + k * 16 * kRowX, ok ? gX + (size_t)k * 16 * HP : p.x, ok);
        }
        if (tid < 3 * Q / 4)
            cp_async16(st + Lay::PR + tid * 16, p.prep + (((size_t)b * H + h) * nC + c) * 3 * Q + tid * 4, true);
    };
    auto issue_g = [&](int c) {
        const float* gG = p.G + ((size_t)b * nC + c) * Q * Q + rBC * Q + pBC * 4;
#pragma unroll
        for (int k = 0; k < 8; ++k) cp_async16(smem + Lay::GS + sG + k * 8 * 256, gG + k * 8 * Q, true);
    };

    // ---- per-lane parts of the ldmatrix addresses
    const int rowL = (((lane >> 3) & 1) << 3) + (lane & 7), chL = lane >> 4;
    const unsigned offCB = rowL * kRowCB + chL * 16;                 // C (A operand), B (transposed B operand)
    const unsigned offM = rowL * kRowX + chL * 16;                   // M (A operand)
    const unsigned offX = ((((lane >> 4) << 3) + (lane & 7)) * kRowX) + (2 * w + ((lane >> 3) & 1)) * 16;

    // ---- the carried state: rows p = 16w + g (+8), columns n = 8t + 2tq (+1)
    float S[16][4];
    const size_t hoff = (((size_t)b * H + h) * P + 16 * w) * N;
    auto load_state = [&](const float* src) {
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const float2 u = *reinterpret_cast<const float2*>(src + hoff + g * N + 8 * t + 2 * tq);
            const float2 v = *reinterpret_cast<const float2*>(src + hoff + (g + 8) * N + 8 * t + 2 * tq);
            S[t][0] = u.x; S[t][1] = u.y; S[t][2] = v.x; S[t][3] = v.y;
        }
    };
    auto store_state = [&](float* dst) {
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            *reinterpret_cast<float2*>(dst + hoff + g * N + 8 * t + 2 * tq) = make_float2(S[t][0], S[t][1]);
            *reinterpret_cast<float2*>(dst + hoff + (g + 8) * N + 8 * t + 2 * tq) = make_float2(S[t][2], S[t][3]);
        }
    };
    auto zero_state = [&]() {
#pragma unroll
        for (int t = 0; t < 16; ++t) S[t][0] = S[t][1] = S[t][2] = S[t][3] = 0.f;
    };
    const size_t BHPN = (size_t)p.B * H * P * N;
    bool s_nonzero;
    if constexpr (!kFull) {
        s_nonzero = seg == 0 && p.h0 != nullptr;
        if (s_nonzero) {
            load_state(p.h0);
            if (p.h0c) store_state(p.h0c);
        } else {
            zero_state();
        }
    } else {
        if (seg == 0) {
            const float* src = p.h0c ? p.h0c : p.h0;
            s_nonzero = src != nullptr;
            if (s_nonzero) load_state(src);
            else zero_state();
        } else {
            s_nonzero = true;
            load_state(p.sloc);                                      // the first piece ran from h0
            for (int j = 1; j < seg * p.pcs; ++j) {
                const float dj = ex2_approx(p.sega[((size_t)j * p.B + b) * H + h]);
                const float* src = p.sloc + (size_t)j * BHPN;
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const float2 u = *reinterpret_cast<const float2*>(src + hoff + g * N + 8 * t + 2 * tq);
                    const float2 v = *reinterpret_cast<const float2*>(src + hoff + (g + 8) * N + 8 * t + 2 * tq);
                    S[t][0] = fmaf(dj, S[t][0], u.x); S[t][1] = fmaf(dj, S[t][1], u.y);
                    S[t][2] = fmaf(dj, S[t][2], v.x); S[t][3] = fmaf(dj, S[t][3], v.y);
                }
            }
        }
    }

    float seg_decay = 0.f;
    if (c_begin < c_end) {
        issue_stage(c_begin, 0);
        if constexpr (kFull) issue_g(c_begin);
        cp_async_commit();
    }
    float Dh = 0.f;
    if constexpr (kFull) Dh = __ldg(p.D + h);
    // M build: thread -> row tid/8 of a 16x16 block, column pair tid%8
    const int rr = tid >> 3, k2 = 2 * (tid & 7);
    int gcol[4];                               // byte offset of G[rr][16jb + k2] within a row pair
#pragma unroll
    for (int jb = 0; jb < 4; ++jb) gcol[jb] = ((((jb ^ (rr & 1)) << 2) + (k2 >> 2)) << 4) + (k2 & 3) * 4;

    for (int c = c_begin; c < c_end; ++c) {
        const int s = (c - c_begin) & 1;
        const unsigned st = sbase + s * Lay::STAGE;
        const float* pr = reinterpret_cast<const float*>(smem + s * Lay::STAGE + Lay::PR);  // acum, e, w
        cp_async_wait_0();
        __syncthreads();                       // this chunk's rows landed; chunk c-1 is done everywhere
        if (c + 1 < c_end) {
            issue_stage(c + 1, s ^ 1);
            cp_async_commit();
        }

        if constexpr (kFull) {
            // ---- M = mask(G_ij 2^(acum_i + e_j)) + D on the diagonal, bf16: the ten 16x16
            // blocks on or below the diagonal
            float2 ej[4];
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) ej[jb] = *reinterpret_cast<const float2*>(pr + Q + 16 * jb + k2);
#pragma unroll
            for (int ib = 0; ib < 4; ++ib) {
                const int i = 16 * ib + rr;
                const float ai = pr[i];
#pragma unroll
                for (int jb = 0; jb <= ib; ++jb) {
                    const int j = 16 * jb + k2;
                    const float2 gv = *reinterpret_cast<const float2*>(smem + Lay::GS + i * 256 + gcol[jb]);
                    float m0 = gv.x * ex2_approx(ai + ej[jb].x);
                    float m1 = gv.y * ex2_approx(ai + ej[jb].y);
                    if (jb == ib) {
                        m0 = j < i ? m0 : (j == i ? m0 + Dh : 0.f);
                        m1 = j + 1 < i ? m1 : (j + 1 == i ? m1 + Dh : 0.f);
                    }
                    *reinterpret_cast<uint32_t*>(smem + Lay::MS + i * kRowX + j * 2) = pack_bf16(m0, m1);
                }
            }
            __syncthreads();                   // M complete; G free
            if (c + 1 < c_end) {
                issue_g(c + 1);
                cp_async_commit();
            }
        }

        // ---- x of this warp's 16 head columns: ks -> tokens 16ks .. 16ks+15
        uint32_t xr[4][4];
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) ldsm_x4_t(xr[ks], st + Lay::XS + offX + ks * 16 * kRowX);

        if constexpr (kFull) {
            float yacc[4][2][4];
#pragma unroll
            for (int rb = 0; rb < 4; ++rb)
#pragma unroll
                for (int pt = 0; pt < 2; ++pt) yacc[rb][pt][0] = yacc[rb][pt][1] = yacc[rb][pt][2] = yacc[rb][pt][3] = 0.f;
            if (s_nonzero || c > c_begin) {
                // exp(acum_i) C_i . S_in: K = the state columns, B operand = the state registers
#pragma unroll
                for (int ks = 0; ks < N / 16; ++ks) {
                    uint32_t bh[2][2], bl[2][2];
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const float* v = S[2 * ks + half];
                        split_bf16(v[0], v[1], bh[0][half], bl[0][half]);
                        split_bf16(v[2], v[3], bh[1][half], bl[1][half]);
                    }
                    uint32_t a[4][4];
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb) ldsm_x4(a[rb], st + Lay::CS + offCB + rb * 16 * kRowCB + ks * 32);
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb)
#pragma unroll
                        for (int pt = 0; pt < 2; ++pt) mma_16816(yacc[rb][pt], a[rb], bl[pt][0], bl[pt][1]);
#pragma unroll
                    for (int rb = 0; rb < 4; ++rb)
#pragma unroll
                        for (int pt = 0; pt < 2; ++pt) mma_16816(yacc[rb][pt], a[rb], bh[pt][0], bh[pt][1]);
                }
#pragma unroll
                for (int rb = 0; rb < 4; ++rb) {
                    const unsigned long long e =
                        f2_pack(ex2_approx(pr[16 * rb + g]), ex2_approx(pr[16 * rb + g + 8]));
#pragma unroll
                    for (int pt = 0; pt < 2; ++pt) {
                        const unsigned long long u = f2_mul(f2_pack(yacc[rb][pt][0], yacc[rb][pt][2]), e);
                        const unsigned long long v = f2_mul(f2_pack(yacc[rb][pt][1], yacc[rb][pt][3]), e);
                        yacc[rb][pt][0] = f2_lo(u); yacc[rb][pt][2] = f2_hi(u);
                        yacc[rb][pt][1] = f2_lo(v); yacc[rb][pt][3] = f2_hi(v);
                    }
                }
            }
            // + M x: K = the chunk's tokens, blocks on or below the diagonal
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                uint32_t a[4][4];
#pragma unroll
                for (int rb = kb; rb < 4; ++rb) ldsm_x4(a[rb], sbase + Lay::MS + offM + rb * 16 * kRowX + kb * 32);
#pragma unroll
                for (int rb = kb; rb < 4; ++rb) {
                    mma_16816(yacc[rb][0], a[rb], xr[kb][0], xr[kb][2]);
                    mma_16816(yacc[rb][1], a[rb], xr[kb][1], xr[kb][3]);
                }
            }
            // ---- y rows inside the sequence
            const int left = L - c * Q;
            __nv_bfloat16* yb = p.y + (((size_t)b * L + (size_t)c * Q + g) * H + h) * P + 16 * w + 2 * tq;
#pragma unroll
            for (int rb = 0; rb < 4; ++rb)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    if (16 * rb + g + 8 * r < left) {
                        __nv_bfloat16* yo = yb + (size_t)(16 * rb + 8 * r) * HP;
#pragma unroll
                        for (int pt = 0; pt < 2; ++pt)
                            *reinterpret_cast<uint32_t*>(yo + 8 * pt) = pack_bf16(yacc[rb][pt][2 * r], yacc[rb][pt][2 * r + 1]);
                    }
                }
        }

        // ---- S = exp(acum_last) S + (w x)^T B: K = the chunk's tokens
        const float alast = pr[Q - 1];
        seg_decay += alast;
        const float el = ex2_approx(alast);
        const unsigned long long el2 = f2_pack(el, el);
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const unsigned long long u = f2_mul(f2_pack(S[t][0], S[t][1]), el2);
            const unsigned long long v = f2_mul(f2_pack(S[t][2], S[t][3]), el2);
            S[t][0] = f2_lo(u); S[t][1] = f2_hi(u); S[t][2] = f2_lo(v); S[t][3] = f2_hi(v);
        }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const float4 wv = make_float4(pr[2 * Q + 16 * ks + 2 * tq], pr[2 * Q + 16 * ks + 2 * tq + 1],
                                          pr[2 * Q + 16 * ks + 8 + 2 * tq], pr[2 * Q + 16 * ks + 9 + 2 * tq]);
            const unsigned long long wa = f2_pack(wv.x, wv.y), wb = f2_pack(wv.z, wv.w);
            uint32_t a[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const unsigned long long xv = f2_mul(f2_pack(bf16_lo(xr[ks][r]), bf16_hi(xr[ks][r])), r < 2 ? wa : wb);
                a[r] = pack_bf16(f2_lo(xv), f2_hi(xv));
            }
            constexpr int kBatch = kFull ? 8 : 4;             // fragments loaded ahead of their MMAs
#pragma unroll
            for (int q0 = 0; q0 < 8; q0 += kBatch) {
                uint32_t bb[kBatch][4];
#pragma unroll
                for (int q = 0; q < kBatch; ++q)
                    ldsm_x4_t(bb[q], st + Lay::BS + offCB + ks * 16 * kRowCB + (q0 + q) * 32);
#pragma unroll
                for (int q = 0; q < kBatch; ++q) {
                    mma_16816(S[2 * (q0 + q)], a, bb[q][0], bb[q][1]);
                    mma_16816(S[2 * (q0 + q) + 1], a, bb[q][2], bb[q][3]);
                }
            }
        }
    }

    if constexpr (kFull) {
        if (seg == p.segs - 1) store_state(p.h_out);
    } else {
        store_state(p.sloc + (size_t)seg * BHPN);
        if (tid == 0) p.sega[((size_t)seg * p.B + b) * H + h] = seg_decay;
    }
}

}  // namespace axon
