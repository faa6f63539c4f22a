// ssd.cuh -- the Mamba-2 (SSD) layer core, one scalar decay per head, as a
// chunked scan on the tcgen05 tensor cores (the SSD article: inside a chunk
// the recurrence is a masked matrix product on fast on-chip memory, between
// chunks a carried state; wiki page "Selective State Space Models (Mamba)",
// section "Mamba-2 block (SSD)": d_state 128, headdim 64).
//
// Per batch row b, head h, chunk of Q = 128 tokens starting at t0, with
// a_t = dt_t A_h and acum_i = sum_{k<=i} a_k inside the chunk:
//   G        = C B^T                                   (Q x Q)
//   M        = mask(G_ij exp(acum_i - acum_j) dt_j) + D_h I
//   y        = diag(exp(acum)) C S_in^T + M x
//   S_out^T  = exp(acum_{Q-1}) S_in^T + B^T (w x),    w_j = exp(acum_{Q-1} - acum_j) dt_j
//
// Launches: ssd_chunk_prep_kernel (per chunk and head: acum, log2(dt_j) -
// acum_j, w_j, and the in-block decay factors v_j), then the chunk walks.  To fill the GPU when B * H is small,
// the sequence is cut into segments of whole chunks and the carried state
// crosses them as in the chunked associative scan of the SSD article: a first
// walk over pieces of every segment but the last, from a zero state (state
// products only), gives each piece's local end state and total decay; the full
// walk of segment k starts from the fold S_end(j) = exp(sum a over piece j)
// S_end(j-1) + S_loc(j) over the pieces before it.
//
// The four products of a chunk are tcgen05 MMAs (kind::f16, bf16 operands,
// float32 accumulators in tensor memory, M = 128), issued by one thread and
// tracked by mbarriers.  Operands sit in shared memory as 128-byte-swizzled
// tiles of 64-element rows; one copy of each input tile serves every product
// (the B rows are the K-major B operand of C B^T and the MN-major A operand of
// B^T (w x); the x rows are the MN-major B operand of M x), except M, which
// each thread writes as its row into tensor memory, the A operand of M x, as
// two bf16 parts (hi, and the rounding residual lo: about 16 significant
// bits), both multiplied by x into the same accumulator -- a single bf16 copy
// of M costs up to 2.8% of |y| at the Mamba-2 shape, the split about 0.6%.
// Tensor-memory lane i holds row i of G, M, y and of the transposed state; the
// full walk gives each lane two threads, each taking half of the row's head
// columns and of M's column blocks.  M's entries below the diagonal 32-token
// blocks come from the factorised decay (one exponential per row and block);
// only the diagonal block takes one per entry.  The full walk double-buffers
// its input rows: chunk c+1's copies are in flight while chunk c computes.
// The carried state stays float32 in registers (row n of S^T with the threads
// of lane n) and enters C S^T as two bf16 parts (hi + lo, about 16
// significant bits), because that product can cancel heavily for long-memory
// heads.
#pragma once

#include <cuda_bf16.h>

#include "device_math.cuh"
#include "scan_chunked.cuh"   // cp.async helpers
#include "tc_ops.cuh"         // tcgen05, tensor-memory and mbarrier primitives

namespace axon {

constexpr int kSsdQ = 128;    // tokens per chunk
constexpr int kSsdP = 64;     // head dimension
constexpr int kSsdN = 128;    // state size
constexpr int kSsdThreads = 128;      // the preliminary launch and the state-only walk
constexpr int kSsdFullThreads = 256;  // the full walk: two threads per tensor-memory lane
constexpr int kSsdMaxSegs = 64;
// Iterations of an mbarrier poll before a walk gives up and records an error.
constexpr int kSsdWaitLimit = kTcWaitLimit;

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
    float* prep;                 // (B, H, nC, 4, Q): acum (log2 units), log2(dt) - acum, w, v
    float* sloc;                 // ((segs - 1) pcs, B, H, P, N): local end states of the pieces
    float* sega;                 // ((segs - 1) pcs, B, H): total decay of a piece (log2 units)
    float* h0c;                  // (B, H, P, N): copy of h0 (h_out may overwrite h0) when segs > 1
    int* err;                    // set to 1 when a wait gave up
};

// The walks' failure path in isolation: one warp polls, `limit` times, an
// mbarrier that nothing arrives on, as a walk does when a product never
// completes, and thread 0 writes 1 to *status when the wait gave up (0 if it
// completed, which cannot happen here).  grid = 1, 32 threads.
__global__ void __launch_bounds__(32) ssd_wait_probe_kernel(int* status, int limit) {
    __shared__ __align__(8) unsigned long long bar;
    const uint32_t mbar = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
    if (threadIdx.x == 0) mbar_init(mbar, 1);
    __syncwarp();
    const bool done = mbar_wait(mbar, 0u, limit);
    if (threadIdx.x == 0) *status = done ? 0 : 1;
}

// Byte offset of the 16-byte piece `pc` (8 bf16) of row r in a tile of 128
// rows stored as 64-column blocks of 128-byte rows, 128-byte swizzle (the
// piece index XORed by the row mod 8; the tile base is 1024-byte aligned).
__device__ __forceinline__ int tile_off(int r, int pc) {
    return (pc >> 3) * (128 * 128) + r * 128 + (((pc & 7) ^ (r & 7)) << 4);
}

// Per (b, chunk, head): dt_j, acum_j (log2 units: exp(acum) = 2^acum2),
// e_j = log2(dt_j) - acum2_j (so dt_j exp(acum_i - acum_j) = 2^(acum2_i + e_j),
// whose exponent never exceeds log2(dt_j) for j <= i), the state weights
// w_j = dt_j 2^(acum2_{Q-1} - acum2_j), and v_j = dt_j 2^(acum2_r - acum2_j)
// with r the last token of j's 32-token block: below the diagonal blocks,
// dt_j exp(acum_i - acum_j) = 2^(acum2_i - acum2_r) v_j, both factors at most
// 1 (acum decreases), so neither overflows and an underflow only drops a term
// below 2^-126 of G_ij dt_j.  Tokens past L get dt = 0, e = -inf, v = 0.
// grid = (nC, ceil(H / 4), B), 128 threads: warp -> head, lane -> 4 tokens.
__global__ void __launch_bounds__(kSsdThreads) ssd_chunk_prep_kernel(SsdParams p) {
    grid_dep_launch();
    grid_dep_wait();
    const int c = blockIdx.x, b = blockIdx.z;
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.y * 4 + (threadIdx.x >> 5);
    if (c == 0 && b == 0 && threadIdx.x == 0 && blockIdx.y == 0) *p.err = 0;
    if (h >= p.H) return;                      // whole warps
    const int L = p.L, H = p.H;
    const float A2 = -expf(__ldg(p.A_log + h)) * kLog2e;
    const float bias = __ldg(p.dt_bias + h);
    const int t0 = c * kSsdQ + 4 * lane;
    float dt[4], cum[4];
    float run = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int t = t0 + k;
        dt[k] = t < L ? dt_from_raw(__bfloat162float(p.dt_raw[((size_t)b * L + t) * H + h]) + bias) : 0.f;
        run += dt[k] * A2;
        cum[k] = run;
    }
    float s = run;                             // inclusive scan of the lanes' totals
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const float o = __shfl_up_sync(0xffffffffu, s, d);
        if (lane >= d) s += o;
    }
    const float before = s - run;
    const float alast = __shfl_sync(0xffffffffu, s, 31);
    const float ablock = __shfl_sync(0xffffffffu, s, lane | 7);   // acum2 at the last token of this 32-token block
    float a[4], e[4], wv[4], vv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        a[k] = before + cum[k];
        e[k] = t0 + k < L ? lg2_approx(dt[k]) - a[k] : -INFINITY;
        wv[k] = dt[k] * ex2_approx(alast - a[k]);
        vv[k] = dt[k] * ex2_approx(ablock - a[k]);
    }
    float* out = p.prep + (((size_t)b * H + h) * p.nC + c) * 4 * kSsdQ + 4 * lane;
    *reinterpret_cast<float4*>(out) = make_float4(a[0], a[1], a[2], a[3]);
    *reinterpret_cast<float4*>(out + kSsdQ) = make_float4(e[0], e[1], e[2], e[3]);
    *reinterpret_cast<float4*>(out + 2 * kSsdQ) = make_float4(wv[0], wv[1], wv[2], wv[3]);
    *reinterpret_cast<float4*>(out + 3 * kSsdQ) = make_float4(vv[0], vv[1], vv[2], vv[3]);
}

// Shared memory of the chunk walk (bytes from a 1024-byte-aligned base).
// STAGES copies of the input rows (C, B, x), STAGE bytes apart.
template <bool kFull> struct SsdSmem;
template <> struct SsdSmem<true> {
    static constexpr int STAGES = 2;
    static constexpr int CT = 0;                 // C rows: 128 x 128 bf16
    static constexpr int BT = CT + 32768;        // B rows: 128 x 128 bf16
    static constexpr int XT = BT + 32768;        // x rows of this head: 128 x 64 bf16
    static constexpr int STAGE = XT + 16384 - CT;
    static constexpr int XW = STAGES * STAGE;    // w_j x_j rows
    static constexpr int SH = XW + 16384;        // S^T rows, hi part: 128 (n) x 64 (p) bf16
    static constexpr int SL = SH + 16384;        // lo part
    static constexpr int PR = SL + 16384;        // two buffers of (acum, e, w, v) x 128 floats
    static constexpr int MB = PR + 2 * 4 * kSsdQ * 4;   // mbarriers: Gram, state, outputs, drain
    static constexpr int SLOT = MB + 32;         // tensor-memory address
    static constexpr int BYTES = SLOT + 8;
    static constexpr int TOTAL = BYTES + 1024;   // with the alignment pad
    // tensor memory: G (0..127); the state product (128..191); M as the A
    // operand, two bf16 per column, hi part (192..255); C S^T, hi part
    // (256..319) and lo part (320..383); M x (384..447); M's lo part (448..511)
    static constexpr int TMEM_COLS = 512;
};
template <> struct SsdSmem<false> {
    static constexpr int STAGES = 1;
    static constexpr int CT = -1;
    static constexpr int BT = 0;
    static constexpr int XT = BT + 32768;
    static constexpr int STAGE = XT + 16384 - BT;
    static constexpr int XW = STAGES * STAGE;
    static constexpr int SH = -1, SL = -1;
    static constexpr int PR = XW + 16384;
    static constexpr int MB = PR + 2 * 4 * kSsdQ * 4;
    static constexpr int SLOT = MB + 32;
    static constexpr int BYTES = SLOT + 8;
    static constexpr int TOTAL = BYTES + 1024;
    static constexpr int TMEM_COLS = 64;
};

// The chunk walk of one (head h, run of chunks, batch row b).
// kFull = false, the first walk (128 threads): grid = (H, (segs - 1) pcs, B),
// one piece of cpp chunks of a segment but the last, state products only, from
// h0 for the first piece and zeros otherwise, writing the piece's local end
// state and total decay.  kFull = true (256 threads): grid = (H, segs, B), one
// segment, entering with the fold of the pieces before it; the outputs y and,
// for the last segment, the final state.  Thread t serves row r = t % 128
// (tensor-memory lane r, reachable from warps r/32 and r/32 + 4) and half
// hf = t / 128 of that row's work: head columns 32 hf .. 32 hf + 31 of the
// state, w x and y, and the column blocks jb = hf, hf + 2 of M.
template <bool kFull>
__global__ void __launch_bounds__(kFull ? kSsdFullThreads : kSsdThreads, kFull ? 1 : 3)
    ssd_chunk_scan_kernel(SsdParams p) {
    grid_dep_launch();
    using Lay = SsdSmem<kFull>;
    constexpr int Q = kSsdQ, P = kSsdP, N = kSsdN;
    constexpr int NT = kFull ? kSsdFullThreads : kSsdThreads;
    constexpr int HALVES = NT / 128;
    constexpr int PH = P / HALVES;             // head columns per thread
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const uint32_t raw = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    unsigned char* sm = smem_raw + pad;
    const uint32_t sb = raw + pad;
    const int h = blockIdx.x, seg = blockIdx.y, b = blockIdx.z;     // seg: segment, or piece of the first walk
    const int H = p.H, L = p.L, nC = p.nC;
    const int tid = threadIdx.x, w = tid >> 5;
    const int r = tid & 127, hf = tid >> 7, qd = w & 3;             // row, half, lane quadrant
    int c_begin, c_end;
    if constexpr (kFull) {
        c_begin = seg * p.cps;
        c_end = min(nC, c_begin + p.cps);
    } else {
        const int k = seg / p.pcs, m = seg - k * p.pcs;
        c_begin = k * p.cps + m * p.cpp;
        c_end = min(min(nC, (k + 1) * p.cps), c_begin + p.cpp);
    }
    const uint32_t mbG = sb + Lay::MB, mbS = sb + Lay::MB + 8, mbY = sb + Lay::MB + 16;
    const uint32_t mbF = sb + Lay::MB + 24;   // drain: every product thread 0 issued has completed

    // ---- copies of chunk c's rows: B/C rows rBC + (NT/16) k, piece tid%16; x rows
    // rX + (NT/8) k, piece tid%8; the prep values into buffer `slot`
    const int rBC = tid >> 4, pBC = tid & 15, rX = tid >> 3, pX = tid & 7;
    const int sBC = tile_off(rBC, pBC), sX = tile_off(rX, pX);
    auto issue_chunk = [&](int c, int slot) {
        unsigned char* st = sm + (Lay::STAGES > 1 ? slot : 0) * Lay::STAGE;   // input rows of this chunk
        const int t0 = c * Q;
        const int left = L - t0;
        const size_t rowBC = (size_t)b * L + t0 + rBC;
#pragma unroll
        for (int k = 0; k < 128 * 16 / NT; ++k) {
            const int dr = (NT / 16) * k;
            const bool ok = rBC + dr < left;
            const size_t go = (rowBC + dr) * N + pBC * 8;
            cp_async16(st + Lay::BT + sBC + dr * 128, ok ? p.Bm + go : p.Bm, ok);
            if constexpr (kFull) cp_async16(st + Lay::CT + sBC + dr * 128, ok ? p.Cm + go : p.Cm, ok);
        }
        const size_t rowX = (size_t)b * L + t0 + rX;
#pragma unroll
        for (int k = 0; k < 128 * 8 / NT; ++k) {
            const int dr = (NT / 8) * k;
            const bool ok = rX + dr < left;
            cp_async16(st + Lay::XT + sX + dr * 128, ok ? p.x + ((rowX + dr) * H + h) * P + pX * 8 : p.x, ok);
        }
        if (tid < Q)
            cp_async16(sm + Lay::PR + slot * 4 * Q * 4 + tid * 16,
                       p.prep + (((size_t)b * H + h) * nC + c) * 4 * Q + tid * 4, true);
        cp_async_commit();
    };

    // ---- tensor memory and mbarriers
    if (tid == 0) {
        mbar_init(mbG, 1);
        mbar_init(mbS, 1);
        mbar_init(mbY, 1);
        mbar_init(mbF, 1);
    }
    if (w == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sb + Lay::SLOT),
                     "r"(Lay::TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    grid_dep_wait();                    // the prep values and the first walk's states are written
    if (c_begin < c_end) issue_chunk(c_begin, 0);

    // ---- the carried state, transposed: thread (n, hf) holds S[p][n] for its PH head columns
    float S[PH];
    const size_t hoff = ((size_t)b * H + h) * P * N + (size_t)(PH * hf) * N + r;
    const size_t BHPN = (size_t)p.B * H * P * N;
    bool s_nonzero;
    if constexpr (!kFull) {
        s_nonzero = seg == 0 && p.h0 != nullptr;
#pragma unroll
        for (int q = 0; q < PH; ++q) S[q] = s_nonzero ? p.h0[hoff + (size_t)q * N] : 0.f;
        if (s_nonzero && p.h0c) {
#pragma unroll
            for (int q = 0; q < PH; ++q) p.h0c[hoff + (size_t)q * N] = S[q];
        }
    } else {
        if (seg == 0) {
            const float* src = p.h0c ? p.h0c : p.h0;
            s_nonzero = src != nullptr;
#pragma unroll
            for (int q = 0; q < PH; ++q) S[q] = s_nonzero ? src[hoff + (size_t)q * N] : 0.f;
        } else {
            s_nonzero = true;
#pragma unroll
            for (int q = 0; q < PH; ++q) S[q] = p.sloc[hoff + (size_t)q * N];     // the first piece ran from h0
            for (int j = 1; j < seg * p.pcs; ++j) {
                const float dj = ex2_approx(p.sega[((size_t)j * p.B + b) * H + h]);
                const float* src = p.sloc + (size_t)j * BHPN + hoff;
#pragma unroll
                for (int q = 0; q < PH; ++q) S[q] = fmaf(dj, S[q], src[(size_t)q * N]);
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(sm + Lay::SLOT);
    const uint32_t tlane = tbase + ((uint32_t)(qd * 32) << 16);     // this warp's lanes
    bool ok_all = true;
    float Dh = 0.f;
    if constexpr (kFull) Dh = __ldg(p.D + h);
    float seg_decay = 0.f;
    // instruction descriptors
    constexpr uint32_t kIdGram = umma_idesc(128, 128, 0, 0);     // C (K-major) x B rows (K-major)
    constexpr uint32_t kIdState = umma_idesc(128, 64, 1, 1);     // B rows as B^T (MN-major) x w x (MN-major)
    constexpr uint32_t kIdOff = umma_idesc(128, 128, 0, 1);      // C (K-major) x [S^T hi | S^T lo] (MN-major)
    constexpr uint32_t kIdDiag = umma_idesc(128, 64, 0, 1);      // M (tensor memory, K-major) x x (MN-major)
    constexpr uint32_t kColState = kFull ? 128 : 0;

    for (int c = c_begin; c < c_end; ++c) {
        const int k = c - c_begin;
        const uint32_t par = (uint32_t)(k & 1);
        const float* pr = reinterpret_cast<const float*>(sm + Lay::PR + (k & 1) * 4 * Q * 4);   // acum, e, w, v
        const int so = (Lay::STAGES > 1 ? (k & 1) : 0) * Lay::STAGE;                              // this chunk's rows
        cp_async_wait_0();
        fence_async_smem();
        tc_fence_before();
        // chunk c's rows landed; the previous chunk's tensor reads done; a wait that
        // gave up anywhere ends the walk for the whole CTA
        if (__syncthreads_or(!ok_all)) break;
        tc_fence_after();
        if constexpr (kFull) {
            // the other stage was last read by the previous chunk, whose products are done
            if (c + 1 < c_end) issue_chunk(c + 1, (k + 1) & 1);
            if (tid == 0) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = so + (ks >> 2) * 16384 + (ks & 3) * 32;
                    umma(tbase, umma_desc(sb + Lay::CT + off, 16, 1024), umma_desc(sb + Lay::BT + off, 16, 1024),
                         kIdGram, ks > 0);
                }
                umma_commit(mbG);
            }
        }
        // ---- w_j x_j (thread (j, hf): its 16-byte pieces of row j)
        {
            const float wj = pr[2 * Q + r];
#pragma unroll
            for (int pc = (8 / HALVES) * hf; pc < (8 / HALVES) * (hf + 1); ++pc) {
                const uint4 v = *reinterpret_cast<const uint4*>(sm + so + Lay::XT + tile_off(r, pc));
                uint4 o;
                o.x = pack_bf16(bf16_lo(v.x) * wj, bf16_hi(v.x) * wj);
                o.y = pack_bf16(bf16_lo(v.y) * wj, bf16_hi(v.y) * wj);
                o.z = pack_bf16(bf16_lo(v.z) * wj, bf16_hi(v.z) * wj);
                o.w = pack_bf16(bf16_lo(v.w) * wj, bf16_hi(v.w) * wj);
                *reinterpret_cast<uint4*>(sm + Lay::XW + tile_off(r, pc)) = o;
            }
        }
        if constexpr (kFull) {
            // the state product needs only w x: issue it now, to run during the M build
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
            if (tid == 0) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma(tbase + kColState, umma_desc(sb + so + Lay::BT + ks * 2048, 16384, 1024),
                         umma_desc(sb + Lay::XW + ks * 2048, 16384, 1024), kIdState, ks > 0);
                umma_commit(mbS);
            }
            // ---- S_in^T row n as hi + lo bf16 parts (thread (n, hf): its head columns), when nonzero
            if (s_nonzero || k > 0) {
#pragma unroll
                for (int pq = 0; pq < PH / 8; ++pq) {
                    const int pc = (PH / 8) * hf + pq;
                    uint32_t hi[4], lo[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float v0 = S[8 * pq + 2 * q], v1 = S[8 * pq + 2 * q + 1];
                        hi[q] = __byte_perm(__float_as_uint(v0), __float_as_uint(v1), 0x7632);
                        lo[q] = pack_bf16(v0 - bf16_lo(hi[q]), v1 - bf16_hi(hi[q]));
                    }
                    *reinterpret_cast<uint4*>(sm + Lay::SH + tile_off(r, pc)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    *reinterpret_cast<uint4*>(sm + Lay::SL + tile_off(r, pc)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                }
            }
            // ---- M row i from G row i into tensor memory (the A operand of M x): thread
            // (i, hf) takes the 32-column blocks jb = hf, hf + 2; zeros above the diagonal
            ok_all &= mbar_wait(mbG, par);
            tc_fence_after();
            const int i = r;
            const float ai = pr[i];
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                const int jb = hf + 2 * bb;
                uint32_t m[16], ml[16];        // M as bf16 hi + lo parts
                if (jb <= qd) {                // warp-uniform: rows 32 qd .. 32 qd + 31
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb) {
                        float g[16];
                        tmem_ld16(tlane + 32 * jb + 16 * hb, g);
                        const int j0 = 32 * jb + 16 * hb;
                        if (jb < qd) {         // below the diagonal: G u_i v_j
                            const float ui = ex2_approx(ai - pr[32 * jb + 31]);
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const float2 v2 = *reinterpret_cast<const float2*>(pr + 3 * Q + j0 + 2 * q);
                                const float m0 = g[2 * q] * ui * v2.x, m1 = g[2 * q + 1] * ui * v2.y;
                                m[8 * hb + q] = pack_bf16(m0, m1);
                                ml[8 * hb + q] = pack_bf16(m0 - bf16_lo(m[8 * hb + q]), m1 - bf16_hi(m[8 * hb + q]));
                            }
                        } else {               // the diagonal block: masked, D on the diagonal
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                const int j = j0 + 2 * q;
                                const float2 e2 = *reinterpret_cast<const float2*>(pr + Q + j);
                                float m0 = g[2 * q] * ex2_approx(ai + e2.x);
                                float m1 = g[2 * q + 1] * ex2_approx(ai + e2.y);
                                m0 = j < i ? m0 : (j == i ? m0 + Dh : 0.f);
                                m1 = j + 1 < i ? m1 : (j + 1 == i ? m1 + Dh : 0.f);
                                m[8 * hb + q] = pack_bf16(m0, m1);
                                ml[8 * hb + q] = pack_bf16(m0 - bf16_lo(m[8 * hb + q]), m1 - bf16_hi(m[8 * hb + q]));
                            }
                        }
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) m[q] = ml[q] = 0u;
                }
                tmem_st16(tlane + 192 + 16 * jb, m);
                tmem_st16(tlane + 448 + 16 * jb, ml);
            }
            tmem_st_wait();
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(!ok_all)) break;  // w x, S parts and M written; G read
        tc_fence_after();
        if (tid == 0) {
            if constexpr (!kFull) {
                // state: S^T += B^T (w x): A = B rows (MN-major, two 64-column blocks), K = the tokens
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma(tbase + kColState, umma_desc(sb + so + Lay::BT + ks * 2048, 16384, 1024),
                         umma_desc(sb + Lay::XW + ks * 2048, 16384, 1024), kIdState, ks > 0);
                umma_commit(mbS);
            } else {
                // outputs: C [S_in^T hi | lo] (N = 128, the lo part 16 KB after the hi part)
                // into columns 256..383, M x into 384..447 (M's hi part, then its lo part)
                if (s_nonzero || k > 0) {
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t off = so + (ks >> 2) * 16384 + (ks & 3) * 32;
                        umma(tbase + 256, umma_desc(sb + Lay::CT + off, 16, 1024),
                             umma_desc(sb + Lay::SH + ks * 2048, 16384, 1024), kIdOff, ks > 0);
                    }
                }
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_ts(tbase + 384, tbase + 192 + 8 * ks, umma_desc(sb + so + Lay::XT + ks * 2048, 16384, 1024),
                            kIdDiag, ks > 0);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    umma_ts(tbase + 384, tbase + 448 + 8 * ks, umma_desc(sb + so + Lay::XT + ks * 2048, 16384, 1024),
                            kIdDiag, 1);
                umma_commit(mbY);
            }
        }
        // ---- state update (thread (n, hf): its head columns of row n of S^T)
        ok_all &= mbar_wait(mbS, par);
        tc_fence_after();
        const float alast = pr[Q - 1];
        seg_decay += alast;
        const float el = ex2_approx(alast);
        if constexpr (!kFull) {
            if (c + 1 < c_end) issue_chunk(c + 1, (k + 1) & 1);     // every tensor read of this chunk is done
        }
#pragma unroll
        for (int q0 = 0; q0 < PH; q0 += 16) {
            float d[16];
            tmem_ld16(tlane + kColState + PH * hf + q0, d);
#pragma unroll
            for (int q = 0; q < 16; ++q) S[q0 + q] = fmaf(el, S[q0 + q], d[q]);
        }
        if constexpr (kFull) {
            // ---- y row i, head columns of this half: 2^acum_i (C S_in^T)_i + (M x)_i
            ok_all &= mbar_wait(mbY, par);
            tc_fence_after();
            const int i = r;
            const bool with_state = s_nonzero || k > 0;
            const float ea = ex2_approx(pr[i]);
            const bool inside = c * Q + i < L;
            __nv_bfloat16* yo = p.y + (((size_t)b * L + (size_t)c * Q + i) * H + h) * P + PH * hf;
#pragma unroll
            for (int q0 = 0; q0 < PH; q0 += 16) {
                float yd[16], yh[16], yl[16];
                tmem_ld16(tlane + 384 + PH * hf + q0, yd);     // warp-wide: rows past L take part too
                if (with_state) {
                    tmem_ld16(tlane + 256 + PH * hf + q0, yh);
                    tmem_ld16(tlane + 320 + PH * hf + q0, yl);
                }
                uint32_t o[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float y0 = with_state ? fmaf(ea, yh[2 * q] + yl[2 * q], yd[2 * q]) : yd[2 * q];
                    const float y1 = with_state ? fmaf(ea, yh[2 * q + 1] + yl[2 * q + 1], yd[2 * q + 1]) : yd[2 * q + 1];
                    o[q] = pack_bf16(y0, y1);
                }
                if (inside) {
                    *reinterpret_cast<uint4*>(yo + q0) = make_uint4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<uint4*>(yo + q0 + 8) = make_uint4(o[4], o[5], o[6], o[7]);
                }
            }
        }
    }

    cp_async_wait_0();                         // this thread's copies in flight
    // A wait that gave up (in the loop, or in the last chunk after its final
    // barrier) leaves products thread 0 issued possibly still running: before
    // the tensor memory is freed, one more commit from thread 0 on the drain
    // barrier tracks the completion of all of them, waited for with the same
    // bound.  If that wait gives up too, the tensor memory is not freed (a
    // late product must not land in columns another CTA has allocated).
    const bool failed = __syncthreads_or(!ok_all);
    bool drained = true;
    if (failed) {
        if (tid == 0) {
            tc_fence_after();
            umma_commit(mbF);
        }
        drained = mbar_wait(mbF, 0u);
        drained = !__syncthreads_or(!drained);
        if (tid == 0) atomicExch(p.err, 1);
    }
    if constexpr (kFull) {
        if (seg == p.segs - 1) {
#pragma unroll
            for (int q = 0; q < PH; ++q) p.h_out[hoff + (size_t)q * N] = S[q];
        }
    } else {
        float* dst = p.sloc + (size_t)seg * BHPN + hoff;
#pragma unroll
        for (int q = 0; q < PH; ++q) dst[(size_t)q * N] = S[q];
        if (tid == 0) p.sega[((size_t)seg * p.B + b) * H + h] = seg_decay;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (w == 0 && drained)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(Lay::TMEM_COLS));
}

}  // namespace axon
