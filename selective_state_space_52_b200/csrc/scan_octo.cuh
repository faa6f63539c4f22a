// scan_octo.cuh -- warp-independent selective scan, states split in eighths.
//
// The quadrant scan's structure (scan_quad.cuh) with twice the warps: every
// warp owns 4 consecutive channels of one batch row for the whole sequence,
// and lane = 8 * c + g handles channel c and the state pair g (states 2g,
// 2g+1).  A quarter warp is one channel, so the per-token (dt, f) read is
// uniform per quarter warp; the B and C pairs are 8 consecutive 4-byte words
// (bf16) per quarter.  Per chunk of T tokens the warp
//
//   1. copies (cp.async, one chunk ahead, double buffered) the 16-byte aligned
//      window holding its 4 channels (8 bf16 or 4 fp32 channels per row) of
//      the x rows with a 3-token halo, the z and dt_raw rows, and the chunk's
//      B, C rows into its own shared memory;
//   2. runs the prologue once per (token, channel): lane (c, g) takes tokens
//      g*T/8 .. g*T/8 + T/8 - 1 of channel c, writes (dt, f) to shared memory
//      and keeps D*u and SiLU(z) of its tokens in registers;
//   3. walks the T tokens: a = 2^(dt * A log2 e) for its 2 states, h = a h +
//      f B (packed fp32x2), partial_t = C . h over the pair;
//   4. sums the eight partials of each (token, channel) with a seven-shuffle
//      reduce-scatter over tokens (t, t + T/8, ..., t + 7T/8): lane (c, g)
//      ends with the full C . h of token g*T/8 + j and stores
//      y = (C . h + D u) SiLU(z) straight to global memory.
//
// Recurrence and gating: Axon-SSM page, recurrence equation, "Selective
// mechanism", "Diagonal state matrix", "Gating"; with kZoh the exact
// zero-order-hold Bbar of section "ZOH discretisation".
#pragma once

#include "device_math.cuh"
#include "scan_chunked.cuh"   // ChunkParams, SmemIo, cp.async helpers, f2

namespace axon {

constexpr int kOctoCh = 4;   // channels per warp

// Byte layout of one warp's shared memory; identical on host and device.
// Staged rows are one 16-byte piece; rows read by the eight state pairs at
// once are padded one row per T/8 rows.
struct OctoSmem {
    int xs, zs, ds, bs, cs, stage, pf, total;
    __host__ __device__ static int pad(int r, int TE) { return r + r / TE; }
    __host__ __device__ OctoSmem(int T, int io_bytes) {
        const int TE = T / 8;
        int off = 0;
        xs = off; off += (pad(T + kK - 2, TE) + 1) * 16;
        zs = off; off += (pad(T - 1, TE) + 1) * 16;
        ds = off; off += (pad(T - 1, TE) + 1) * 16;
        bs = off; off += T * kN * io_bytes;
        cs = off; off += T * kN * io_bytes;
        stage = (off + 15) & ~15;
        off = 2 * stage;
        pf = off; off += (pad(T - 1, TE) + 1) * kOctoCh * 8;
        total = (off + 127) & ~127;
    }
};

// The state pair g of a staged B/C row as float32.
template <class Io> struct OctoRow;
template <> struct OctoRow<IoF32> {
    __device__ __forceinline__ static float2 ld(const unsigned char* row, int g) {
        return *reinterpret_cast<const float2*>(row + g * 8);
    }
};
template <> struct OctoRow<IoBF16> {
    __device__ __forceinline__ static float2 ld(const unsigned char* row, int g) {
        const uint32_t q = *reinterpret_cast<const uint32_t*>(row + g * 4);
        return f2(__uint_as_float(q << 16), __uint_as_float(q & 0xffff0000u));
    }
};

template <class Io, int T, bool kZoh = false, int kBlk = 4>
__global__ void __launch_bounds__(256) scan_octo_kernel(ChunkParams p) {
    static_assert(T % 32 == 0 && T % kBlk == 0, "T: multiple of 32 and of the walk block");
    using TT = typename Io::T;
    using SI = SmemIo<Io>;
    constexpr int S = Io::kBytes;
    constexpr int TE = T / 8;                // tokens per state pair in the prologue
    constexpr int PB = kN * S / 16;          // 16-byte pieces per B/C row
    constexpr int NXP = T + kK - 1, NX = (NXP + 31) / 32;   // x pieces per chunk, per lane
    constexpr int NZ = (T + 31) / 32;                       // z (and dt) pieces
    constexpr int NBP = T * PB, NB = (NBP + 31) / 32;       // B (and C) pieces
    extern __shared__ __align__(16) unsigned char smem[];

    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int tiles = p.E / kOctoCh;         // E is a multiple of 4 (fp32) or 8 (bf16)
    if (gw >= p.B * tiles) return;           // the whole warp leaves; warps never wait for each other
    const int b = gw / tiles;
    const int e0 = (gw - b * tiles) * kOctoCh;
    const int c = lane >> 3;                 // channel in the tile (a quarter warp)
    const int g = lane & 7;                  // state pair
    const int e = e0 + c;
    const OctoSmem lay(T, S);
    unsigned char* ws = smem + (threadIdx.x >> 5) * lay.total;

    const unsigned char* xg = static_cast<const unsigned char*>(p.x);
    const unsigned char* zg = static_cast<const unsigned char*>(p.z);
    const unsigned char* dg = static_cast<const unsigned char*>(p.dt_raw);
    const unsigned char* bg = static_cast<const unsigned char*>(p.Bm);
    const unsigned char* cg = static_cast<const unsigned char*>(p.Cm);
    const unsigned char* ccg = static_cast<const unsigned char*>(p.conv_cache_in);
    const int row_bytes = p.E * S;           // the host keeps (T + K) * E * S below 2^31
    const int wb0 = (e0 * S) & ~15;          // the 16-byte window holding the tile
    const int coff = e0 * S - wb0 + c * S;   // this channel's bytes in a staged row
    const size_t win_off = (size_t)b * p.L * row_bytes + wb0;

    // ---- this lane's share of a chunk's copies (fixed for all chunks)
    int xsd[NX], xgo[NX], bso[NB];
    bool xok[NX], bok[NB];
#pragma unroll
    for (int i = 0; i < NX; ++i) {
        const int r = lane + 32 * i;
        xok[i] = r < NXP;
        xsd[i] = lay.xs + OctoSmem::pad(r, TE) * 16;
        xgo[i] = (r - (kK - 1)) * row_bytes;
    }
#pragma unroll
    for (int i = 0; i < NB; ++i) {
        const int w = lane + 32 * i;
        bok[i] = w < NBP;
        bso[i] = (w / PB) * (kN * S) + (w % PB) * 16;
    }

    auto prefetch = [&](int k, int st) {
        unsigned char* sb = ws + st * lay.stage;
        const int t0 = k * T;
        if (k > 0 && t0 + T <= p.L) {
            // every row of the chunk and its halo lies inside the sequence
            const unsigned char* xr = xg + win_off + (size_t)t0 * row_bytes;
            const size_t zo = win_off + (size_t)t0 * row_bytes;
            const size_t bc0 = ((size_t)b * p.L + t0) * (kN * S);
#pragma unroll
            for (int i = 0; i < NX; ++i)
                if (xok[i]) cp_async16(sb + xsd[i], xr + xgo[i], true);
#pragma unroll
            for (int i = 0; i < NZ; ++i) {
                const int r = lane + 32 * i;
                if (r < T) {
                    const int so = OctoSmem::pad(r, TE) * 16;
                    cp_async16(sb + lay.zs + so, zg + zo + (size_t)r * row_bytes, true);
                    cp_async16(sb + lay.ds + so, dg + zo + (size_t)r * row_bytes, true);
                }
            }
#pragma unroll
            for (int i = 0; i < NB; ++i)
                if (bok[i]) {
                    cp_async16(sb + lay.bs + bso[i], bg + bc0 + bso[i], true);
                    cp_async16(sb + lay.cs + bso[i], cg + bc0 + bso[i], true);
                }
            return;
        }
        // first chunk (halo from the conv cache or zeros) or a ragged last chunk
        for (int r = lane; r < NXP; r += 32) {
            const int t = t0 - (kK - 1) + r;
            const void* src = xg;
            bool ok = false;
            if (t >= 0 && t < p.L) {
                src = xg + win_off + (size_t)t * row_bytes;
                ok = true;
            } else if (t < 0 && ccg != nullptr) {
                src = ccg + ((size_t)b * (kK - 1) + (kK - 1 + t)) * row_bytes + wb0;
                ok = true;
            }
            cp_async16(sb + lay.xs + OctoSmem::pad(r, TE) * 16, src, ok);
        }
        for (int r = lane; r < T; r += 32) {
            const int t = t0 + r;
            const bool ok = t < p.L;
            const size_t go = ok ? win_off + (size_t)t * row_bytes : 0;
            const int so = OctoSmem::pad(r, TE) * 16;
            cp_async16(sb + lay.zs + so, zg + go, ok);
            cp_async16(sb + lay.ds + so, dg + go, ok);
        }
        for (int w = lane; w < NBP; w += 32) {
            const int r = w / PB, pc = w % PB;
            const int t = t0 + r;
            const bool ok = t < p.L;
            const size_t go = ok ? ((size_t)b * p.L + t) * (kN * S) + pc * 16 : 0;
            cp_async16(sb + lay.bs + r * (kN * S) + pc * 16, bg + go, ok);
            cp_async16(sb + lay.cs + r * (kN * S) + pc * 16, cg + go, ok);
        }
    };

    // ---- per-lane constants: the channel's conv / dt / D parameters, the
    // pair's A log2 e (and 1/A for ZOH) and initial states
    const float w0 = __ldg(p.conv_w + (size_t)e * kK + 0);
    const float w1 = __ldg(p.conv_w + (size_t)e * kK + 1);
    const float w2 = __ldg(p.conv_w + (size_t)e * kK + 2);
    const float w3 = __ldg(p.conv_w + (size_t)e * kK + 3);
    const float cb = __ldg(p.conv_b + e);
    const float db = __ldg(p.dt_bias + e);
    const float Dv = __ldg(p.D + e);
    float2 s01, iA01 = f2(0.f, 0.f), h01;
    {
        const float2 al = __ldg(reinterpret_cast<const float2*>(p.A_log + (size_t)e * kN) + g);
        s01 = f2(-expf(al.x) * kLog2e, -expf(al.y) * kLog2e);
        if constexpr (kZoh) iA01 = f2(kLog2e / s01.x, kLog2e / s01.y);
        h01 = p.ssm_state_in ? reinterpret_cast<const float2*>(p.ssm_state_in + ((size_t)b * p.E + e) * kN)[g]
                             : f2(0.f, 0.f);
    }

    // y of token t0 + g*TE + j, channel e: ybase + (t0 + j) * row_bytes
    unsigned char* ybase = static_cast<unsigned char*>(p.y) + (size_t)b * p.L * row_bytes +
                           (size_t)(g * TE) * row_bytes + (size_t)e * S;
    const int nck = (p.L + T - 1) / T;
    float2* pf = reinterpret_cast<float2*>(ws + lay.pf);   // [padded token][channel] (dt, f)
    float part[T];

    prefetch(0, 0);
    cp_async_commit();
    for (int k = 0; k < nck; ++k) {
        const int st = k & 1;
        const int t0 = k * T;
        const bool full = t0 + T <= p.L;
        __syncwarp();                        // every lane is done with the stage refilled below and with pf
        if (k + 1 < nck) prefetch(k + 1, st ^ 1);
        cp_async_commit();
        cp_async_wait_1();                   // this lane's copies of chunk k have landed
        __syncwarp();                        // ... and every lane's
        const unsigned char* sb = ws + st * lay.stage;

        // ---- prologue: tokens g*TE .. g*TE + TE - 1 of channel c
        float Du[TE], gz[TE];
        {
            const int tb = g * TE;
            const unsigned char* xc = sb + lay.xs + coff;
            float xm3 = SI::ld(xc + OctoSmem::pad(tb + 0, TE) * 16);
            float xm2 = SI::ld(xc + OctoSmem::pad(tb + 1, TE) * 16);
            float xm1 = SI::ld(xc + OctoSmem::pad(tb + 2, TE) * 16);
#pragma unroll
            for (int i = 0; i < TE; ++i) {
                const int t = tb + i;
                const float xt = SI::ld(xc + OctoSmem::pad(t + 3, TE) * 16);
                float xv = fmaf(w0, xm3, cb);
                xv = fmaf(w1, xm2, xv);
                xv = fmaf(w2, xm1, xv);
                xv = fmaf(w3, xt, xv);
                xm3 = xm2; xm2 = xm1; xm1 = xt;
                const float u = silu(xv);
                const int tp = t + g;        // padded row of token t (t / TE == g)
                const float dt = dt_from_raw(SI::ld(sb + lay.ds + tp * 16 + coff) + db);
                const bool live = full || (t0 + t) < p.L;
                const float dtl = live ? dt : 0.0f;          // dt = 0: decay 1, no input
                const float f = live ? (kZoh ? u : dt * u) : 0.0f;
                pf[tp * kOctoCh + c] = make_float2(dtl, f);
                Du[i] = Dv * u;
                gz[i] = silu(SI::ld(sb + lay.zs + tp * 16 + coff));
            }
        }
        __syncwarp();

        // ---- walk: 2 states per lane, partial C . h per token
#pragma unroll
        for (int tb = 0; tb < T; tb += kBlk) {
            float2 a[kBlk], u[kBlk];
#pragma unroll
            for (int i = 0; i < kBlk; ++i) {
                const int t = tb + i;
                const float2 v = pf[(t + t / TE) * kOctoCh + c];
                const float2 arg = __fmul2_rn(f2(v.x, v.x), s01);
                a[i] = f2(ex2_approx(arg.x), ex2_approx(arg.y));
                u[i] = __fmul2_rn(f2(v.y, v.y), OctoRow<Io>::ld(sb + lay.bs + t * (kN * S), g));
                if constexpr (kZoh)
                    u[i] = __fmul2_rn(u[i], f2(zoh_bbar(v.x, arg.x * kLn2, a[i].x, iA01.x),
                                               zoh_bbar(v.x, arg.y * kLn2, a[i].y, iA01.y)));
            }
#pragma unroll
            for (int i = 0; i < kBlk; ++i) {
                const int t = tb + i;
                h01 = __ffma2_rn(a[i], h01, u[i]);
                const float2 cq = OctoRow<Io>::ld(sb + lay.cs + t * (kN * S), g);
                part[t] = fmaf(cq.x, h01.x, cq.y * h01.y);
            }
        }

        // ---- reduce-scatter over the eight pairs (lanes 4, 2, 1 apart) and store y
        const bool b2 = (g & 4) != 0, b1 = (g & 2) != 0, b0 = (g & 1) != 0;
        unsigned char* yrow = ybase + (size_t)t0 * row_bytes;
#pragma unroll
        for (int j = 0; j < TE; ++j) {
            float m[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float lo4 = part[i * TE + j], hi4 = part[(4 + i) * TE + j];
                const float keep = b2 ? hi4 : lo4, send = b2 ? lo4 : hi4;
                m[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);      // pair 4*b2 + i
            }
            float n[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float keep = b1 ? m[2 + i] : m[i], send = b1 ? m[i] : m[2 + i];
                n[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);      // pair 4*b2 + 2*b1 + i
            }
            const float keep = b0 ? n[1] : n[0], send = b0 ? n[0] : n[1];
            const float tot = keep + __shfl_xor_sync(0xffffffffu, send, 1);   // token g*TE + j
            if (full || t0 + g * TE + j < p.L)
                Io::store(reinterpret_cast<TT*>(yrow + j * row_bytes), (tot + Du[j]) * gz[j]);
        }
    }

    // ---- final caches
    reinterpret_cast<float2*>(p.ssm_state_out + ((size_t)b * p.E + e) * kN)[g] = h01;
    if (g == 0) {
        // the last K-1 raw inputs of conv_cache_in ++ x (all read before any write: may alias)
        const TT* xs = static_cast<const TT*>(p.x);
        const TT* cc = static_cast<const TT*>(p.conv_cache_in);
        TT v[kK - 1];
#pragma unroll
        for (int j = 0; j < kK - 1; ++j) {
            const int t = p.L - (kK - 1) + j;
            if (t >= 0) v[j] = xs[((size_t)b * p.L + t) * p.E + e];
            else if (cc) v[j] = cc[((size_t)b * (kK - 1) + (kK - 1 + t)) * p.E + e];
            else v[j] = TT(0.0f);
        }
        TT* co = static_cast<TT*>(p.conv_cache_out);
#pragma unroll
        for (int j = 0; j < kK - 1; ++j) co[((size_t)b * (kK - 1) + j) * p.E + e] = v[j];
    }
}

}  // namespace axon
