// scan_quad.cuh -- warp-independent selective scan, states split in quadrants.
//
// Every warp owns 8 consecutive channels of one batch row for the whole
// sequence and never waits for another warp (no CTA barrier): lane
// = 8 * g + c handles channel c and the state quadrant g (states 4g .. 4g+3).
// Per chunk of T tokens the warp
//
//   1. copies (cp.async, one chunk ahead, double buffered) the x rows with a
//      3-token halo, the z and dt_raw rows of its 8 channels (one 16-byte
//      piece per row for bf16, two for fp32) and the chunk's B, C rows into
//      its own shared memory;
//   2. runs the per-(token, channel) prologue once: lane (g, c) takes tokens
//      g*T/4 .. g*T/4 + T/4 - 1 of channel c (the causal conv window slides in
//      registers), writes (dt, f) -- f = dt*u first order, u for ZOH -- to
//      shared memory and keeps D*u and SiLU(z) of its tokens in registers;
//   3. walks the T tokens: a = 2^(dt * A log2 e) for the lane's 4 states,
//      h = a h + f B (packed fp32x2), partial_t = C . h over the quadrant;
//   4. sums the four quadrant partials of each (token, channel) with a
//      three-shuffle reduce-scatter over tokens (t, t+T/4, t+T/2, t+3T/4):
//      lane (g, c) ends with the full C . h of token g*T/4 + j -- exactly the
//      token whose D*u and SiLU(z) it computed -- and stores
//      y = (C . h + D u) SiLU(z) straight to global memory.
//
// Shared-memory reads are laid out for the sm_100 wavefront rules: B and C
// quads are uniform per quarter warp (one quadrant per quarter); rows read by
// the four quadrants at once are padded one row per T/4 rows.
//
// Recurrence and gating: Axon-SSM page, recurrence equation, "Selective
// mechanism", "Diagonal state matrix", "Gating"; with kZoh the exact
// zero-order-hold Bbar of section "ZOH discretisation".
#pragma once

#include "device_math.cuh"
#include "scan_chunked.cuh"   // ChunkParams, SmemIo, cp.async helpers, f2

namespace axon {

constexpr int kQuadCh = 8;   // channels per warp

// Byte layout of one warp's shared memory; identical on host and device.
struct QuadSmem {
    int xs, zs, ds, bs, cs, stage, pf, total;
    __host__ __device__ static int pad(int r, int TQ) { return r + r / TQ; }
    __host__ __device__ QuadSmem(int T, int io_bytes) {
        const int TQ = T / 4;
        const int XB = kQuadCh * io_bytes;
        int off = 0;
        xs = off; off += (pad(T + kK - 2, TQ) + 1) * XB;
        zs = off; off += (pad(T - 1, TQ) + 1) * XB;
        ds = off; off += (pad(T - 1, TQ) + 1) * XB;
        bs = off; off += T * kN * io_bytes;
        cs = off; off += T * kN * io_bytes;
        stage = (off + 15) & ~15;
        off = 2 * stage;
        pf = off; off += (pad(T - 1, TQ) + 1) * kQuadCh * 8;
        total = (off + 127) & ~127;
    }
};

// Four consecutive values of a staged B/C row as float32 (quadrant g).
template <class Io> struct QuadRow;
template <> struct QuadRow<IoF32> {
    __device__ __forceinline__ static void ld(const unsigned char* row, int g, float (&v)[4]) {
        const float4 q = *reinterpret_cast<const float4*>(row + g * 16);
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
};
template <> struct QuadRow<IoBF16> {
    __device__ __forceinline__ static void ld(const unsigned char* row, int g, float (&v)[4]) {
        const uint2 q = *reinterpret_cast<const uint2*>(row + g * 8);
        v[0] = __uint_as_float(q.x << 16); v[1] = __uint_as_float(q.x & 0xffff0000u);
        v[2] = __uint_as_float(q.y << 16); v[3] = __uint_as_float(q.y & 0xffff0000u);
    }
};

// The walk goes in blocks of kBlk tokens: the decays and inputs of a block
// (independent of the state) first, then its state updates.
template <class Io, int T, bool kZoh = false, int kBlk = 4>
__global__ void __launch_bounds__(256) scan_quad_kernel(ChunkParams p) {
    static_assert(T % 16 == 0 && T % kBlk == 0, "T: multiple of 16 and of the walk block");
    using TT = typename Io::T;
    using SI = SmemIo<Io>;
    constexpr int S = Io::kBytes;
    constexpr int XB = kQuadCh * S;          // bytes of one staged row (8 channels)
    constexpr int TQ = T / 4;                // tokens per quadrant in the prologue
    constexpr int P = XB / 16;               // 16-byte pieces per staged row
    constexpr int PB = kN * S / 16;          // 16-byte pieces per B/C row
    constexpr int NXP = (T + kK - 1) * P, NX = (NXP + 31) / 32;   // x pieces per chunk, per lane
    constexpr int NZP = T * P, NZ = (NZP + 31) / 32;               // z (and dt) pieces
    constexpr int NBP = T * PB, NB = (NBP + 31) / 32;              // B (and C) pieces
    extern __shared__ __align__(16) unsigned char smem[];

    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int tiles = (p.E + kQuadCh - 1) / kQuadCh;
    if (gw >= p.B * tiles) return;           // the whole warp leaves; warps never wait for each other
    const int b = gw / tiles;
    const int e0 = (gw - b * tiles) * kQuadCh;
    const int ne = min(kQuadCh, p.E - e0);   // 8, or 4 for an fp32 tail
    const int g = lane >> 3;                 // state quadrant
    const int c = lane & 7;                  // channel in the tile
    const bool active = c < ne;
    const int e = e0 + (active ? c : 0);
    const QuadSmem lay(T, S);
    unsigned char* ws = smem + (threadIdx.x >> 5) * lay.total;

    const unsigned char* xg = static_cast<const unsigned char*>(p.x);
    const unsigned char* zg = static_cast<const unsigned char*>(p.z);
    const unsigned char* dg = static_cast<const unsigned char*>(p.dt_raw);
    const unsigned char* bg = static_cast<const unsigned char*>(p.Bm);
    const unsigned char* cg = static_cast<const unsigned char*>(p.Cm);
    const unsigned char* ccg = static_cast<const unsigned char*>(p.conv_cache_in);
    const int row_bytes = p.E * S;           // the host keeps (T + K) * E * S below 2^31
    const int npc = (ne * S + 15) / 16;      // pieces of a row inside the tile
    const size_t tile_off = (size_t)b * p.L * row_bytes + (size_t)e0 * S;

    // ---- this lane's share of a chunk's copies: shared-memory destinations
    // and byte offsets from the chunk's first row (t0), fixed for all chunks
    int xsd[NX], xgo[NX], zsd[NZ], zgo[NZ], bso[NB];
    bool xok[NX], zok[NZ], bok[NB];
#pragma unroll
    for (int i = 0; i < NX; ++i) {
        const int w = lane + 32 * i, r = w / P, pc = w % P;
        xok[i] = w < NXP && pc < npc;
        xsd[i] = lay.xs + QuadSmem::pad(r, TQ) * XB + pc * 16;
        xgo[i] = (r - (kK - 1)) * row_bytes + pc * 16;
    }
#pragma unroll
    for (int i = 0; i < NZ; ++i) {
        const int w = lane + 32 * i, r = w / P, pc = w % P;
        zok[i] = w < NZP && pc < npc;
        zsd[i] = QuadSmem::pad(r, TQ) * XB + pc * 16;
        zgo[i] = r * row_bytes + pc * 16;
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
            const unsigned char* xr = xg + tile_off + (size_t)t0 * row_bytes;
            const unsigned char* zr = zg + tile_off + (size_t)t0 * row_bytes;
            const unsigned char* dr = dg + tile_off + (size_t)t0 * row_bytes;
            const size_t bc0 = ((size_t)b * p.L + t0) * (kN * S);
#pragma unroll
            for (int i = 0; i < NX; ++i)
                if (xok[i]) cp_async16(sb + xsd[i], xr + xgo[i], true);
#pragma unroll
            for (int i = 0; i < NZ; ++i)
                if (zok[i]) {
                    cp_async16(sb + lay.zs + zsd[i], zr + zgo[i], true);
                    cp_async16(sb + lay.ds + zsd[i], dr + zgo[i], true);
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
        for (int w = lane; w < NXP; w += 32) {
            const int r = w / P, pc = w % P;
            const int t = t0 - (kK - 1) + r;
            const void* src = xg;
            bool ok = false;
            if (pc < npc) {
                if (t >= 0 && t < p.L) {
                    src = xg + tile_off + (size_t)t * row_bytes + pc * 16;
                    ok = true;
                } else if (t < 0 && ccg != nullptr) {
                    src = ccg + ((size_t)b * (kK - 1) + (kK - 1 + t)) * row_bytes + (size_t)e0 * S + pc * 16;
                    ok = true;
                }
            }
            cp_async16(sb + lay.xs + QuadSmem::pad(r, TQ) * XB + pc * 16, src, ok);
        }
        for (int w = lane; w < NZP; w += 32) {
            const int r = w / P, pc = w % P;
            const int t = t0 + r;
            const bool ok = t < p.L && pc < npc;
            const size_t go = ok ? tile_off + (size_t)t * row_bytes + pc * 16 : 0;
            const int so = QuadSmem::pad(r, TQ) * XB + pc * 16;
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
    // quadrant's A log2 e (and 1/A for ZOH) and initial states
    const float w0 = __ldg(p.conv_w + (size_t)e * kK + 0);
    const float w1 = __ldg(p.conv_w + (size_t)e * kK + 1);
    const float w2 = __ldg(p.conv_w + (size_t)e * kK + 2);
    const float w3 = __ldg(p.conv_w + (size_t)e * kK + 3);
    const float cb = __ldg(p.conv_b + e);
    const float db = __ldg(p.dt_bias + e);
    const float Dv = __ldg(p.D + e);
    float2 s01, s23, iA01 = f2(0.f, 0.f), iA23 = f2(0.f, 0.f), h01, h23;
    {
        const float4 al = __ldg(reinterpret_cast<const float4*>(p.A_log + (size_t)e * kN) + g);
        s01 = f2(-expf(al.x) * kLog2e, -expf(al.y) * kLog2e);
        s23 = f2(-expf(al.z) * kLog2e, -expf(al.w) * kLog2e);
        if constexpr (kZoh) {
            iA01 = f2(kLog2e / s01.x, kLog2e / s01.y);
            iA23 = f2(kLog2e / s23.x, kLog2e / s23.y);
        }
        float4 h0 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p.ssm_state_in && active)
            h0 = reinterpret_cast<const float4*>(p.ssm_state_in + ((size_t)b * p.E + e) * kN)[g];
        h01 = f2(h0.x, h0.y);
        h23 = f2(h0.z, h0.w);
    }

    // y of token t0 + g*TQ + j, channel e: ybase + (t0 + j) * row_bytes
    unsigned char* ybase = static_cast<unsigned char*>(p.y) + tile_off + (size_t)(g * TQ) * row_bytes + c * S;
    const int nck = (p.L + T - 1) / T;

    // ---- prologue, one token at a time: lane (g, c) takes tokens g*TQ ..
    // g*TQ + TQ - 1 of channel c; the conv window slides in registers
    struct Window { float xm3, xm2, xm1; };
    auto pro_begin = [&](const unsigned char* sb) {
        const int tb = g * TQ;
        const unsigned char* xc = sb + lay.xs + c * S;
        return Window{SI::ld(xc + QuadSmem::pad(tb + 0, TQ) * XB), SI::ld(xc + QuadSmem::pad(tb + 1, TQ) * XB),
                      SI::ld(xc + QuadSmem::pad(tb + 2, TQ) * XB)};
    };
    auto pro_token = [&](Window& wd, const unsigned char* sb, float2* pfb, int t0, bool full, int i,
                         float& du, float& gzv) {
        const int t = g * TQ + i;
        const float xt = SI::ld(sb + lay.xs + c * S + QuadSmem::pad(t + 3, TQ) * XB);
        float xv = fmaf(w0, wd.xm3, cb);
        xv = fmaf(w1, wd.xm2, xv);
        xv = fmaf(w2, wd.xm1, xv);
        xv = fmaf(w3, xt, xv);
        wd.xm3 = wd.xm2; wd.xm2 = wd.xm1; wd.xm1 = xt;
        const float u = silu(xv);
        const int tp = t + g;            // padded row of token t (t / TQ == g)
        const float dt = dt_from_raw(SI::ld(sb + lay.ds + tp * XB + c * S) + db);
        const bool live = full || (t0 + t) < p.L;
        const float dtl = live ? dt : 0.0f;          // dt = 0: decay 1, no input
        const float f = live ? (kZoh ? u : dt * u) : 0.0f;
        pfb[tp * kQuadCh + c] = make_float2(dtl, f);
        du = Dv * u;
        gzv = silu(SI::ld(sb + lay.zs + tp * XB + c * S));
    };

    // ---- walk pieces: decays and inputs of token t (state-independent), then
    // the state update and the quadrant's partial C . h
    float part[T];
    auto decay_input = [&](const unsigned char* sb, const float2* pfb, int t,
                           float2& a01, float2& a23, float2& u01, float2& u23) {
        const float2 v = pfb[(t + t / TQ) * kQuadCh + c];
        const float2 dd = f2(v.x, v.x), ff = f2(v.y, v.y);
        float Bq[4];
        QuadRow<Io>::ld(sb + lay.bs + t * (kN * S), g, Bq);
        const float2 arg01 = __fmul2_rn(dd, s01);
        const float2 arg23 = __fmul2_rn(dd, s23);
        a01 = f2(ex2_approx(arg01.x), ex2_approx(arg01.y));
        a23 = f2(ex2_approx(arg23.x), ex2_approx(arg23.y));
        u01 = __fmul2_rn(ff, f2(Bq[0], Bq[1]));
        u23 = __fmul2_rn(ff, f2(Bq[2], Bq[3]));
        if constexpr (kZoh) {
            u01 = __fmul2_rn(u01, f2(zoh_bbar(v.x, arg01.x * kLn2, a01.x, iA01.x),
                                     zoh_bbar(v.x, arg01.y * kLn2, a01.y, iA01.y)));
            u23 = __fmul2_rn(u23, f2(zoh_bbar(v.x, arg23.x * kLn2, a23.x, iA23.x),
                                     zoh_bbar(v.x, arg23.y * kLn2, a23.y, iA23.y)));
        }
    };
    auto update = [&](const unsigned char* sb, int t, float2 a01, float2 a23, float2 u01, float2 u23) {
        float Cq[4];
        QuadRow<Io>::ld(sb + lay.cs + t * (kN * S), g, Cq);
        h01 = __ffma2_rn(a01, h01, u01);
        h23 = __ffma2_rn(a23, h23, u23);
        const float2 pq = __ffma2_rn(f2(Cq[2], Cq[3]), h23, __fmul2_rn(f2(Cq[0], Cq[1]), h01));
        part[t] = pq.x + pq.y;
    };
    auto walk_block = [&](const unsigned char* sb, const float2* pfb, int tb) {
        float2 a01[kBlk], a23[kBlk], u01[kBlk], u23[kBlk];
#pragma unroll
        for (int i = 0; i < kBlk; ++i) decay_input(sb, pfb, tb + i, a01[i], a23[i], u01[i], u23[i]);
#pragma unroll
        for (int i = 0; i < kBlk; ++i) update(sb, tb + i, a01[i], a23[i], u01[i], u23[i]);
    };

    // ---- reduce-scatter over the quadrants (lanes 8 and 16 apart) and store y
    auto finish = [&](int t0, bool full, const float (&Du)[TQ], const float (&gz)[TQ]) {
        const bool hi = (g & 2) != 0, lo = (g & 1) != 0;
        unsigned char* yrow = ybase + (size_t)t0 * row_bytes;
#pragma unroll
        for (int j = 0; j < TQ; ++j) {
            const float v0 = part[j], v1 = part[TQ + j], v2 = part[2 * TQ + j], v3 = part[3 * TQ + j];
            const float k0 = hi ? v2 : v0, k1 = hi ? v3 : v1;     // pair this lane keeps
            const float s0 = hi ? v0 : v2, s1 = hi ? v1 : v3;     // pair its partner keeps
            const float m0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 16);
            const float m1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 16);
            const float keep = lo ? m1 : m0, send = lo ? m0 : m1;
            const float tot = keep + __shfl_xor_sync(0xffffffffu, send, 8);   // token g*TQ + j
            if (active && (full || t0 + g * TQ + j < p.L))
                Io::store(reinterpret_cast<TT*>(yrow + j * row_bytes), (tot + Du[j]) * gz[j]);
        }
    };

    float2* pf = reinterpret_cast<float2*>(ws + lay.pf);   // [padded token][channel] (dt, f)
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
        float Du[TQ], gz[TQ];
        Window wd = pro_begin(sb);
#pragma unroll
        for (int i = 0; i < TQ; ++i) pro_token(wd, sb, pf, t0, full, i, Du[i], gz[i]);
        __syncwarp();
#pragma unroll
        for (int tb = 0; tb < T; tb += kBlk) walk_block(sb, pf, tb);
        finish(t0, full, Du, gz);
    }

    // ---- final caches
    if (active) {
        reinterpret_cast<float4*>(p.ssm_state_out + ((size_t)b * p.E + e) * kN)[g] =
            make_float4(h01.x, h01.y, h23.x, h23.y);
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
}

}  // namespace axon
