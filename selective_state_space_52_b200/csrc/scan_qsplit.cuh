// scan_qsplit.cuh -- quadrant scan with each chunk split in time over W warps.
//
// A CTA of W warps owns 8 consecutive channels of one batch row for the whole
// sequence.  In every warp lane = 8 g + c handles channel c and the state
// quadrant g (states 4g .. 4g+3), so the B and C values a lane needs are the
// same for the 8 lanes of its quarter warp.  The sequence is walked in chunks
// of W * R tokens; warp w takes the run of R tokens w*R .. w*R + R - 1 of each
// chunk.  Per chunk and warp:
//
//   1. copies (cp.async, one chunk ahead, double buffered) of its run's x
//      rows with a 3-token halo, the z and dt_raw rows of the 8 channels and
//      the B, C rows into the warp's own shared memory;
//   2. the per-(token, channel) prologue, once: lane (g, c) takes tokens
//      g*R/4 .. g*R/4 + R/4 - 1 of channel c (conv window in registers), writes
//      (dt, dt, f, f) -- f = dt*u first order, u for ZOH -- and keeps D*u and
//      SiLU(z) of its tokens in registers;
//   3. W > 1: a first pass from a zero state over the run computes the
//      decays a = 2^(dt * A log2 e), the local states H_t, the decay products
//      P_t, and keeps per token C_t . H_t and C_t P_t; its end (P, H) is the
//      run's aggregate.  After one CTA barrier each warp folds the
//      aggregates of the runs before it into the chunk's entering state,
//      h = P_j h + H_j (the intra-block pass and inter-block carry of the SSD
//      article's chunked scan, applied to the diagonal recurrence), and the
//      second pass needs no recurrence and no exponential:
//      C_t . h_t = C_t . H_t + (C_t P_t) . h_in;
//      W == 1: one pass with the carried state, decays computed on the way;
//   4. the partial C . h of each token (sum over the lane's quadrant) is summed
//      over the four quadrants by a shuffle reduce-scatter that leaves each
//      lane with the tokens whose prologue it ran, and the lane stores
//      y = (C . h + D u) SiLU(z).
// The last warp's end state is the next chunk's entering state (shared
// memory, double buffered by chunk parity, so one barrier per chunk suffices).
//
// Recurrence and gating: Axon-SSM page, recurrence equation, "Selective
// mechanism", "Diagonal state matrix", "Gating"; with kZoh the exact
// zero-order-hold Bbar of section "ZOH discretisation".
#pragma once

#include "device_math.cuh"
#include "scan_chunked.cuh"   // ChunkParams, cp.async helpers, SmemIo, f2

namespace axon {

constexpr int kQsCh = 8;   // channels per CTA

// Byte layout of the shared memory: W per-warp areas, then the CTA's
// aggregate and entering-state slots.  Identical on host and device.
struct QsplitSmem {
    int xs, zs, ds, bs, cs, stage;   // one staging buffer (io dtype); two per warp
    int pf;                          // (dt, f) per (token, channel)
    int dz;                          // (D u, SiLU(z)) per (token, channel), W > 1
    int warp_bytes;
    int agg, entry, dts, total;
    __host__ __device__ static int pad(int r, int RQ) { return r + r / RQ; }
    __host__ __device__ QsplitSmem(int W, int R, int io_bytes) {
        const int RQ = R / 4;
        const int XB = kQsCh * io_bytes;
        const int RB = kN * io_bytes;
        int off = 0;
        xs = off; off += (pad(R + kK - 2, RQ) + 1) * XB;
        zs = off; off += (pad(R - 1, RQ) + 1) * XB;
        ds = off; off += (pad(R - 1, RQ) + 1) * XB;
        bs = off; off += R * RB;
        cs = off; off += R * RB;
        stage = (off + 15) & ~15;
        off = 2 * stage;
        pf = off; off += R * kQsCh * 8;
        dz = off; off += W > 1 ? R * kQsCh * 8 : 0;
        warp_bytes = (off + 127) & ~127;
        off = W * warp_bytes;
        agg = off; off += W > 1 ? 2 * W * 2 * 32 * 16 : 0;   // [parity][warp][A | H][lane] float4
        entry = off; off += W > 1 ? 2 * 32 * 16 : 0;         // [parity][lane] h0..3
        dts = off; off += W * kQsCh * 4;                     // state-only: [warp][channel] dt sums
        total = off;
    }
};

// kState (first order only): the state-only form for a time split's first
// pass -- no z, C, D, y: it walks the states to the end and writes the final
// caches and, per channel, the sum of the step sizes (p.dt_sum).
template <class Io, int W, int R, bool kZoh, bool kState = false>
__global__ void __launch_bounds__(32 * W, kZoh ? 1 : 16 / W) scan_qsplit_kernel(ChunkParams p) {
    static_assert(!(kZoh && kState), "the state-only form is first order");
    static_assert(R == 16 || R == 32, "R: 16 or 32 tokens per run");
    static_assert(W == 1 || W == 2 || W == 4 || W == 8, "W: 1, 2, 4 or 8 runs per chunk");
    using TT = typename Io::T;
    using SI = SmemIo<Io>;
    constexpr int S = Io::kBytes;
    constexpr int XB = kQsCh * S;            // bytes of one staged x/z/dt row (8 channels)
    constexpr int RB = kN * S;               // bytes of one staged B/C row
    constexpr int RQ = R / 4;                // tokens per lane in the prologue
    static_assert(RQ % 2 == 0, "the prologue runs tokens in pairs");
    constexpr int T = W * R;                 // tokens per chunk
    constexpr int P = XB / 16;               // 16-byte pieces per staged x/z/dt row
    constexpr int PB = RB / 16;              // 16-byte pieces per B/C row
    constexpr int NXP = (R + kK - 1) * P, NX = (NXP + 31) / 32;
    constexpr int NZP = R * P, NZ = (NZP + 31) / 32;
    constexpr int NBP = R * PB, NB = (NBP + 31) / 32;
    extern __shared__ __align__(16) unsigned char smem[];
    // a kernel launched after this one with programmatic serialization (the
    // whole layer's output projection) may be scheduled now: it waits for
    // this grid's completion before it reads y
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;          // run of the chunk
    const int tiles = (p.E + kQsCh - 1) / kQsCh;
    const int b = blockIdx.x / tiles;
    const int e0 = (blockIdx.x - b * tiles) * kQsCh;
    const int ne = min(kQsCh, p.E - e0);     // 8, or 4 for an fp32 tail
    const int g = lane >> 3;                 // state quadrant
    const int c = lane & 7;                  // channel in the tile
    const bool active = c < ne;
    const int e = e0 + (active ? c : 0);
    const QsplitSmem lay(W, R, S);
    unsigned char* ws = smem + w * lay.warp_bytes;

    const unsigned char* xg = static_cast<const unsigned char*>(p.x);
    const unsigned char* zg = static_cast<const unsigned char*>(p.z);
    const unsigned char* dg = static_cast<const unsigned char*>(p.dt_raw);
    const unsigned char* bg = static_cast<const unsigned char*>(p.Bm);
    const unsigned char* cg = static_cast<const unsigned char*>(p.Cm);
    const unsigned char* ccg = static_cast<const unsigned char*>(p.conv_cache_in);
    const int row_bytes = p.E * S;           // the host keeps (T + K) * E * S below 2^31
    const int npc = (ne * S + 15) / 16;      // pieces of a row inside the tile
    const size_t tile_off = (size_t)b * p.L * row_bytes + (size_t)e0 * S;

    // copies of chunk k's run of this warp into stage st
    auto prefetch = [&](int k, int st) {
        unsigned char* sb = ws + st * lay.stage;
        const int t0 = k * T + w * R;
        if (t0 >= kK - 1 && t0 + R <= p.L) {
            // every row of the run and its halo lies inside the sequence;
            // this lane's pieces: x (with halo), z and dt rows, B and C rows
            const unsigned char* xr = xg + tile_off + (size_t)t0 * row_bytes;
            const unsigned char* zr = zg + tile_off + (size_t)t0 * row_bytes;
            const unsigned char* dr = dg + tile_off + (size_t)t0 * row_bytes;
            const size_t bc0 = ((size_t)b * p.L + t0) * RB;
#pragma unroll
            for (int i = 0; i < NX; ++i) {
                const int q = lane + 32 * i, r = q / P, pc = q % P;
                if (q < NXP && pc < npc)
                    cp_async16(sb + lay.xs + QsplitSmem::pad(r, RQ) * XB + pc * 16,
                               xr + (r - (kK - 1)) * row_bytes + pc * 16, true);
            }
#pragma unroll
            for (int i = 0; i < NZ; ++i) {
                const int q = lane + 32 * i, r = q / P, pc = q % P;
                if (q < NZP && pc < npc) {
                    const int so = QsplitSmem::pad(r, RQ) * XB + pc * 16, go = r * row_bytes + pc * 16;
                    if constexpr (!kState) cp_async16(sb + lay.zs + so, zr + go, true);
                    cp_async16(sb + lay.ds + so, dr + go, true);
                }
            }
#pragma unroll
            for (int i = 0; i < NB; ++i) {
                const int q = lane + 32 * i;
                if (q < NBP) {
                    const int o = (q / PB) * RB + (q % PB) * 16;
                    cp_async16(sb + lay.bs + o, bg + bc0 + o, true);
                    if constexpr (!kState) cp_async16(sb + lay.cs + o, cg + bc0 + o, true);
                }
            }
            return;
        }
        // the sequence's first rows (halo from the conv cache or zeros) or a
        // ragged end (rows past L zero-filled)
        for (int q = lane; q < NXP; q += 32) {
            const int r = q / P, pc = q % P;
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
            cp_async16(sb + lay.xs + QsplitSmem::pad(r, RQ) * XB + pc * 16, src, ok);
        }
        for (int q = lane; q < NZP; q += 32) {
            const int r = q / P, pc = q % P;
            const int t = t0 + r;
            const bool ok = t < p.L && pc < npc;
            const size_t go = ok ? tile_off + (size_t)t * row_bytes + pc * 16 : 0;
            const int so = QsplitSmem::pad(r, RQ) * XB + pc * 16;
            if constexpr (!kState) cp_async16(sb + lay.zs + so, zg + go, ok);
            cp_async16(sb + lay.ds + so, dg + go, ok);
        }
        for (int q = lane; q < NBP; q += 32) {
            const int r = q / PB, pc = q % PB;
            const int t = t0 + r;
            const bool ok = t < p.L;
            const size_t go = ok ? ((size_t)b * p.L + t) * RB + pc * 16 : 0;
            cp_async16(sb + lay.bs + r * RB + pc * 16, bg + go, ok);
            if constexpr (!kState) cp_async16(sb + lay.cs + r * RB + pc * 16, cg + go, ok);
        }
    };

    // ---- per-lane constants: the channel's conv / dt / D parameters, the
    // quadrant's A log2 e (and 1/A for ZOH) and the initial state
    const float w0 = __ldg(p.conv_w + (size_t)e * kK + 0);
    const float w1 = __ldg(p.conv_w + (size_t)e * kK + 1);
    const float w2 = __ldg(p.conv_w + (size_t)e * kK + 2);
    const float w3 = __ldg(p.conv_w + (size_t)e * kK + 3);
    const float cb = __ldg(p.conv_b + e);
    const float db = __ldg(p.dt_bias + e);
    const float Dv = kState ? 0.0f : __ldg(p.D + e);     // D may be null for the state-only form
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

    // y of token (chunk start) + w*R + g*RQ + j, channel e: ybase + (t0 + j) * row_bytes
    unsigned char* ybase = static_cast<unsigned char*>(p.y) + tile_off + (size_t)(w * R + g * RQ) * row_bytes + c * S;
    const int nck = (p.L + T - 1) / T;
    float2* pf = reinterpret_cast<float2*>(ws + lay.pf);          // [token][channel] (dt, f)

    // B / C values of token t for this lane's quadrant, from the staged rows
    // (a float4, or four bf16 values widened in registers: the 8 lanes of a
    // quarter warp read the same 8 bytes, one shared-memory wavefront)
    auto quad_of = [&](const unsigned char* row) -> float4 {
        if constexpr (S == 4) {
            return *reinterpret_cast<const float4*>(row + 16 * g);
        } else {
            const uint2 q = *reinterpret_cast<const uint2*>(row + 8 * g);
            return make_float4(__uint_as_float(q.x << 16), __uint_as_float(q.x & 0xffff0000u),
                               __uint_as_float(q.y << 16), __uint_as_float(q.y & 0xffff0000u));
        }
    };
    auto bq = [&](const unsigned char* sb, int t) -> float4 { return quad_of(sb + lay.bs + t * RB); };
    auto cq = [&](const unsigned char* sb, int t) -> float4 { return quad_of(sb + lay.cs + t * RB); };
    // the ZOH input factor of token t's 4 states from dt and the decays
    auto zoh4 = [&](float dt, float2 a01, float2 a23, float2& z01, float2& z23) {
        const float2 x01 = __fmul2_rn(f2(dt, dt), s01), x23 = __fmul2_rn(f2(dt, dt), s23);
        z01 = f2(zoh_bbar(dt, x01.x * kLn2, a01.x, iA01.x), zoh_bbar(dt, x01.y * kLn2, a01.y, iA01.y));
        z23 = f2(zoh_bbar(dt, x23.x * kLn2, a23.x, iA23.x), zoh_bbar(dt, x23.y * kLn2, a23.y, iA23.y));
    };

    float4* agg = reinterpret_cast<float4*>(smem + lay.agg);       // W > 1: [parity][warp][A | H][lane]
    float4* entry = reinterpret_cast<float4*>(smem + lay.entry);   // W > 1

    float dt_acc = 0.0f;                     // state-only: sum of this lane's step sizes
    prefetch(0, 0);
    cp_async_commit();
    for (int k = 0; k < nck; ++k) {
        const int st = k & 1;
        const int t0 = k * T;                // chunk start
        const int tr = t0 + w * R;           // this warp's run start
        const bool full = tr + R <= p.L;
        __syncwarp();                        // every lane is done with the stage refilled below
        if (k + 1 < nck) prefetch(k + 1, st ^ 1);
        cp_async_commit();
        cp_async_wait_1();                   // this lane's copies of chunk k have landed
        __syncwarp();                        // ... and every lane's
        const unsigned char* sb = ws + st * lay.stage;

        // ---- prologue: lane (g, c) takes tokens g*RQ .. g*RQ + RQ - 1 of channel c
        // D u and SiLU(z) of the lane's prologue tokens: registers for one run
        // per chunk, shared memory for several (their walk keeps more live)
        constexpr int RQr = W == 1 ? RQ : 1;
        float Du[RQr], gz[RQr];
        float2* dzs = reinterpret_cast<float2*>(ws + lay.dz);
        {
            const unsigned char* xc = sb + lay.xs + c * S;
            const int tb = g * RQ;
            float xm3 = SI::ld(xc + QsplitSmem::pad(tb + 0, RQ) * XB);
            float xm2 = SI::ld(xc + QsplitSmem::pad(tb + 1, RQ) * XB);
            float xm1 = SI::ld(xc + QsplitSmem::pad(tb + 2, RQ) * XB);
#pragma unroll
            for (int i = 0; i < RQ; i += 2) {   // tokens t and t + 1 as one float32 pair
                const int t = tb + i;
                const float xt0 = SI::ld(xc + QsplitSmem::pad(t + 3, RQ) * XB);
                const float xt1 = SI::ld(xc + QsplitSmem::pad(t + 4, RQ) * XB);
                float xv0 = fmaf(w0, xm3, cb);
                xv0 = fmaf(w1, xm2, xv0);
                xv0 = fmaf(w2, xm1, xv0);
                xv0 = fmaf(w3, xt0, xv0);
                float xv1 = fmaf(w0, xm2, cb);
                xv1 = fmaf(w1, xm1, xv1);
                xv1 = fmaf(w2, xt0, xv1);
                xv1 = fmaf(w3, xt1, xv1);
                xm3 = xm1; xm2 = xt0; xm1 = xt1;
                const float2 u = silu2(make_float2(xv0, xv1));
                const int tp = t + g;            // padded row of token t (t / RQ == g)
                const float2 dt = dt_from_raw2(__fadd2_rn(make_float2(SI::ld(sb + lay.ds + tp * XB + c * S),
                                                                      SI::ld(sb + lay.ds + (tp + 1) * XB + c * S)),
                                                          make_float2(db, db)));
                // dt = 0 past the sequence end: decay 1, no input
                const bool live0 = full || tr + t < p.L, live1 = full || tr + t + 1 < p.L;
                const float2 fu = kZoh ? u : __fmul2_rn(dt, u);
                pf[t * kQsCh + c] = make_float2(live0 ? dt.x : 0.0f, live0 ? fu.x : 0.0f);
                pf[(t + 1) * kQsCh + c] = make_float2(live1 ? dt.y : 0.0f, live1 ? fu.y : 0.0f);
                if constexpr (kState) {            // the step sizes of the lane's tokens
                    dt_acc += (live0 ? dt.x : 0.0f);
                    dt_acc += (live1 ? dt.y : 0.0f);
                } else {
                    const float2 du = __fmul2_rn(make_float2(Dv, Dv), u);
                    const float2 gzv = silu2(make_float2(SI::ld(sb + lay.zs + tp * XB + c * S),
                                                         SI::ld(sb + lay.zs + (tp + 1) * XB + c * S)));
                    if constexpr (W == 1) { Du[i] = du.x; gz[i] = gzv.x; Du[i + 1] = du.y; gz[i + 1] = gzv.y; }
                    else {
                        dzs[t * kQsCh + c] = make_float2(du.x, gzv.x);
                        dzs[(t + 1) * kQsCh + c] = make_float2(du.y, gzv.y);
                    }
                }
            }
        }
        __syncwarp();

        float part[R];
        if constexpr (W == 1) {
            // ---- one pass from the carried state, in blocks of kBlk tokens:
            // the block's decays and inputs first, then its state updates
            constexpr int kBlk = 4;
#pragma unroll
            for (int tb = 0; tb < R; tb += kBlk) {
                float2 a01[kBlk], a23[kBlk], u01[kBlk], u23[kBlk];
#pragma unroll
                for (int i = 0; i < kBlk; ++i) {
                    const int t = tb + i;
                    const float2 v = pf[t * kQsCh + c];
                    const float4 Bq = bq(sb, t);
                    const float2 dd = f2(v.x, v.x), ff = f2(v.y, v.y);
                    const float2 arg01 = __fmul2_rn(dd, s01);
                    const float2 arg23 = __fmul2_rn(dd, s23);
                    a01[i] = f2(ex2_approx(arg01.x), ex2_approx(arg01.y));
                    a23[i] = f2(ex2_approx(arg23.x), ex2_approx(arg23.y));
                    u01[i] = __fmul2_rn(ff, f2(Bq.x, Bq.y));
                    u23[i] = __fmul2_rn(ff, f2(Bq.z, Bq.w));
                    if constexpr (kZoh) {
                        float2 z01, z23;
                        zoh4(v.x, a01[i], a23[i], z01, z23);
                        u01[i] = __fmul2_rn(u01[i], z01);
                        u23[i] = __fmul2_rn(u23[i], z23);
                    }
                }
#pragma unroll
                for (int i = 0; i < kBlk; ++i) {
                    const int t = tb + i;
                    h01 = __ffma2_rn(a01[i], h01, u01[i]);
                    h23 = __ffma2_rn(a23[i], h23, u23[i]);
                    if constexpr (!kState) {
                        const float4 Cq = cq(sb, t);
                        const float2 pq = __ffma2_rn(f2(Cq.z, Cq.w), h23, __fmul2_rn(f2(Cq.x, Cq.y), h01));
                        part[t] = pq.x + pq.y;
                    }
                }
            }
        } else {
            // ---- first pass: the run from a zero state.  With h_in the state
            // entering the run, P_t the product of its decays up to t and
            // H_t the state reached from zero, h_t = P_t h_in + H_t, so
            // C_t . h_t = C_t . H_t + (C_t P_t) . h_in: keep the local partial
            // C_t . H_t and Q_t = C_t P_t of every token, and (P, H) at the end.
            float2 q01[R], q23[R];
            float pl[R];
            float2 H01 = f2(0.f, 0.f), H23 = f2(0.f, 0.f);
            float2 P01 = f2(1.f, 1.f), P23 = f2(1.f, 1.f);
#pragma unroll
            for (int t = 0; t < R; ++t) {
                const float2 v = pf[t * kQsCh + c];
                const float4 Bq = bq(sb, t);
                const float2 dd = f2(v.x, v.x), ff = f2(v.y, v.y);
                const float2 arg01 = __fmul2_rn(dd, s01);
                const float2 arg23 = __fmul2_rn(dd, s23);
                const float2 a01 = f2(ex2_approx(arg01.x), ex2_approx(arg01.y));
                const float2 a23 = f2(ex2_approx(arg23.x), ex2_approx(arg23.y));
                float2 i01 = __fmul2_rn(ff, f2(Bq.x, Bq.y));
                float2 i23 = __fmul2_rn(ff, f2(Bq.z, Bq.w));
                if constexpr (kZoh) {
                    float2 z01, z23;
                    zoh4(v.x, a01, a23, z01, z23);
                    i01 = __fmul2_rn(i01, z01);
                    i23 = __fmul2_rn(i23, z23);
                }
                H01 = __ffma2_rn(a01, H01, i01);
                H23 = __ffma2_rn(a23, H23, i23);
                P01 = __fmul2_rn(P01, a01);
                P23 = __fmul2_rn(P23, a23);
                if constexpr (!kState) {
                    const float4 Cq = cq(sb, t);
                    const float2 c01 = f2(Cq.x, Cq.y), c23 = f2(Cq.z, Cq.w);
                    const float2 pq = __ffma2_rn(c23, H23, __fmul2_rn(c01, H01));
                    pl[t] = pq.x + pq.y;
                    q01[t] = __fmul2_rn(c01, P01);
                    q23[t] = __fmul2_rn(c23, P23);
                }
            }
            // the run's aggregate (prod a, H) for the other warps
            {
                float4* slot = agg + ((k & 1) * W + w) * 64 + lane;
                slot[0] = make_float4(P01.x, P01.y, P23.x, P23.y);
                slot[32] = make_float4(H01.x, H01.y, H23.x, H23.y);
            }
            __syncthreads();                 // every run's aggregate of chunk k is written
            // ---- the state entering this run: the chunk's entering state (the
            // last run's end state of chunk k-1) folded through runs 0 .. w-1
            if (k > 0) {
                const float4 he = entry[(k & 1) * 32 + lane];
                h01 = f2(he.x, he.y);
                h23 = f2(he.z, he.w);
            }
            for (int j = 0; j < w; ++j) {
                const float4* slot = agg + ((k & 1) * W + j) * 64 + lane;
                const float4 A = slot[0], H = slot[32];
                h01 = __ffma2_rn(f2(A.x, A.y), h01, f2(H.x, H.y));
                h23 = __ffma2_rn(f2(A.z, A.w), h23, f2(H.z, H.w));
            }
            // ---- second pass: every token's C . h from the entering state,
            // no chain; then the run's end state
            if constexpr (!kState) {
#pragma unroll
                for (int t = 0; t < R; ++t) {
                    const float2 pq = __ffma2_rn(q23[t], h23, __fmul2_rn(q01[t], h01));
                    part[t] = pl[t] + (pq.x + pq.y);
                }
            }
            h01 = __ffma2_rn(P01, h01, H01);
            h23 = __ffma2_rn(P23, h23, H23);
            if (w == W - 1) entry[((k + 1) & 1) * 32 + lane] = make_float4(h01.x, h01.y, h23.x, h23.y);
        }

        // ---- reduce-scatter of the quadrant partials over lanes 16 and 8
        // apart: quadrants {0, 1} keep the first half of the run's tokens and
        // {2, 3} the second, then each quadrant keeps its own R/4 tokens, so
        // lane (g, c) ends with the totals of tokens g*RQ .. g*RQ + RQ - 1
        if constexpr (!kState) {
            const bool hi = (g & 2) != 0, lo = (g & 1) != 0;
            float half[R / 2];
#pragma unroll
            for (int i = 0; i < R / 2; ++i) {
                const float keep = hi ? part[R / 2 + i] : part[i];
                const float send = hi ? part[i] : part[R / 2 + i];
                half[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
            }
            float tot[RQ];
#pragma unroll
            for (int j = 0; j < RQ; ++j) {
                const float keep = lo ? half[RQ + j] : half[j];
                const float send = lo ? half[j] : half[RQ + j];
                tot[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
            }
            unsigned char* yrow = ybase + (size_t)t0 * row_bytes;
#pragma unroll
            for (int j = 0; j < RQ; ++j) {
                if (!active || (!full && tr + g * RQ + j >= p.L)) continue;
                float du, gzv;
                if constexpr (W == 1) { du = Du[j]; gzv = gz[j]; }
                else { const float2 v = dzs[(g * RQ + j) * kQsCh + c]; du = v.x; gzv = v.y; }
                Io::store(reinterpret_cast<TT*>(yrow + j * row_bytes), (tot[j] + du) * gzv);
            }
        }
    }

    // ---- final caches: the last run holds the sequence's end state
    if (active && w == W - 1)
        reinterpret_cast<float4*>(p.ssm_state_out + ((size_t)b * p.E + e) * kN)[g] =
            make_float4(h01.x, h01.y, h23.x, h23.y);
    if (active && w == 0 && g == 0) {
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
    if constexpr (kState) {
        // the channel's sum of step sizes: its four quadrant lanes in every warp
        // hold the sums of disjoint tokens; added in a fixed order
        float v = dt_acc;
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        float* dts = reinterpret_cast<float*>(smem + lay.dts);
        if (g == 0) dts[w * kQsCh + c] = v;
        __syncthreads();
        if (active && w == 0 && g == 0) {
            float tot = 0.0f;
            for (int j = 0; j < W; ++j) tot += dts[j * kQsCh + c];
            p.dt_sum[(size_t)b * p.E + e] = tot;
        }
    }
}

}  // namespace axon
