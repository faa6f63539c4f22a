// gemm_pair.cuh -- the layer's projection GEMM on CTA pairs: the same product
// as gemm_tc.cuh (C = A W, bf16 in and out, float32 accumulation; Axon-SSM
// page, "Gating" and "Selective mechanism"), with each output tile of 256 x 256
// computed by a cluster of two CTAs on two SMs through tcgen05.mma.cta_group::2
// (M 256, N 256, K 16).
//
// Why pairs: a single CTA's 128 x 256 product reads its whole W stage (64 x
// 256) from its own shared memory for only 128 rows of A, and every stage is
// also written there by the TMA: per 64-deep K block 48 KB in and 48 KB out
// of one SM's shared memory, more than it moves in the block's product time.
// In a pair each CTA stages its 128 rows of A and HALF of the W columns (the
// tensor cores read the other half from the peer), so per SM and K block the
// traffic is 32 KB in and 32 KB out for the same product rate.
//
// Roles in each CTA (192 threads, one CTA per SM):
//   warp 0 (one thread)  TMA producer: per K block, this CTA's A tile (128 rows
//                        x 64) and its W half (64 x 128, two 64-column boxes)
//                        into a ring of 6 stages; the copies complete on the
//                        stage's "full" barrier of CTA 0 (each producer first
//                        arrives there expecting its own 32 KB);
//   warp 1               allocates the pair's tensor memory (both CTAs); in
//                        CTA 0, one thread issues the products and commits
//                        each stage back to both CTAs' "empty" barriers and
//                        each finished accumulator to both "ready" barriers;
//   warps 2-5            epilogue: this CTA's 128 accumulator rows (tensor
//                        memory -> registers, 64 columns a round -> bf16 ->
//                        a swizzled per-warp shared buffer -> global, 128
//                        contiguous bytes of four rows per store
//                        instruction), then one arrival per warp on CTA 0's
//                        "drained" barrier (8 in all), so the issuer may
//                        refill that accumulator.
// Work: whole tiles round-robin over the pairs, M fastest (pairs running at
// once share W tiles in L2).  With a stream-K scratch, only the tiles of all
// full waves but the last go whole; the (tile, K block) iterations of the
// rest are cut into equal contiguous ranges, one per pair, so the last wave
// ends with every pair busy.  A tile split between pairs is finished by the
// pair holding its first K blocks (the end of that pair's range, so the
// others' parts -- the starts of their ranges -- are ready by then): the
// others store float32 partial sums (chunk-major, coalesced) and raise a
// flag per epilogue warp; the owner waits for the flags, copies a single
// partial into its now idle stage ring with one bulk copy (several: read from
// global memory), adds the partials in pair order and stores bf16, so results
// do not depend on timing.
// Every mbarrier and flag wait gives up after a bounded number of polls;
// both CTAs always reach the final cluster barrier, and the tensor memory is
// freed only once CTA 0 has seen every product finish.  No load is multicast.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "gemm_tc.cuh"
#include "tc_ops.cuh"

namespace axon {

constexpr int kGpTileM = 2 * kGmBM;     // output rows of a pair's tile
constexpr int kGpTileN = 256;           // output columns of a pair's tile (the MMA's N)
constexpr int kGpHalfN = kGpTileN / 2;  // W columns staged by each CTA

struct GemmPairCfg {
    static constexpr int kBBytes = kGmBK * kGpHalfN * 2;             // 16 KB
    static constexpr int kStageBytes = kGmABytes + kBBytes;           // 32 KB per CTA
    static constexpr int kStages = 6;
    static constexpr int kAccs = 2;                                    // 256-column accumulators
    static constexpr int kBarOff = kStages * kStageBytes;
    static constexpr int kEpiOff = kBarOff + 256;                      // after the barriers, slot, flags
    static constexpr int kEpiBytes = 4 * 32 * 128;                     // per epilogue warp: 32 rows x 64 bf16
    static constexpr int kSmem = kEpiOff + kEpiBytes + 1024;           // + alignment pad
};

__global__ void __launch_bounds__(kGmThreads, 1)
    gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                          GemmParams p) {
    using Cfg = GemmPairCfg;
    constexpr int kStages = Cfg::kStages, kStageBytes = Cfg::kStageBytes, kAccs = Cfg::kAccs;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    // the same offsets in both CTAs: the products address the peer's tiles
    // through this CTA's descriptors
    const uint32_t raw = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    unsigned char* sm = smem_raw + pad;
    const uint32_t sb = raw + pad;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();            // 0 issues the products
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const uint32_t bar = sb + Cfg::kBarOff;
    auto full = [&](int s) { return bar + 8u * s; };                       // CTA 0: both halves of a stage loaded
    auto empty = [&](int s) { return bar + 8u * (kStages + s); };          // stage consumed (both CTAs)
    auto tfull = [&](int a) { return bar + 8u * (2 * kStages + a); };      // accumulator ready (both CTAs)
    auto tempty = [&](int a) { return bar + 8u * (2 * kStages + kAccs + a); };  // CTA 0: drained by 8 warps
    const uint32_t drain = bar + 8u * (2 * kStages + 2 * kAccs);
    const uint32_t slot = bar + 8u * (2 * kStages + 2 * kAccs + 1);
    const uint32_t flags = bar + 8u * (2 * kStages + 2 * kAccs + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Cfg::kBarOff + 8 * (2 * kStages + 2 * kAccs + 2));
    volatile int* drained = abort_flag + 1;     // CTA 0 sets it in both CTAs once every product has finished

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full(s), 2);               // one expect-arrival per CTA
            mbar_init(empty(s), 1);
        }
        for (int a = 0; a < kAccs; ++a) {
            mbar_init(tfull(a), 1);
            mbar_init(tempty(a), 8);             // four epilogue warps per CTA
        }
        mbar_init(drain, 1);
        mbar_init(bar + 8u * (2 * kStages + 2 * kAccs + 3), 1);   // a stream-K partial copied in
        *abort_flag = 0;
        *drained = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc_pair(slot, 512);
    tc_fence_before();
    cluster_sync_all();                          // both CTAs' barriers and tensor memory exist
    tc_fence_after();
    grid_dep_launch();
    grid_dep_wait();                             // the operands' producers have finished
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(sm + Cfg::kBarOff + 8 * (2 * kStages + 2 * kAccs + 1));

    const int kblocks = (p.K + kGmBK - 1) / kGmBK;
    auto fail = [&]() {
        *abort_flag = 1;
        if (p.err) atomicExch(p.err, 1);
    };
    // The pair's work as segments (tile, K blocks kb0 .. kb1 - 1), the same
    // sequence for the producer, the issuer and the epilogue; f returns false
    // to stop.  Whole tiles round-robin (neighbouring pairs share W tiles in
    // L2); with sk_partial only the first sk_dp_tiles tiles, and the
    // iterations (tile, K block) of the rest are split evenly, tile-major:
    // pair i takes [T i / P, T (i+1) / P) of their T, so at most its first
    // segment of them starts inside a tile and at most its last one ends
    // inside one (stream-K).
    const int ntiles = p.tiles_m * p.tiles_n;
    const int dp_tiles = p.sk_partial ? p.sk_dp_tiles : ntiles;
    const long long iters = (long long)(ntiles - dp_tiles) * kblocks;
    auto range_begin = [&](int i) { return iters * i / npairs; };
    auto for_segments = [&](auto&& f) {
        for (int tile = pair; tile < dp_tiles; tile += npairs)
            if (!f(tile, 0, kblocks)) return;
        long long it = range_begin(pair);
        const long long e = range_begin(pair + 1);
        while (it < e) {
            const int t = (int)(it / kblocks), kb0 = (int)(it % kblocks);
            const int kb1 = (int)min((long long)kblocks, kb0 + (e - it));
            if (!f(dp_tiles + t, kb0, kb1)) return;
            it += kb1 - kb0;
        }
    };

    if (warp == 0) {
        // ---- TMA producer (both CTAs)
        if (lane == 0) {
            int s = 0, issued = 0;
            uint32_t ph = 0;
            for_segments([&](int tile, int kb0, int kb1) {
                const int m0 = (tile % p.tiles_m) * kGpTileM + kGmBM * (int)rank;
                const int n0 = (tile / p.tiles_m) * kGpTileN + kGpHalfN * (int)rank;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(empty(s), ph ^ 1u)) { fail(); return false; }
                    if (*abort_flag) return false;
                    const uint32_t a_dst = sb + s * kStageBytes, b_dst = a_dst + kGmABytes;
                    const uint32_t fb = cluster_map(full(s), 0);
                    mbar_arrive_expect_tx_remote(fb, kStageBytes);
                    tma_load_2d_pair(a_dst, &tmA, kb * kGmBK, m0, fb);
#pragma unroll
                    for (int j = 0; j < kGpHalfN / 64; ++j)
                        tma_load_2d_pair(b_dst + j * (kGmBK * 128), &tmW, n0 + 64 * j, kb * kGmBK, fb);
                    ++issued;
                    if (++s == kStages) { s = 0; ph ^= 1u; }
                }
                return !*abort_flag;
            });
            // CTA 0: every copy of both CTAs has landed before either may exit
            // (the last stages' phases completed; the final cluster barrier
            // holds CTA 1 until then)
            if (rank == 0) {
                int s2 = s;
                uint32_t ph2 = ph;
                for (int i = 0; i < kStages && i < issued; ++i) {
                    if (--s2 < 0) { s2 = kStages - 1; ph2 ^= 1u; }
                    if (!mbar_wait(full(s2), ph2)) fail();
                }
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer (CTA 0)
        if (lane == 0 && rank == 0) {
            constexpr uint32_t idesc = umma_idesc(kGpTileM, kGpTileN, 0, 1);   // A K-major, W N-major
            int s = 0, a = 0;
            uint32_t ph = 0, aph = 0;
            for_segments([&](int, int kb0, int kb1) {
                if (*abort_flag || !mbar_wait(tempty(a), aph ^ 1u)) { fail(); return false; }
                tc_fence_after();
                const uint32_t d = tbase + (uint32_t)(a * kGpTileN);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(full(s), ph) || *abort_flag) { fail(); return false; }
                    tc_fence_after();
                    const uint32_t a_s = sb + s * kStageBytes, b_s = a_s + kGmABytes;
#pragma unroll
                    for (int ks = 0; ks < kGmBK / 16; ++ks)
                        umma_pair(d, umma_desc(a_s + ks * 32, 16, 1024), umma_desc(b_s + ks * 16 * 128, kGmBK * 128, 1024),
                                  idesc, (kb != kb0) | (ks != 0));
                    umma_pair_commit_both(empty(s));     // both CTAs may refill the stage
                    if (++s == kStages) { s = 0; ph ^= 1u; }
                }
                umma_pair_commit_both(tfull(a));         // both halves of the accumulator are complete
                if (++a == kAccs) { a = 0; aph ^= 1u; }
                return true;
            });
            // every product issued has finished before the tensor memory is freed
            umma_pair_commit(drain);
            if (mbar_wait(drain, 0u)) {
                *drained = 1;
                st_cluster_u32(cluster_map(flags + 4u, 1), 1u);
            } else {
                fail();
            }
        }
    } else {
        // ---- epilogue (both CTAs): warp w reads tensor-memory lanes 32 (w % 4) .. + 31
        const int q = warp & 3;
        const int row = 32 * q + lane;
        constexpr int kSlot = kGmBM * kGpTileN;  // floats of one CTA's partial
        int a = 0;
        uint32_t aph = 0;
        for_segments([&](int tile, int kb0, int kb1) {
            // the warp decides together: the tensor-memory loads below are warp-wide
            const bool ready = mbar_wait(tfull(a), aph) && !*abort_flag;
            if (!__all_sync(0xffffffffu, ready)) { fail(); return false; }
            tc_fence_after();
            const int n0 = (tile / p.tiles_m) * kGpTileN;
            const uint32_t tl = tbase + (uint32_t)(a * kGpTileN) + ((uint32_t)(32 * q) << 16);
            // 64 accumulator columns per round: two 32-column loads in flight
            // (warp-wide: rows past M take part too)
            auto load64 = [&](int c0, float (&v)[64]) {
                uint32_t r0[32], r1[32];
                tmem_ld32_async(tl + c0, r0);
                tmem_ld32_async(tl + c0 + 32, r1);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    v[j] = __uint_as_float(r0[j]);
                    v[32 + j] = __uint_as_float(r1[j]);
                }
            };
            // 64 columns of the warp's 32 rows as bf16, through the warp's
            // shared-memory buffer (16-byte chunks XOR-swizzled by row: both
            // the row-wise writes and the reads below are conflict-free), so
            // that each store instruction writes 128 contiguous bytes of four
            // rows instead of 16 bytes of 32
            unsigned char* ebuf = sm + Cfg::kEpiOff + q * (32 * 128);
            const int mrow0 = (tile % p.tiles_m) * kGpTileM + kGmBM * (int)rank + 32 * q;
            auto store64 = [&](int c0, const float (&v)[64]) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 pk;
                    pk.x = pack_bf16(v[8 * j + 0], v[8 * j + 1]);
                    pk.y = pack_bf16(v[8 * j + 2], v[8 * j + 3]);
                    pk.z = pack_bf16(v[8 * j + 4], v[8 * j + 5]);
                    pk.w = pack_bf16(v[8 * j + 6], v[8 * j + 7]);
                    *reinterpret_cast<uint4*>(ebuf + lane * 128 + ((j ^ (lane & 7)) * 16)) = pk;
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int r = (lane >> 3) + 4 * i, ch = lane & 7;
                    const uint4 pk = *reinterpret_cast<const uint4*>(ebuf + r * 128 + ((ch ^ (r & 7)) * 16));
                    const int mm = mrow0 + r, col = n0 + c0 + 8 * ch;
                    if (mm < p.M && col < p.N) gemm_store8(p, mm, col, pk);
                }
                __syncwarp();
            };
            if (kb0 > 0) {
                // a later part of the tile: publish the float32 partial for the
                // pair that holds the tile's first K blocks, chunk-major
                // ([16-column chunk][quad][row] float4: one warp's stores are
                // 512 contiguous bytes)
                float4* dst = reinterpret_cast<float4*>(p.sk_partial + ((size_t)pair * 2 + rank) * kSlot) + row;
#pragma unroll 1
                for (int c0 = 0; c0 < kGpTileN; c0 += 64) {
                    float v[64];
                    load64(c0, v);
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        dst[(c0 / 4 + k) * kGmBM] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
                }
                __threadfence();
                __syncwarp();
                if (lane == 0) st_release_gpu(p.sk_flag + ((size_t)pair * 2 + rank) * 4 + q, 1);
            } else {
                // the tile's first K blocks: add the partials of the pairs that
                // took the rest (their first segments of the split tiles,
                // published early), in pair order, then store
                int nparts = 0;
                if (kb1 < kblocks) {
                    const long long tile_end = (long long)(tile - dp_tiles + 1) * kblocks;
                    while (pair + 1 + nparts < npairs && range_begin(pair + 1 + nparts) < tile_end) ++nparts;
                    // every contributor's four warps have published (each
                    // warp checks all four: one partial may be copied whole)
                    bool ok = true;
                    for (int idx = lane; idx < 4 * nparts && ok; idx += 32) {
                        const int* f = p.sk_flag + ((size_t)(pair + 1 + idx / 4) * 2 + rank) * 4 + (idx & 3);
                        int it = 0;
                        while (ld_acquire_gpu(f) == 0 && ++it < kTcWaitLimit) __nanosleep(64);
                        ok = it < kTcWaitLimit;
                    }
                    if (!__all_sync(0xffffffffu, ok)) { fail(); return false; }
                }
                // one partial: copied whole into the stage ring (free once
                // this last segment's products are done) by one thread, then
                // read from shared memory; several: read from global memory
                const float4* part = nullptr;
                if (nparts == 1) {
                    const uint32_t pbar = bar + 8u * (2 * kStages + 2 * kAccs + 3);
                    constexpr uint32_t kPartBytes = kSlot * 4, kPiece = kPartBytes / 4;   // 128 KB in 4 copies
                    static_assert(kPartBytes <= kStages * kStageBytes, "a partial fits the stage ring");
                    if (q == 0 && lane == 0) {
                        fence_proxy_async();
                        mbar_arrive_expect_tx(pbar, kPartBytes);
                        const unsigned char* src = reinterpret_cast<const unsigned char*>(
                            p.sk_partial + ((size_t)(pair + 1) * 2 + rank) * kSlot);
                        for (uint32_t c = 0; c < 4; ++c) bulk_load(sb + c * kPiece, src + c * kPiece, kPiece, pbar);
                    }
                    const bool got = mbar_wait(pbar, 0u);
                    if (!__all_sync(0xffffffffu, got)) { fail(); return false; }
                    part = reinterpret_cast<const float4*>(sm) + row;
                }
#pragma unroll 1
                for (int c0 = 0; c0 < kGpTileN; c0 += 64) {
                    float v[64];
                    load64(c0, v);
                    if (nparts == 1) {
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const float4 w = part[(c0 / 4 + k) * kGmBM];
                            v[4 * k] += w.x; v[4 * k + 1] += w.y; v[4 * k + 2] += w.z; v[4 * k + 3] += w.w;
                        }
                    } else {
                        for (int j = 1; j <= nparts; ++j) {
                            const float4* src = reinterpret_cast<const float4*>(
                                p.sk_partial + ((size_t)(pair + j) * 2 + rank) * kSlot) + row;
#pragma unroll
                            for (int k = 0; k < 16; ++k) {
                                const float4 w = __ldcg(src + (c0 / 4 + k) * kGmBM);
                                v[4 * k] += w.x; v[4 * k + 1] += w.y; v[4 * k + 2] += w.z; v[4 * k + 3] += w.w;
                            }
                        }
                    }
                    store64(c0, v);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(cluster_map(tempty(a), 0));   // CTA 0 may refill it
            if (++a == kAccs) { a = 0; aph ^= 1u; }
            return true;
        });
    }

    tc_fence_before();
    __syncwarp();
    cluster_sync_all();                          // both CTAs done; CTA 0's drain flag is visible in both
    tc_fence_after();
    // free the pair's tensor memory (both CTAs together) unless a product may
    // still be writing it
    if (warp == 1 && *drained) {
        __syncwarp();
        tmem_dealloc_pair(tbase, 512);
    }
}

}  // namespace axon
