// gemm_tc.cuh -- the layer's dense projections as a bf16 GEMM on the sm_100a
// tensor cores: C (M x N) = A (M x K) W (K x N), A and W row-major bf16,
// float32 accumulation, bf16 out (Axon-SSM page, "Gating": the input and
// output projections; "Selective mechanism": f_proj, one linear map of the
// conv output).
//
// Persistent, warp-specialised, one CTA per SM (192 threads), output tiles of
// 128 x BN, BN = 256 or 192 (whichever fills the SMs in less time; 128-column
// tiles measured slower):
//   warp 0 (one thread)  TMA producer: per 64-deep K block, the A tile
//                        (128 rows x 64, K-major) and the W tile (64 x BN,
//                        N-major, 64-column boxes), 128-byte swizzle, into a
//                        ring of shared-memory stages (4 for BN 256, 5 for 192);
//   warp 1 (one thread)  MMA issuer: four tcgen05.mma (M 128, N BN, K 16)
//                        per stage into one of 512 / BN float32 accumulators
//                        in tensor memory; each stage is handed back to the
//                        producer by a tcgen05.commit;
//   warps 2-5            epilogue: tensor memory -> registers (thread = row)
//                        -> bf16, stored straight to global memory, while the
//                        MMA issuer fills the other accumulator.
// Output tiles go round-robin over the CTAs, M fastest, so the
// CTAs running at once share W tiles in L2.  The output columns may be split
// over up to three row-major destinations (columns [c_k, c_{k+1}) go to
// destination k at column - c_k), so one GEMM writes x and z, or dt_raw, B
// and C, into separate arrays.  Every mbarrier wait gives up after a bounded
// number of polls; the block then stops, waits (bounded) for its copies and
// products in flight, records an error in *err and frees its tensor memory.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "tc_ops.cuh"

namespace axon {

constexpr int kGmBM = 128;          // rows of an output tile (the MMA's M)
constexpr int kGmBK = 64;           // K per stage: one 128-byte swizzle row of bf16
constexpr int kGmThreads = 192;
constexpr int kGmABytes = kGmBM * kGmBK * 2;          // 16 KB

// Shared-memory plan for output tiles of BN columns (the MMA's N): as many
// stages of (A 16 KB + W BN x 128 bytes) as fit, then the mbarriers.
template <int BN>
struct GemmCfg {
    static constexpr int kBBytes = kGmBK * BN * 2;
    static constexpr int kStageBytes = kGmABytes + kBBytes;
    static constexpr int kStages = BN == 256 ? 4 : (BN == 192 ? 5 : 6);
    static constexpr int kAccs = 512 / BN;            // tensor-memory accumulators (of 512 columns)
    static constexpr int kAccStride = BN > 128 ? 256 : 128;   // their first columns: 0, 256 (or 128 apart)
    static constexpr int kBarOff = kStages * kStageBytes;
    static constexpr int kSmem = kBarOff + 256 + 1024;  // + barriers, slot, flags + alignment pad
};

struct GemmOut {
    __nv_bfloat16* ptr;   // row-major destination
    int ld;               // its row stride (elements)
    int col0;             // first GEMM column it receives
};

struct GemmParams {
    int M, N, K;
    int tiles_m, tiles_n;
    int nout;             // destinations (1..3), sorted by col0, out[0].col0 == 0
    GemmOut out[3];
    int* err;             // set to 1 when a wait gave up (may be null)
    // CTA-pair kernel, stream-K split (null: whole tiles round-robin):
    float* sk_partial;    // [pair][CTA][16 column chunks][4 quads][128 rows] float4 partial sums
    int* sk_flag;         // [pair][CTA][4 epilogue warps], zero at launch; 1 once published
    int sk_dp_tiles;      // the first tiles (a multiple of the pairs) go whole, round-robin
};

// Output row m, columns col .. col + 7: one 16-byte piece of bf16 into the
// destination that owns those columns (col < N).
__device__ __forceinline__ void gemm_store8(const GemmParams& p, int m, int col, uint4 pk) {
    const int k = (p.nout > 2 && col >= p.out[2].col0) ? 2 : ((p.nout > 1 && col >= p.out[1].col0) ? 1 : 0);
    const GemmOut o = k == 2 ? p.out[2] : (k == 1 ? p.out[1] : p.out[0]);
    *reinterpret_cast<uint4*>(o.ptr + (size_t)m * o.ld + (col - o.col0)) = pk;
}

// Output row m, columns n .. n + 15 (bf16), as two 8-column (16-byte)
// pieces, each into the destination that owns its columns; columns past N
// are dropped.
__device__ __forceinline__ void gemm_store16(const GemmParams& p, int m, int n, const float (&v)[16]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int col = n + 8 * h;
        if (col < p.N) {
            const int k = (p.nout > 2 && col >= p.out[2].col0) ? 2 : ((p.nout > 1 && col >= p.out[1].col0) ? 1 : 0);
            const GemmOut o = k == 2 ? p.out[2] : (k == 1 ? p.out[1] : p.out[0]);
            uint4 pk;
            pk.x = pack_bf16(v[8 * h + 0], v[8 * h + 1]);
            pk.y = pack_bf16(v[8 * h + 2], v[8 * h + 3]);
            pk.z = pack_bf16(v[8 * h + 4], v[8 * h + 5]);
            pk.w = pack_bf16(v[8 * h + 6], v[8 * h + 7]);
            *reinterpret_cast<uint4*>(o.ptr + (size_t)m * o.ld + (col - o.col0)) = pk;
        }
    }
}

template <int kGmBN>
__global__ void __launch_bounds__(kGmThreads, 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW,
                        GemmParams p) {
    using Cfg = GemmCfg<kGmBN>;
    constexpr int kGmStages = Cfg::kStages, kGmStageBytes = Cfg::kStageBytes, kGmBarOff = Cfg::kBarOff;
    constexpr int kAccs = Cfg::kAccs;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const uint32_t raw = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;   // swizzled tiles want 1024-byte alignment
    unsigned char* sm = smem_raw + pad;
    const uint32_t sb = raw + pad;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar = sb + kGmBarOff;
    auto full = [&](int s) { return bar + 8u * s; };                       // stage loaded
    auto empty = [&](int s) { return bar + 8u * (kGmStages + s); };        // stage consumed
    auto tfull = [&](int a) { return bar + 8u * (2 * kGmStages + a); };    // accumulator ready
    auto tempty = [&](int a) { return bar + 8u * (2 * kGmStages + kAccs + a); };  // accumulator drained
    const uint32_t drain = bar + 8u * (2 * kGmStages + 2 * kAccs);
    const uint32_t slot = bar + 8u * (2 * kGmStages + 2 * kAccs + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kGmBarOff + 8 * (2 * kGmStages + 2 * kAccs + 2));
    volatile int* drained = abort_flag + 1;     // set once every issued product has finished

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGmStages; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        for (int a = 0; a < kAccs; ++a) {
            mbar_init(tfull(a), 1);
            mbar_init(tempty(a), 4);             // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        *drained = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    grid_dep_launch();
    grid_dep_wait();                             // the operands' producers have finished
    const uint32_t tbase = *reinterpret_cast<volatile uint32_t*>(sm + kGmBarOff + 8 * (2 * kGmStages + 2 * kAccs + 1));

    const int ntiles = p.tiles_m * p.tiles_n;
    const int kblocks = (p.K + kGmBK - 1) / kGmBK;
    auto fail = [&]() {
        *abort_flag = 1;
        if (p.err) atomicExch(p.err, 1);
    };

    if (warp == 0) {
        // ---- TMA producer
        int issued = 0;                          // stages filled so far
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
                const int m0 = (tile % p.tiles_m) * kGmBM, n0 = (tile / p.tiles_m) * kGmBN;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(empty(s), ph ^ 1u)) { fail(); break; }
                    if (*abort_flag) break;
                    const uint32_t a_dst = sb + s * kGmStageBytes, b_dst = a_dst + kGmABytes;
                    mbar_arrive_expect_tx(full(s), kGmStageBytes);
                    tma_load_2d(a_dst, &tmA, kb * kGmBK, m0, full(s));
#pragma unroll
                    for (int j = 0; j < kGmBN / 64; ++j)
                        tma_load_2d(b_dst + j * (kGmBK * 128), &tmW, n0 + 64 * j, kb * kGmBK, full(s));
                    ++issued;
                    if (++s == kGmStages) { s = 0; ph ^= 1u; }
                }
            }
            // every copy issued has landed before the block may exit: the last
            // (up to kGmStages) stages' loads completed their phases
            int s2 = s;
            uint32_t ph2 = ph;
            for (int i = 0; i < kGmStages && i < issued; ++i) {
                if (--s2 < 0) { s2 = kGmStages - 1; ph2 ^= 1u; }
                if (!mbar_wait(full(s2), ph2)) fail();
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc(kGmBM, kGmBN, 0, 1);   // A K-major, W N-major
            int s = 0, a = 0;
            uint32_t ph = 0, aph = 0;
            for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
                if (!mbar_wait(tempty(a), aph ^ 1u)) { fail(); break; }
                tc_fence_after();
                const uint32_t d = tbase + (uint32_t)(a * Cfg::kAccStride);
                bool ok = true;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(full(s), ph) || *abort_flag) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_s = sb + s * kGmStageBytes, b_s = a_s + kGmABytes;
#pragma unroll
                    for (int ks = 0; ks < kGmBK / 16; ++ks)
                        umma(d, umma_desc(a_s + ks * 32, 16, 1024), umma_desc(b_s + ks * 16 * 128, kGmBK * 128, 1024),
                             idesc, (kb | ks) != 0);
                    umma_commit(empty(s));           // the stage returns to the producer once read
                    if (++s == kGmStages) { s = 0; ph ^= 1u; }
                }
                if (!ok) { fail(); break; }
                umma_commit(tfull(a));               // the accumulator is complete
                if (++a == kAccs) { a = 0; aph ^= 1u; }
            }
            // every product issued has finished before the tensor memory is freed
            umma_commit(drain);
            if (mbar_wait(drain, 0u)) *drained = 1;
            else fail();
        }
    } else {
        // ---- epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31
        const int q = warp & 3;
        const int row = 32 * q + lane;
        int a = 0;
        uint32_t aph = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            // the warp decides together: the tensor-memory loads below are warp-wide
            const bool ready = mbar_wait(tfull(a), aph) && !*abort_flag;
            if (!__all_sync(0xffffffffu, ready)) { fail(); break; }
            tc_fence_after();
            const int m = (tile % p.tiles_m) * kGmBM + row;
            const int n0 = (tile / p.tiles_m) * kGmBN;
            const uint32_t tl = tbase + (uint32_t)(a * Cfg::kAccStride) + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
            for (int c0 = 0; c0 < kGmBN; c0 += 16) {
                float v[16];
                tmem_ld16(tl + c0, v);               // warp-wide: rows past M take part too
                if (m < p.M) gemm_store16(p, m, n0 + c0, v);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty(a));   // the MMA issuer may refill this accumulator
            if (++a == kAccs) { a = 0; aph ^= 1u; }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // free the tensor memory unless a product may still be writing it
    if (warp == 1 && *drained) tmem_dealloc(tbase, 512);
}

}  // namespace axon
