// axon_block.cu -- the whole Axon-SSM layer around the scan (C ABI in
// include/axon_ssm.h): input projection, conv stage, projection to the SSM
// parameters, the fused scan, output projection.
//
// Axon-SSM page, "Gating": (x, z) = split(W_in X) and y_out = W_out (y_ssm *
// SiLU(z)); "Selective mechanism": (dt, B, C) = f_proj(conv output), read as
// one linear map E -> E + 2N.  The three projections are this library's
// tcgen05 GEMMs (gemm_pair.cuh on CTA pairs from 256 rows, with the stream-K
// tail where whole tiles would leave the last wave a tenth idle; gemm_tc.cuh
// below): one launch writes x and z, one writes dt_raw, B and C, one the
// output; the conv stage and the scan are this library's kernels too.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "axon_ssm.h"
#include "conv_silu.cuh"
#include "device_math.cuh"
#include "gemm_pair.cuh"
#include "gemm_tc.cuh"

namespace axon {
namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxBlockDevices = 64;

size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

// Stream-K scratch of the CTA-pair GEMM: one float32 partial tile (two CTAs x
// 128 x 256) and four flags per CTA for each of at most kGpMaxPairs pairs.
constexpr int kGpMaxPairs = 128;
constexpr size_t kSkPartialBytes = (size_t)kGpMaxPairs * 2 * kGmBM * kGpTileN * 4;
constexpr size_t kSkFlagBytes = (size_t)kGpMaxPairs * 2 * 4 * sizeof(int);
struct GemmScratch {
    float* partial;       // kSkPartialBytes
    int* flag;            // kSkFlagBytes, zero when the GEMM is enqueued
};

// Byte offsets of the intermediates inside the caller's workspace; the first
// 256 bytes hold the GEMMs' error flag, then the three GEMMs' stream-K flags
// (all cleared by one memset per call) and the stream-K partials they share.
struct BlockPlan {
    size_t flag, sk_flag, sk_partial, x, z, u, dt, bm, cm, y, scan_ws, scan_ws_bytes, total;
};

bool plan_block(int B, int L, int E, int N, int K, BlockPlan* p) {
    const size_t M = (size_t)B * L;
    const size_t act = round_up(M * E * 2), bc = round_up(M * N * 2);
    size_t off = 0;
    p->flag = off; off += kAlign;
    p->sk_flag = off; off += round_up(3 * kSkFlagBytes);
    p->sk_partial = off; off += round_up(kSkPartialBytes);
    p->x = off; off += act;
    p->z = off; off += act;
    p->u = off; off += act;
    p->dt = off; off += act;
    p->bm = off; off += bc;
    p->cm = off; off += bc;
    p->y = off; off += act;
    p->scan_ws_bytes = axon_ssm_scan_workspace_bytes(B, L, E, N, K, AXON_BF16);
    p->scan_ws = off; off += round_up(p->scan_ws_bytes);
    p->total = off;
    return true;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// A 2-D bf16 tensor map over a row-major (rows x cols, row stride ld
// elements) array, boxes of box_cols x box_rows, 128-byte swizzle,
// out-of-bounds elements read as zero.
bool tensor_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_cols,
                uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {ld * 2};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

std::atomic<int> g_gemm_sms[kMaxBlockDevices];
std::atomic<unsigned long long> g_gemm_smem_set[2];   // per tile width: 256, 192

template <int BN>
axon_status launch_gemm(int M, int N, int K, const CUtensorMap& ta, const void* W, int ldw, GemmParams p, int sms,
                        cudaStream_t st) {
    using Cfg = GemmCfg<BN>;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxBlockDevices) return AXON_ERR_CUDA;
    const unsigned long long bit = 1ull << dev;
    std::atomic<unsigned long long>& set = g_gemm_smem_set[BN == 256 ? 0 : 1];
    static_assert(BN == 256 || BN == 192, "tile widths of the layer's GEMM");
    if (!(set.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(gemm_bf16_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem) !=
            cudaSuccess)
            return AXON_ERR_CUDA;
        set.fetch_or(bit, std::memory_order_acq_rel);
    }
    CUtensorMap tw;
    if (!tensor_map(&tw, W, (uint64_t)K, (uint64_t)N, (uint64_t)ldw, 64, kGmBK)) return AXON_ERR_CUDA;
    p.tiles_m = (M + kGmBM - 1) / kGmBM;
    p.tiles_n = (N + BN - 1) / BN;
    const long long tiles = (long long)p.tiles_m * p.tiles_n;
    const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kGmThreads, 1, 1);
    cfg.dynamicSmemBytes = Cfg::kSmem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, gemm_bf16_tc_kernel<BN>, ta, tw, p) != cudaSuccess) return AXON_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

std::atomic<int> g_gemm_pairs[kMaxBlockDevices];   // pairs resident at once; 0 unknown, -1 none
std::atomic<unsigned long long> g_pair_smem_set;

cudaLaunchConfig_t pair_config(unsigned pairs, cudaStream_t st, cudaLaunchAttribute* attr) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    cfg.blockDim = dim3(kGmThreads, 1, 1);
    cfg.dynamicSmemBytes = GemmPairCfg::kSmem;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cfg;
}

// CTA pairs of the pair GEMM that fit on the device at once (its clusters
// take one SM each side), or -1 when none does.
int gemm_pair_slots(int dev) {
    int n = g_gemm_pairs[dev].load(std::memory_order_relaxed);
    if (n != 0) return n;
    const unsigned long long bit = 1ull << dev;
    if (!(g_pair_smem_set.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(gemm_bf16_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 GemmPairCfg::kSmem) != cudaSuccess) {
            cudaGetLastError();
            g_gemm_pairs[dev].store(-1, std::memory_order_relaxed);
            return -1;
        }
        g_pair_smem_set.fetch_or(bit, std::memory_order_acq_rel);
    }
    cudaLaunchAttribute attr[2];
    const cudaLaunchConfig_t cfg = pair_config(1, nullptr, attr);
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, gemm_bf16_pair_kernel, &cfg) != cudaSuccess || clusters <= 0) {
        cudaGetLastError();
        clusters = -1;
    }
    g_gemm_pairs[dev].store(clusters, std::memory_order_relaxed);
    return clusters;
}

// With `sk` (flags zero) the tiles of all full waves but the last go whole,
// round-robin, and the iterations of the rest are split evenly (stream-K):
// the tiles' last wave then ends with all pairs; below one wave the split
// takes min(resident pairs, iterations / 8) pairs.  Without `sk` whole tiles
// round-robin.
axon_status launch_gemm_pair(int M, int N, int K, const CUtensorMap& ta, const void* W, int ldw, GemmParams p,
                             int pairs, const GemmScratch* sk, cudaStream_t st) {
    CUtensorMap tw;
    if (!tensor_map(&tw, W, (uint64_t)K, (uint64_t)N, (uint64_t)ldw, 64, kGmBK)) return AXON_ERR_CUDA;
    p.tiles_m = (M + kGpTileM - 1) / kGpTileM;
    p.tiles_n = (N + kGpTileN - 1) / kGpTileN;
    const long long tiles = (long long)p.tiles_m * p.tiles_n;
    long long np = tiles < pairs ? tiles : pairs;
    if (sk) {
        np = pairs < kGpMaxPairs ? pairs : kGpMaxPairs;
        long long dp;
        if (tiles < np) {
            const long long iters = tiles * ((K + kGmBK - 1) / kGmBK);
            np = iters / 8 < np ? (iters / 8 > 0 ? iters / 8 : 1) : np;
            dp = 0;
        } else {
            dp = tiles % np == 0 ? tiles : (tiles / np - 1) * np;
        }
        p.sk_partial = sk->partial;
        p.sk_flag = sk->flag;
        p.sk_dp_tiles = (int)dp;
    }
    cudaLaunchAttribute attr[2];
    const cudaLaunchConfig_t cfg = pair_config((unsigned)np, st, attr);
    if (cudaLaunchKernelEx(&cfg, gemm_bf16_pair_kernel, ta, tw, p) != cudaSuccess) return AXON_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

// Launches after the layer's first kernel carry the programmatic-serialization
// attribute: each kernel signals griddepcontrol.launch_dependents early and
// waits (griddepcontrol.wait) for its predecessor before touching global
// memory, so a kernel's launch and its local set-up (barriers, tensor memory)
// overlap the previous kernel's tail.

// Row-major outputs (M x N) = A (M x K, row stride lda) * W (K x N, row
// stride ldw), bf16 in and out, float32 accumulation, on the tcgen05 GEMM.
// Strides, base addresses and column splits must be 16-byte multiples.  Tiles
// are 256 columns wide unless 192-column tiles cut waves x width by a quarter
// or more: a tile's time is about proportional to its width and the last wave
// runs as long as a full one, but 192-column tiles run a little less
// efficiently (measured on the layer: the 2048 x 2560 output projection gains,
// 160 tiles of 256 taking two waves on 148 SMs; the wider ones lose).
axon_status gemm_tc(int M, int N, int K, const void* A, int lda, const void* W, int ldw, const GemmOut* outs,
                    int nout, int* err, cudaStream_t st, int plan = AXON_GEMM_AUTO, const GemmScratch* sk = nullptr) {
    if (M == 0 || N == 0) return AXON_OK;
    if (K == 0 || nout < 1 || nout > 3) return AXON_ERR_UNSUPPORTED;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxBlockDevices) return AXON_ERR_CUDA;
    int sms = g_gemm_sms[dev].load(std::memory_order_relaxed);
    if (sms <= 0) {
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return AXON_ERR_CUDA;
        g_gemm_sms[dev].store(sms, std::memory_order_relaxed);
    }
    CUtensorMap ta;
    if (!tensor_map(&ta, A, (uint64_t)M, (uint64_t)K, (uint64_t)lda, kGmBK, kGmBM)) return AXON_ERR_CUDA;
    GemmParams p{};
    p.M = M; p.N = N; p.K = K;
    p.nout = nout;
    for (int i = 0; i < nout; ++i) p.out[i] = outs[i];
    p.err = err;
    if (plan == AXON_GEMM_PAIR || plan == AXON_GEMM_PAIR_STREAMK) {
        if (plan == AXON_GEMM_PAIR_STREAMK && !sk) return AXON_ERR_WORKSPACE;
        const int pairs = gemm_pair_slots(dev);
        if (pairs <= 0) return AXON_ERR_UNSUPPORTED;
        return launch_gemm_pair(M, N, K, ta, W, ldw, p, pairs, plan == AXON_GEMM_PAIR_STREAMK ? sk : nullptr, st);
    }
    const long long tm = (M + kGmBM - 1) / kGmBM;
    const long long w256 = (tm * ((N + 255) / 256) + sms - 1) / sms;
    const long long w192 = (tm * ((N + 191) / 192) + sms - 1) / sms;
    if (plan == AXON_GEMM_SINGLE_256) return launch_gemm<256>(M, N, K, ta, W, ldw, p, sms, st);
    if (plan == AXON_GEMM_SINGLE_192) return launch_gemm<192>(M, N, K, ta, W, ldw, p, sms, st);
    if (plan != AXON_GEMM_AUTO) return AXON_ERR_INVALID_ARG;
    // automatic: CTA pairs from 256 rows (their tiles are 256 rows high), with
    // the stream-K tail when whole tiles would leave a tenth or more of the
    // pairs' last wave idle (measured on the layer's projections: 2048 x 15360
    // x 2560 runs best on whole pair tiles, 7712- and 2560-column ones with
    // the split); single CTAs below 256 rows
    if (M >= kGpTileM) {
        const int pairs = gemm_pair_slots(dev);
        if (pairs > 0) {
            const long long pt = (long long)((M + kGpTileM - 1) / kGpTileM) * ((N + kGpTileN - 1) / kGpTileN);
            const long long np = pairs < kGpMaxPairs ? pairs : kGpMaxPairs;
            const long long slots = (pt + np - 1) / np * np;
            const bool split = sk != nullptr && 10 * pt < 9 * slots;
            return launch_gemm_pair(M, N, K, ta, W, ldw, p, pairs, split ? sk : nullptr, st);
        }
    }
    if (4 * w192 * 192 <= 3 * w256 * 256) return launch_gemm<192>(M, N, K, ta, W, ldw, p, sms, st);
    return launch_gemm<256>(M, N, K, ta, W, ldw, p, sms, st);
}

}  // namespace
}  // namespace axon

using namespace axon;

extern "C" {

size_t axon_ssm_block_workspace_bytes(int B, int L, int Dm, int E, int N, int K, axon_dtype io) {
    if (B < 0 || L < 0 || Dm < 0 || E < 0 || N != kN || K != kK || io != AXON_BF16) return 0;
    BlockPlan p;
    plan_block(B, L, E, N, K, &p);
    return p.total;
}

axon_status axon_ssm_block_fwd(int B, int L, int Dm, int E, int N, int K, axon_dtype io,
                               const void* X, const void* W_in, const void* W_x, const void* W_out,
                               const float* conv_w, const float* conv_b,
                               const float* dt_bias, const float* A_log, const float* D,
                               const void* conv_cache_in, const float* ssm_state_in,
                               void* out, void* conv_cache_out, float* ssm_state_out,
                               void* workspace, size_t workspace_bytes, axon_stream_t stream) {
    if (B < 0 || L < 0 || Dm < 0 || E < 0) return AXON_ERR_INVALID_ARG;
    if (N != kN || K != kK || io != AXON_BF16) return AXON_ERR_UNSUPPORTED;
    if ((long long)B * L > (1LL << 31) || (long long)B * E > (1LL << 31) ||
        (long long)(E + 2 * N) > (1LL << 30) || (long long)Dm > (1LL << 30))
        return AXON_ERR_UNSUPPORTED;
    if (Dm % 8 != 0 || E % 8 != 0) return AXON_ERR_ALIGNMENT;
    if (B == 0 || E == 0) return AXON_OK;
    if (!W_in || !W_x || !W_out || !conv_w || !conv_b || !dt_bias || !A_log || !D ||
        !conv_cache_out || !ssm_state_out || !workspace)
        return AXON_ERR_INVALID_ARG;
    if (L > 0 && (!X || !out)) return AXON_ERR_INVALID_ARG;
    const void* ptrs[] = {X, W_in, W_x, W_out, conv_w, conv_b, dt_bias, A_log, D, conv_cache_in,
                          ssm_state_in, out, conv_cache_out, ssm_state_out, workspace};
    for (const void* q : ptrs)
        if (q && !aligned16(q)) return AXON_ERR_ALIGNMENT;
    BlockPlan plan;
    plan_block(B, L, E, N, K, &plan);
    if (workspace_bytes < plan.total) return AXON_ERR_WORKSPACE;
    const size_t M = (size_t)B * L;
    const size_t n_out = M * Dm * 2;
    const size_t n_cc = (size_t)B * (K - 1) * E * 2, n_ss = (size_t)B * E * N * 4;
    // out and the workspace must not overlap any input, weight or each other
    const void* ins[] = {X, W_in, W_x, W_out};
    const size_t nin[] = {M * Dm * 2, (size_t)Dm * 2 * E * 2, (size_t)E * (E + 2 * N) * 2, (size_t)E * Dm * 2};
    for (int i = 0; i < 4; ++i)
        if (overlaps(ins[i], nin[i], out, n_out) || overlaps(ins[i], nin[i], workspace, plan.total))
            return AXON_ERR_INVALID_ARG;
    if (overlaps(out, n_out, workspace, plan.total) || overlaps(out, n_out, conv_cache_out, n_cc) ||
        overlaps(out, n_out, ssm_state_out, n_ss) || overlaps(workspace, plan.total, conv_cache_out, n_cc) ||
        overlaps(workspace, plan.total, ssm_state_out, n_ss) ||
        overlaps(workspace, plan.total, conv_cache_in, n_cc) || overlaps(workspace, plan.total, ssm_state_in, n_ss))
        return AXON_ERR_INVALID_ARG;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned char* ws = static_cast<unsigned char*>(workspace);
    int* err = reinterpret_cast<int*>(ws + plan.flag);
    __nv_bfloat16* x = reinterpret_cast<__nv_bfloat16*>(ws + plan.x);
    __nv_bfloat16* z = reinterpret_cast<__nv_bfloat16*>(ws + plan.z);
    __nv_bfloat16* u = reinterpret_cast<__nv_bfloat16*>(ws + plan.u);
    __nv_bfloat16* dt = reinterpret_cast<__nv_bfloat16*>(ws + plan.dt);
    __nv_bfloat16* bm = reinterpret_cast<__nv_bfloat16*>(ws + plan.bm);
    __nv_bfloat16* cm = reinterpret_cast<__nv_bfloat16*>(ws + plan.cm);
    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(ws + plan.y);
    const int Mi = (int)M;
    axon_status rc = AXON_OK;
    if (cudaMemsetAsync(err, 0, plan.sk_partial - plan.flag, st) != cudaSuccess) return AXON_ERR_CUDA;
    GemmScratch sk[3];
    for (int i = 0; i < 3; ++i) {
        sk[i].partial = reinterpret_cast<float*>(ws + plan.sk_partial);
        sk[i].flag = reinterpret_cast<int*>(ws + plan.sk_flag + i * kSkFlagBytes);
    }
    if (L > 0) {
        // (x, z) = split(X W_in): one GEMM over the 2E columns of W_in
        const GemmOut xz[2] = {{x, E, 0}, {z, E, E}};
        if ((rc = gemm_tc(Mi, 2 * E, Dm, X, Dm, W_in, 2 * E, xz, 2, err, st, AXON_GEMM_AUTO, &sk[0])) != AXON_OK)
            return rc;
        // u = SiLU(conv(x))
        ConvParams cp{B, L, E, x, conv_w, conv_b, conv_cache_in, u};
        const dim3 grid((unsigned)((E / kConvCh + kConvThreads - 1) / kConvThreads),
                        (unsigned)((L + kConvRun - 1) / kConvRun), (unsigned)B);
        if (grid.y > 65535u || grid.z > 65535u) return AXON_ERR_UNSUPPORTED;
        cudaLaunchConfig_t ccfg{};
        ccfg.gridDim = grid;
        ccfg.blockDim = dim3(kConvThreads, 1, 1);
        ccfg.stream = st;
        cudaLaunchAttribute cat[1];
        cat[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        cat[0].val.programmaticStreamSerializationAllowed = 1;
        ccfg.attrs = cat;
        ccfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&ccfg, conv_silu_kernel<IoBF16>, cp) != cudaSuccess) return AXON_ERR_CUDA;
        if (cudaGetLastError() != cudaSuccess) return AXON_ERR_CUDA;
        // (dt_raw, B, C) = split(u W_x): columns [0, E), [E, E+N), [E+N, E+2N), one GEMM
        const GemmOut dbc[3] = {{dt, E, 0}, {bm, N, E}, {cm, N, E + N}};
        if ((rc = gemm_tc(Mi, E + 2 * N, E, u, E, W_x, E + 2 * N, dbc, 3, err, st, AXON_GEMM_AUTO, &sk[1])) != AXON_OK)
            return rc;
    }
    // the fused layer core: conv, SiLU, dt, recurrence, D skip, SiLU(z) gate, caches
    rc = axon_ssm_scan_fwd_segments(B, L, E, N, K, AXON_BF16, x, z, dt, bm, cm, conv_w, conv_b, dt_bias,
                                    A_log, D, conv_cache_in, ssm_state_in, y, conv_cache_out, ssm_state_out,
                                    plan.scan_ws_bytes ? ws + plan.scan_ws : nullptr, plan.scan_ws_bytes, 0,
                                    stream);
    if (rc != AXON_OK || L == 0) return rc;
    // out = y W_out
    const GemmOut o[1] = {{static_cast<__nv_bfloat16*>(out), Dm, 0}};
    return gemm_tc(Mi, Dm, E, y, E, W_out, Dm, o, 1, err, st, AXON_GEMM_AUTO, &sk[2]);
}

axon_status axon_gemm_bf16(int M, int N, int K, const void* A, int lda, const void* W, int ldw, void* C, int ldc,
                           int* err, axon_stream_t stream) {
    return axon_gemm_bf16_plan(M, N, K, A, lda, W, ldw, C, ldc, err, AXON_GEMM_AUTO, nullptr, 0, stream);
}

size_t axon_gemm_workspace_bytes(void) { return kSkFlagBytes + kSkPartialBytes; }

axon_status axon_gemm_bf16_plan(int M, int N, int K, const void* A, int lda, const void* W, int ldw, void* C,
                                int ldc, int* err, int plan, void* workspace, size_t workspace_bytes,
                                axon_stream_t stream) {
    if (plan < AXON_GEMM_AUTO || plan > AXON_GEMM_PAIR_STREAMK) return AXON_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 0 || lda < K || ldw < N || ldc < N) return AXON_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return AXON_OK;
    if (K == 0 || !A || !W || !C) return AXON_ERR_INVALID_ARG;
    if (N % 8 || lda % 8 || ldw % 8 || ldc % 8 || !aligned16(A) || !aligned16(W) || !aligned16(C) ||
        (err && (reinterpret_cast<uintptr_t>(err) & 3u)))
        return AXON_ERR_ALIGNMENT;
    if (overlaps(C, (size_t)M * ldc * 2, A, (size_t)M * lda * 2) || overlaps(C, (size_t)M * ldc * 2, W, (size_t)K * ldw * 2))
        return AXON_ERR_INVALID_ARG;
    const GemmOut o[1] = {{static_cast<__nv_bfloat16*>(C), ldc, 0}};
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    GemmScratch sk{};
    const bool have_ws = workspace != nullptr && workspace_bytes >= axon_gemm_workspace_bytes();
    if (workspace && !aligned16(workspace)) return AXON_ERR_ALIGNMENT;
    if (have_ws) {
        const size_t nw = axon_gemm_workspace_bytes();
        if (overlaps(workspace, nw, A, (size_t)M * lda * 2) || overlaps(workspace, nw, W, (size_t)K * ldw * 2) ||
            overlaps(workspace, nw, C, (size_t)M * ldc * 2))
            return AXON_ERR_INVALID_ARG;
        sk.flag = static_cast<int*>(workspace);
        sk.partial = reinterpret_cast<float*>(static_cast<unsigned char*>(workspace) + kSkFlagBytes);
        if (cudaMemsetAsync(sk.flag, 0, kSkFlagBytes, st) != cudaSuccess) return AXON_ERR_CUDA;
    } else if (plan == AXON_GEMM_PAIR_STREAMK) {
        return AXON_ERR_WORKSPACE;
    }
    return gemm_tc(M, N, K, A, lda, W, ldw, o, 1, err, st, plan, have_ws ? &sk : nullptr);
}

}  // extern "C"
