// axon_block.cu -- the whole Axon-SSM layer around the scan (C ABI in
// include/axon_ssm.h): input projection, conv stage, projection to the SSM
// parameters, the fused scan, output projection.
//
// Axon-SSM page, "Gating": (x, z) = split(W_in X) and y_out = W_out (y_ssm *
// SiLU(z)); "Selective mechanism": (dt, B, C) = f_proj(conv output), read as
// one linear map E -> E + 2N.  The four projections are plain bf16 GEMMs with
// float32 accumulation, run by cuBLASLt; the conv stage and the scan are this
// library's kernels.
#include <cublasLt.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "axon_ssm.h"
#include "conv_silu.cuh"
#include "device_math.cuh"

namespace axon {
namespace {

constexpr size_t kGemmWorkspace = size_t(32) << 20;   // cuBLASLt scratch inside the caller's workspace
constexpr size_t kAlign = 256;
constexpr int kMaxBlockDevices = 64;

size_t round_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

// Byte offsets of the intermediates inside the caller's workspace.
struct BlockPlan {
    size_t x, z, u, dt, bm, cm, y, scan_ws, scan_ws_bytes, gemm_ws, total;
};

bool plan_block(int B, int L, int E, int N, int K, BlockPlan* p) {
    const size_t M = (size_t)B * L;
    const size_t act = round_up(M * E * 2), bc = round_up(M * N * 2);
    size_t off = 0;
    p->x = off; off += act;
    p->z = off; off += act;
    p->u = off; off += act;
    p->dt = off; off += act;
    p->bm = off; off += bc;
    p->cm = off; off += bc;
    p->y = off; off += act;
    p->scan_ws_bytes = axon_ssm_scan_workspace_bytes(B, L, E, N, K, AXON_BF16);
    p->scan_ws = off; off += round_up(p->scan_ws_bytes);
    p->gemm_ws = off; off += kGemmWorkspace;
    p->total = off;
    return true;
}

// One cuBLASLt handle per device, created on first use with that device current.
std::mutex g_lt_mu;
cublasLtHandle_t g_lt[kMaxBlockDevices] = {};

axon_status lt_handle(cublasLtHandle_t* out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return AXON_ERR_CUDA;
    if (dev < 0 || dev >= kMaxBlockDevices) return AXON_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_lt_mu);
    if (!g_lt[dev] && cublasLtCreate(&g_lt[dev]) != CUBLAS_STATUS_SUCCESS) {
        g_lt[dev] = nullptr;
        return AXON_ERR_CUDA;
    }
    *out = g_lt[dev];
    return AXON_OK;
}

// Row-major C (M x Nc, ldc) = A (M x Kd, lda) * W (Kd x Nc, ldw), bf16 in and
// out, float32 accumulation.  In cuBLASLt's column-major terms this is
// C^T (Nc x M) = W^T (Nc x Kd) * A^T (Kd x M), no transposes.
axon_status gemm_rm(cublasLtHandle_t lt, int M, int Nc, int Kd, const void* A, int lda,
                    const void* W, int ldw, void* C, int ldc, void* ws, size_t ws_bytes,
                    cudaStream_t st) {
    if (M == 0 || Nc == 0) return AXON_OK;
    cublasLtMatmulDesc_t op = nullptr;
    cublasLtMatrixLayout_t dw = nullptr, da = nullptr, dc = nullptr;
    cublasLtMatmulPreference_t pref = nullptr;
    axon_status rc = AXON_ERR_CUDA;
    const float alpha = 1.0f, beta = 0.0f;
    cublasLtMatmulHeuristicResult_t heur{};
    int found = 0;
    if (cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS) goto done;
    if (cublasLtMatrixLayoutCreate(&dw, CUDA_R_16BF, Nc, Kd, ldw) != CUBLAS_STATUS_SUCCESS) goto done;
    if (cublasLtMatrixLayoutCreate(&da, CUDA_R_16BF, Kd, M, lda) != CUBLAS_STATUS_SUCCESS) goto done;
    if (cublasLtMatrixLayoutCreate(&dc, CUDA_R_16BF, Nc, M, ldc) != CUBLAS_STATUS_SUCCESS) goto done;
    if (cublasLtMatmulPreferenceCreate(&pref) != CUBLAS_STATUS_SUCCESS) goto done;
    if (cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws_bytes,
                                             sizeof(ws_bytes)) != CUBLAS_STATUS_SUCCESS) goto done;
    if (cublasLtMatmulAlgoGetHeuristic(lt, op, dw, da, dc, dc, pref, 1, &heur, &found) != CUBLAS_STATUS_SUCCESS ||
        found == 0) {
        rc = AXON_ERR_UNSUPPORTED;
        goto done;
    }
    if (cublasLtMatmul(lt, op, &alpha, W, dw, A, da, &beta, C, dc, C, dc, &heur.algo, ws, ws_bytes, st) ==
        CUBLAS_STATUS_SUCCESS)
        rc = AXON_OK;
done:
    if (pref) cublasLtMatmulPreferenceDestroy(pref);
    if (dc) cublasLtMatrixLayoutDestroy(dc);
    if (da) cublasLtMatrixLayoutDestroy(da);
    if (dw) cublasLtMatrixLayoutDestroy(dw);
    if (op) cublasLtMatmulDescDestroy(op);
    return rc;
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
    void* x = ws + plan.x;
    void* z = ws + plan.z;
    void* u = ws + plan.u;
    void* dt = ws + plan.dt;
    void* bm = ws + plan.bm;
    void* cm = ws + plan.cm;
    void* y = ws + plan.y;
    void* gws = ws + plan.gemm_ws;
    const int Mi = (int)M;
    const unsigned char* wx = static_cast<const unsigned char*>(W_x);
    const unsigned char* win = static_cast<const unsigned char*>(W_in);
    axon_status rc = AXON_OK;
    if (L > 0) {
        cublasLtHandle_t lt = nullptr;
        if ((rc = lt_handle(&lt)) != AXON_OK) return rc;
        // (x, z) = split(X W_in): the two column halves of W_in
        if ((rc = gemm_rm(lt, Mi, E, Dm, X, Dm, win, 2 * E, x, E, gws, kGemmWorkspace, st)) != AXON_OK) return rc;
        if ((rc = gemm_rm(lt, Mi, E, Dm, X, Dm, win + (size_t)E * 2, 2 * E, z, E, gws, kGemmWorkspace, st)) != AXON_OK)
            return rc;
        // u = SiLU(conv(x))
        ConvParams cp{B, L, E, x, conv_w, conv_b, conv_cache_in, u};
        const dim3 grid((unsigned)((E / 8 + kConvThreads - 1) / kConvThreads),
                        (unsigned)((L + kConvRun - 1) / kConvRun), (unsigned)B);
        if (grid.y > 65535u || grid.z > 65535u) return AXON_ERR_UNSUPPORTED;
        conv_silu_kernel<IoBF16><<<grid, kConvThreads, 0, st>>>(cp);
        if (cudaGetLastError() != cudaSuccess) return AXON_ERR_CUDA;
        // (dt_raw, B, C) = split(u W_x): columns [0, E), [E, E+N), [E+N, E+2N)
        const int ldx = E + 2 * N;
        if ((rc = gemm_rm(lt, Mi, E, E, u, E, wx, ldx, dt, E, gws, kGemmWorkspace, st)) != AXON_OK) return rc;
        if ((rc = gemm_rm(lt, Mi, N, E, u, E, wx + (size_t)E * 2, ldx, bm, N, gws, kGemmWorkspace, st)) != AXON_OK)
            return rc;
        if ((rc = gemm_rm(lt, Mi, N, E, u, E, wx + (size_t)(E + N) * 2, ldx, cm, N, gws, kGemmWorkspace, st)) !=
            AXON_OK)
            return rc;
    }
    // the fused layer core: conv, SiLU, dt, recurrence, D skip, SiLU(z) gate, caches
    rc = axon_ssm_scan_fwd_segments(B, L, E, N, K, AXON_BF16, x, z, dt, bm, cm, conv_w, conv_b, dt_bias,
                                    A_log, D, conv_cache_in, ssm_state_in, y, conv_cache_out, ssm_state_out,
                                    plan.scan_ws_bytes ? ws + plan.scan_ws : nullptr, plan.scan_ws_bytes, 0,
                                    stream);
    if (rc != AXON_OK || L == 0) return rc;
    // out = y W_out
    cublasLtHandle_t lt = nullptr;
    if ((rc = lt_handle(&lt)) != AXON_OK) return rc;
    return gemm_rm(lt, Mi, Dm, E, y, E, W_out, Dm, out, Dm, gws, kGemmWorkspace, st);
}

}  // extern "C"
