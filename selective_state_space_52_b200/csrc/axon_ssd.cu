// axon_ssd.cu -- C ABI of the Mamba-2 (SSD) layer core (include/axon_ssm.h):
// argument checks, the chunk-Gram workspace, and the two launches of ssd.cuh.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "axon_ssm.h"
#include "ssd.cuh"

namespace axon {
namespace {

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ovl(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}
size_t gram_bytes(int B, int L) {
    const size_t nC = ((size_t)L + kSsdQ - 1) / kSsdQ;
    return (size_t)B * nC * kSsdQ * kSsdQ * sizeof(float);
}

}  // namespace
}  // namespace axon

using namespace axon;

extern "C" {

size_t axon_ssd_workspace_bytes(int B, int L, int H, int P, int N) {
    if (B < 0 || L < 0 || H < 0 || P != kSsdP || N != kSsdN) return 0;
    return gram_bytes(B, L);
}

axon_status axon_ssd_scan_fwd(int B, int L, int H, int P, int N, axon_dtype io,
                              const void* x, const void* dt_raw, const float* dt_bias, const float* A_log,
                              const void* Bm, const void* Cm, const float* D, const float* h0,
                              void* y, float* h_out, void* workspace, size_t workspace_bytes,
                              axon_stream_t stream) {
    if (B < 0 || L < 0 || H < 0) return AXON_ERR_INVALID_ARG;
    if (P != kSsdP || N != kSsdN || io != AXON_BF16) return AXON_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535 || (long long)B * L * H > (1LL << 31)) return AXON_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return AXON_OK;
    if (!dt_bias || !A_log || !D || !h_out) return AXON_ERR_INVALID_ARG;
    if (L > 0 && (!x || !dt_raw || !Bm || !Cm || !y || !workspace)) return AXON_ERR_INVALID_ARG;
    const void* ptrs[] = {x, dt_raw, dt_bias, A_log, Bm, Cm, D, h0, y, h_out, workspace};
    for (const void* q : ptrs)
        if (q && !al16(q)) return AXON_ERR_ALIGNMENT;
    const size_t n_x = (size_t)B * L * H * kSsdP * 2, n_dt = (size_t)B * L * H * 2, n_bc = (size_t)B * L * kSsdN * 2;
    const size_t n_h = (size_t)B * H * kSsdP * kSsdN * 4, n_ws = gram_bytes(B, L);
    if (L > 0 && workspace_bytes < n_ws) return AXON_ERR_WORKSPACE;
    // y and the workspace overlap no input; h_out is h0 itself or disjoint from it
    const void* ins[] = {x, dt_raw, Bm, Cm, h0};
    const size_t nin[] = {n_x, n_dt, n_bc, n_bc, n_h};
    for (int i = 0; i < 5; ++i)
        if (ovl(ins[i], nin[i], y, n_x) || (L > 0 && ovl(ins[i], nin[i], workspace, n_ws))) return AXON_ERR_INVALID_ARG;
    if ((const void*)h0 != (const void*)h_out && ovl(h0, n_h, h_out, n_h)) return AXON_ERR_INVALID_ARG;
    if (ovl(h_out, n_h, y, n_x) || ovl(h_out, n_h, x, n_x) || ovl(h_out, n_h, dt_raw, n_dt) ||
        ovl(h_out, n_h, Bm, n_bc) || ovl(h_out, n_h, Cm, n_bc) || (L > 0 && ovl(h_out, n_h, workspace, n_ws)))
        return AXON_ERR_INVALID_ARG;

    SsdParams p;
    p.B = B; p.L = L; p.H = H;
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.dt_raw = static_cast<const __nv_bfloat16*>(dt_raw);
    p.dt_bias = dt_bias; p.A_log = A_log;
    p.Bm = static_cast<const __nv_bfloat16*>(Bm);
    p.Cm = static_cast<const __nv_bfloat16*>(Cm);
    p.D = D; p.h0 = h0;
    p.y = static_cast<__nv_bfloat16*>(y);
    p.h_out = h_out;
    p.G = static_cast<float*>(workspace);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int nC = (L + kSsdQ - 1) / kSsdQ;
    if (nC > 0) {
        ssd_gram_kernel<<<dim3((unsigned)nC, (unsigned)B), kSsdThreads, 0, st>>>(p);
        if (cudaGetLastError() != cudaSuccess) return AXON_ERR_CUDA;
    }
    static std::atomic<unsigned long long> smem_set{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return AXON_ERR_CUDA;
    const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
    if (!bit || !(smem_set.load(std::memory_order_acquire) & bit)) {
        if (cudaFuncSetAttribute(ssd_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SsdSmem::TOTAL) !=
            cudaSuccess)
            return AXON_ERR_CUDA;
        if (bit) smem_set.fetch_or(bit, std::memory_order_acq_rel);
    }
    ssd_scan_kernel<<<dim3((unsigned)H, kSsdP / kSsdPB, (unsigned)B), kSsdThreads, SsdSmem::TOTAL, st>>>(p);
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

}  // extern "C"
