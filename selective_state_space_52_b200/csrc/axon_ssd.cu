// axon_ssd.cu -- C ABI of the Mamba-2 (SSD) layer core (include/axon_ssm.h):
// argument checks, the segment plan, the workspace, and the launches of
// ssd.cuh (per-chunk decays, the chunk walks).
#include <cuda_runtime.h>

#include <algorithm>
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
size_t up256(size_t n) { return (n + 255) & ~size_t(255); }

// Resident chunk walks per SM: one full walk (217 KB of shared memory, 512
// tensor-memory columns), three state-only walks (70 KB, 64 columns each).
constexpr int kWalksPerSm = 1;
constexpr int kStateWalksPerSm = 3;

int sm_count() {
    static std::atomic<int> cached[64];   // zero-initialised (static storage)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64) {
        const int v = cached[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < 64) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

// Segments of whole chunks: enough (head, segment) walks to give every SM
// kWalksPerSm of them, at most one per chunk and kSsdMaxSegs; `requested` > 0
// asks for that many (still capped).  Returns segments and chunks per segment.
void plan_segments(int B, int H, int nC, int requested, int& segs, int& cps) {
    if (nC <= 1) {
        segs = 1;
        cps = std::max(nC, 1);
        return;
    }
    long long want = requested > 0 ? requested
                                   : std::max<long long>(1, (long long)kWalksPerSm * sm_count() / std::max(1LL, (long long)B * H));
    want = std::min<long long>(want, std::min(nC, kSsdMaxSegs));
    cps = (int)((nC + want - 1) / want);
    segs = (nC + cps - 1) / cps;
}

// Pieces per segment for the first (state-only) walk: enough walks over the
// segments but the last to give every SM kStateWalksPerSm of them.  Returns
// pieces per segment and chunks per piece (no piece is empty).
void plan_pieces(int B, int H, int segs, int cps, int& pcs, int& cpp) {
    pcs = 1;
    if (segs > 1) {
        const long long walks = (long long)(segs - 1) * B * H;
        pcs = (int)std::max<long long>(1, (long long)kStateWalksPerSm * sm_count() / walks);
        pcs = std::min(pcs, cps);
    }
    cpp = (cps + pcs - 1) / pcs;
    pcs = (cps + cpp - 1) / cpp;
}

struct SsdWs {
    size_t err, prep, sloc, sega, h0c, total;
};
SsdWs ws_layout(int B, int L, int H, int segs, int pcs) {
    const size_t nC = ((size_t)L + kSsdQ - 1) / kSsdQ;
    SsdWs w{};
    w.err = 0;
    w.prep = w.err + 256;
    w.sloc = w.prep + up256((size_t)B * H * nC * 4 * kSsdQ * 4);
    const size_t extra = segs > 1 ? (size_t)(segs - 1) * pcs : 0;
    w.sega = w.sloc + up256(extra * B * H * kSsdP * kSsdN * 4);
    w.h0c = w.sega + up256(extra * B * H * 4);
    w.total = w.h0c + (segs > 1 ? up256((size_t)B * H * kSsdP * kSsdN * 4) : 0);
    if (nC == 0) w.total = 0;                  // an empty sequence only copies the state
    return w;
}

template <bool kFull>
bool allow_smem() {
    static std::atomic<unsigned long long> done{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return true;
    if (cudaFuncSetAttribute(ssd_chunk_scan_kernel<kFull>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SsdSmem<kFull>::TOTAL) != cudaSuccess)
        return false;
    if (bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return true;
}

}  // namespace
}  // namespace axon

using namespace axon;

extern "C" {

axon_status axon_ssd_wait_probe(int* status, int limit, axon_stream_t stream) {
    if (!status || (reinterpret_cast<uintptr_t>(status) & 3u) || limit < 1 || limit > (1 << 16))
        return AXON_ERR_INVALID_ARG;
    ssd_wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status, limit);
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

size_t axon_ssd_workspace_bytes(int B, int L, int H, int P, int N, int segments) {
    if (B < 0 || L < 0 || H < 0 || segments < 0 || P != kSsdP || N != kSsdN) return 0;
    int segs = 1, cps = 1, pcs = 1, cpp = 1;
    plan_segments(B, H, (L + kSsdQ - 1) / kSsdQ, segments, segs, cps);
    plan_pieces(B, H, segs, cps, pcs, cpp);
    return ws_layout(B, L, H, segs, pcs).total;
}

axon_status axon_ssd_scan_fwd(int B, int L, int H, int P, int N, axon_dtype io,
                              const void* x, const void* dt_raw, const float* dt_bias, const float* A_log,
                              const void* Bm, const void* Cm, const float* D, const float* h0,
                              void* y, float* h_out, int segments, void* workspace, size_t workspace_bytes,
                              axon_stream_t stream) {
    if (B < 0 || L < 0 || H < 0 || segments < 0) return AXON_ERR_INVALID_ARG;
    if (P != kSsdP || N != kSsdN || io != AXON_BF16) return AXON_ERR_UNSUPPORTED;
    if (B > 65535 || H > 65535 || (long long)B * L * H > (1LL << 31)) return AXON_ERR_UNSUPPORTED;
    if (B == 0 || H == 0) return AXON_OK;
    if (!dt_bias || !A_log || !D || !h_out) return AXON_ERR_INVALID_ARG;
    if (L > 0 && (!x || !dt_raw || !Bm || !Cm || !y)) return AXON_ERR_INVALID_ARG;
    const void* ptrs[] = {x, dt_raw, dt_bias, A_log, Bm, Cm, D, h0, y, h_out, workspace};
    for (const void* q : ptrs)
        if (q && !al16(q)) return AXON_ERR_ALIGNMENT;
    const int nC = (L + kSsdQ - 1) / kSsdQ;
    int segs = 1, cps = 1, pcs = 1, cpp = 1;
    plan_segments(B, H, nC, segments, segs, cps);
    plan_pieces(B, H, segs, cps, pcs, cpp);
    const SsdWs lay = ws_layout(B, L, H, segs, pcs);
    const size_t n_x = (size_t)B * L * H * kSsdP * 2, n_dt = (size_t)B * L * H * 2, n_bc = (size_t)B * L * kSsdN * 2;
    const size_t n_h = (size_t)B * H * kSsdP * kSsdN * 4, n_ws = lay.total;
    if (workspace_bytes < n_ws) return AXON_ERR_WORKSPACE;
    if (n_ws > 0 && !workspace) return AXON_ERR_INVALID_ARG;
    // y and the workspace overlap no input; h_out is h0 itself or disjoint from it
    const void* ins[] = {x, dt_raw, Bm, Cm, h0};
    const size_t nin[] = {n_x, n_dt, n_bc, n_bc, n_h};
    for (int i = 0; i < 5; ++i)
        if (ovl(ins[i], nin[i], y, n_x) || ovl(ins[i], nin[i], workspace, n_ws)) return AXON_ERR_INVALID_ARG;
    if (ovl(y, n_x, workspace, n_ws)) return AXON_ERR_INVALID_ARG;
    if ((const void*)h0 != (const void*)h_out && ovl(h0, n_h, h_out, n_h)) return AXON_ERR_INVALID_ARG;
    if (ovl(h_out, n_h, y, n_x) || ovl(h_out, n_h, x, n_x) || ovl(h_out, n_h, dt_raw, n_dt) ||
        ovl(h_out, n_h, Bm, n_bc) || ovl(h_out, n_h, Cm, n_bc) || ovl(h_out, n_h, workspace, n_ws))
        return AXON_ERR_INVALID_ARG;

    unsigned char* ws = static_cast<unsigned char*>(workspace);
    SsdParams p;
    p.B = B; p.L = L; p.H = H;
    p.nC = nC; p.segs = segs; p.cps = cps; p.pcs = pcs; p.cpp = cpp;
    p.x = static_cast<const __nv_bfloat16*>(x);
    p.dt_raw = static_cast<const __nv_bfloat16*>(dt_raw);
    p.dt_bias = dt_bias; p.A_log = A_log;
    p.Bm = static_cast<const __nv_bfloat16*>(Bm);
    p.Cm = static_cast<const __nv_bfloat16*>(Cm);
    p.D = D; p.h0 = h0;
    p.y = static_cast<__nv_bfloat16*>(y);
    p.h_out = h_out;
    p.err = reinterpret_cast<int*>(ws + lay.err);
    p.prep = reinterpret_cast<float*>(ws + lay.prep);
    p.sloc = reinterpret_cast<float*>(ws + lay.sloc);
    p.sega = reinterpret_cast<float*>(ws + lay.sega);
    p.h0c = (segs > 1 && h0) ? reinterpret_cast<float*>(ws + lay.h0c) : nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (nC > 0) {
        ssd_chunk_prep_kernel<<<dim3((unsigned)nC, (unsigned)((H + 3) / 4), (unsigned)B), kSsdThreads, 0, st>>>(p);
        if (cudaGetLastError() != cudaSuccess) return AXON_ERR_CUDA;
    }
    if (!allow_smem<true>() || !allow_smem<false>()) return AXON_ERR_CUDA;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    auto config = [&](dim3 grid, unsigned threads, size_t smem) {
        cudaLaunchConfig_t c{};
        c.gridDim = grid;
        c.blockDim = dim3(threads, 1, 1);
        c.dynamicSmemBytes = smem;
        c.stream = st;
        c.attrs = pdl;
        c.numAttrs = 1;
        return c;
    };
    if (segs > 1) {
        const cudaLaunchConfig_t c = config(dim3((unsigned)H, (unsigned)((segs - 1) * pcs), (unsigned)B), kSsdThreads,
                                            SsdSmem<false>::TOTAL);
        if (cudaLaunchKernelEx(&c, ssd_chunk_scan_kernel<false>, p) != cudaSuccess) return AXON_ERR_CUDA;
    }
    const cudaLaunchConfig_t c = config(dim3((unsigned)H, (unsigned)segs, (unsigned)B), kSsdFullThreads,
                                        SsdSmem<true>::TOTAL);
    if (cudaLaunchKernelEx(&c, ssd_chunk_scan_kernel<true>, p) != cudaSuccess) return AXON_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

}  // extern "C"
