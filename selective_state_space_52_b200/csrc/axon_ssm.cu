// axon_ssm.cu -- host side of the C ABI declared in include/axon_ssm.h:
// argument checks (nothing is launched on any error), the launch plan, and the
// kernel launches on the caller's stream.  The library allocates no device
// memory: scratch comes from the caller's workspace.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "axon_ssm.h"
#include "carry.cuh"
#include "probe.cuh"
#include "device_math.cuh"
#include "scan_chunked.cuh"
#include "scan_octo.cuh"
#include "scan_qsplit.cuh"
#include "scan_quad.cuh"
#include "scan_seq.cuh"
#include "step.cuh"

namespace axon {
namespace {

constexpr int kAbiVersion = 1;
constexpr int kMaxSegments = 64;      // time segments of a split scan
constexpr int kMinSegLen = 128;       // shortest segment the planner picks
constexpr int kScanThreads = 128;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

size_t io_bytes(axon_dtype io) { return io == AXON_BF16 ? 2 : 4; }

// Common size/dtype checks shared by prefill and decode.
axon_status check_shape(int B, int L, int E, int N, int K, axon_dtype io) {
    if (B < 0 || L < 0 || E < 0) return AXON_ERR_INVALID_ARG;
    if (N != kN || K != kK) return AXON_ERR_UNSUPPORTED;
    if (io != AXON_F32 && io != AXON_BF16) return AXON_ERR_UNSUPPORTED;
    // element counts must stay well inside 64-bit offsets and grid limits
    if ((long long)B * (long long)E > (1LL << 31)) return AXON_ERR_UNSUPPORTED;
    if (B > 65535) return AXON_ERR_UNSUPPORTED;
    if ((E % (io == AXON_BF16 ? 8 : 4)) != 0) return AXON_ERR_ALIGNMENT;
    return AXON_OK;
}

// Longest split the planner may use for a sequence of L tokens.
int max_segments_for(int L) {
    int p = L / kMinSegLen;
    if (p > kMaxSegments) p = kMaxSegments;
    return p < 1 ? 1 : p;
}

size_t ws_bytes_for(int B, int E, int P) {
    if (P <= 1) return 0;
    return (size_t)(P - 1) * (size_t)B * (size_t)E * (kN + 1) * sizeof(float);
}

// Per-device attributes, queried once per device (the values never change).
constexpr int kMaxDevices = 64;
std::atomic<int> g_sms[kMaxDevices];
std::atomic<int> g_max_smem[kMaxDevices];

int cached_attribute(std::atomic<int>* table, cudaDeviceAttr attr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return -1;
    if (dev < kMaxDevices) {
        const int v = table[dev].load(std::memory_order_relaxed);
        if (v > 0) return v;
    }
    int v = 0;
    if (cudaDeviceGetAttribute(&v, attr, dev) != cudaSuccess) return -1;
    if (dev < kMaxDevices && v > 0) table[dev].store(v, std::memory_order_relaxed);
    return v;
}

int device_sm_count() { return cached_attribute(g_sms, cudaDevAttrMultiProcessorCount); }

// Channel-parallel scan: one thread per (b, e).  Split the sequence only when
// the channels alone cannot give every SM a few warps.
int plan_segments(int B, int L, int E, int sms) {
    const long long channels = (long long)B * E;
    const long long want = (long long)sms * 1024;   // resident threads to aim for
    if (channels >= want / 2) return 1;
    long long p = (want + channels - 1) / channels;
    const int pmax = max_segments_for(L);
    if (p > pmax) p = pmax;
    return (int)(p < 1 ? 1 : p);
}

// Few channels and a long sequence: the channel tiles alone cannot occupy the
// GPU, so split the sequence into segments and carry between them.
bool use_time_split(int B, int L, int E, int sms) {
    return (long long)B * E < (long long)sms * 4 && L >= 2 * kMinSegLen;
}

int device_max_smem_optin() { return cached_attribute(g_max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin); }

// Raises a kernel's dynamic shared-memory limit to the device's opt-in maximum
// once per device (the limit only permits; each launch asks for what it uses).
template <class Kern>
bool allow_max_smem(Kern kern, std::atomic<unsigned long long>& done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
    const unsigned long long bit = dev < kMaxDevices ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return true;
    const int max_smem = device_max_smem_optin();
    if (max_smem <= 0) return false;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem) != cudaSuccess)
        return false;
    if (bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return true;
}

struct ChunkPlan {
    int W, R, ET, tiles_per_b, pitch, smem;
};

// Chunked scan plan: channel tiles of ET channels (about one CTA per SM when
// channels are scarce, 128-channel tiles when they are plentiful) and W runs of
// R tokens per chunk, the largest that fits the shared memory.
bool plan_chunked(int B, int E, int io_bytes, int sms, int max_smem, ChunkPlan* out) {
    const long long channels = (long long)B * E;
    ChunkPlan c{};
    if (channels >= (long long)sms * 256) {
        c.W = 1; c.R = 16;
        c.ET = E < 128 ? E : 128;
    } else {
        // about one tile per SM; all W runs of a channel share a warp, so ET
        // is a multiple of the 32/W channels a warp holds
        int tpb = sms / (B > 0 ? B : 1);
        if (tpb < 1) tpb = 1;
        const int et_ideal = (E + tpb - 1) / tpb;
        static const int opts[][2] = {{2, 16}, {4, 16}, {8, 16}, {16, 16}, {8, 8}, {16, 8}, {32, 8}};
        int best_score = -1;
        for (const auto& o : opts) {
            const int W = o[0], R = o[1];
            const int cpw = 32 / W;
            const int ET = (et_ideal + cpw - 1) / cpw * cpw;
            const int threads = ET * W;
            if (threads > 512) continue;
            const int pitch = ((ET * io_bytes + 15) & ~15) + 16;
            if (ChunkSmem(W, R, ET, pitch, io_bytes).total > max_smem) continue;
            // enough warps to hide latency first, then the fewest runs per channel
            const int score = (threads < 256 ? threads : 256) * 64 - W;
            if (score > best_score) { best_score = score; c.W = W; c.R = R; c.ET = ET; }
        }
        if (best_score < 0) {
            c.W = 1; c.R = 16;
            c.ET = et_ideal < 512 ? et_ideal : 512;
        }
    }
    if (c.ET * c.W > 512) return false;   // the kernel's launch bound
    c.tiles_per_b = (E + c.ET - 1) / c.ET;
    c.pitch = ((c.ET * io_bytes + 15) & ~15) + 16;
    c.smem = ChunkSmem(c.W, c.R, c.ET, c.pitch, io_bytes).total;
    if (c.smem > max_smem) return false;
    *out = c;
    return true;
}

// Warp-per-8-channels scan with the states split in quadrants.  Measured on
// B200: it beats the run-split chunked kernel from 48 channels per SM (first
// order; from 128 with exact ZOH, whose heavier input factor favours the
// chunked kernel's wider tiles a little longer) and the one-thread-per-channel
// walk up to 512 channels per SM.  The per-chunk byte offsets it keeps are
// 32-bit.
constexpr int kQuadT = 32;
bool use_quad(int B, int E, int io_bytes, int sms, bool zoh) {
    const long long channels = (long long)B * E;
    if (channels < (long long)sms * (zoh ? 128 : 48) || channels >= (long long)sms * 512) return false;
    return (long long)(kQuadT + kK) * E * io_bytes < (1LL << 31);
}

// Warp-per-4-channels scan with the states split in eighths: twice the warps
// of the quadrant scan for fewer channels.  Measured on B200: it beats the
// run-split chunked kernel from kOctoMinPerSm channels per SM, and the
// quadrant scan below 48 (first order) or 128 (exact ZOH) channels per SM.
constexpr int kOctoT = 32;
constexpr int kOctoMinPerSm = 8;
bool use_octo(int B, int E, int io_bytes, int sms, bool zoh) {
    const long long channels = (long long)B * E;
    if (channels < (long long)sms * kOctoMinPerSm || channels >= (long long)sms * (zoh ? 128 : 48)) return false;
    return (long long)(kOctoT + kK) * E * io_bytes < (1LL << 31);
}

template <class Io, bool Z>
axon_status launch_octo(const ChunkParams& prm, cudaStream_t st) {
    auto kern = scan_octo_kernel<Io, kOctoT, Z, 1>;
    const int smem = OctoSmem(kOctoT, Io::kBytes).total;       // one warp per CTA
    const long long warps = (long long)prm.B * (prm.E / kOctoCh);
    if (warps > 0x7fffffffLL) return AXON_ERR_UNSUPPORTED;
    kern<<<(unsigned)warps, 32, smem, st>>>(prm);
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

template <class Io, bool Z>
axon_status launch_quad(const ChunkParams& prm, cudaStream_t st) {
    auto kern = scan_quad_kernel<Io, kQuadT, Z>;
    const int smem = QuadSmem(kQuadT, Io::kBytes).total;       // one warp per CTA
    const long long warps = (long long)prm.B * ((prm.E + kQuadCh - 1) / kQuadCh);
    if (warps > 0x7fffffffLL) return AXON_ERR_UNSUPPORTED;
    kern<<<(unsigned)warps, 32, smem, st>>>(prm);
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

// Split-chunk quadrant scan: W warps per 8 channels, each chunk cut into W
// runs (R = 32 tokens per run for W = 1, else 8).
template <class Io, int W, int R, bool Z, bool S = false>
axon_status launch_qsplit_t(const ChunkParams& prm, cudaStream_t st) {
    auto kern = scan_qsplit_kernel<Io, W, R, Z, S>;
    static std::atomic<unsigned long long> smem_set{0};
    if (!allow_max_smem(kern, smem_set)) return AXON_ERR_CUDA;
    const int smem = QsplitSmem(W, R, Io::kBytes).total;
    const long long ctas = (long long)prm.B * ((prm.E + kQsCh - 1) / kQsCh);
    if (ctas > 0x7fffffffLL) return AXON_ERR_UNSUPPORTED;
    kern<<<(unsigned)ctas, 32 * W, smem, st>>>(prm);
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

// W runs per chunk: one run of 32 tokens, or W runs of 16 (S: the state-only form)
template <class Io, bool Z, bool S = false>
axon_status launch_qsplit(const ChunkParams& prm, int W, cudaStream_t st) {
    switch (W) {
        case 1: return launch_qsplit_t<Io, 1, 32, Z, S>(prm, st);
        case 2: return launch_qsplit_t<Io, 2, 16, Z, S>(prm, st);
        case 4: return launch_qsplit_t<Io, 4, 16, Z, S>(prm, st);
        case 8: return launch_qsplit_t<Io, 8, 16, Z, S>(prm, st);
    }
    return AXON_ERR_UNSUPPORTED;
}

// Tokens per run of the split-chunk scan with W runs per chunk.
int qsplit_run_len(int W) { return W == 1 ? 32 : 16; }

bool qsplit_fits(int B, int L, int E, int io_bytes, int W) {
    (void)B; (void)L;
    const int R = qsplit_run_len(W);
    return (long long)(W * R + kK) * E * io_bytes < (1LL << 31) &&
           QsplitSmem(W, R, io_bytes).total <= device_max_smem_optin();
}

// Shape code of the split-chunk quadrant scan for an unsplit first-order
// prefill, or 0 where another kernel is faster.  Measured on B200 (prefill
// time against the eighths / quadrant scans and the run-split chunked
// kernel): eight runs of 16 tokens per chunk win below about 20 channels per
// SM (where the CTAs of 8 channels alone leave the SMs nearly idle), one run of 32 tokens per
// chunk from 48 to 511 channels per SM; the eighths scan keeps 20 to 47, and
// the one-thread-per-channel walk 512 and up.
int plan_qsplit(int B, int L, int E, int io_bytes, int sms) {
    const long long channels = (long long)B * E;
    int W = 0;
    if (channels < (long long)sms * 20) W = 8;
    else if (channels >= (long long)sms * 48 && channels < (long long)sms * 512) W = 1;
    if (W == 0 || device_max_smem_optin() <= 0 || !qsplit_fits(B, L, E, io_bytes, W)) return 0;
    return W;
}

template <class Io, int W, int R, bool Z>
axon_status launch_chunked_t(const ChunkParams& prm, int smem, cudaStream_t st) {
    auto kern = scan_chunked_kernel<Io, W, R, Z>;
    static std::atomic<unsigned long long> smem_set{0};
    if (!allow_max_smem(kern, smem_set)) return AXON_ERR_CUDA;
    const unsigned grid = (unsigned)((long long)prm.B * prm.tiles_per_b);
    kern<<<grid, prm.ET * W, smem, st>>>(prm);
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

template <class Io, bool Z>
axon_status launch_chunked(const ChunkParams& prm, const ChunkPlan& c, cudaStream_t st) {
    switch (c.W * 100 + c.R) {
        case 116: return launch_chunked_t<Io, 1, 16, Z>(prm, c.smem, st);
        case 216: return launch_chunked_t<Io, 2, 16, Z>(prm, c.smem, st);
        case 416: return launch_chunked_t<Io, 4, 16, Z>(prm, c.smem, st);
        case 808: return launch_chunked_t<Io, 8, 8, Z>(prm, c.smem, st);
        case 816: return launch_chunked_t<Io, 8, 16, Z>(prm, c.smem, st);
        case 1608: return launch_chunked_t<Io, 16, 8, Z>(prm, c.smem, st);
        case 1616: return launch_chunked_t<Io, 16, 16, Z>(prm, c.smem, st);
        case 3208: return launch_chunked_t<Io, 32, 8, Z>(prm, c.smem, st);
    }
    return AXON_ERR_UNSUPPORTED;
}

template <class Io, bool Z>
axon_status launch_scan(ScanParams& prm, cudaStream_t st) {
    const dim3 block(kScanThreads);
    const unsigned gx = (unsigned)((prm.E + kScanThreads - 1) / kScanThreads);
    if (prm.L == 0) {
        copy_state_kernel<Io><<<dim3(gx, prm.B), block, 0, st>>>(prm);
    } else {
        const unsigned gz = (unsigned)(prm.num_seg > 1 ? prm.num_seg - 1 : 1);
        scan_seq_phase1<Io, Z><<<dim3(gx, prm.B, gz), block, 0, st>>>(prm);
        if (prm.num_seg > 1)
            scan_seq_phase2<Io, Z><<<dim3(gx, prm.B, prm.num_seg - 1), block, 0, st>>>(prm);
    }
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

axon_status scan_impl(int B, int L, int E, int N, int K, axon_dtype io,
                      const void* x, const void* z, const void* dt_raw,
                      const void* Bm, const void* Cm,
                      const float* conv_w, const float* conv_b,
                      const float* dt_bias, const float* A_log, const float* D,
                      const void* conv_cache_in, const float* ssm_state_in,
                      void* y, void* conv_cache_out, float* ssm_state_out,
                      void* workspace, size_t workspace_bytes, int num_segments,
                      cudaStream_t stream, bool zoh = false, int forced_qsplit = 0) {
    axon_status st = check_shape(B, L, E, N, K, io);
    if (st != AXON_OK) return st;
    if (num_segments < 0) return AXON_ERR_INVALID_ARG;
    if (B == 0 || E == 0) return AXON_OK;
    if (!conv_w || !conv_b || !dt_bias || !A_log || !D || !conv_cache_out || !ssm_state_out)
        return AXON_ERR_INVALID_ARG;
    if (L > 0 && (!x || !z || !dt_raw || !Bm || !Cm || !y)) return AXON_ERR_INVALID_ARG;
    const void* ptrs[] = {x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
                          conv_cache_in, ssm_state_in, y, conv_cache_out, ssm_state_out};
    for (const void* q : ptrs)
        if (q && !aligned16(q)) return AXON_ERR_ALIGNMENT;

    const size_t sio = io_bytes(io);
    const size_t n_seq = (size_t)B * L * E * sio;
    const size_t n_bc = (size_t)B * L * kN * sio;
    const size_t n_cc = (size_t)B * (kK - 1) * E * sio;
    const size_t n_ss = (size_t)B * E * kN * sizeof(float);
    // outputs: caches either exactly in place or disjoint; y disjoint from all
    if (conv_cache_in != conv_cache_out && overlaps(conv_cache_in, n_cc, conv_cache_out, n_cc))
        return AXON_ERR_INVALID_ARG;
    if ((const void*)ssm_state_in != (const void*)ssm_state_out &&
        overlaps(ssm_state_in, n_ss, ssm_state_out, n_ss))
        return AXON_ERR_INVALID_ARG;
    if (L > 0) {
        const void* ins[] = {x, z, dt_raw};
        for (const void* q : ins) if (overlaps(q, n_seq, y, n_seq)) return AXON_ERR_INVALID_ARG;
        if (overlaps(Bm, n_bc, y, n_seq) || overlaps(Cm, n_bc, y, n_seq)) return AXON_ERR_INVALID_ARG;
        if (overlaps(conv_cache_in, n_cc, y, n_seq) || overlaps(conv_cache_out, n_cc, y, n_seq) ||
            overlaps(ssm_state_in, n_ss, y, n_seq) || overlaps(ssm_state_out, n_ss, y, n_seq))
            return AXON_ERR_INVALID_ARG;
    }
    if (overlaps(conv_cache_out, n_cc, ssm_state_out, n_ss)) return AXON_ERR_INVALID_ARG;

    int P = 1;
    int seg = L > 0 ? L : 1;
    bool chunked = false, quad = false, octo = false;
    int qsplit = 0;                              // runs per chunk of the split-chunk quadrant scan
    ChunkPlan cplan{};
    if (forced_qsplit != 0) {
        if (forced_qsplit != 1 && forced_qsplit != 2 && forced_qsplit != 4 && forced_qsplit != 8)
            return AXON_ERR_INVALID_ARG;
        if (num_segments != 1) return AXON_ERR_INVALID_ARG;
        if (L > 0) {
            if (device_max_smem_optin() <= 0) return AXON_ERR_CUDA;
            if (!qsplit_fits(B, L, E, (int)io_bytes(io), forced_qsplit)) return AXON_ERR_UNSUPPORTED;
            qsplit = forced_qsplit;
        }
    } else if (L > 0) {
        if (num_segments > kMaxSegments) return AXON_ERR_INVALID_ARG;
        if (num_segments > 1) {
            P = num_segments;                  // forced time split (segment carry)
        } else {
            const int sms = device_sm_count();
            if (sms <= 0) return AXON_ERR_CUDA;
            if (num_segments == 0 && use_time_split(B, L, E, sms)) {
                P = plan_segments(B, L, E, sms);
            } else if (!zoh && (qsplit = plan_qsplit(B, L, E, (int)io_bytes(io), sms)) > 0) {
                // the split-chunk quadrant scan (first order)
            } else if (use_quad(B, E, (int)io_bytes(io), sms, zoh)) {
                quad = true;                   // unsplit: the quadrant scan
            } else if (use_octo(B, E, (int)io_bytes(io), sms, zoh)) {
                octo = true;                   // unsplit: the eighths scan
            } else {
                // unsplit: the chunked kernel (the channel walk is the fallback)
                const int max_smem = device_max_smem_optin();
                if (max_smem <= 0) return AXON_ERR_CUDA;
                chunked = plan_chunked(B, E, (int)io_bytes(io), sms, max_smem, &cplan);
            }
        }
        if (P > 1) {
            seg = (L + P - 1) / P;
            if (seg < kK) return AXON_ERR_INVALID_ARG;   // each segment must cover the conv window
            P = (L + seg - 1) / seg;                       // drop empty trailing segments
        }
    }
    const size_t need = ws_bytes_for(B, E, P);
    if (need > 0) {
        if (!workspace || workspace_bytes < need) return AXON_ERR_WORKSPACE;
        if (!aligned16(workspace)) return AXON_ERR_ALIGNMENT;
        if (overlaps(workspace, need, y, n_seq) || overlaps(workspace, need, ssm_state_out, n_ss) ||
            overlaps(workspace, need, conv_cache_out, n_cc))
            return AXON_ERR_INVALID_ARG;
    }

    if (chunked || quad || octo || qsplit) {
        ChunkParams cp{};
        cp.B = B; cp.L = L; cp.E = E;
        cp.ET = quad ? kQuadCh : (octo ? kOctoCh : cplan.ET);
        cp.tiles_per_b = quad ? (E + kQuadCh - 1) / kQuadCh : (octo ? E / kOctoCh : cplan.tiles_per_b);
        cp.pitch = (quad || octo) ? 0 : cplan.pitch;
        cp.x = x; cp.z = z; cp.dt_raw = dt_raw; cp.Bm = Bm; cp.Cm = Cm;
        cp.conv_w = conv_w; cp.conv_b = conv_b; cp.dt_bias = dt_bias; cp.A_log = A_log; cp.D = D;
        cp.conv_cache_in = conv_cache_in; cp.ssm_state_in = ssm_state_in;
        cp.y = y; cp.conv_cache_out = conv_cache_out; cp.ssm_state_out = ssm_state_out;
        if (qsplit) {
            if (io == AXON_BF16)
                return zoh ? launch_qsplit<IoBF16, true>(cp, qsplit, stream) : launch_qsplit<IoBF16, false>(cp, qsplit, stream);
            return zoh ? launch_qsplit<IoF32, true>(cp, qsplit, stream) : launch_qsplit<IoF32, false>(cp, qsplit, stream);
        }
        if (octo) {
            if (io == AXON_BF16) return zoh ? launch_octo<IoBF16, true>(cp, stream) : launch_octo<IoBF16, false>(cp, stream);
            return zoh ? launch_octo<IoF32, true>(cp, stream) : launch_octo<IoF32, false>(cp, stream);
        }
        if (quad) {
            if (io == AXON_BF16) return zoh ? launch_quad<IoBF16, true>(cp, stream) : launch_quad<IoBF16, false>(cp, stream);
            return zoh ? launch_quad<IoF32, true>(cp, stream) : launch_quad<IoF32, false>(cp, stream);
        }
        if (io == AXON_BF16) return zoh ? launch_chunked<IoBF16, true>(cp, cplan, stream)
                                        : launch_chunked<IoBF16, false>(cp, cplan, stream);
        return zoh ? launch_chunked<IoF32, true>(cp, cplan, stream) : launch_chunked<IoF32, false>(cp, cplan, stream);
    }

    ScanParams prm;
    prm.B = B; prm.L = L; prm.E = E;
    prm.x = x; prm.z = z; prm.dt_raw = dt_raw; prm.Bm = Bm; prm.Cm = Cm;
    prm.conv_w = conv_w; prm.conv_b = conv_b; prm.dt_bias = dt_bias; prm.A_log = A_log; prm.D = D;
    prm.conv_cache_in = conv_cache_in; prm.ssm_state_in = ssm_state_in;
    prm.y = y; prm.conv_cache_out = conv_cache_out; prm.ssm_state_out = ssm_state_out;
    prm.num_seg = P;
    prm.seg_len = seg;   // segments [s*seg, min(L, (s+1)*seg)), s < P, all non-empty
    prm.ws_h = P > 1 ? static_cast<float*>(workspace) : nullptr;
    prm.ws_sdt = P > 1 ? static_cast<float*>(workspace) + (size_t)(P - 1) * B * E * kN : nullptr;

    if (io == AXON_BF16) return zoh ? launch_scan<IoBF16, true>(prm, stream) : launch_scan<IoBF16, false>(prm, stream);
    return zoh ? launch_scan<IoF32, true>(prm, stream) : launch_scan<IoF32, false>(prm, stream);
}

// ---- scratch for axon_ssm_scan_fwd_noalloc --------------------------------
// Library-owned device scratch for callers that cannot pass a workspace.  It
// is a file-scope __device__ array, so every GPU that loads this library holds
// it until the process exits.  In host code `g_static_scratch` is only a
// host-side stand-in for the symbol: its device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kMaxScratchDevices = 64;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxScratchDevices] = {};

// Device address of g_static_scratch on the current device (set up on first use).
axon_status static_scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return AXON_ERR_CUDA;
    if (dev < 0 || dev >= kMaxScratchDevices) return AXON_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
            return AXON_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return AXON_OK;
}

}  // namespace
}  // namespace axon

using namespace axon;

namespace axon {
// y = 2^x through exp2_fma2 (the FMA-pipe exp2), two values per thread.
__global__ void exp2_fma_kernel(const float* x, float* y, long long n) {
    const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const bool pair = i + 1 < n;
    const float2 v = exp2_fma2(make_float2(x[i], pair ? x[i + 1] : x[i]));
    y[i] = v.x;
    if (pair) y[i + 1] = v.y;
}
}  // namespace axon

extern "C" {

int axon_ssm_abi_version(void) { return kAbiVersion; }

const char* axon_status_string(axon_status s) {
    switch (s) {
        case AXON_OK: return "AXON_OK";
        case AXON_ERR_INVALID_ARG: return "AXON_ERR_INVALID_ARG";
        case AXON_ERR_UNSUPPORTED: return "AXON_ERR_UNSUPPORTED";
        case AXON_ERR_ALIGNMENT: return "AXON_ERR_ALIGNMENT";
        case AXON_ERR_WORKSPACE: return "AXON_ERR_WORKSPACE";
        case AXON_ERR_CUDA: return "AXON_ERR_CUDA";
        case AXON_ERR_TIMEOUT: return "AXON_ERR_TIMEOUT";
    }
    return "AXON_ERR_UNKNOWN";
}

size_t axon_ssm_scan_workspace_bytes(int B, int L, int E, int N, int K, axon_dtype io) {
    if (check_shape(B, L, E, N, K, io) != AXON_OK) return 0;
    return ws_bytes_for(B, E, max_segments_for(L));
}

int axon_ssm_scan_launch_count(int B, int L, int E, int N, int K, axon_dtype io) {
    if (check_shape(B, L, E, N, K, io) != AXON_OK) return -1;
    if (B == 0 || E == 0) return 0;
    if (L == 0) return 1;
    const int sms = device_sm_count();
    if (sms <= 0) return -1;
    if (use_time_split(B, L, E, sms)) return plan_segments(B, L, E, sms) > 1 ? 2 : 1;
    return 1;
}

axon_status axon_ssm_scan_fwd(int B, int L, int E, int N, int K, axon_dtype io,
                              const void* x, const void* z, const void* dt_raw,
                              const void* Bm, const void* Cm,
                              const float* conv_w, const float* conv_b,
                              const float* dt_bias, const float* A_log, const float* D,
                              const void* conv_cache_in, const float* ssm_state_in,
                              void* y, void* conv_cache_out, float* ssm_state_out,
                              void* workspace, size_t workspace_bytes, axon_stream_t stream) {
    return scan_impl(B, L, E, N, K, io, x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
                     conv_cache_in, ssm_state_in, y, conv_cache_out, ssm_state_out,
                     workspace, workspace_bytes, 0, reinterpret_cast<cudaStream_t>(stream));
}

axon_status axon_ssm_scan_fwd_segments(int B, int L, int E, int N, int K, axon_dtype io,
                                       const void* x, const void* z, const void* dt_raw,
                                       const void* Bm, const void* Cm,
                                       const float* conv_w, const float* conv_b,
                                       const float* dt_bias, const float* A_log, const float* D,
                                       const void* conv_cache_in, const float* ssm_state_in,
                                       void* y, void* conv_cache_out, float* ssm_state_out,
                                       void* workspace, size_t workspace_bytes, int num_segments,
                                       axon_stream_t stream) {
    return scan_impl(B, L, E, N, K, io, x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
                     conv_cache_in, ssm_state_in, y, conv_cache_out, ssm_state_out,
                     workspace, workspace_bytes, num_segments,
                     reinterpret_cast<cudaStream_t>(stream));
}

namespace {
// Batch rows per decode block: the fewest, in rounds of four, whose grid of
// ceil(E / 32) x ceil(B / rows) blocks fits the resident slots in one wave.
int step_rows(int B, int E, long long slots) {
    const long long bx = (E + kStepChan - 1) / kStepChan;
    int rows = B < 4 ? B : 4;
    while (rows < kStepMaxRows && rows < B && bx * ((B + rows - 1) / rows) > slots) rows += 4;
    return rows;
}

axon_status step_impl(int B, int E, int N, int K, axon_dtype io,
                      const void* x, const void* z, const void* dt_raw,
                      const void* Bm, const void* Cm,
                      const float* conv_w, const float* conv_b,
                      const float* dt_bias, const float* A_log, const float* D,
                      void* conv_cache, float* ssm_state, void* y, axon_stream_t stream, bool zoh) {
    axon_status st = check_shape(B, 1, E, N, K, io);
    if (st != AXON_OK) return st;
    if (B == 0 || E == 0) return AXON_OK;
    if (!x || !z || !dt_raw || !Bm || !Cm || !conv_w || !conv_b || !dt_bias || !A_log || !D ||
        !conv_cache || !ssm_state || !y)
        return AXON_ERR_INVALID_ARG;
    const void* ptrs[] = {x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
                          conv_cache, ssm_state, y};
    for (const void* q : ptrs)
        if (!aligned16(q)) return AXON_ERR_ALIGNMENT;
    const size_t sio = io_bytes(io);
    const size_t n_y = (size_t)B * E * sio;
    const size_t n_cc = (size_t)B * (kK - 1) * E * sio;
    const size_t n_ss = (size_t)B * E * kN * sizeof(float);
    const size_t n_bc = (size_t)B * kN * sio;
    if (overlaps(y, n_y, conv_cache, n_cc) || overlaps(y, n_y, ssm_state, n_ss) ||
        overlaps(conv_cache, n_cc, ssm_state, n_ss))
        return AXON_ERR_INVALID_ARG;
    const void* ins[] = {x, z, dt_raw};
    for (const void* q : ins)
        if (overlaps(q, n_y, y, n_y) || overlaps(q, n_y, conv_cache, n_cc) || overlaps(q, n_y, ssm_state, n_ss))
            return AXON_ERR_INVALID_ARG;
    if (overlaps(Bm, n_bc, y, n_y) || overlaps(Cm, n_bc, y, n_y)) return AXON_ERR_INVALID_ARG;

    StepParams prm;
    prm.B = B; prm.E = E;
    prm.x = x; prm.z = z; prm.dt_raw = dt_raw; prm.Bm = Bm; prm.Cm = Cm;
    prm.conv_w = conv_w; prm.conv_b = conv_b; prm.dt_bias = dt_bias; prm.A_log = A_log; prm.D = D;
    prm.conv_cache = conv_cache; prm.ssm_state = ssm_state; prm.y = y;
    const int sms = device_sm_count();
    if (sms <= 0) return AXON_ERR_CUDA;
    void (*kern)(StepParams, int);
    if (io == AXON_BF16) kern = zoh ? step_kernel<IoBF16, true> : step_kernel<IoBF16, false>;
    else kern = zoh ? step_kernel<IoF32, true> : step_kernel<IoF32, false>;
    // resident blocks per SM of this instance (a property of the compiled
    // kernel, queried once)
    static std::atomic<int> occupancy[4];
    const int ki = (io == AXON_BF16 ? 2 : 0) + (zoh ? 1 : 0);
    int per_sm = occupancy[ki].load(std::memory_order_relaxed);
    if (per_sm <= 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kStepThreads, 0) != cudaSuccess || per_sm <= 0)
            return AXON_ERR_CUDA;
        occupancy[ki].store(per_sm, std::memory_order_relaxed);
    }
    const int rows = step_rows(B, E, (long long)per_sm * sms);
    const dim3 grid((unsigned)((E + kStepChan - 1) / kStepChan), (unsigned)((B + rows - 1) / rows));
    kern<<<grid, kStepThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(prm, rows);
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}
}  // namespace

axon_status axon_ssm_step(int B, int E, int N, int K, axon_dtype io,
                          const void* x, const void* z, const void* dt_raw,
                          const void* Bm, const void* Cm,
                          const float* conv_w, const float* conv_b,
                          const float* dt_bias, const float* A_log, const float* D,
                          void* conv_cache, float* ssm_state, void* y, axon_stream_t stream) {
    return step_impl(B, E, N, K, io, x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
                     conv_cache, ssm_state, y, stream, false);
}

axon_status axon_ssm_step_ex(int B, int E, int N, int K, axon_dtype io, axon_discretization disc,
                             const void* x, const void* z, const void* dt_raw,
                             const void* Bm, const void* Cm,
                             const float* conv_w, const float* conv_b,
                             const float* dt_bias, const float* A_log, const float* D,
                             void* conv_cache, float* ssm_state, void* y, axon_stream_t stream) {
    if (disc != AXON_DISC_FIRST_ORDER && disc != AXON_DISC_ZOH) return AXON_ERR_UNSUPPORTED;
    return step_impl(B, E, N, K, io, x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
                     conv_cache, ssm_state, y, stream, disc == AXON_DISC_ZOH);
}

axon_status axon_ssm_scan_fwd_ex(int B, int L, int E, int N, int K, axon_dtype io,
                                 axon_discretization disc,
                                 const void* x, const void* z, const void* dt_raw,
                                 const void* Bm, const void* Cm,
                                 const float* conv_w, const float* conv_b,
                                 const float* dt_bias, const float* A_log, const float* D,
                                 const void* conv_cache_in, const float* ssm_state_in,
                                 void* y, void* conv_cache_out, float* ssm_state_out,
                                 void* workspace, size_t workspace_bytes, int num_segments,
                                 axon_stream_t stream) {
    if (disc != AXON_DISC_FIRST_ORDER && disc != AXON_DISC_ZOH) return AXON_ERR_UNSUPPORTED;
    return scan_impl(B, L, E, N, K, io, x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
                     conv_cache_in, ssm_state_in, y, conv_cache_out, ssm_state_out,
                     workspace, workspace_bytes, num_segments,
                     reinterpret_cast<cudaStream_t>(stream), disc == AXON_DISC_ZOH);
}

axon_status axon_ssm_scan_fwd_qsplit(int B, int L, int E, int N, int K, axon_dtype io,
                                     axon_discretization disc, int runs,
                                     const void* x, const void* z, const void* dt_raw,
                                     const void* Bm, const void* Cm,
                                     const float* conv_w, const float* conv_b,
                                     const float* dt_bias, const float* A_log, const float* D,
                                     const void* conv_cache_in, const float* ssm_state_in,
                                     void* y, void* conv_cache_out, float* ssm_state_out,
                                     axon_stream_t stream) {
    if (disc != AXON_DISC_FIRST_ORDER && disc != AXON_DISC_ZOH) return AXON_ERR_UNSUPPORTED;
    if (runs == 0) return AXON_ERR_INVALID_ARG;
    return scan_impl(B, L, E, N, K, io, x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
                     conv_cache_in, ssm_state_in, y, conv_cache_out, ssm_state_out,
                     nullptr, 0, 1, reinterpret_cast<cudaStream_t>(stream), disc == AXON_DISC_ZOH, runs);
}

axon_status axon_ssm_scan_fwd_noalloc(int B, int L, int E, int N, int K, axon_dtype io,
                                      const void* x, const void* z, const void* dt_raw,
                                      const void* Bm, const void* Cm,
                                      const float* conv_w, const float* conv_b,
                                      const float* dt_bias, const float* A_log, const float* D,
                                      const void* conv_cache_in, const float* ssm_state_in,
                                      void* y, void* conv_cache_out, float* ssm_state_out,
                                      int num_segments, axon_stream_t stream) {
    // Size checks first, on the host: nothing touches the device on rejection.
    const axon_status shape = check_shape(B, L, E, N, K, io);
    if (shape != AXON_OK) return shape;
    if (num_segments < 0 || num_segments > kMaxSegments) return AXON_ERR_INVALID_ARG;
    // Worst-case scratch of any plan for this call: the caller's forced split,
    // or the library's largest split for a sequence of L tokens.
    const int worst = num_segments > 0 ? num_segments : max_segments_for(L);
    if (ws_bytes_for(B, E, worst) > kStaticScratchBytes) return AXON_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    if (B > 0 && E > 0 && L > 0) {
        const axon_status st = static_scratch_address(&scratch);
        if (st != AXON_OK) return st;
    }
    // Every scratch word the split reads is written earlier in the same call
    // (segment end states and dt sums by the first phase), so stale contents
    // left by a previous call need no clearing.
    return scan_impl(B, L, E, N, K, io, x, z, dt_raw, Bm, Cm, conv_w, conv_b, dt_bias, A_log, D,
                     conv_cache_in, ssm_state_in, y, conv_cache_out, ssm_state_out,
                     scratch, scratch ? kStaticScratchBytes : 0, num_segments,
                     reinterpret_cast<cudaStream_t>(stream));
}

axon_status axon_ssm_dt_sum(int B, int L, int E, axon_dtype io, const void* dt_raw,
                            const float* dt_bias, float* dt_sum, axon_stream_t stream) {
    if (B < 0 || L < 0 || E < 0) return AXON_ERR_INVALID_ARG;
    if (io != AXON_F32 && io != AXON_BF16) return AXON_ERR_UNSUPPORTED;
    if (B > 65535 || (long long)B * E > (1LL << 31)) return AXON_ERR_UNSUPPORTED;
    if (B == 0 || E == 0) return AXON_OK;
    if (!dt_bias || !dt_sum || (L > 0 && !dt_raw)) return AXON_ERR_INVALID_ARG;
    if ((dt_raw && !aligned16(dt_raw)) || !aligned16(dt_bias) || !aligned16(dt_sum)) return AXON_ERR_ALIGNMENT;
    if (L > 0 && overlaps(dt_raw, (size_t)B * L * E * io_bytes(io), dt_sum, (size_t)B * E * 4))
        return AXON_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(dt_sum, 0, (size_t)B * E * sizeof(float), st) != cudaSuccess) return AXON_ERR_CUDA;
    if (L == 0) return AXON_OK;
    const dim3 grid((unsigned)((E + kDtSumThreads - 1) / kDtSumThreads),
                    (unsigned)((L + kDtSumRun - 1) / kDtSumRun), (unsigned)B);
    if (grid.y > 65535u) return AXON_ERR_UNSUPPORTED;
    if (io == AXON_BF16) dt_sum_kernel<IoBF16><<<grid, kDtSumThreads, 0, st>>>(L, E, dt_raw, dt_bias, dt_sum);
    else dt_sum_kernel<IoF32><<<grid, kDtSumThreads, 0, st>>>(L, E, dt_raw, dt_bias, dt_sum);
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

axon_status axon_ssm_carry_fold(int P, int r, int B, int E, int N, const float* A_log,
                                const float* h_loc, const float* dt_sum, float* h_in,
                                axon_stream_t stream) {
    if (P < 1 || r < 1 || r >= P || B < 0 || E < 0) return AXON_ERR_INVALID_ARG;
    if (N != kN) return AXON_ERR_UNSUPPORTED;
    if ((long long)B * E > (1LL << 31) / kN) return AXON_ERR_UNSUPPORTED;
    if (B == 0 || E == 0) return AXON_OK;
    if (!A_log || !h_loc || !dt_sum || !h_in) return AXON_ERR_INVALID_ARG;
    if (!aligned16(A_log) || !aligned16(h_loc) || !aligned16(dt_sum) || !aligned16(h_in))
        return AXON_ERR_ALIGNMENT;
    const size_t state = (size_t)B * E * kN * 4;
    if (overlaps(h_in, state, h_loc, (size_t)P * state) || overlaps(h_in, state, dt_sum, (size_t)P * B * E * 4))
        return AXON_ERR_INVALID_ARG;
    const size_t total = (size_t)B * E * kN;
    carry_fold_kernel<<<(unsigned)((total + 127) / 128), 128, 0, static_cast<cudaStream_t>(stream)>>>(
        r, B, E, A_log, h_loc, dt_sum, h_in);
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

axon_status axon_exp2_fma(const float* x, float* y, long long n, axon_stream_t stream) {
    if (n < 0) return AXON_ERR_INVALID_ARG;
    if (n == 0) return AXON_OK;
    if (!x || !y) return AXON_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(y)) return AXON_ERR_ALIGNMENT;
    if (overlaps(x, (size_t)n * 4, y, (size_t)n * 4) && x != y) return AXON_ERR_INVALID_ARG;
    const long long threads = (n + 1) / 2;
    if ((threads + 255) / 256 > 0x7fffffffLL) return AXON_ERR_UNSUPPORTED;
    exp2_fma_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

axon_status axon_ssm_scan_state(int B, int L, int E, int N, int K, axon_dtype io,
                                const void* x, const void* dt_raw, const void* Bm,
                                const float* conv_w, const float* conv_b,
                                const float* dt_bias, const float* A_log,
                                const void* conv_cache_in, const float* ssm_state_in,
                                void* conv_cache_out, float* ssm_state_out, float* dt_sum,
                                axon_stream_t stream) {
    axon_status st = check_shape(B, L, E, N, K, io);
    if (st != AXON_OK) return st;
    if (B == 0 || E == 0) return AXON_OK;
    if (!conv_w || !conv_b || !dt_bias || !A_log || !conv_cache_out || !ssm_state_out || !dt_sum)
        return AXON_ERR_INVALID_ARG;
    if (L > 0 && (!x || !dt_raw || !Bm)) return AXON_ERR_INVALID_ARG;
    const void* ptrs[] = {x, dt_raw, Bm, conv_w, conv_b, dt_bias, A_log, conv_cache_in, ssm_state_in,
                          conv_cache_out, ssm_state_out, dt_sum};
    for (const void* q : ptrs)
        if (q && !aligned16(q)) return AXON_ERR_ALIGNMENT;
    const size_t sio = io_bytes(io);
    const size_t n_in = (size_t)B * L * E * sio, n_b = (size_t)B * L * kN * sio;
    const size_t n_cc = (size_t)B * (kK - 1) * E * sio, n_ss = (size_t)B * E * kN * sizeof(float);
    const size_t n_dt = (size_t)B * E * sizeof(float);
    // outputs: disjoint from each other and from every input, except each cache
    // may be updated in place (conv_cache_out == conv_cache_in, state likewise)
    const void* outs[] = {conv_cache_out, ssm_state_out, dt_sum};
    const size_t nouts[] = {n_cc, n_ss, n_dt};
    for (int i = 0; i < 3; ++i) {
        for (int j = i + 1; j < 3; ++j)
            if (overlaps(outs[i], nouts[i], outs[j], nouts[j])) return AXON_ERR_INVALID_ARG;
        if (overlaps(outs[i], nouts[i], x, n_in) || overlaps(outs[i], nouts[i], dt_raw, n_in) ||
            overlaps(outs[i], nouts[i], Bm, n_b))
            return AXON_ERR_INVALID_ARG;
    }
    if (conv_cache_in != conv_cache_out && overlaps(conv_cache_in, n_cc, conv_cache_out, n_cc))
        return AXON_ERR_INVALID_ARG;
    if (ssm_state_in != ssm_state_out && overlaps(ssm_state_in, n_ss, ssm_state_out, n_ss))
        return AXON_ERR_INVALID_ARG;
    if (overlaps(conv_cache_in, n_cc, ssm_state_out, n_ss) || overlaps(conv_cache_in, n_cc, dt_sum, n_dt) ||
        overlaps(ssm_state_in, n_ss, conv_cache_out, n_cc) || overlaps(ssm_state_in, n_ss, dt_sum, n_dt))
        return AXON_ERR_INVALID_ARG;
    const int sms = device_sm_count();
    if (sms <= 0) return AXON_ERR_CUDA;
    // the prefill's split-chunk plan, or (where the prefill prefers another
    // kernel) eight runs per chunk for few channels and one run for many
    int W = plan_qsplit(B, L, E, (int)sio, sms);
    if (W == 0) W = (long long)B * E < (long long)sms * 48 ? 8 : 1;
    if (!qsplit_fits(B, L, E, (int)sio, W)) return AXON_ERR_UNSUPPORTED;
    ChunkParams cp{};
    cp.B = B; cp.L = L; cp.E = E;
    cp.x = x; cp.z = nullptr; cp.dt_raw = dt_raw; cp.Bm = Bm; cp.Cm = nullptr;
    cp.conv_w = conv_w; cp.conv_b = conv_b; cp.dt_bias = dt_bias; cp.A_log = A_log; cp.D = nullptr;
    cp.conv_cache_in = conv_cache_in; cp.ssm_state_in = ssm_state_in;
    cp.y = nullptr; cp.conv_cache_out = conv_cache_out; cp.ssm_state_out = ssm_state_out;
    cp.dt_sum = dt_sum;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return io == AXON_BF16 ? launch_qsplit<IoBF16, false, true>(cp, W, s) : launch_qsplit<IoF32, false, true>(cp, W, s);
}

axon_status axon_peak_probe(int kind, float* out, int blocks, long long iters, axon_stream_t stream) {
    if (kind != 0 && kind != 1) return AXON_ERR_UNSUPPORTED;
    if (blocks <= 0 || iters < 0 || !out) return AXON_ERR_INVALID_ARG;
    if (!aligned16(out)) return AXON_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (kind == 0) peak_probe_kernel<0><<<(unsigned)blocks, 256, 0, st>>>(out, iters);
    else peak_probe_kernel<1><<<(unsigned)blocks, 256, 0, st>>>(out, iters);
    return cudaGetLastError() == cudaSuccess ? AXON_OK : AXON_ERR_CUDA;
}

}  // extern "C"
