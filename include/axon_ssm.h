/*
 * axon_ssm.h -- C ABI of the B200 (sm_100a) selective-scan (S6) layer core.
 *
 * The operation is the Axon-SSM layer core of the page "Axon-SSM: Selective
 * State Space Model for Apple Silicon" (bit-axon docs), between its input and
 * output projections (axon_ssm_block_fwd, at the end of this file, adds the
 * projections around it):
 *
 *   xc_t  = conv_b + sum_{k<K} conv_w[k] * xpad[t+k]     causal depthwise conv1d,
 *           xpad = conv_cache ++ x, tap K-1 meets x_t    (section "Implementation
 *                                                         in Bit-Axon", code map
 *                                                         `_causal_conv1d`)
 *   u_t   = SiLU(xc_t)
 *   dt_t  = clip(softplus(dt_raw_t + dt_bias), 1e-4, 100) (section "Selective
 *                                                         mechanism")
 *   A     = -exp(A_log), diagonal                         (section "Diagonal state
 *                                                         matrix")
 *   h_t   = exp(dt_t*A) (.) h_{t-1} + dt_t*B_t*u_t        (section "ZOH
 *                                                         discretisation": the
 *                                                         first-order form used by
 *                                                         Axon-SSM, and the
 *                                                         recurrence equation)
 *   y_t   = (C_t . h_t + D*u_t) * SiLU(z_t)               (recurrence output and
 *                                                         section "Gating")
 *
 * and the cached decode of section "Autoregressive decoding": the cache pair
 * [conv_cache (B,K-1,E), ssm_state (B,E,N)] carries the conv padding and the
 * hidden state from one call to the next.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Sizes: B batch rows, L tokens, E channels (d_inner), N states, K conv taps.
 *    This build supports N == 16 and K == 4 only (the layer configuration table
 *    of the Axon-SSM page); other values return AXON_ERR_UNSUPPORTED.
 *  - Layouts are dense row-major, last index fastest:
 *      x, z, dt_raw, y        (B, L, E)   io dtype
 *      Bm, Cm                 (B, L, N)   io dtype, shared by all channels
 *      conv_w                 (E, K)      float32
 *      conv_b, dt_bias, D     (E)         float32
 *      A_log                  (E, N)      float32
 *      conv_cache             (B, K-1, E) io dtype; index 0 is the oldest input
 *      ssm_state              (B, E, N)   float32
 *    For axon_ssm_step the L axis is absent: x, z, dt_raw, y are (B, E) and
 *    Bm, Cm are (B, N).
 *  - io dtype: AXON_F32 (float) or AXON_BF16 (bfloat16 bits, round-to-nearest-
 *    even on output).  Arithmetic is float32 throughout; the state is float32.
 *  - Pointers are DEVICE pointers owned by the caller.  The library never
 *    allocates, frees or retains them; scratch memory comes from the caller
 *    through `workspace` (axon_ssm_block_fwd's cuBLASLt handle is the one
 *    library-owned object).  Every pointer must be 16-byte aligned, and E must be
 *    a multiple of 8 (bf16) or 4 (f32), else AXON_ERR_ALIGNMENT.  There is no
 *    fallback path.
 *  - Work is enqueued on `stream` and runs asynchronously.  Arguments are
 *    checked on the host before anything is enqueued: an error return means
 *    nothing was launched and no output was touched.  AXON_ERR_CUDA reports a
 *    failed launch; faults that occur later surface at the caller's next
 *    synchronisation, as for any CUDA kernel.
 *  - Global state: per-device caches of read-only facts (SM count, shared-
 *    memory limit, each kernel's raised shared-memory limit) and, for
 *    axon_ssm_block_fwd, one cuBLASLt handle per device, all set up once under
 *    a lock or with atomics; and the scratch array of
 *    axon_ssm_scan_fwd_noalloc (below).  Otherwise concurrent calls on
 *    different streams with disjoint outputs are safe.
 *  - `axon_stream_t` is the CUDA runtime's cudaStream_t (a CUstream_st
 *    pointer); NULL means the legacy default stream.
 */
#ifndef AXON_SSM_H
#define AXON_SSM_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define AXON_API __attribute__((visibility("default")))
#else
#define AXON_API
#endif

struct CUstream_st;
typedef struct CUstream_st *axon_stream_t;

typedef enum {
    AXON_F32 = 0,
    AXON_BF16 = 1
} axon_dtype;

/* Discretisation of B (Axon-SSM page, section "ZOH discretisation"). */
typedef enum {
    AXON_DISC_FIRST_ORDER = 0,  /* Bbar = dt * B: the form Axon-SSM uses (default) */
    AXON_DISC_ZOH = 1           /* Bbar = (exp(dt*A) - 1) / A * B: exact zero-order hold */
} axon_discretization;

typedef enum {
    AXON_OK = 0,
    AXON_ERR_INVALID_ARG = 1,   /* negative size, NULL required pointer, bad aliasing */
    AXON_ERR_UNSUPPORTED = 2,   /* N != 16, K != 4, unknown dtype, size beyond limits */
    AXON_ERR_ALIGNMENT = 3,     /* pointer not 16-byte aligned, E not a multiple of 8/4 */
    AXON_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
    AXON_ERR_CUDA = 5,          /* a kernel launch (or device query) failed */
    AXON_ERR_TIMEOUT = 6        /* reserved: no entry point waits on the device */
} axon_status;

/* Version of this ABI (bumped on any incompatible change). */
AXON_API int axon_ssm_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
AXON_API const char *axon_status_string(axon_status status);

/*
 * Bytes of device scratch memory `axon_ssm_scan_fwd` may need for a problem of
 * this size: an upper bound over every launch plan the library can choose for
 * it, independent of the device.  Returns 0 when no plan needs scratch, and 0
 * for arguments axon_ssm_scan_fwd would reject.
 *
 * The scratch holds, per sequence segment after the first and per (b, e)
 * channel, the segment's local end state (N floats) and its summed dt (one
 * float): the chunk-carry summaries of a time-split scan (the chunked
 * associative scan of the SSD article, intra-block pass plus inter-block
 * carry).
 */
AXON_API size_t axon_ssm_scan_workspace_bytes(int B, int L, int E, int N, int K, axon_dtype io);

/*
 * Number of kernel launches axon_ssm_scan_fwd enqueues for a problem of this
 * size on the current device (its launch plan), or -1 for arguments it would
 * reject or when the device cannot be queried.  Lets a caller count the work
 * it put on a stream; it launches nothing.
 */
AXON_API int axon_ssm_scan_launch_count(int B, int L, int E, int N, int K, axon_dtype io);

/*
 * Prefill: run the layer core over L tokens of B sequences.
 *
 *   x, z, dt_raw        (B,L,E) io   inputs (post-projection x branch, gate branch,
 *                                    raw step size); required when L > 0
 *   Bm, Cm              (B,L,N) io   input-dependent B_t and C_t; required when L > 0
 *   conv_w, conv_b, dt_bias, A_log, D  float32 parameters; required
 *   conv_cache_in       (B,K-1,E) io or NULL (NULL: zero padding)
 *   ssm_state_in        (B,E,N) f32  or NULL (NULL: zero initial state)
 *   y                   (B,L,E) io   output; required when L > 0; must not
 *                                    overlap any input
 *   conv_cache_out      (B,K-1,E) io the last K-1 entries of conv_cache_in ++ x
 *                                    (raw inputs, bit-exact copies); required;
 *                                    either the same pointer as conv_cache_in
 *                                    (updated in place) or disjoint from it
 *   ssm_state_out       (B,E,N) f32  h after the last token; required; same
 *                                    pointer as ssm_state_in or disjoint
 *   workspace, workspace_bytes       caller-owned device scratch of at least
 *                                    axon_ssm_scan_workspace_bytes(...) bytes;
 *                                    may be NULL when that query returns 0
 *   stream                           stream to enqueue on
 *
 * L == 0 copies the initial caches (or zeros) to the outputs.  B == 0 or
 * E == 0 is a no-op.  Passing the returned caches to the next call continues
 * the sequence exactly (the streaming `model.step(chunk, state)` pattern of
 * the wiki page "Selective State Space Models (Mamba)").
 */
AXON_API axon_status axon_ssm_scan_fwd(
    int B, int L, int E, int N, int K, axon_dtype io,
    const void *x, const void *z, const void *dt_raw,
    const void *Bm, const void *Cm,
    const float *conv_w, const float *conv_b,
    const float *dt_bias, const float *A_log, const float *D,
    const void *conv_cache_in, const float *ssm_state_in,
    void *y, void *conv_cache_out, float *ssm_state_out,
    void *workspace, size_t workspace_bytes, axon_stream_t stream);

/*
 * The prefill with an explicit time split: `num_segments` >= 2 forces the
 * sequence to be cut into that many segments processed in parallel, with the
 * chunk carry passed through `workspace` (which must then hold at least
 * (num_segments-1) * B * E * (N+1) floats; num_segments <= 64 and every
 * segment at least K tokens long, else AXON_ERR_INVALID_ARG).
 * num_segments == 1 runs the sequence unsplit (one kernel walks every
 * channel's whole sequence, no workspace); num_segments == 0 lets the
 * library choose, exactly as
 * axon_ssm_scan_fwd does.  Same arguments and errors as axon_ssm_scan_fwd
 * otherwise.  Intended for tests and tuning; results agree with the library's
 * own plan to float32 rounding.
 */
AXON_API axon_status axon_ssm_scan_fwd_segments(
    int B, int L, int E, int N, int K, axon_dtype io,
    const void *x, const void *z, const void *dt_raw,
    const void *Bm, const void *Cm,
    const float *conv_w, const float *conv_b,
    const float *dt_bias, const float *A_log, const float *D,
    const void *conv_cache_in, const float *ssm_state_in,
    void *y, void *conv_cache_out, float *ssm_state_out,
    void *workspace, size_t workspace_bytes, int num_segments, axon_stream_t stream);

/*
 * The prefill with one kernel forced, for tests and tuning: the split-chunk
 * quadrant scan (a block of `runs` warps per 8 channels; each chunk of the
 * sequence is cut into `runs` runs of consecutive tokens, one per warp, whose
 * aggregates (decay product, local end state) are folded into every run's
 * entering state -- the chunked associative scan of the SSD article applied
 * to the diagonal recurrence of the Axon-SSM page).  runs is 1, 2, 4 or 8
 * (one run per chunk: 32-token runs; several: 16-token runs; else
 * AXON_ERR_INVALID_ARG); shapes whose staging does not fit return
 * AXON_ERR_UNSUPPORTED.  `disc` as for axon_ssm_scan_fwd_ex.  No workspace.
 * Other arguments, layouts and errors are those of axon_ssm_scan_fwd; results
 * agree with the library's own plan to float32 rounding.
 */
AXON_API axon_status axon_ssm_scan_fwd_qsplit(
    int B, int L, int E, int N, int K, axon_dtype io, axon_discretization disc, int runs,
    const void *x, const void *z, const void *dt_raw,
    const void *Bm, const void *Cm,
    const float *conv_w, const float *conv_b,
    const float *dt_bias, const float *A_log, const float *D,
    const void *conv_cache_in, const float *ssm_state_in,
    void *y, void *conv_cache_out, float *ssm_state_out, axon_stream_t stream);

/*
 * The prefill (axon_ssm_scan_fwd_segments semantics) for callers that cannot
 * provide scratch memory.  The pages have no counterpart; this is a
 * convenience of the library.
 *
 * Who needs it: a serving process whose memory pool reserved nearly all of
 * HBM up front has no room for a cudaMalloc of its own, and a host program
 * that must not call cudaMalloc/cudaFree inside its token loop (those calls
 * can synchronise the device) has no workspace to hand over.  Both still own
 * and pass every input and output buffer; only the time-split scratch moves
 * into the library.
 *
 *  - The scratch is one library-owned 16 MiB device array
 *    (AXON_NOALLOC_SCRATCH_BYTES).  Every GPU that loads the library holds it
 *    until the process exits.  The entry point itself calls no cudaMalloc,
 *    cudaFree or other allocating routine.
 *  - Limit: a call is rejected with AXON_ERR_UNSUPPORTED, before anything is
 *    launched, when its worst-case scratch exceeds that size, i.e. when
 *    (P - 1) * B * E * (N + 1) * 4 bytes > 16 MiB, with P = num_segments if it
 *    is > 0, else min(64, max(1, L / 128)) (the largest split the library plans
 *    for L tokens; axon_ssm_scan_workspace_bytes gives the same bound).
 *  - num_segments as for axon_ssm_scan_fwd_segments (0 = library's plan).
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current); make that first call before any
 *    stream capture on that device.
 *  - All calls share the one array and it keeps the last call's contents;
 *    every scratch word a call reads was written earlier in the same call, so
 *    nothing needs clearing.  Calls whose executions overlap on the GPU (on
 *    different streams, or from different threads) race on the array: order
 *    them, e.g. keep them on one stream.
 * Other arguments, layouts and errors are those of axon_ssm_scan_fwd.
 */
#define AXON_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
AXON_API axon_status axon_ssm_scan_fwd_noalloc(
    int B, int L, int E, int N, int K, axon_dtype io,
    const void *x, const void *z, const void *dt_raw,
    const void *Bm, const void *Cm,
    const float *conv_w, const float *conv_b,
    const float *dt_bias, const float *A_log, const float *D,
    const void *conv_cache_in, const float *ssm_state_in,
    void *y, void *conv_cache_out, float *ssm_state_out,
    int num_segments, axon_stream_t stream);

/*
 * axon_ssm_scan_fwd_segments with a choice of discretisation: `disc` selects
 * the first-order Bbar = dt*B (AXON_DISC_FIRST_ORDER, what every other entry
 * point uses) or the exact zero-order hold Bbar = (exp(dt*A) - 1)/A * B
 * (AXON_DISC_ZOH) of the Axon-SSM page's "ZOH discretisation" section.  The
 * decay exp(dt*A) is the same in both.  An unknown `disc` returns
 * AXON_ERR_UNSUPPORTED; all other arguments and errors are those of
 * axon_ssm_scan_fwd_segments (num_segments == 0: the library's plan).
 */
AXON_API axon_status axon_ssm_scan_fwd_ex(
    int B, int L, int E, int N, int K, axon_dtype io, axon_discretization disc,
    const void *x, const void *z, const void *dt_raw,
    const void *Bm, const void *Cm,
    const float *conv_w, const float *conv_b,
    const float *dt_bias, const float *A_log, const float *D,
    const void *conv_cache_in, const float *ssm_state_in,
    void *y, void *conv_cache_out, float *ssm_state_out,
    void *workspace, size_t workspace_bytes, int num_segments, axon_stream_t stream);

/*
 * Cached single-token decode (section "Autoregressive decoding"): one step of
 * the layer core for B sequences, caches updated in place.
 *
 *   x, z, dt_raw        (B,E) io     this token's inputs
 *   Bm, Cm              (B,N) io     this token's B_t, C_t
 *   conv_w ... D                     float32 parameters, as for the prefill
 *   conv_cache          (B,K-1,E) io read, then shifted by one with x appended
 *   ssm_state           (B,E,N) f32  read-modify-written
 *   y                   (B,E) io     output; must not overlap the other buffers
 *
 * Equivalent to axon_ssm_scan_fwd with L == 1 and in-place caches; its cost
 * does not depend on how many tokens came before (O(1) state per token).
 */
AXON_API axon_status axon_ssm_step(
    int B, int E, int N, int K, axon_dtype io,
    const void *x, const void *z, const void *dt_raw,
    const void *Bm, const void *Cm,
    const float *conv_w, const float *conv_b,
    const float *dt_bias, const float *A_log, const float *D,
    void *conv_cache, float *ssm_state, void *y, axon_stream_t stream);

/*
 * axon_ssm_step with a choice of discretisation (see axon_ssm_scan_fwd_ex).
 * A decode that continues a prefill must use the same `disc` as the prefill.
 */
AXON_API axon_status axon_ssm_step_ex(
    int B, int E, int N, int K, axon_dtype io, axon_discretization disc,
    const void *x, const void *z, const void *dt_raw,
    const void *Bm, const void *Cm,
    const float *conv_w, const float *conv_b,
    const float *dt_bias, const float *A_log, const float *D,
    void *conv_cache, float *ssm_state, void *y, axon_stream_t stream);

/*
 * A sequence split by time across P devices (slice r = tokens [r*L/P, ...)),
 * with one exchange of per-slice summaries (the chunked associative scan of
 * the SSD article, devices as blocks; the recurrence's decay over a run of
 * tokens is exp(A * sum dt), Axon-SSM page, recurrence equation):
 *   1. every slice r >= 1 runs axon_ssm_scan_state from a ZERO state (its
 *      conv cache = the last K-1 inputs of slice r-1) for its end state
 *      h_loc_r and dt_sum_r in one pass (or axon_ssm_scan_fwd and
 *      axon_ssm_dt_sum); slice 0 runs axon_ssm_scan_fwd from the true
 *      initial state, its end state is h_loc_0 and its output is final;
 *   2. the P (h_loc, dt_sum) pairs are exchanged (one all-gather);
 *   3. axon_ssm_carry_fold gives slice r its entering state
 *      h = h_loc_0; h = exp(A * dt_sum_j) * h + h_loc_j for j = 1 .. r-1;
 *   4. slice r runs axon_ssm_scan_fwd again from that state: its y and end
 *      caches are final (the last slice's caches are the sequence's).
 *
 * axon_ssm_dt_sum: dt_sum (B,E) float32 = sum over t of clip(softplus(dt_raw
 * + dt_bias), 1e-4, 100) (section "Selective mechanism"); dt_raw (B,L,E) io.
 * dt_sum is zeroed on the stream first and accumulated with atomic adds, so
 * its last bits may vary from run to run.
 * axon_ssm_carry_fold: h_loc (P,B,E,N) and dt_sum (P,B,E) float32 as
 * gathered (index = slice), A_log (E,N); writes h_in (B,E,N) for slice r,
 * 1 <= r < P (AXON_ERR_INVALID_ARG otherwise).  Conventions as above; h_in
 * must not overlap the inputs.
 */
AXON_API axon_status axon_ssm_dt_sum(int B, int L, int E, axon_dtype io, const void *dt_raw,
                                     const float *dt_bias, float *dt_sum, axon_stream_t stream);

AXON_API axon_status axon_ssm_carry_fold(int P, int r, int B, int E, int N, const float *A_log,
                                         const float *h_loc, const float *dt_sum, float *h_in,
                                         axon_stream_t stream);

/*
 * The state-only prefill of step 1 above: the conv + SiLU, dt and recurrence
 * of axon_ssm_scan_fwd (first order) without the output side -- no z, C, D
 * or y -- writing only the final caches (conv_cache_out: the last K-1 raw
 * inputs; ssm_state_out: h_L) and dt_sum (B,E) float32 = the sum over t of the
 * same step sizes the recurrence used, added in a fixed order (the same bits
 * on every run).  Layouts, ownership and the NULL conventions of
 * conv_cache_in / ssm_state_in as in axon_ssm_scan_fwd; L == 0 copies the
 * caches and zeroes dt_sum.  Each cache may be updated in place
 * (conv_cache_out == conv_cache_in, ssm_state_out == ssm_state_in); the
 * outputs must not otherwise overlap each other or the inputs
 * (AXON_ERR_INVALID_ARG); every pointer 16-byte aligned (AXON_ERR_ALIGNMENT).
 * Enqueued on `stream`; needs no workspace.
 */
AXON_API axon_status axon_ssm_scan_state(int B, int L, int E, int N, int K, axon_dtype io,
                                         const void *x, const void *dt_raw, const void *Bm,
                                         const float *conv_w, const float *conv_b,
                                         const float *dt_bias, const float *A_log,
                                         const void *conv_cache_in, const float *ssm_state_in,
                                         void *conv_cache_out, float *ssm_state_out, float *dt_sum,
                                         axon_stream_t stream);

/*
 * The Mamba-2 (SSD) layer core: one scalar decay per head (wiki page
 * "Selective State Space Models (Mamba)", section "Mamba-2 block (SSD)":
 * d_state 128, headdim 64), computed as a chunked scan on the tensor cores
 * (the SSD article: masked matrix products inside chunks of tokens, a carried
 * state between them; this library's chunks are 128 tokens).  Per batch row b and head h, state S (P x N):
 *   dt = clip(softplus(dt_raw[b,t,h] + dt_bias[h]), 1e-4, 100),
 *   S  = exp(dt * A_h) S + dt * x[b,t,h,:] B[b,t,:]^T,  A_h = -exp(A_log[h]),
 *   y[b,t,h,:] = S C[b,t,:] + D[h] x[b,t,h,:].
 * Layouts: x, y (B,L,H,P) bf16; dt_raw (B,L,H) bf16; Bm, Cm (B,L,N) bf16,
 * shared by all heads; dt_bias, A_log, D (H) float32; h0 (B,H,P,N) float32 or
 * NULL (zeros); h_out (B,H,P,N) float32, may be h0 itself.  P == 64, N == 128
 * and io == AXON_BF16 only (else AXON_ERR_UNSUPPORTED).  The products run on
 * the tcgen05 tensor cores with bf16 operands (the decayed chunk Gram matrix
 * with D on its diagonal and the carried state, each split in two bf16 parts,
 * hi and the rounding residual lo; the dt-weighted x) and float32
 * accumulators; the carried state itself is float32.  To fill the GPU when B * H is small the sequence is cut into
 * `segments` runs of whole 128-token chunks (0: chosen for the current
 * device, about one walk per SM; capped at one per chunk and 64): a first
 * walk over pieces of every segment but the last gives their local end
 * states from a zero state, and the full walk of each segment starts from
 * the fold of those.  `workspace` (16-byte aligned; may be NULL when the size
 * is 0) holds axon_ssd_workspace_bytes(B, L, H, P, N, segments) bytes for the
 * same `segments` on the current device: an error flag (its first 4 bytes,
 * an int), the per-chunk decays and weights, and the pieces' local states.
 * The flag is cleared by each call and set to 1 if a wait of the walk for its
 * tensor-core products gave up (the outputs are then undefined); it is
 * written on the stream, so read it after the call completes (the Python
 * binding's ssd_scan reads it and raises).  A walk that gave up first waits,
 * with the same bound, for every product it issued to finish, and only then
 * frees its tensor memory; if that wait gives up as well, it leaves the
 * tensor memory allocated rather than risk a late product writing into
 * columns another block has since allocated.  Other
 * conventions as above.
 */
AXON_API size_t axon_ssd_workspace_bytes(int B, int L, int H, int P, int N, int segments);

/*
 * A check of the SSD walks' failure path, for tests: one warp polls, `limit`
 * times (1 .. 65536), an mbarrier that nothing arrives on, exactly as a walk
 * waits for its tensor-core products, and writes 1 to *status (a device int,
 * 4-byte aligned) when the wait gave up.  AXON_ERR_INVALID_ARG for a NULL or
 * misaligned status or a limit out of range.  Enqueued on `stream`.
 */
AXON_API axon_status axon_ssd_wait_probe(int *status, int limit, axon_stream_t stream);

AXON_API axon_status axon_ssd_scan_fwd(
    int B, int L, int H, int P, int N, axon_dtype io,
    const void *x, const void *dt_raw, const float *dt_bias, const float *A_log,
    const void *Bm, const void *Cm, const float *D, const float *h0,
    void *y, float *h_out, int segments, void *workspace, size_t workspace_bytes, axon_stream_t stream);

/*
 * The whole Axon-SSM layer around the layer core (Axon-SSM page, sections
 * "Gating" and "Selective mechanism"), bf16 io only:
 *
 *   (x, z)          = split(X W_in)       X (B,L,Dm); W_in (Dm, 2E): x = columns
 *                                         [0, E), z = columns [E, 2E)
 *   u               = SiLU(conv(x))       the conv output (conv_w, conv_b, cache)
 *   (dt_raw, B, C)  = split(u W_x)        f_proj, one linear map of the conv
 *                                         output; W_x (E, E+2N): dt_raw = columns
 *                                         [0, E), B = [E, E+N), C = [E+N, E+2N)
 *   y               = layer core          axon_ssm_scan_fwd on (x, z, dt_raw, B, C)
 *   out             = y W_out             W_out (E, Dm); out (B,L,Dm)
 *
 * Weights are row-major bf16 ("activations times weights").  The three
 * projections run on this library's tcgen05 GEMM (axon_gemm_bf16_plan's
 * automatic tiling with the workspace's stream-K scratch; float32
 * accumulation): one launch writes x and z, one writes dt_raw, B and C, one
 * the output.  The conv stage and the layer core run in this library's
 * kernels too.  The intermediates x, z, u, dt_raw, B, C and y are stored in
 * bf16 inside `workspace`, which must hold at least
 * axon_ssm_block_workspace_bytes(...) bytes (16-byte aligned; it also serves
 * as the scan's scratch and the GEMMs' stream-K scratch).  Its first 4 bytes (an int) are an error flag,
 * cleared by each call and set to 1 if a wait of a GEMM for its copies or
 * tensor-core products gave up (the outputs are then undefined); read it
 * after the call completes.  Caches and parameters as for
 * axon_ssm_scan_fwd (in == out allowed); conv_cache_out receives the last K-1
 * rows of x.  Dm and E must be multiples of 8 (AXON_ERR_ALIGNMENT); io other
 * than AXON_BF16, N != 16 or K != 4 return AXON_ERR_UNSUPPORTED; out and the
 * workspace must not overlap each other, X, the weights or the caches
 * (AXON_ERR_INVALID_ARG).  L == 0 copies the caches in -> out.
 */
AXON_API size_t axon_ssm_block_workspace_bytes(int B, int L, int Dm, int E, int N, int K, axon_dtype io);

AXON_API axon_status axon_ssm_block_fwd(
    int B, int L, int Dm, int E, int N, int K, axon_dtype io,
    const void *X, const void *W_in, const void *W_x, const void *W_out,
    const float *conv_w, const float *conv_b,
    const float *dt_bias, const float *A_log, const float *D,
    const void *conv_cache_in, const float *ssm_state_in,
    void *out, void *conv_cache_out, float *ssm_state_out,
    void *workspace, size_t workspace_bytes, axon_stream_t stream);

/*
 * The projection GEMM the whole layer uses, on its own (tests and timing):
 * C (M x N) = A (M x K) W (K x N), all row-major bf16 with row strides lda,
 * ldw, ldc (elements), float32 accumulation, written as bf16.  Runs on the
 * tcgen05 tensor cores (TMA-fed, accumulators in tensor memory): from 256
 * rows on CTA pairs, 256 x 256 tiles, whole tiles; below on single CTAs,
 * 128 x 256 or 128 x 192 tiles.  N, lda, ldw and ldc must be multiples of 8 and A, W, C 16-byte
 * aligned (AXON_ERR_ALIGNMENT); C must not overlap A or W; K == 0 with M, N
 * > 0 is AXON_ERR_INVALID_ARG.  `err` (a device int, or NULL) is set to 1 if
 * a wait of the kernel for its copies or products gave up (C is then
 * undefined); it is not cleared by the call.  Enqueued on `stream`.
 */
AXON_API axon_status axon_gemm_bf16(int M, int N, int K, const void *A, int lda, const void *W, int ldw,
                                    void *C, int ldc, int *err, axon_stream_t stream);

/*
 * axon_gemm_bf16 with its tiling chosen by the caller (tests and timing):
 *   AXON_GEMM_AUTO          what axon_gemm_bf16 picks (given the workspace);
 *   AXON_GEMM_SINGLE_256    one CTA per 128 x 256 output tile;
 *   AXON_GEMM_SINGLE_192    one CTA per 128 x 192 output tile;
 *   AXON_GEMM_PAIR          a cluster of two CTAs (two SMs) per 256 x 256
 *                           output tile, the tensor cores of both running one
 *                           product of 256 rows (each CTA stages half of the
 *                           W tile), whole tiles round-robin over the pairs;
 *   AXON_GEMM_PAIR_STREAMK  the same tiles with the tiles x K-blocks
 *                           iterations split evenly over the pairs
 *                           (stream-K): a tile split between pairs is
 *                           finished by the pair holding its first K blocks,
 *                           which adds the others' float32 partial sums
 *                           (kept in `workspace`) in a fixed order, so the
 *                           result does not depend on timing.
 * The pair plans return AXON_ERR_UNSUPPORTED if no two-CTA cluster fits on
 * the device.  `workspace` (device, 16-byte aligned, not overlapping A, W or
 * C) may be NULL except for AXON_GEMM_PAIR_STREAMK, which needs
 * axon_gemm_workspace_bytes() bytes (AXON_ERR_WORKSPACE otherwise); the
 * call clears its first bytes (flags) on `stream` before the product.  The
 * stream-K pairs wait (bounded) on one another's flags: the grid holds as
 * many pairs as fit on the device, so when other work occupies SMs at the
 * same time a wait may give up, and `err` is then set (C undefined).  Any
 * other plan is AXON_ERR_INVALID_ARG; the other arguments and errors are those
 * of axon_gemm_bf16.
 */
enum {
    AXON_GEMM_AUTO = 0,
    AXON_GEMM_SINGLE_256 = 1,
    AXON_GEMM_SINGLE_192 = 2,
    AXON_GEMM_PAIR = 3,
    AXON_GEMM_PAIR_STREAMK = 4
};
AXON_API size_t axon_gemm_workspace_bytes(void);
AXON_API axon_status axon_gemm_bf16_plan(int M, int N, int K, const void *A, int lda, const void *W, int ldw,
                                         void *C, int ldc, int *err, int plan, void *workspace,
                                         size_t workspace_bytes, axon_stream_t stream);

/*
 * The FMA-pipe exp2 on its own (tests): y[i] = 2^x[i] for x[i] <= 0, computed
 * with float32 fused multiply-adds instead of the MUFU unit -- Cody and
 * Waite's reduction 2^x = 2^n 2^f, n = round(x), f in [-1/2, 1/2], 2^f by a
 * degree-6 minimax polynomial with constant term 1 (relative error within
 * 1.3 * 2^-24; 2^0 is exactly 1), 2^n added to the exponent field; x below
 * -126 gives 2^-126.  Kernels whose MUFU pipe is their busiest can take part
 * of their decays exp(dt A) = 2^(dt A log2 e) this way (page "Axon-SSM:
 * Selective State Space Model for Apple Silicon", "ZOH discretisation").
 * x and y are n float32 device values, 16-byte aligned; y may be x itself,
 * not otherwise overlap it.  n < 0 or a NULL pointer with n > 0 is
 * AXON_ERR_INVALID_ARG.  Enqueued on `stream`.
 */
AXON_API axon_status axon_exp2_fma(const float *x, float *y, long long n, axon_stream_t stream);

/*
 * Throughput probes for the roofline's compute denominators, measured in the
 * same run as the kernels they rate (bench.py): `blocks` blocks of 256
 * threads, each thread running 8 independent chains for `iters` steps --
 * kind 0: y = 2^(y * c) on the MUFU unit (one exp2 per step), kind 1: y =
 * y * a + b (one float32 FMA per step).  Ops executed = blocks * 256 * 8 *
 * iters.  `out` (blocks * 256 float32 device values, 16-byte aligned)
 * receives one sum per thread so the work is kept.  Other kinds are
 * AXON_ERR_UNSUPPORTED, blocks <= 0, iters < 0 or out == NULL
 * AXON_ERR_INVALID_ARG.  Enqueued on `stream`.
 */
AXON_API axon_status axon_peak_probe(int kind, float *out, int blocks, long long iters, axon_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* AXON_SSM_H */
