/*
 * m3.h -- C ABI of the B200 (sm_100a) Mamba-3 SSM sequence-mixer forward.
 *
 * The method (per batch b, head h, token t; state H_t in R^{N x P}):
 *
 *   h_t = a_t h_{t-1} + (1 - lam_t) dt_t a_t B~_{t-1} x_{t-1}^T + lam_t dt_t B~_t x_t^T,
 *   a_t = exp(dt_t A_h),      y_t = h_t^T C~_t + D_h x_t,
 *
 * the three-term exponential-trapezoidal recurrence displayed in
 * "Знакомство с Mamba-3" (chernovdev.ru), section 1; with B~, C~ the inputs
 * rotated pair-wise by the cumulative data-dependent angle
 * phi_t[k] = sum_{s<=t} dt_s theta_s[k] (the complex-state "RoPE trick":
 * same page, section 2, and "La dualità: Mamba-2 e Mamba-3", section
 * "Mamba-3"); and MIMO rank R: x_t in R^{P x R}, B_t, C_t in R^{N x R}, the
 * write a sum of R outer products (same chapter, MIMO paragraph).
 *
 * Conventions fixed by this library where the pages are silent:
 *   - state pairs are interleaved: pair k = rows (2k, 2k+1); theta has N/2
 *     angle rates per token-head;
 *   - rotation sign: B and C are rotated by +phi (standard RoPE), i.e. the
 *     state transition on pair k is the complex eigenvalue
 *     exp(dt (A - i theta[k])) acting on z = h[2k] + i h[2k+1];
 *   - the state handed between calls is the plain-frame h_{T-1} together with
 *     the raw last inputs (b_prev = B_{T-1}, x_prev = x_{T-1}), so that the
 *     next call's t-1 trapezoid term is exact; a zero / absent initial state
 *     means h = 0, b_prev = 0, x_prev = 0;
 *   - B and C are per head; A and D are per head (fp32).
 *
 * Memory: every pointer is a DEVICE pointer owned by the caller (except the
 * sequence and state pointers of m3_scan_fwd_host, which are host memory);
 * the library never allocates memory on these paths.  Tensors are dense, row-major (last index
 * fastest), base addresses 16-byte aligned.  "io" tensors are fp32 or bf16
 * according to m3_dims.io; A, D and all state buffers are fp32.
 *
 *   x, y      [batch, seqlen, nheads, rank, headdim]   io
 *   B, C      [batch, seqlen, nheads, rank, dstate]    io
 *   dt, lam   [batch, seqlen, nheads]                  io
 *   theta     [batch, seqlen, nheads, dstate/2]        io
 *   A, D      [nheads]                                 fp32
 *             (A: [batch, seqlen, nheads] with M3_FLAG_A_PER_TOKEN)
 *   theta with M3_FLAG_THETA_PER_HEAD: [nheads, dstate/2]      io
 *   h         [batch, nheads, dstate, headdim]         fp32
 *   b_prev    [batch, nheads, rank, dstate]            fp32
 *   x_prev    [batch, nheads, rank, headdim]           fp32
 *
 * Execution: every call is asynchronous on the given CUDA stream (a
 * cudaStream_t passed as void*, NULL = legacy default stream) and never
 * synchronises the device.  m3_scan_fwd / m3_scan_fwd_algo (whole and split
 * sequences) and m3_step can be captured into a CUDA graph and replayed; the
 * arguments (pointers included) are fixed at capture.  Errors are returned as m3_status; the message of
 * the calling thread's last failure is available from m3_last_error().  No
 * C++ exception crosses this boundary and no kernel traps.
 */
#ifndef M3_H
#define M3_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define M3_API __attribute__((visibility("default")))
#else
#define M3_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum m3_status {
    M3_OK = 0,
    M3_ERR_INVALID_ARG = 1,  /* null/misaligned/overlapping pointer, bad size */
    M3_ERR_UNSUPPORTED = 2,  /* valid sizes outside what the kernels support   */
    M3_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed          */
    M3_ERR_TIMEOUT = 4,      /* a bounded device-side wait gave up            */
    M3_ERR_BOUNDS = 5        /* a device-side index check failed (bounds build) */
} m3_status;

typedef enum m3_dtype { M3_F32 = 0, M3_BF16 = 1 } m3_dtype;

typedef struct m3_dims {
    int64_t batch;    /* Bt >= 0                                   */
    int64_t seqlen;   /* T >= 0 (ignored by m3_step)               */
    int64_t nheads;   /* H >= 1                                    */
    int64_t headdim;  /* P >= 1                                    */
    int64_t dstate;   /* N >= 2, even                              */
    int64_t rank;     /* R >= 1 (MIMO rank; 1 = SISO)              */
    int32_t io;       /* m3_dtype of x, B, C, dt, lam, theta, y    */
    int32_t flags;    /* 0 or M3_FLAG_* bits                       */
} m3_dims;

/* A is data-dependent: one fp32 value per token-head, [batch, seqlen, nheads]
 * for m3_scan_fwd and [batch, nheads] for m3_step, instead of one per head.
 * Mamba-3 produces the transition scalar A_t from the input at every token
 * ("La dualità: Mamba-2 e Mamba-3", section "Mamba-3", paragraph on the
 * exponential-trapezoidal rule; Mamba-2 held it fixed per head); the decay
 * of token t is exp(dt_t A_t) and everything else is unchanged. */
#define M3_FLAG_A_PER_TOKEN 1

/* theta fixed per head: [nheads, dstate/2] (io dtype) for m3_scan_fwd and
 * m3_step alike, instead of one set of angle rates per token-head.  The
 * angle of pair k at token t is then dt_t theta[h][k] -- the time-constant
 * rotation of a complex-diagonal SSM, the form the complex-state equivalence
 * starts from ("La dualità: Mamba-2 e Mamba-3", section "Mamba-3", paragraph
 * on complex transitions).  It saves reading theta per token. */
#define M3_FLAG_THETA_PER_HEAD 2

typedef struct m3_state {
    float *h;       /* [batch, nheads, dstate, headdim] */
    float *b_prev;  /* [batch, nheads, rank, dstate]    */
    float *x_prev;  /* [batch, nheads, rank, headdim]   */
} m3_state;

/* BC-norm prologue (optional).  Mamba-3 normalises the B and C projections
 * with an RMS norm, as QKNorm does for queries and keys, and adds learnable
 * head-specific biases after the norm ("Знакомство с Mamba-3", section
 * "Архитектура и нормализация"; "Mamba-3, parte 1", paragraphs on the
 * normalisations and on dropping the short convolution).  With it, every
 * (token, head, rank) row of B -- and of C -- over its dstate entries becomes
 *     B^ = B / sqrt(mean_n B^2 + eps) * wB + bB[head][rank]
 * before anything else uses it (the rotation included), and the state's
 * b_prev holds the last token's B^.  All device pointers, fp32, caller-owned:
 *     wB, wC  [dstate]                      (shared by heads and ranks)
 *     bB, bC  [nheads, rank, dstate]        (head-specific biases)
 * eps > 0.  The pages give the norm and the biases, not their shapes or eps;
 * these are this library's reading. */
typedef struct m3_bcnorm {
    const float *wB, *wC;
    const float *bB, *bC;
    float eps;
} m3_bcnorm;

/* Prefill kernel selection for m3_scan_fwd_algo. */
typedef enum m3_algo {
    M3_ALGO_AUTO = 0,   /* tensor-core path where supported, else SIMT            */
    M3_ALGO_SIMT = 1,   /* fp32 CUDA-core chunked scan (any supported size)      */
    M3_ALGO_TC = 2      /* tcgen05/TMEM chunked scan: bf16 I/O (headdim 64,
                         * dstate 64 or 128, rank 1, 2 or 4), or fp32 I/O
                         * (headdim 64, dstate 64, rank 1, 2 or 4, no forced
                         * segments)                                           */
} m3_algo;

/* The tensor-core path forced to split every sequence into s >= 1 segments
 * (fewer if the sequence has fewer chunks); M3_ALGO_TC and M3_ALGO_AUTO
 * choose the number themselves.  A split sequence runs as two launches, so
 * that a few long sequences still fill every SM: a summary pass (each
 * segment's local end state from a zero state and its transition
 * exp(sum dt A) Rot(-sum dt theta), published with a release flag) and the
 * full pass of every segment, launched as a programmatic dependent of the
 * summary pass (its CTAs take SMs as summary CTAs finish), in which the CTA
 * of segment j first scans the published summaries of segments 0 .. j-1
 * into its initial state -- the chunk-state recurrence of "La dualità:
 * Mamba-2 e Mamba-3", section "Perché conviene: i tensor core", applied one
 * level up -- waiting (bounded, error 0x8 on expiry) for any not yet
 * published. */
#define M3_ALGO_TC_SEGMENTS(s) (M3_ALGO_TC | ((int)(s) << 8))

/* MIMO projections, as read from "Mamba-3, parte 1" (architecture paragraph:
 * the projections widen B and C to the shape the MIMO SSM needs; TileLang
 * paragraph: the extra projections let the MIMO prefill save I/O through the
 * memory hierarchy) and "Знакомство с Mamba-3", section 3 (rank-R input and
 * output projections, B_t in R^{N x R}, x_t in R^{P x R}); the pages give no
 * shapes, so this is the plainest form: per head h and rank r, elementwise
 * fp32 weights widen the token-head's one row of x [P], B [N], C [N] to rank
 * R -- X[.., r, p] = wx[h, r, p] x[p], likewise B with wB and C with wC --
 * the rank-R scan runs on them, and the output row is y[p] = sum_r
 * wy[h, r, p] Y[.., r, p] (Y including its D x term).  Layouts: wx, wy
 * [H, R, P], wB, wC [H, R, N], fp32, 4-byte aligned, owned by the caller.
 * The kernels widen on chip, so x, B, C and y cross HBM at one row per
 * token-head. */
typedef struct m3_mimo_proj {
    const float *wx, *wB, *wC, *wy;
} m3_mimo_proj;

/* m3_scan_fwd_algo with the MIMO projections: x [B,T,H,P], B and C
 * [B,T,H,N], y [B,T,H,P] (one row per token-head; dt, lam, theta, A, D as
 * usual); d->rank is the rank R the projections widen to; the states (init,
 * final_state) keep the rank-R layout, their pending term widened.  bf16
 * I/O on the tensor-core prefill only (headdim 64, dstate 64 or 128, rank 1,
 * 2 or 4; split sequences and the per-token A and per-head theta layouts
 * included), M3_ERR_UNSUPPORTED otherwise and with algo M3_ALGO_SIMT; not
 * combined with the BC-norm prologue.  The workspace is the same as for
 * m3_scan_fwd_algo with these dims. */
M3_API m3_status m3_scan_fwd_proj(int algo, const m3_dims *d, const m3_mimo_proj *proj, const void *x,
                                  const void *B, const void *C, const void *dt, const void *lam,
                                  const void *theta, const float *A, const float *D, const m3_state *init,
                                  void *y, const m3_state *final_state, void *workspace,
                                  size_t workspace_bytes, void *stream);

/* m3_step with the MIMO projections: x [B,H,P], B and C [B,H,N], y [B,H,P];
 * the state in the rank-R layout, updated in place (b_prev, x_prev widened).
 * The register-tiled and streaming decode sizes only ((dstate, headdim) in
 * {64, 128} x {64, 128} or (256, 64); rank 1, 2 or 4): M3_ERR_UNSUPPORTED
 * otherwise. */
M3_API m3_status m3_step_proj(const m3_dims *d, const m3_mimo_proj *proj, const void *x, const void *B,
                              const void *C, const void *dt, const void *lam, const void *theta,
                              const float *A, const float *D, const m3_state *state, void *y, void *stream);

/* Bytes of device workspace m3_scan_fwd needs for these dims (0 = none; the
 * workspace pointer may then be NULL).  Host function; the answer depends on
 * the current CUDA device's SM count (it sets how sequences are split).  The
 * workspace (16-byte aligned) holds fp32 per-segment states of split
 * sequences, [segments][batch*nheads][dstate][headdim + 1], and one 32-bit
 * flag per segment and sequence (zeroed by the call itself, on its stream);
 * it needs no initialisation, its contents are meaningless after the call,
 * and calls that may run at the same time (other streams) must not share
 * one. */
M3_API m3_status m3_scan_workspace_size(const m3_dims *d, size_t *bytes);

/* How m3_scan_fwd_algo(algo, d, ...) will run on the current device:
 * workspace bytes, segments per sequence (1 = not split) and the number of
 * kernel launches of one call.  Any output pointer may be NULL.
 * M3_ERR_UNSUPPORTED if `algo` names the tensor-core path for sizes it does
 * not cover.  (m3_scan_plan_info also names the kernel, and tells how
 * m3_scan_fwd_static runs.) */
M3_API m3_status m3_scan_plan(int algo, const m3_dims *d, size_t *workspace_bytes, int *segments,
                              int *launches);

/* The prefill kernel a call runs. */
typedef enum m3_kernel {
    M3_KERNEL_NONE = 0,  /* nothing to run (batch = 0)                    */
    M3_KERNEL_SIMT = 1,  /* the fp32 CUDA-core chunked scan               */
    M3_KERNEL_TC = 2,    /* the tcgen05/TMEM/TMA chunked scan (bf16 I/O)  */
    M3_KERNEL_TC32 = 3   /* the tcgen05/TMEM chunked scan for fp32 I/O:
                          * every product operand split into bf16 high and
                          * low halves, three MMAs per product (about 2^-16
                          * relative error), one CTA per sequence and head,
                          * no workspace                                    */
} m3_kernel;

typedef struct m3_plan_info {
    size_t workspace_bytes;  /* device workspace the call needs (0: none)          */
    int32_t kernel;          /* m3_kernel that runs                                 */
    int32_t segments;        /* segments per sequence (1 = not split)               */
    int32_t launches;        /* kernel launches of one call                         */
    int32_t reserved;        /* 0                                                   */
    int64_t ctas;            /* CTAs of the (main) launch                           */
} m3_plan_info;

/* Flag of m3_scan_plan_info: describe the call as m3_scan_fwd_static runs it
 * (the library's 24 MiB scratch bounds its choice of segments, so it may
 * differ from m3_scan_fwd's). */
#define M3_PLAN_STATIC 1

/* Which kernel and schedule m3_scan_fwd_algo(algo, d, ...) -- or, with
 * M3_PLAN_STATIC, m3_scan_fwd_static -- runs on the current device.  Host
 * function.  So that a bf16 call that runs the SIMT kernel (for sizes the
 * tensor-core kernel does not cover: headdim != 64, dstate not 64 or 128,
 * rank not 1, 2 or 4) is visible to the caller. */
M3_API m3_status m3_scan_plan_info(int algo, const m3_dims *d, int flags, m3_plan_info *info);

/* Prefill: the chunked scan over a whole sequence (the four-piece chunked
 * algorithm of "La dualità: Mamba-2 e Mamba-3", section "Perché conviene: i
 * tensor core", extended with the trapezoid's previous-token term and the
 * pair rotations).  Reads x, B, C, dt, lam, theta, A, D and the optional
 * initial state `init` (NULL = zero state; its three buffers all required
 * when given); writes y and, when `final_state` is non-NULL, the state after
 * the last token.  `init` and `final_state` may be the same buffers only if
 * they are identical (in-place resume); partial overlaps are rejected, as is
 * any overlap of y with an input.  seqlen = 0 copies init to final_state.
 * With batch = 0 nothing is read or written and every pointer may be NULL. */
M3_API m3_status m3_scan_fwd(const m3_dims *d,
                      const void *x, const void *B, const void *C,
                      const void *dt, const void *lam, const void *theta,
                      const float *A, const float *D,
                      const m3_state *init, void *y, const m3_state *final_state,
                      void *workspace, size_t workspace_bytes, void *stream);

/* Same as m3_scan_fwd with an explicit kernel choice (for cross-checks):
 * an m3_algo value or M3_ALGO_TC_SEGMENTS(s); the workspace must be at
 * least m3_scan_plan's answer for the same `algo`.  The tensor-core choices
 * return M3_ERR_UNSUPPORTED for sizes that path does not cover. */
M3_API m3_status m3_scan_fwd_algo(int algo, const m3_dims *d,
                           const void *x, const void *B, const void *C,
                           const void *dt, const void *lam, const void *theta,
                           const float *A, const float *D,
                           const m3_state *init, void *y, const m3_state *final_state,
                           void *workspace, size_t workspace_bytes, void *stream);

/* m3_scan_fwd_algo with the BC-norm prologue fused in (`bcn` required). */
M3_API m3_status m3_scan_fwd_bcnorm(int algo, const m3_dims *d, const m3_bcnorm *bcn,
                             const void *x, const void *B, const void *C,
                             const void *dt, const void *lam, const void *theta,
                             const float *A, const float *D,
                             const m3_state *init, void *y, const m3_state *final_state,
                             void *workspace, size_t workspace_bytes, void *stream);

/* m3_scan_fwd_algo without a workspace argument: the per-segment states of
 * split sequences go to a scratch area the library itself holds in device
 * memory (a static 24 MiB array, reserved on each device when the library's
 * code is loaded there).  The pages have no counterpart to this entry point;
 * it exists for callers that cannot hand over device memory.
 *   - Size limit: the library's own segment choice is capped so that it fits
 *     the 24 MiB; a forced M3_ALGO_TC_SEGMENTS(s) whose states would not fit
 *     returns M3_ERR_UNSUPPORTED.  m3_scan_plan_info with M3_PLAN_STATIC
 *     tells how such a call runs.
 *   - Nothing in the scratch needs to start at zero: every value a call reads
 *     there was written earlier in the same call.
 *   - Calls that may overlap in time on one device (other streams, other host
 *     threads) race on the single scratch area: serialise them.
 *   - The first call on each device looks the scratch address up
 *     (cudaGetSymbolAddress): make one call outside CUDA-graph stream capture
 *     before capturing calls to this entry point. */
M3_API m3_status m3_scan_fwd_static(int algo, const m3_dims *d,
                             const void *x, const void *B, const void *C,
                             const void *dt, const void *lam, const void *theta,
                             const float *A, const float *D,
                             const m3_state *init, void *y, const m3_state *final_state,
                             void *stream);

/* How m3_scan_fwd_host will run `d` (with the BC-norm prologue when
 * `with_bcnorm` is non-zero) on the current device: the device
 * workspace it needs (bytes), the tokens per time slice (of every group but
 * the last, and of the last), the sequences per group and the number of
 * (group, slice) units.  Any output pointer may be NULL.  Slices are
 * multiples of 128 tokens (one slice when seqlen <= 128); the plan aims for 8
 * units: groups of whole sequences first, then time slices when there are
 * fewer than 8 groups; the last group is cut into at least 4 slices (when
 * seqlen allows), so that little work is left once the last copy-in ends. */
M3_API m3_status m3_scan_host_plan(const m3_dims *d, int with_bcnorm, size_t *workspace_bytes,
                                   int64_t *slice_tokens, int64_t *last_slice_tokens, int64_t *group_batch,
                                   int64_t *units);

/* m3_scan_fwd for sequences held in HOST memory: x, B, C, dt, lam, theta, A,
 * D, y and the optional init / final_state buffers are host pointers (same
 * shapes, dtypes and m3_dims flags as m3_scan_fwd); `workspace` is DEVICE
 * memory of at least m3_scan_host_plan's size, 16-byte aligned.  The result
 * is the scan of the whole sequence, as m3_scan_fwd computes it (as
 * m3_scan_fwd_bcnorm when `bcn` is non-NULL: its four arrays are then host
 * memory too, copied to the device once per call).  The pages have no
 * counterpart to this entry point: it is the end-to-end call for data that
 * starts and ends in host memory.  Errors: M3_ERR_INVALID_ARG for missing or
 * overlapping host buffers or a small or misaligned workspace (nothing is
 * queued then), the scan's own errors for its units, M3_ERR_CUDA for a failed
 * copy, event or stream call.
 *   - Pipelining: the call cuts the problem into (group of sequences) x
 *     (time slice) units and chains the slices of a group through the
 *     recurrent state (each slice resumes from the state the previous one
 *     left, exactly as a caller resumes one m3_scan_fwd with the previous
 *     call's final_state).  Copies in, kernels and copies out of successive
 *     units overlap on two copy streams of the library's own (created once
 *     per device on first use) and the caller's `stream`.
 *   - Asynchronous on `stream`: all of the call's work, copies included, is
 *     ordered after the work queued on `stream` before the call, and work
 *     queued on `stream` afterwards runs after all of it (y and final_state
 *     are complete once `stream` has reached that point).  Host buffers must
 *     stay valid and unmodified until then.  Pinned (page-locked) host memory
 *     lets the copies overlap; pageable memory works but serialises them.
 *   - Calls on one device are serialised while they enqueue; two calls must
 *     not share a workspace unless `stream` orders them.
 *   - Host buffers: y must not overlap an input; final_state must not overlap
 *     the inputs or y; init and final_state may be identical (in-place
 *     resume), not partially overlapping.
 *   - No explicit kernel choice (m3_scan_fwd's automatic choice runs every
 *     unit).  On an error returned after some units were queued, y and
 *     final_state are undefined. */
M3_API m3_status m3_scan_fwd_host(const m3_dims *d, const m3_bcnorm *bcn,
                           const void *x, const void *B, const void *C,
                           const void *dt, const void *lam, const void *theta,
                           const float *A, const float *D,
                           const m3_state *init, void *y, const m3_state *final_state,
                           void *workspace, size_t workspace_bytes, void *stream);

/* Decode: one token per (batch, head) against a resident state, updated in
 * place -- the three-term recurrence of "Знакомство с Mamba-3", section 1,
 * applied to a single token: h += beta' b_prev x_prev^T, h <- a Rot(-dt theta) h,
 * h += gamma B x^T, y = h^T C + D x, then b_prev <- B, x_prev <- x.
 * x [batch,nheads,rank,headdim], B/C [batch,nheads,rank,dstate],
 * dt/lam [batch,nheads], theta [batch,nheads,dstate/2] (io dtype);
 * y [batch,nheads,rank,headdim] (io).  `state` buffers are read and written
 * once each; y must not overlap anything else.  Errors: M3_ERR_INVALID_ARG
 * (null, misaligned or overlapping buffers, bad dims), M3_ERR_UNSUPPORTED
 * (sizes outside the compiled set), M3_ERR_CUDA (launch failure); nothing
 * is queued on an error. */
M3_API m3_status m3_step(const m3_dims *d,
                  const void *x, const void *B, const void *C,
                  const void *dt, const void *lam, const void *theta,
                  const float *A, const float *D,
                  const m3_state *state, void *y, void *stream);

/* m3_step with the BC-norm prologue fused in (`bcn` required); the state's
 * b_prev must hold normalised B (as m3_scan_fwd_bcnorm leaves it). */
M3_API m3_status m3_step_bcnorm(const m3_dims *d, const m3_bcnorm *bcn,
                         const void *x, const void *B, const void *C,
                         const void *dt, const void *lam, const void *theta,
                         const float *A, const float *D,
                         const m3_state *state, void *y, void *stream);

/* Wait for all work queued on `stream` (blocking the calling host thread),
 * then report any device-side failure recorded since the previous call:
 * M3_ERR_TIMEOUT if a bounded wait inside a kernel gave up (the kernel
 * drained its own copies and returned without trapping; its outputs are then
 * incomplete), M3_ERR_CUDA if the stream itself reported an error.  The
 * recorded failure is cleared.  Failures are recorded per device, not per
 * stream: the call reports (and clears) a wait that gave up in a kernel of
 * any stream of the current device, whatever `stream` is.  The code in the
 * message tells which wait: 0x1 a tile copy, 0x2 a tensor-core MMA (of either
 * prefill kernel), 0x4 the other warps of the prefill CTA, 0x8 a split
 * sequence's wait for an earlier segment (or, in its last segment, for the
 * first to have read the initial state), 0x10 the
 * self-test; the same bits shifted
 * left by 8 come from the decode kernels.  In the bounds build it also
 * returns M3_ERR_BOUNDS (after any timeout) if a device index check failed
 * (m3_device_checks).  A device-side wait gives up only on
 * a library bug; this call exists so that such a failure surfaces as a status
 * instead of a hang.
 * The library keeps, per device and for the life of the process, the
 * address of its scratch array and the host-buffer entry point's two streams
 * and events: do not use it across a cudaDeviceReset (or other teardown of
 * the device's primary context). */
M3_API m3_status m3_stream_status(void *stream);

/* Failure-path self-test: queues on `stream` one kernel whose bounded
 * device-side wait is made to give up (about 1 ms; nothing ever completes the
 * awaited phase).  The next m3_stream_status on that stream then returns
 * M3_ERR_TIMEOUT, and the device stays usable: the same path a stuck wait in
 * the prefill or decode kernels takes, without a fault, trap or hang.  The
 * pages have no counterpart to this call. */
M3_API m3_status m3_selftest_wait_timeout(void *stream);

/* Failure-path self-test of split sequences: the same call as
 * m3_scan_fwd_algo(M3_ALGO_TC_SEGMENTS(segments), ...) (bf16 I/O, sizes the
 * tensor-core path covers, segments >= 2, a workspace of
 * m3_scan_workspace_size for that algo) but without the summary pass, so
 * that the flags the main pass's look-back waits for are never published:
 * the CTAs of segments 1 .. segments-1 give up after their bounded wait
 * (about 1 s), record code 0x8, drain what they issued and return.  The next
 * m3_stream_status then returns M3_ERR_TIMEOUT, y and the final state are
 * incomplete, and the device stays usable.  The pages have no counterpart to
 * this call. */
M3_API m3_status m3_selftest_segment_timeout(const m3_dims *d, int segments, const void *x, const void *B,
                                             const void *C, const void *dt, const void *lam, const void *theta,
                                             const float *A, const float *D, const m3_state *init, void *y,
                                             const m3_state *final_state, void *workspace,
                                             size_t workspace_bytes, void *stream);

/* Message describing the calling thread's most recent failure ("" if none). */
M3_API const char *m3_last_error(void);

/* 1 in the bounds build of the library (libm3_bounds.so, compiled with
 * M3_DEVICE_CHECKS), 0 in the normal build.  In the bounds build every
 * kernel checks each global-memory access it makes through a plain pointer
 * against the extent of its buffer (computed from the call's dims); a failed
 * check skips the access (a read gives 0; a bulk copy reads from the
 * buffer's start instead) and records the site, the index and the extent of
 * the first failure, and m3_stream_status then returns M3_ERR_BOUNDS with
 * them in m3_last_error (and clears the record).  Tile copies (TMA) carry
 * their own extents and are not checked.  Same ABI and results as the normal
 * build, slower.  The pages have no counterpart to it. */
M3_API int m3_device_checks(void);

/* ABI version of this header (major * 100 + minor): 101 adds m3_scan_plan_info,
 * 102 the fp32 tensor-core prefill (M3_KERNEL_TC32), 103 the bounds build
 * (m3_device_checks, M3_ERR_BOUNDS), split sequences in two launches and the
 * MIMO projections (m3_scan_fwd_proj, m3_step_proj). */
M3_API int m3_version(void);

#ifdef __cplusplus
}
#endif
#endif /* M3_H */
