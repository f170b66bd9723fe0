// Internal interface between the C ABI layer (api.cpp) and the kernel
// translation units.  Not installed, not part of the public ABI.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/m3.h"

namespace m3 {

// Validated problem description handed to the launchers.
struct Problem {
    int64_t Bt, T, H, P, N, R;
    bool bf16;
    bool a_tok;                   // A per token-head ([Bt,T,H]; decode [Bt,H]) instead of per head
    bool th_head;                 // theta fixed per head ([H,N/2]) instead of per token-head
    const float *wB, *wC, *bB, *bC;  // BC-norm prologue (wB == nullptr: off)
    float eps;
    // MIMO projections (pwx == nullptr: off): x, B, C, y hold one row per
    // token-head; wx, wy [H, R, P] and wB, wC [H, R, N] widen them to rank R
    const float *pwx, *pwB, *pwC, *pwy;
    const void *x, *B, *C, *dt, *lam, *theta;
    const float *A, *D;
    const float *h0, *bp0, *xp0;  // nullable (zero initial state)
    void *y;
    float *hT, *bpT, *xpT;        // nullable (no final state wanted)
    void *ws;
    size_t ws_bytes;
    int segments;                 // tensor-core prefill: segments per sequence (0 = chosen by the library)
    size_t ws_cap;                // > 0: the library's choice of segments must fit this workspace
    bool skip_summary;            // failure-path self-test: split sequences without their summary pass
    cudaStream_t stream;
};

// How the tensor-core prefill runs one problem: every sequence in `nseg`
// segments of `cpseg` chunks (nseg = 1: one CTA per sequence, one launch;
// nseg > 1: summary pass, then the main pass with its look-back = two
// launches and a workspace of ws_bytes); `ctas` CTAs in the (main) launch.
struct TcPlan {
    int nchunks, cpseg, nseg, launches;
    int64_t ctas;
    size_t ws_bytes;
};

// Each launcher returns cudaSuccess or the launch error; `why` receives a
// static message for M3_ERR_UNSUPPORTED-style refusals (returned as
// cudaErrorNotSupported).
cudaError_t launch_prefill_simt(const Problem &p, const char **why);
bool prefill_tc_supported(const Problem &p, const char **why);
TcPlan prefill_tc_plan(const Problem &p);
size_t prefill_tc_workspace(const Problem &p);
cudaError_t launch_prefill_tc(const Problem &p, const char **why);
// fp32 I/O on the tensor cores (bf16 hi/lo operand halves); no workspace.
bool prefill_tc32_supported(const Problem &p, const char **why);
cudaError_t launch_prefill_tc32(const Problem &p, const char **why);
cudaError_t launch_step(const Problem &p, const char **why);
// The library's own device scratch for m3_scan_fwd_static: its address on the
// current device (looked up once per device) and its size.
cudaError_t static_scratch(void **ptr, size_t *bytes);
size_t static_scratch_bytes();
// One bounded device wait that is made to give up (failure-path self-test).
cudaError_t launch_wait_selftest(cudaStream_t stream);
// Synchronise `stream`, then read and clear the device error word that the
// tensor-core kernel's bounded waits set when they give up.
cudaError_t read_device_error(unsigned *code, cudaStream_t stream);
// Read and clear the decode kernels' device error word (after a sync).
cudaError_t read_decode_error(unsigned *code);
// Read and clear the fp32 tensor-core prefill's device error word (after a sync).
cudaError_t read_tc32_error(unsigned *code);
// First failed device index check recorded by one kernel file (the bounds
// build, compiled with M3_DEVICE_CHECKS; the normal build records none).
struct DcheckRecord {
    unsigned count;      // failed checks since the last read
    unsigned site;       // site code of the first failure (kernel file in the high byte)
    long long index;     // first element index of the failed access
    long long extent;    // elements in the buffer
};
// Read and clear each kernel file's record, after a sync.
cudaError_t read_dcheck_tc(DcheckRecord *r);
cudaError_t read_dcheck_tc32(DcheckRecord *r);
cudaError_t read_dcheck_simt(DcheckRecord *r);
cudaError_t read_dcheck_decode(DcheckRecord *r);
// Record the calling thread's failure message (m3_last_error) and return `s`.
m3_status set_error(m3_status s, const char *msg);
m3_status set_cuda_error(cudaError_t e, const char *where);

}  // namespace m3
