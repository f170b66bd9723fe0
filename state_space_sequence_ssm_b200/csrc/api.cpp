// api.cpp -- the C ABI of include/m3.h: argument validation, dispatch to the
// kernels, and thread-local error reporting.  No exception crosses the
// boundary; nothing here allocates device memory.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <exception>
#include <string>

#include "m3_internal.h"

namespace {

thread_local std::string g_err;

constexpr int kMaxForcedSegments = 4096;  // upper bound of M3_ALGO_TC_SEGMENTS(s)

m3_status fail(m3_status s, const char *fmt, const char *a = nullptr) {
    char buf[512];
    std::snprintf(buf, sizeof buf, fmt, a ? a : "");
    g_err = buf;
    return s;
}

m3_status cuda_fail(cudaError_t e, const char *where) {
    char buf[512];
    std::snprintf(buf, sizeof buf, "%s: %s (%s)", where, cudaGetErrorString(e), cudaGetErrorName(e));
    g_err = buf;
    return M3_ERR_CUDA;
}

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
    bool empty() const { return hi <= lo; }
};
Range range(const void *p, size_t bytes) {
    uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    return {lo, lo + (p ? bytes : 0)};
}
bool overlap(Range a, Range b) { return !a.empty() && !b.empty() && a.lo < b.hi && b.lo < a.hi; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

m3_status check_dims(const m3_dims *d, bool decode) {
    if (!d) return fail(M3_ERR_INVALID_ARG, "dims is NULL");
    if (d->batch < 0 || (!decode && d->seqlen < 0))
        return fail(M3_ERR_INVALID_ARG, "batch and seqlen must be >= 0");
    if (d->nheads < 1 || d->headdim < 1 || d->rank < 1)
        return fail(M3_ERR_INVALID_ARG, "nheads, headdim and rank must be >= 1");
    if (d->dstate < 2 || (d->dstate & 1))
        return fail(M3_ERR_INVALID_ARG, "dstate must be even and >= 2 (state pairs)");
    if (d->io != M3_F32 && d->io != M3_BF16) return fail(M3_ERR_INVALID_ARG, "io must be M3_F32 or M3_BF16");
    if (d->flags & ~(M3_FLAG_A_PER_TOKEN | M3_FLAG_THETA_PER_HEAD))
        return fail(M3_ERR_INVALID_ARG, "unknown bits in flags");
    if (d->dstate > 256 || d->headdim > 256 || d->rank > 8)
        return fail(M3_ERR_UNSUPPORTED, "supported sizes: dstate <= 256, headdim <= 256, rank <= 8");
    if (d->headdim % 4 != 0 && d->headdim != 1 && d->headdim != 2)
        return fail(M3_ERR_UNSUPPORTED, "headdim must be a multiple of 4 (or 1, 2)");
    // every flat index must fit comfortably in int64
    const double elems = double(d->batch) * double(decode ? 1 : d->seqlen) * double(d->nheads) *
                         double(d->rank) * double(d->dstate > d->headdim ? d->dstate : d->headdim);
    if (elems > 4.0e18) return fail(M3_ERR_INVALID_ARG, "problem too large");
    return M3_OK;
}

// Shared validation of tensor pointers.  `tok` = number of token-heads.
// proj: the MIMO projections' layout (x, B, C and y with one row per
// token-head instead of R).
m3_status check_tensors(const m3_dims *d, int64_t tok, const void *x, const void *B, const void *C,
                        const void *dt, const void *lam, const void *theta, const float *A,
                        const float *D, const void *y, Range *ins, int *nin, Range *yr, bool proj = false) {
    const size_t es = d->io == M3_BF16 ? 2 : 4;
    const int64_t R = proj ? 1 : d->rank, P = d->headdim, N = d->dstate;
    if (tok > 0) {
        if (!x || !B || !C || !dt || !lam || !theta || !y)
            return fail(M3_ERR_INVALID_ARG, "x, B, C, dt, lam, theta and y are required");
        const void *ptrs[] = {x, B, C, theta, y};
        for (const void *p : ptrs)
            if (!aligned16(p)) return fail(M3_ERR_INVALID_ARG, "x, B, C, theta and y must be 16-byte aligned");
        if ((reinterpret_cast<uintptr_t>(dt) | reinterpret_cast<uintptr_t>(lam)) % es)
            return fail(M3_ERR_INVALID_ARG, "dt and lam must be aligned to their element size");
    }
    if (!A || !D) return fail(M3_ERR_INVALID_ARG, "A and D are required");
    if ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(D)) % 4)
        return fail(M3_ERR_INVALID_ARG, "A and D must be 4-byte aligned");
    int n = 0;
    ins[n++] = range(x, tok * R * P * es);
    ins[n++] = range(B, tok * R * N * es);
    ins[n++] = range(C, tok * R * N * es);
    ins[n++] = range(dt, tok * es);
    ins[n++] = range(lam, tok * es);
    ins[n++] = range(theta, ((d->flags & M3_FLAG_THETA_PER_HEAD) ? d->nheads : tok) * (N / 2) * es);
    ins[n++] = range(A, ((d->flags & M3_FLAG_A_PER_TOKEN) ? tok : d->nheads) * 4);
    ins[n++] = range(D, d->nheads * 4);
    *nin = n;
    *yr = range(y, tok * R * P * es);
    for (int i = 0; i < n; ++i)
        if (overlap(*yr, ins[i])) return fail(M3_ERR_INVALID_ARG, "y overlaps an input tensor");
    return M3_OK;
}

m3_status check_state(const m3_dims *d, const m3_state *s, const char *what, Range out[3]) {
    const int64_t BH = d->batch * d->nheads;
    const int64_t N = d->dstate, P = d->headdim, R = d->rank;
    if (BH == 0) {  // zero-sized state: nothing is read or written, pointers may be NULL
        out[0] = out[1] = out[2] = Range{0, 0};
        return M3_OK;
    }
    if (!s->h || !s->b_prev || !s->x_prev) {
        g_err = std::string(what) + ": h, b_prev and x_prev are all required";
        return M3_ERR_INVALID_ARG;
    }
    if (!aligned16(s->h) || !aligned16(s->b_prev) || !aligned16(s->x_prev)) {
        g_err = std::string(what) + ": state buffers must be 16-byte aligned";
        return M3_ERR_INVALID_ARG;
    }
    out[0] = range(s->h, BH * N * P * 4);
    out[1] = range(s->b_prev, BH * R * N * 4);
    out[2] = range(s->x_prev, BH * R * P * 4);
    for (int i = 0; i < 3; ++i)
        for (int j = i + 1; j < 3; ++j)
            if (overlap(out[i], out[j])) {
                g_err = std::string(what) + ": state buffers overlap each other";
                return M3_ERR_INVALID_ARG;
            }
    return M3_OK;
}

m3::Problem make_problem(const m3_dims *d, const void *x, const void *B, const void *C, const void *dt,
                         const void *lam, const void *theta, const float *A, const float *D, void *y,
                         void *stream) {
    m3::Problem p{};
    p.Bt = d->batch; p.T = d->seqlen; p.H = d->nheads; p.P = d->headdim; p.N = d->dstate; p.R = d->rank;
    p.bf16 = d->io == M3_BF16;
    p.a_tok = (d->flags & M3_FLAG_A_PER_TOKEN) != 0;
    p.th_head = (d->flags & M3_FLAG_THETA_PER_HEAD) != 0;
    p.x = x; p.B = B; p.C = C; p.dt = dt; p.lam = lam; p.theta = theta; p.A = A; p.D = D; p.y = y;
    p.stream = static_cast<cudaStream_t>(stream);
    return p;
}

// BC-norm parameters: all four arrays, 4-byte aligned, eps > 0, no overlap with y.
m3_status check_bcnorm(const m3_dims *d, const m3_bcnorm *bcn, Range yr) {
    if (!bcn) return fail(M3_ERR_INVALID_ARG, "bcn is NULL");
    if (!bcn->wB || !bcn->wC || !bcn->bB || !bcn->bC)
        return fail(M3_ERR_INVALID_ARG, "bcn: wB, wC, bB and bC are all required");
    if ((reinterpret_cast<uintptr_t>(bcn->wB) | reinterpret_cast<uintptr_t>(bcn->wC) |
         reinterpret_cast<uintptr_t>(bcn->bB) | reinterpret_cast<uintptr_t>(bcn->bC)) % 4)
        return fail(M3_ERR_INVALID_ARG, "bcn arrays must be 4-byte aligned");
    if (!(bcn->eps > 0.f)) return fail(M3_ERR_INVALID_ARG, "bcn eps must be > 0");
    const Range rs[4] = {range(bcn->wB, d->dstate * 4), range(bcn->wC, d->dstate * 4),
                         range(bcn->bB, d->nheads * d->rank * d->dstate * 4),
                         range(bcn->bC, d->nheads * d->rank * d->dstate * 4)};
    for (const Range &r : rs)
        if (overlap(r, yr)) return fail(M3_ERR_INVALID_ARG, "y overlaps a bcn array");
    return M3_OK;
}

m3_status check_proj(const m3_dims *d, const m3_mimo_proj *pr, Range yr) {
    if (!pr) return fail(M3_ERR_INVALID_ARG, "proj is NULL");
    if (!pr->wx || !pr->wB || !pr->wC || !pr->wy)
        return fail(M3_ERR_INVALID_ARG, "proj: wx, wB, wC and wy are all required");
    if ((reinterpret_cast<uintptr_t>(pr->wx) | reinterpret_cast<uintptr_t>(pr->wB) |
         reinterpret_cast<uintptr_t>(pr->wC) | reinterpret_cast<uintptr_t>(pr->wy)) % 4)
        return fail(M3_ERR_INVALID_ARG, "proj arrays must be 4-byte aligned");
    const int64_t hr = d->nheads * d->rank;
    const Range rs[4] = {range(pr->wx, hr * d->headdim * 4), range(pr->wB, hr * d->dstate * 4),
                         range(pr->wC, hr * d->dstate * 4), range(pr->wy, hr * d->headdim * 4)};
    for (const Range &r : rs)
        if (overlap(r, yr)) return fail(M3_ERR_INVALID_ARG, "y overlaps a proj array");
    return M3_OK;
}

// The tensor-core kernel for p's I/O type (bf16: prefill_tc, fp32:
// prefill_tc32) and whether it covers p.
bool tc_supported(const m3::Problem &p, const char **why) {
    return p.bf16 ? m3::prefill_tc_supported(p, why) : m3::prefill_tc32_supported(p, why);
}

m3_status scan_impl(int algo, const m3_dims *d, const void *x, const void *B, const void *C, const void *dt,
                    const void *lam, const void *theta, const float *A, const float *D, const m3_state *init,
                    void *y, const m3_state *fin, void *ws, size_t ws_bytes, void *stream,
                    bool static_ws = false, const m3_bcnorm *bcn = nullptr, bool skip_summary = false,
                    const m3_mimo_proj *proj = nullptr) {
    m3_status s = check_dims(d, false);
    if (s != M3_OK) return s;
    const int segments = algo >> 8;
    algo &= 0xff;
    if (algo != M3_ALGO_AUTO && algo != M3_ALGO_SIMT && algo != M3_ALGO_TC)
        return fail(M3_ERR_INVALID_ARG, "unknown algo");
    if (segments < 0 || segments > kMaxForcedSegments || (segments && algo != M3_ALGO_TC))
        return fail(M3_ERR_INVALID_ARG, "bad segment count in algo");
    const int64_t tok = d->batch * d->seqlen * d->nheads;
    Range ins[8], yr;
    int nin = 0;
    s = check_tensors(d, tok, x, B, C, dt, lam, theta, A, D, y, ins, &nin, &yr, proj != nullptr);
    if (s != M3_OK) return s;
    Range ir[3] = {}, fr[3] = {};
    if (init && (s = check_state(d, init, "init", ir)) != M3_OK) return s;
    if (fin && (s = check_state(d, fin, "final_state", fr)) != M3_OK) return s;
    for (int i = 0; i < 3; ++i) {
        if (overlap(fr[i], yr)) return fail(M3_ERR_INVALID_ARG, "final_state overlaps y");
        for (int j = 0; j < nin; ++j)
            if (overlap(fr[i], ins[j]) || overlap(ir[i], yr))
                return fail(M3_ERR_INVALID_ARG, "state buffers overlap the sequence tensors");
        for (int j = 0; j < 3; ++j) {
            // in-place resume (identical buffers) is allowed; partial overlap is not
            const bool same = i == j && fr[i].lo == ir[j].lo && fr[i].hi == ir[j].hi;
            if (!same && overlap(fr[i], ir[j]))
                return fail(M3_ERR_INVALID_ARG, "final_state partially overlaps init");
        }
    }
    if (bcn && (s = check_bcnorm(d, bcn, yr)) != M3_OK) return s;
    if (proj) {
        if ((s = check_proj(d, proj, yr)) != M3_OK) return s;
        if (bcn) return fail(M3_ERR_UNSUPPORTED, "the MIMO projections do not combine with the BC-norm prologue");
        if (d->io != M3_BF16 || algo == M3_ALGO_SIMT)
            return fail(M3_ERR_UNSUPPORTED, "the MIMO projections run on the bf16 tensor-core prefill only");
    }
    if (d->batch == 0) return M3_OK;  // nothing to read or write, whichever kernel was asked for
    m3::Problem p = make_problem(d, x, B, C, dt, lam, theta, A, D, y, stream);
    if (bcn) { p.wB = bcn->wB; p.wC = bcn->wC; p.bB = bcn->bB; p.bC = bcn->bC; p.eps = bcn->eps; }
    if (proj) { p.pwx = proj->wx; p.pwB = proj->wB; p.pwC = proj->wC; p.pwy = proj->wy; }
    if (init) { p.h0 = init->h; p.bp0 = init->b_prev; p.xp0 = init->x_prev; }
    if (fin) { p.hT = fin->h; p.bpT = fin->b_prev; p.xpT = fin->x_prev; }
    p.ws = ws;
    p.ws_bytes = ws_bytes;
    p.segments = segments;
    p.skip_summary = skip_summary;

    const char *why = nullptr;
    const char *tc_why = nullptr;
    const bool tc_ok = tc_supported(p, &tc_why);
    bool use_tc = false;
    if (algo == M3_ALGO_TC || proj) {
        if (!tc_ok) return fail(M3_ERR_UNSUPPORTED, "%s", tc_why ? tc_why : "tensor-core path unsupported");
        use_tc = true;
    } else if (algo == M3_ALGO_AUTO) {
        use_tc = tc_ok;
    }
    if (use_tc && p.bf16) {  // the fp32 kernel needs no workspace
        if (static_ws) {
            p.ws_cap = m3::static_scratch_bytes();
            const size_t need = m3::prefill_tc_workspace(p);
            if (need > p.ws_cap)
                return fail(M3_ERR_UNSUPPORTED,
                            "m3_scan_fwd_static: this segment count needs more than the library's 24 MiB scratch "
                            "(use m3_scan_fwd_algo with a workspace)");
            if (need) {
                const cudaError_t e = m3::static_scratch(&p.ws, &p.ws_bytes);
                if (e != cudaSuccess) return cuda_fail(e, "m3_scan_fwd_static (scratch address)");
            }
        } else {
            const size_t need = m3::prefill_tc_workspace(p);
            if (need > ws_bytes || (need && !ws))
                return fail(M3_ERR_INVALID_ARG, "workspace too small (query m3_scan_workspace_size)");
            if (need && !aligned16(ws)) return fail(M3_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
        }
    }
    cudaError_t e = !use_tc ? m3::launch_prefill_simt(p, &why)
                    : p.bf16 ? m3::launch_prefill_tc(p, &why)
                             : m3::launch_prefill_tc32(p, &why);
    if (e == cudaErrorNotSupported && why) return fail(M3_ERR_UNSUPPORTED, "%s", why);
    if (e != cudaSuccess)
        return cuda_fail(e, !use_tc ? "m3_scan_fwd (SIMT kernel)"
                            : p.bf16 ? "m3_scan_fwd (tensor-core kernel)"
                                     : "m3_scan_fwd (fp32 tensor-core kernel)");
    return M3_OK;
}

}  // namespace

namespace m3 {
m3_status set_error(m3_status s, const char *msg) { return fail(s, "%s", msg); }
m3_status set_cuda_error(cudaError_t e, const char *where) { return cuda_fail(e, where); }
}  // namespace m3

extern "C" {

int m3_version(void) { return 103; }

int m3_device_checks(void) {
#ifdef M3_DEVICE_CHECKS
    return 1;
#else
    return 0;
#endif
}

const char *m3_last_error(void) { return g_err.c_str(); }

m3_status m3_scan_plan_info(int algo, const m3_dims *d, int flags, m3_plan_info *info) {
    try {
        if (!info) return fail(M3_ERR_INVALID_ARG, "info is NULL");
        m3_status s = check_dims(d, false);
        if (s != M3_OK) return s;
        if (flags & ~M3_PLAN_STATIC) return fail(M3_ERR_INVALID_ARG, "unknown plan flags");
        const int forced = algo >> 8;
        const int base = algo & 0xff;
        if (base != M3_ALGO_AUTO && base != M3_ALGO_SIMT && base != M3_ALGO_TC)
            return fail(M3_ERR_INVALID_ARG, "unknown algo");
        if (forced < 0 || forced > kMaxForcedSegments || (forced && base != M3_ALGO_TC))
            return fail(M3_ERR_INVALID_ARG, "bad segment count in algo");
        *info = m3_plan_info{};
        info->segments = 1;
        if (d->batch == 0) return M3_OK;  // nothing to run, whichever kernel was asked for
        m3::Problem p{};
        p.Bt = d->batch; p.T = d->seqlen; p.H = d->nheads; p.P = d->headdim; p.N = d->dstate; p.R = d->rank;
        p.bf16 = d->io == M3_BF16;
        p.segments = forced;
        const char *why = nullptr;
        const bool tc = base != M3_ALGO_SIMT && tc_supported(p, &why);
        if (base == M3_ALGO_TC && !tc)
            return fail(M3_ERR_UNSUPPORTED, "%s", why ? why : "tensor-core path unsupported");
        if (!tc) {
            info->kernel = M3_KERNEL_SIMT;
            info->launches = 1;
            info->ctas = d->batch * d->nheads;
            return M3_OK;
        }
        if (!p.bf16) {  // fp32 tensor-core kernel: one CTA per sequence and head, no workspace
            info->kernel = M3_KERNEL_TC32;
            info->launches = 1;
            info->ctas = d->batch * d->nheads;
            return M3_OK;
        }
        if (flags & M3_PLAN_STATIC) p.ws_cap = m3::static_scratch_bytes();
        const m3::TcPlan plan = m3::prefill_tc_plan(p);
        if ((flags & M3_PLAN_STATIC) && plan.ws_bytes > p.ws_cap)
            return fail(M3_ERR_UNSUPPORTED, "m3_scan_fwd_static: this segment count needs more than the "
                                            "library's 24 MiB scratch");
        info->kernel = M3_KERNEL_TC;
        info->workspace_bytes = plan.ws_bytes;
        info->segments = plan.nseg;
        info->launches = plan.launches;
        info->ctas = plan.ctas;
        return M3_OK;
    } catch (const std::exception &ex) {
        return fail(M3_ERR_INVALID_ARG, "internal error: %s", ex.what());
    } catch (...) {
        return fail(M3_ERR_INVALID_ARG, "internal error");
    }
}

m3_status m3_scan_plan(int algo, const m3_dims *d, size_t *workspace_bytes, int *segments, int *launches) {
    m3_plan_info info{};
    const m3_status s = m3_scan_plan_info(algo, d, 0, &info);
    if (s != M3_OK) return s;
    if (workspace_bytes) *workspace_bytes = info.workspace_bytes;
    if (segments) *segments = info.segments;
    if (launches) *launches = info.launches;
    return M3_OK;
}

m3_status m3_scan_workspace_size(const m3_dims *d, size_t *bytes) {
    if (!bytes) return fail(M3_ERR_INVALID_ARG, "bytes is NULL");
    return m3_scan_plan(M3_ALGO_AUTO, d, bytes, nullptr, nullptr);
}

m3_status m3_scan_fwd(const m3_dims *d, const void *x, const void *B, const void *C, const void *dt,
                      const void *lam, const void *theta, const float *A, const float *D, const m3_state *init,
                      void *y, const m3_state *final_state, void *workspace, size_t workspace_bytes,
                      void *stream) {
    try {
        return scan_impl(M3_ALGO_AUTO, d, x, B, C, dt, lam, theta, A, D, init, y, final_state, workspace,
                         workspace_bytes, stream);
    } catch (...) {
        return fail(M3_ERR_INVALID_ARG, "internal error");
    }
}

m3_status m3_scan_fwd_algo(int algo, const m3_dims *d, const void *x, const void *B, const void *C,
                           const void *dt, const void *lam, const void *theta, const float *A, const float *D,
                           const m3_state *init, void *y, const m3_state *final_state, void *workspace,
                           size_t workspace_bytes, void *stream) {
    try {
        return scan_impl(algo, d, x, B, C, dt, lam, theta, A, D, init, y, final_state, workspace,
                         workspace_bytes, stream);
    } catch (...) {
        return fail(M3_ERR_INVALID_ARG, "internal error");
    }
}

m3_status m3_scan_fwd_bcnorm(int algo, const m3_dims *d, const m3_bcnorm *bcn, const void *x, const void *B,
                             const void *C, const void *dt, const void *lam, const void *theta, const float *A,
                             const float *D, const m3_state *init, void *y, const m3_state *final_state,
                             void *workspace, size_t workspace_bytes, void *stream) {
    try {
        if (!bcn) return fail(M3_ERR_INVALID_ARG, "bcn is NULL");
        return scan_impl(algo, d, x, B, C, dt, lam, theta, A, D, init, y, final_state, workspace,
                         workspace_bytes, stream, false, bcn);
    } catch (...) {
        return fail(M3_ERR_INVALID_ARG, "internal error");
    }
}

m3_status m3_scan_fwd_proj(int algo, const m3_dims *d, const m3_mimo_proj *proj, const void *x, const void *B,
                           const void *C, const void *dt, const void *lam, const void *theta, const float *A,
                           const float *D, const m3_state *init, void *y, const m3_state *final_state,
                           void *workspace, size_t workspace_bytes, void *stream) {
    try {
        if (!proj) return fail(M3_ERR_INVALID_ARG, "proj is NULL");
        return scan_impl(algo, d, x, B, C, dt, lam, theta, A, D, init, y, final_state, workspace,
                         workspace_bytes, stream, false, nullptr, false, proj);
    } catch (...) {
        return fail(M3_ERR_INVALID_ARG, "internal error");
    }
}

m3_status m3_scan_fwd_static(int algo, const m3_dims *d, const void *x, const void *B, const void *C,
                             const void *dt, const void *lam, const void *theta, const float *A, const float *D,
                             const m3_state *init, void *y, const m3_state *final_state, void *stream) {
    try {
        return scan_impl(algo, d, x, B, C, dt, lam, theta, A, D, init, y, final_state, nullptr, 0, stream, true);
    } catch (...) {
        return fail(M3_ERR_INVALID_ARG, "internal error");
    }
}

m3_status m3_selftest_segment_timeout(const m3_dims *d, int segments, const void *x, const void *B, const void *C,
                                       const void *dt, const void *lam, const void *theta, const float *A,
                                       const float *D, const m3_state *init, void *y, const m3_state *final_state,
                                       void *workspace, size_t workspace_bytes, void *stream) {
    try {
        if (segments < 2) return fail(M3_ERR_INVALID_ARG, "m3_selftest_segment_timeout: segments must be >= 2");
        if (!d || d->io != M3_BF16) return fail(M3_ERR_INVALID_ARG, "m3_selftest_segment_timeout: bf16 I/O only");
        return scan_impl(M3_ALGO_TC_SEGMENTS(segments), d, x, B, C, dt, lam, theta, A, D, init, y, final_state,
                         workspace, workspace_bytes, stream, false, nullptr, true);
    } catch (...) {
        return fail(M3_ERR_INVALID_ARG, "internal error");
    }
}

m3_status m3_selftest_wait_timeout(void *stream) {
    try {
        const cudaError_t e = m3::launch_wait_selftest(static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "m3_selftest_wait_timeout");
        return M3_OK;
    } catch (...) {
        return fail(M3_ERR_INVALID_ARG, "internal error");
    }
}

m3_status m3_stream_status(void *stream) {
    try {
        unsigned code = 0;
        cudaError_t e = m3::read_device_error(&code, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e, "m3_stream_status");
        unsigned dcode = 0;
        e = m3::read_decode_error(&dcode);
        if (e != cudaSuccess) return cuda_fail(e, "m3_stream_status");
        unsigned tcode = 0;
        e = m3::read_tc32_error(&tcode);
        if (e != cudaSuccess) return cuda_fail(e, "m3_stream_status");
        code |= tcode | (dcode << 8);
        // the bounds build's index-check records (all read, so all cleared)
        m3::DcheckRecord rec[4], first{0u, 0u, 0, 0};
        unsigned fails = 0;
        cudaError_t (*const readers[4])(m3::DcheckRecord *) = {m3::read_dcheck_tc, m3::read_dcheck_tc32,
                                                                m3::read_dcheck_simt, m3::read_dcheck_decode};
        for (int i = 0; i < 4; ++i) {
            if ((e = readers[i](&rec[i])) != cudaSuccess) return cuda_fail(e, "m3_stream_status");
            if (rec[i].count && !fails) first = rec[i];
            fails += rec[i].count;
        }
        if (code) {
            char buf[128];
            std::snprintf(buf, sizeof buf, "a bounded device-side wait gave up (code 0x%x)", code);
            g_err = buf;
            return M3_ERR_TIMEOUT;
        }
        if (fails) {
            char buf[192];
            std::snprintf(buf, sizeof buf,
                          "device index check failed: site 0x%x, index %lld, extent %lld (%u failed checks)",
                          first.site, first.index, first.extent, fails);
            g_err = buf;
            return M3_ERR_BOUNDS;
        }
        return M3_OK;
    } catch (...) {
        return fail(M3_ERR_INVALID_ARG, "internal error");
    }
}

m3_status step_impl(const m3_dims *d, const m3_bcnorm *bcn, const void *x, const void *B, const void *C,
                    const void *dt, const void *lam, const void *theta, const float *A, const float *D,
                    const m3_state *state, void *y, void *stream, const m3_mimo_proj *proj = nullptr);

m3_status m3_step_proj(const m3_dims *d, const m3_mimo_proj *proj, const void *x, const void *B, const void *C,
                       const void *dt, const void *lam, const void *theta, const float *A, const float *D,
                       const m3_state *state, void *y, void *stream) {
    if (!proj) return fail(M3_ERR_INVALID_ARG, "proj is NULL");
    return step_impl(d, nullptr, x, B, C, dt, lam, theta, A, D, state, y, stream, proj);
}

m3_status m3_step(const m3_dims *d, const void *x, const void *B, const void *C, const void *dt,
                  const void *lam, const void *theta, const float *A, const float *D, const m3_state *state,
                  void *y, void *stream) {
    return step_impl(d, nullptr, x, B, C, dt, lam, theta, A, D, state, y, stream);
}

m3_status m3_step_bcnorm(const m3_dims *d, const m3_bcnorm *bcn, const void *x, const void *B, const void *C,
                         const void *dt, const void *lam, const void *theta, const float *A, const float *D,
                         const m3_state *state, void *y, void *stream) {
    if (!bcn) return fail(M3_ERR_INVALID_ARG, "bcn is NULL");
    return step_impl(d, bcn, x, B, C, dt, lam, theta, A, D, state, y, stream);
}

m3_status step_impl(const m3_dims *d, const m3_bcnorm *bcn, const void *x, const void *B, const void *C,
                    const void *dt, const void *lam, const void *theta, const float *A, const float *D,
                    const m3_state *state, void *y, void *stream, const m3_mimo_proj *proj) {
    try {
        m3_status s = check_dims(d, true);
        if (s != M3_OK) return s;
        const int64_t tok = d->batch * d->nheads;
        Range ins[8], yr;
        int nin = 0;
        s = check_tensors(d, tok, x, B, C, dt, lam, theta, A, D, y, ins, &nin, &yr, proj != nullptr);
        if (s != M3_OK) return s;
        if (!state) return fail(M3_ERR_INVALID_ARG, "state is required");
        Range sr[3];
        if ((s = check_state(d, state, "state", sr)) != M3_OK) return s;
        for (int i = 0; i < 3; ++i) {
            if (overlap(sr[i], yr)) return fail(M3_ERR_INVALID_ARG, "state overlaps y");
            for (int j = 0; j < nin; ++j)
                if (overlap(sr[i], ins[j])) return fail(M3_ERR_INVALID_ARG, "state overlaps an input tensor");
        }
        if (bcn && (s = check_bcnorm(d, bcn, yr)) != M3_OK) return s;
        if (proj && (s = check_proj(d, proj, yr)) != M3_OK) return s;
        m3::Problem p = make_problem(d, x, B, C, dt, lam, theta, A, D, y, stream);
        if (bcn) { p.wB = bcn->wB; p.wC = bcn->wC; p.bB = bcn->bB; p.bC = bcn->bC; p.eps = bcn->eps; }
        if (proj) { p.pwx = proj->wx; p.pwB = proj->wB; p.pwC = proj->wC; p.pwy = proj->wy; }
        p.T = 1;
        p.hT = state->h; p.bpT = state->b_prev; p.xpT = state->x_prev;
        const char *why = nullptr;
        cudaError_t e = m3::launch_step(p, &why);
        if (e == cudaErrorNotSupported && why) return fail(M3_ERR_UNSUPPORTED, "%s", why);
        if (e != cudaSuccess) return cuda_fail(e, "m3_step");
        return M3_OK;
    } catch (...) {
        return fail(M3_ERR_INVALID_ARG, "internal error");
    }
}

}  // extern "C"
