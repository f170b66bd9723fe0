// host_pipeline.cpp -- m3_scan_fwd_host: the prefill scan over sequences that
// live in host memory.
//
// The problem is cut into units of (a group of whole sequences) x (a slice of
// their tokens).  Within a group the slices are chained through the
// recurrent state: slice i starts from the state slice i-1 left (the same
// resume a caller gets by passing one call's final_state as the next call's
// init), so the result is the scan of the whole sequence.  Every unit runs as
//
//   copy-in stream:   inputs of unit k  -> device slot k % 2
//   caller's stream:  m3_scan_fwd on slot k % 2
//   copy-out stream:  y of unit k (and the final state after a group's last
//                     slice) -> host
//
// so that the host-to-device copy of unit k+1, the kernels of unit k and the
// device-to-host copy of unit k-1 overlap (the two copy directions run on
// separate copy engines).  Two slots suffice because a unit's kernels take a
// small fraction of its copy-in time.  Slices are multiples of 128 tokens, so
// every slice boundary is also a chunk boundary of the tensor-core kernel.
//
// The two copy streams and the events are the library's own, created once
// per device on first use and kept for the life of the process; calls on one
// device are serialised by a mutex while they enqueue.  Nothing here
// allocates device memory: the staging buffers live in the caller's
// workspace.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "m3_internal.h"

namespace {

constexpr int64_t kSliceAlign = 128;   // tokens; a multiple of every chunk length
constexpr int64_t kUnitsTarget = 8;    // units per call the plan aims for
constexpr int64_t kTailSlices = 4;     // the last group is cut into at least this many slices
constexpr size_t kAlign = 256;         // byte alignment of every staging buffer
constexpr int kMaxDevices = 64;

size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct Streams {
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    cudaEvent_t loaded[2] = {}, computed[2] = {}, drained[2] = {};
    std::mutex call;  // one call at a time enqueues on this device's streams
};
Streams g_streams[kMaxDevices];
std::mutex g_create;

cudaError_t streams_for(int dev, Streams **out) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    Streams &s = g_streams[dev];
    std::lock_guard<std::mutex> lk(g_create);
    if (!s.ready) {
        cudaError_t e = cudaStreamCreateWithFlags(&s.in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s.out, cudaStreamNonBlocking);
        cudaEvent_t *evs[] = {&s.fork, &s.join, &s.loaded[0], &s.loaded[1], &s.computed[0], &s.computed[1],
                              &s.drained[0], &s.drained[1]};
        for (cudaEvent_t *ev : evs)
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
        s.ready = true;
    }
    *out = &s;
    return cudaSuccess;
}

// How one call is cut into units, and where its staging buffers sit in the
// workspace (byte offsets from its start).
struct Layout {
    int64_t slice, group, nslice, ngroup;
    int64_t slice_last, nslice_last;    // the last group's slicing (finer: a short pipeline tail)
    size_t A, D, theta;                 // per-head constants (theta only when fixed per head)
    size_t wB, wC, bB, bC;              // BC-norm parameters (when the call has them)
    size_t st[3][3];                    // state sets (initial, ping, pong) x (h, b_prev, x_prev)
    size_t slot[2][8];                  // x, B, C, dt, lam, theta, A, y of each slot
    size_t ws, ws_bytes;                // the scan's own workspace and its size
    size_t total;
};

struct Rows {  // bytes per token of each per-token tensor, in the order of Layout::slot
    size_t b[8];
};

Rows token_rows(const m3_dims *d) {
    const size_t es = d->io == M3_BF16 ? 2 : 4;
    const size_t H = d->nheads, R = d->rank, P = d->headdim, N = d->dstate;
    Rows r{};
    r.b[0] = H * R * P * es;
    r.b[1] = r.b[2] = H * R * N * es;
    r.b[3] = r.b[4] = H * es;
    r.b[5] = (d->flags & M3_FLAG_THETA_PER_HEAD) ? 0 : H * (N / 2) * es;
    r.b[6] = (d->flags & M3_FLAG_A_PER_TOKEN) ? H * 4 : 0;
    r.b[7] = H * R * P * es;
    return r;
}

m3_status plan_layout(const m3_dims *d, bool bcn, Layout *L) {
    const int64_t T = d->seqlen, Bt = d->batch;
    // Whole sequences first (their copies are contiguous: measured 1 % faster
    // than time slices of the full batch), time slices only for the rest.
    const int64_t groups = std::max<int64_t>(1, std::min(Bt, kUnitsTarget));
    L->group = Bt > 0 ? cdiv(Bt, groups) : 0;
    L->ngroup = Bt > 0 ? cdiv(Bt, L->group) : 0;
    const int64_t want = cdiv(kUnitsTarget, std::max<int64_t>(L->ngroup, 1));
    L->nslice = T <= kSliceAlign ? 1 : std::min(cdiv(T, kSliceAlign), want);
    L->slice = T <= kSliceAlign ? T : cdiv(cdiv(T, L->nslice), kSliceAlign) * kSliceAlign;
    if (T > kSliceAlign) L->nslice = cdiv(T, L->slice);
    // What is left after the last copy-in -- the last unit's kernels and its
    // copy-out -- is the pipeline's exposed tail: cut the last group finer.
    L->slice_last = L->slice;
    L->nslice_last = L->nslice;
    if (T > kSliceAlign) {
        const int64_t n = std::min(cdiv(T, kSliceAlign), std::max(L->nslice, kTailSlices));
        L->slice_last = cdiv(cdiv(T, n), kSliceAlign) * kSliceAlign;
        L->nslice_last = cdiv(T, L->slice_last);
    }

    const size_t es = d->io == M3_BF16 ? 2 : 4;
    const size_t H = d->nheads, R = d->rank, P = d->headdim, N = d->dstate;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += up(bytes);
        return at;
    };
    L->A = (d->flags & M3_FLAG_A_PER_TOKEN) ? 0 : take(H * 4);
    L->D = take(H * 4);
    L->theta = (d->flags & M3_FLAG_THETA_PER_HEAD) ? take(H * (N / 2) * es) : 0;
    L->wB = bcn ? take(N * 4) : 0;
    L->wC = bcn ? take(N * 4) : 0;
    L->bB = bcn ? take(H * R * N * 4) : 0;
    L->bC = bcn ? take(H * R * N * 4) : 0;
    const size_t gh = (size_t)L->group * H;
    for (int s = 0; s < 3; ++s) {
        L->st[s][0] = take(gh * N * P * 4);
        L->st[s][1] = take(gh * R * N * 4);
        L->st[s][2] = take(gh * R * P * 4);
    }
    const Rows rows = token_rows(d);
    const size_t toks = (size_t)L->group * (size_t)L->slice;
    for (int j = 0; j < 2; ++j)
        for (int t = 0; t < 8; ++t) L->slot[j][t] = rows.b[t] ? take(toks * rows.b[t]) : 0;
    // the scan's workspace: the largest any unit's shape asks for
    size_t need = 0;
    const int64_t Ts[4] = {L->slice, T - (L->nslice - 1) * L->slice, L->slice_last,
                           T - (L->nslice_last - 1) * L->slice_last};
    const int64_t Bs[2] = {L->group, Bt - (L->ngroup - 1) * L->group};
    for (int64_t b : Bs)
        for (int64_t t : Ts) {
            if (b <= 0) continue;
            m3_dims u = *d;
            u.batch = b;
            u.seqlen = t;
            size_t w = 0;
            const m3_status st = m3_scan_plan(M3_ALGO_AUTO, &u, &w, nullptr, nullptr);
            if (st != M3_OK) return st;
            need = std::max(need, w);
        }
    L->ws_bytes = need;
    L->ws = take(need);
    L->total = off;
    return M3_OK;
}

struct Span {
    uintptr_t lo, hi;
};
Span span(const void *p, size_t n) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return {a, a + (p ? n : 0)};
}
bool overlaps(Span a, Span b) { return a.hi > a.lo && b.hi > b.lo && a.lo < b.hi && b.lo < a.hi; }

// Copy the rows of batch entries [b0, b0+nb), tokens [t0, t0+tl) of a
// [batch, T, row] host tensor to (or from) a dense [nb, tl, row] device block.
cudaError_t copy_tokens(char *dev, const char *host_in, char *host_out, size_t row, int64_t b0, int64_t nb,
                        int64_t T, int64_t t0, int64_t tl, cudaStream_t s) {
    if (row == 0 || tl == 0 || nb == 0) return cudaSuccess;
    const size_t width = (size_t)tl * row, pitch = (size_t)T * row;
    const size_t first = ((size_t)b0 * T + t0) * row;
    const bool to_dev = host_in != nullptr;
    if (nb == 1)
        return to_dev ? cudaMemcpyAsync(dev, host_in + first, width, cudaMemcpyHostToDevice, s)
                      : cudaMemcpyAsync(host_out + first, dev, width, cudaMemcpyDeviceToHost, s);
    if (pitch < ((size_t)1 << 31))
        return to_dev ? cudaMemcpy2DAsync(dev, width, host_in + first, pitch, width, nb, cudaMemcpyHostToDevice, s)
                      : cudaMemcpy2DAsync(host_out + first, pitch, dev, width, width, nb, cudaMemcpyDeviceToHost, s);
    for (int64_t b = 0; b < nb; ++b) {  // pitch beyond what a 2D copy takes: one copy per sequence
        const cudaError_t e =
            to_dev ? cudaMemcpyAsync(dev + b * width, host_in + first + b * pitch, width, cudaMemcpyHostToDevice, s)
                   : cudaMemcpyAsync(host_out + first + b * pitch, dev + b * width, width, cudaMemcpyDeviceToHost, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

m3_status host_impl(const m3_dims *d, const m3_bcnorm *bcn, const void *x, const void *B, const void *C,
                    const void *dt, const void *lam, const void *theta, const float *A, const float *D,
                    const m3_state *init, void *y, const m3_state *fin, void *ws, size_t ws_bytes, void *stream) {
    Layout L{};
    m3_status st = m3_scan_plan(M3_ALGO_AUTO, d, nullptr, nullptr, nullptr);  // validates dims
    if (st != M3_OK) return st;
    if ((st = plan_layout(d, bcn != nullptr, &L)) != M3_OK) return st;
    const int64_t Bt = d->batch, T = d->seqlen, H = d->nheads;
    const int64_t N = d->dstate, P = d->headdim, R = d->rank;
    const size_t es = d->io == M3_BF16 ? 2 : 4;
    const int64_t tok = Bt * T * H;
    const bool a_tok = (d->flags & M3_FLAG_A_PER_TOKEN) != 0;
    const bool th_head = (d->flags & M3_FLAG_THETA_PER_HEAD) != 0;

    // ---- validation (host pointers: presence and overlaps; workspace: size)
    if (tok > 0 && (!x || !B || !C || !dt || !lam || !theta || !y))
        return m3::set_error(M3_ERR_INVALID_ARG, "x, B, C, dt, lam, theta and y are required");
    if (!A || !D) return m3::set_error(M3_ERR_INVALID_ARG, "A and D are required");
    if (bcn && (!bcn->wB || !bcn->wC || !bcn->bB || !bcn->bC))
        return m3::set_error(M3_ERR_INVALID_ARG, "bcn: wB, wC, bB and bC are all required");
    if (bcn && !(bcn->eps > 0.f)) return m3::set_error(M3_ERR_INVALID_ARG, "bcn eps must be > 0");
    const Rows rows = token_rows(d);
    const Span ins[8] = {span(x, tok / H * rows.b[0]), span(B, tok / H * rows.b[1]), span(C, tok / H * rows.b[2]),
                         span(dt, tok / H * rows.b[3]), span(lam, tok / H * rows.b[4]),
                         span(theta, th_head ? H * (N / 2) * es : tok / H * rows.b[5]),
                         span(A, (a_tok ? tok : H) * 4), span(D, H * 4)};
    const Span ys = span(y, tok / H * rows.b[7]);
    for (const Span &s : ins)
        if (overlaps(s, ys)) return m3::set_error(M3_ERR_INVALID_ARG, "y overlaps an input tensor");
    const int64_t BH = Bt * H;
    const size_t sbytes[3] = {(size_t)(BH * N * P * 4), (size_t)(BH * R * N * 4), (size_t)(BH * R * P * 4)};
    auto state_spans = [&](const m3_state *s, Span out[3], const char *what) -> m3_status {
        if (BH == 0) {
            out[0] = out[1] = out[2] = Span{0, 0};
            return M3_OK;
        }
        if (!s->h || !s->b_prev || !s->x_prev)
            return m3::set_error(M3_ERR_INVALID_ARG, what);
        out[0] = span(s->h, sbytes[0]);
        out[1] = span(s->b_prev, sbytes[1]);
        out[2] = span(s->x_prev, sbytes[2]);
        return M3_OK;
    };
    Span is[3] = {}, fs[3] = {};
    if (init && (st = state_spans(init, is, "init: h, b_prev and x_prev are all required")) != M3_OK) return st;
    if (fin && (st = state_spans(fin, fs, "final_state: h, b_prev and x_prev are all required")) != M3_OK)
        return st;
    for (int i = 0; i < 3; ++i) {
        for (const Span &s : ins)
            if (overlaps(fs[i], s) || overlaps(is[i], ys))
                return m3::set_error(M3_ERR_INVALID_ARG, "state buffers overlap the sequence tensors");
        if (overlaps(fs[i], ys)) return m3::set_error(M3_ERR_INVALID_ARG, "final_state overlaps y");
        for (int j = 0; j < 3; ++j) {
            const bool same = i == j && fs[i].lo == is[j].lo && fs[i].hi == is[j].hi;
            if ((i != j && overlaps(fs[i], fs[j])) || (i != j && overlaps(is[i], is[j])))
                return m3::set_error(M3_ERR_INVALID_ARG, "state buffers overlap each other");
            if (!same && overlaps(fs[i], is[j]))
                return m3::set_error(M3_ERR_INVALID_ARG, "final_state partially overlaps init");
        }
    }
    if (Bt == 0) return M3_OK;
    if (!ws || ws_bytes < L.total)
        return m3::set_error(M3_ERR_INVALID_ARG, "workspace too small (query m3_scan_host_plan)");
    if (reinterpret_cast<uintptr_t>(ws) % 16)
        return m3::set_error(M3_ERR_INVALID_ARG, "workspace must be 16-byte aligned");

    // ---- enqueue
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    Streams *S = nullptr;
    if (e == cudaSuccess) e = streams_for(dev, &S);
    if (e != cudaSuccess) return m3::set_cuda_error(e, "m3_scan_fwd_host (copy streams)");
    std::lock_guard<std::mutex> lk(S->call);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    char *w = static_cast<char *>(ws);
#define M3_TRY(call, where)                                          \
    do {                                                             \
        const cudaError_t e_ = (call);                               \
        if (e_ != cudaSuccess) return m3::set_cuda_error(e_, where); \
    } while (0)
    M3_TRY(cudaEventRecord(S->fork, cs), "m3_scan_fwd_host (fork)");
    M3_TRY(cudaStreamWaitEvent(S->in, S->fork, 0), "m3_scan_fwd_host (fork)");
    M3_TRY(cudaStreamWaitEvent(S->out, S->fork, 0), "m3_scan_fwd_host (fork)");
    if (!a_tok) M3_TRY(cudaMemcpyAsync(w + L.A, A, H * 4, cudaMemcpyHostToDevice, S->in), "m3_scan_fwd_host (A)");
    M3_TRY(cudaMemcpyAsync(w + L.D, D, H * 4, cudaMemcpyHostToDevice, S->in), "m3_scan_fwd_host (D)");
    if (th_head)
        M3_TRY(cudaMemcpyAsync(w + L.theta, theta, H * (N / 2) * es, cudaMemcpyHostToDevice, S->in),
               "m3_scan_fwd_host (theta)");
    m3_bcnorm dbcn{};  // the BC-norm parameters' device copies
    if (bcn) {
        const size_t nb = (size_t)N * 4, hb = (size_t)H * R * N * 4;
        M3_TRY(cudaMemcpyAsync(w + L.wB, bcn->wB, nb, cudaMemcpyHostToDevice, S->in), "m3_scan_fwd_host (bcn)");
        M3_TRY(cudaMemcpyAsync(w + L.wC, bcn->wC, nb, cudaMemcpyHostToDevice, S->in), "m3_scan_fwd_host (bcn)");
        M3_TRY(cudaMemcpyAsync(w + L.bB, bcn->bB, hb, cudaMemcpyHostToDevice, S->in), "m3_scan_fwd_host (bcn)");
        M3_TRY(cudaMemcpyAsync(w + L.bC, bcn->bC, hb, cudaMemcpyHostToDevice, S->in), "m3_scan_fwd_host (bcn)");
        dbcn = m3_bcnorm{reinterpret_cast<const float *>(w + L.wB), reinterpret_cast<const float *>(w + L.wC),
                         reinterpret_cast<const float *>(w + L.bB), reinterpret_cast<const float *>(w + L.bC),
                         bcn->eps};
    }
    const void *hin[8] = {x, B, C, dt, lam, theta, A, nullptr};
    int64_t k = 0;
    for (int64_t g = 0; g < L.ngroup; ++g) {
        const int64_t b0 = g * L.group, nb = std::min(L.group, Bt - b0);
        const bool last_group = g == L.ngroup - 1;
        const int64_t ns = last_group ? L.nslice_last : L.nslice, sl = last_group ? L.slice_last : L.slice;
        for (int64_t i = 0; i < ns; ++i, ++k) {
            const int64_t t0 = i * sl, tl = std::min(sl, T - t0);
            const int j = (int)(k & 1);
            // copy-in: wait until unit k-2 no longer reads this slot
            if (k >= 2) M3_TRY(cudaStreamWaitEvent(S->in, S->computed[j], 0), "m3_scan_fwd_host (copy-in wait)");
            if (i == 0 && init) {
                // the initial-state buffer is shared by all groups: wait for the
                // previous unit's kernels, which follow the last reader of it
                if (k >= 1)
                    M3_TRY(cudaStreamWaitEvent(S->in, S->computed[j ^ 1], 0), "m3_scan_fwd_host (copy-in wait)");
                const void *src[3] = {init->h, init->b_prev, init->x_prev};
                for (int q = 0; q < 3; ++q) {
                    const size_t per = sbytes[q] / (size_t)Bt;
                    M3_TRY(cudaMemcpyAsync(w + L.st[0][q], static_cast<const char *>(src[q]) + b0 * per, nb * per,
                                           cudaMemcpyHostToDevice, S->in),
                           "m3_scan_fwd_host (init)");
                }
            }
            for (int t = 0; t < 7; ++t)
                M3_TRY(copy_tokens(w + L.slot[j][t], static_cast<const char *>(hin[t]), nullptr, rows.b[t], b0, nb,
                                   T, t0, tl, S->in),
                       "m3_scan_fwd_host (copy-in)");
            M3_TRY(cudaEventRecord(S->loaded[j], S->in), "m3_scan_fwd_host (copy-in)");

            // kernels, on the caller's stream
            M3_TRY(cudaStreamWaitEvent(cs, S->loaded[j], 0), "m3_scan_fwd_host (compute wait)");
            if (k >= 2) M3_TRY(cudaStreamWaitEvent(cs, S->drained[j], 0), "m3_scan_fwd_host (compute wait)");
            if (i == 0 && k >= 1 && fin)  // the previous group's final state may still be on its way out
                M3_TRY(cudaStreamWaitEvent(cs, S->drained[j ^ 1], 0), "m3_scan_fwd_host (compute wait)");
            m3_dims u = *d;
            u.batch = nb;
            u.seqlen = tl;
            const int pin = i == 0 ? 0 : 1 + (int)((i - 1) & 1), pout = 1 + (int)(i & 1);
            m3_state sin{reinterpret_cast<float *>(w + L.st[pin][0]), reinterpret_cast<float *>(w + L.st[pin][1]),
                         reinterpret_cast<float *>(w + L.st[pin][2])};
            m3_state sout{reinterpret_cast<float *>(w + L.st[pout][0]), reinterpret_cast<float *>(w + L.st[pout][1]),
                          reinterpret_cast<float *>(w + L.st[pout][2])};
            const bool zero_init = i == 0 && !init;
            const void *uth = th_head ? w + L.theta : w + L.slot[j][5];
            const float *uA = reinterpret_cast<const float *>(a_tok ? w + L.slot[j][6] : w + L.A);
            const float *uD = reinterpret_cast<const float *>(w + L.D);
            st = bcn ? m3_scan_fwd_bcnorm(M3_ALGO_AUTO, &u, &dbcn, w + L.slot[j][0], w + L.slot[j][1],
                                          w + L.slot[j][2], w + L.slot[j][3], w + L.slot[j][4], uth, uA, uD,
                                          zero_init ? nullptr : &sin, w + L.slot[j][7], &sout, w + L.ws,
                                          L.ws_bytes, cs)
                     : m3_scan_fwd(&u, w + L.slot[j][0], w + L.slot[j][1], w + L.slot[j][2], w + L.slot[j][3],
                                   w + L.slot[j][4], uth, uA, uD, zero_init ? nullptr : &sin, w + L.slot[j][7],
                                   &sout, w + L.ws, L.ws_bytes, cs);
            if (st != M3_OK) return st;
            M3_TRY(cudaEventRecord(S->computed[j], cs), "m3_scan_fwd_host (compute)");

            // copy-out
            M3_TRY(cudaStreamWaitEvent(S->out, S->computed[j], 0), "m3_scan_fwd_host (copy-out wait)");
            M3_TRY(copy_tokens(w + L.slot[j][7], nullptr, static_cast<char *>(y), rows.b[7], b0, nb, T, t0, tl,
                               S->out),
                   "m3_scan_fwd_host (copy-out)");
            if (i == ns - 1 && fin) {
                void *dst[3] = {fin->h, fin->b_prev, fin->x_prev};
                for (int q = 0; q < 3; ++q) {
                    const size_t per = sbytes[q] / (size_t)Bt;
                    M3_TRY(cudaMemcpyAsync(static_cast<char *>(dst[q]) + b0 * per, w + L.st[pout][q], nb * per,
                                           cudaMemcpyDeviceToHost, S->out),
                           "m3_scan_fwd_host (final state)");
                }
            }
            M3_TRY(cudaEventRecord(S->drained[j], S->out), "m3_scan_fwd_host (copy-out)");
        }
    }
    M3_TRY(cudaEventRecord(S->join, S->out), "m3_scan_fwd_host (join)");
    M3_TRY(cudaStreamWaitEvent(cs, S->join, 0), "m3_scan_fwd_host (join)");
#undef M3_TRY
    return M3_OK;
}

}  // namespace

extern "C" {

m3_status m3_scan_host_plan(const m3_dims *d, int with_bcnorm, size_t *workspace_bytes, int64_t *slice_tokens,
                            int64_t *last_slice_tokens, int64_t *group_batch, int64_t *units) {
    try {
        m3_status st = m3_scan_plan(M3_ALGO_AUTO, d, nullptr, nullptr, nullptr);
        if (st != M3_OK) return st;
        Layout L{};
        if ((st = plan_layout(d, with_bcnorm != 0, &L)) != M3_OK) return st;
        if (workspace_bytes) *workspace_bytes = d->batch > 0 ? L.total : 0;
        if (slice_tokens) *slice_tokens = L.slice;
        if (last_slice_tokens) *last_slice_tokens = L.slice_last;
        if (group_batch) *group_batch = L.group;
        if (units) *units = d->batch > 0 ? L.nslice * (L.ngroup - 1) + L.nslice_last : 0;
        return M3_OK;
    } catch (...) {
        return m3::set_error(M3_ERR_INVALID_ARG, "internal error");
    }
}

m3_status m3_scan_fwd_host(const m3_dims *d, const m3_bcnorm *bcn, const void *x, const void *B, const void *C,
                           const void *dt, const void *lam, const void *theta, const float *A, const float *D,
                           const m3_state *init, void *y, const m3_state *final_state, void *workspace,
                           size_t workspace_bytes, void *stream) {
    try {
        return host_impl(d, bcn, x, B, C, dt, lam, theta, A, D, init, y, final_state, workspace, workspace_bytes,
                         stream);
    } catch (...) {
        return m3::set_error(M3_ERR_INVALID_ARG, "internal error");
    }
}

}  // extern "C"
