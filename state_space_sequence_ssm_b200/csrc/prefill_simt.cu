// prefill_simt.cu -- fp32 CUDA-core chunked prefill scan.
//
// One CTA per (batch, head) walks the sequence chunk by chunk.  Inside a
// chunk it evaluates the four pieces of the chunked SSD algorithm ("La
// dualità: Mamba-2 e Mamba-3", section "Perché conviene: i tensor core"):
// (i) the masked, decay-weighted C~ B~^T block times X, (ii) the chunk's own
// state contribution, (iii) the state carried from chunk to chunk, and
// (iv) that carried state read out through the decay since the chunk start.
// Two extensions carry the method of "Знакомство с Mamba-3" (sections 1-3):
//   - the trapezoid's previous-token write is folded into the per-token
//     coefficient gamma_hat_s = lam_s dt_s + (1 - lam_{s+1}) dt_{s+1} for every
//     off-diagonal (s < t) entry, the diagonal keeping gamma_t = lam_t dt_t;
//   - B and C are rotated pair-wise by the chunk-local cumulative angle
//     phi_t = sum_{s=c0..t} dt_s theta_s, and the carried state is kept in the
//     plain frame: h*_c = Rot(-Phi_c)(exp(cA_end) h*_{c-1} + G_c), so no
//     angle ever exceeds one chunk's sum (fp32 stays accurate at any length).
// All arithmetic is fp32 with accurate expf/sincosf; this is the path for
// fp32 I/O and the in-repo cross-check of the tensor-core kernel.
#include <cuda_bf16.h>

#include "bcnorm.cuh"
#include "dcheck.cuh"
#include "m3_internal.h"

namespace m3 {
namespace {

// Index-check sites of this file (bounds build).
enum : unsigned {
    kSiteScalars = 0x301,  // dt, lam, A, D
    kSiteTheta = 0x302,    // angle rates
    kSiteRows = 0x303,     // x, B, C rows
    kSiteNorm = 0x304,     // BC-norm weights and biases
    kSiteInit = 0x305,     // initial state h0, b_prev, x_prev
    kSiteY = 0x306,        // output rows
    kSiteFinal = 0x307,    // final state
};

// Element i of a buffer of n elements (the bounds build checks i and reads 0
// outside; `site` names the access).
template <typename T>
__device__ __forceinline__ float ldv(const T *p, int64_t i, int64_t n, unsigned site);
template <>
__device__ __forceinline__ float ldv<float>(const float *p, int64_t i, int64_t n, unsigned site) {
    return dchk::in(site, i, 1, n) ? p[i] : 0.f;
}
template <>
__device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i, int64_t n, unsigned site) {
    return dchk::in(site, i, 1, n) ? __bfloat162float(p[i]) : 0.f;
}
// Four consecutive values (i a multiple of 4; the row they lie in starts
// 16-byte aligned for fp32, 8-byte aligned for bf16).
template <typename T>
__device__ __forceinline__ float4 ldv4(const T *p, int64_t i, int64_t n, unsigned site);
template <>
__device__ __forceinline__ float4 ldv4<float>(const float *p, int64_t i, int64_t n, unsigned site) {
    if (!dchk::in(site, i, 4, n)) return make_float4(0.f, 0.f, 0.f, 0.f);
    return __ldg(reinterpret_cast<const float4 *>(p + i));
}
template <>
__device__ __forceinline__ float4 ldv4<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i, int64_t n, unsigned site) {
    if (!dchk::in(site, i, 4, n)) return make_float4(0.f, 0.f, 0.f, 0.f);
    const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p + i));
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}
template <typename T>
__device__ __forceinline__ void stv(T *p, int64_t i, int64_t n, unsigned site, float v);
template <>
__device__ __forceinline__ void stv<float>(float *p, int64_t i, int64_t n, unsigned site, float v) {
    if (dchk::in(site, i, 1, n)) p[i] = v;
}
template <>
__device__ __forceinline__ void stv<__nv_bfloat16>(__nv_bfloat16 *p, int64_t i, int64_t n, unsigned site, float v) {
    if (dchk::in(site, i, 1, n)) p[i] = __float2bfloat16_rn(v);
}

template <typename IO>
struct SimtArgs {
    int64_t Bt, T, H;
    int P, N, R, Q;  // Q tokens per chunk, rows = Q * R
    const IO *x, *B, *C, *dt, *lam, *theta;
    const float *A, *D;
    int a_tok;    // A is [Bt, T, H] (per token-head)
    int th_head;  // theta is [H, N/2] (fixed per head)
    const float *wB, *wC, *bB, *bC;  // BC-norm prologue (wB == nullptr: off)
    float eps;
    const float *h0, *bp0, *xp0;
    IO *y;
    float *hT, *bpT, *xpT;
};

constexpr int kThreads = 256;

// B and C rows are N + 1 floats apart in shared memory: with an odd stride,
// threads that read the same column of consecutive rows hit distinct banks.
__host__ __device__ inline size_t simt_smem_floats(int P, int N, int R, int Q) {
    const size_t rows = (size_t)Q * R;
    return rows * P + 2 * rows * (N + 1) + rows * rows + (size_t)N * P + 6 * (size_t)Q + 3 * (size_t)(N / 2) +
           (size_t)Q * (N / 2);
}

template <typename IO>
__global__ void __launch_bounds__(kThreads) prefill_simt_kernel(const SimtArgs<IO> a) {
    extern __shared__ float smem[];
    const int P = a.P, N = a.N, R = a.R, Q = a.Q, K2 = N / 2, NS = N + 1;
    const int rowsmax = Q * R;
    float *Xs = smem;                       // [rows][P]
    float *Bs = Xs + rowsmax * P;           // [rows][NS]  (rotated in place)
    float *Cs = Bs + rowsmax * NS;          // [rows][NS]  (rotated in place)
    float *Pm = Cs + rowsmax * NS;          // [rows][rows] masked scores
    float *hs = Pm + rowsmax * rowsmax;     // [N][P] carried plain-frame state
    float *dts = hs + N * P;                // [Q] dt
    float *cA = dts + Q;                    // [Q] chunk-local cumulative dt*A
    float *gam = cA + Q;                    // [Q] lam*dt (diagonal weight)
    float *ghat = gam + Q;                  // [Q] lam*dt + (1-lam')dt' (off-diagonal weight)
    float *wst = ghat + Q;                  // [Q] chunk-state weight
    float *scr = wst + Q;                   // [Q] scratch (1-lam)*dt
    float *phiE = scr + Q;                  // [N/2] chunk-end angle
    float *cosE = phiE + K2;                // [N/2]
    float *sinE = cosE + K2;                // [N/2]
    float *phis = sinE + K2;                // [Q][N/2] chunk-local cumulative angles

    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / a.H, h = bh % a.H;
    const int64_t T = a.T, H = a.H;
    auto tok = [&](int64_t t) { return (b * T + t) * H + h; };  // token-head index
    // buffer extents in elements, for the bounds build's index checks
    const int64_t BH = gridDim.x, nTok = BH * T, nX = nTok * R * P, nBC = nTok * R * N, nSt = BH * N * P;
    const float Ah = a.a_tok ? 0.f : ldv(a.A, h, H, kSiteScalars), Dh = ldv(a.D, h, H, kSiteScalars);

    // ---- initial state: h0 + beta'_0 * b_prev x_prev^T (pending write of token -1)
    float betap0 = 0.f;
    if (T > 0) {
        const float d0 = ldv(a.dt, tok(0), nTok, kSiteScalars), l0 = ldv(a.lam, tok(0), nTok, kSiteScalars);
        betap0 = (1.f - l0) * d0;
    }
    for (int idx = tid; idx < N * P; idx += kThreads) {
        const int n = idx / P, p = idx % P;
        float v = a.h0 ? ldv(a.h0, bh * N * P + idx, nSt, kSiteInit) : 0.f;
        if (a.bp0 && a.xp0 && T > 0) {
            float acc = 0.f;
            for (int r = 0; r < R; ++r)
                acc += ldv(a.bp0, (bh * R + r) * N + n, BH * R * N, kSiteInit) *
                       ldv(a.xp0, (bh * R + r) * P + p, BH * R * P, kSiteInit);
            v += betap0 * acc;
        }
        hs[idx] = v;
    }
    __syncthreads();

    for (int64_t t0 = 0; t0 < T; t0 += Q) {
        const int L = (int)((T - t0) < Q ? (T - t0) : Q);
        const int rows = L * R;
        const bool last_chunk = (t0 + L == T);

        // ---- load the chunk (rows = (token, rank)), four values per load where
        //      the rows allow it (every load of a loop is independent)
        if (P % 4 == 0) {
            const int P4 = P / 4;
#pragma unroll 4
            for (int idx = tid; idx < rows * P4; idx += kThreads) {
                const int i = idx / P4, p = 4 * (idx % P4);
                *reinterpret_cast<float4 *>(Xs + i * P + p) =
                    ldv4(a.x, (tok(t0 + i / R) * R + i % R) * P + p, nX, kSiteRows);
            }
        } else {
            for (int idx = tid; idx < rows * P; idx += kThreads) {
                const int i = idx / P, p = idx % P;
                Xs[idx] = ldv(a.x, (tok(t0 + i / R) * R + i % R) * P + p, nX, kSiteRows);
            }
        }
        if (N % 4 == 0) {
            const int N4 = N / 4;
#pragma unroll 4
            for (int idx = tid; idx < rows * N4; idx += kThreads) {
                const int i = idx / N4, n = 4 * (idx % N4);
                const int64_t g = (tok(t0 + i / R) * R + i % R) * N + n;
                const float4 vb = ldv4(a.B, g, nBC, kSiteRows), vc = ldv4(a.C, g, nBC, kSiteRows);
                float *bd = Bs + i * NS + n, *cd = Cs + i * NS + n;
                bd[0] = vb.x; bd[1] = vb.y; bd[2] = vb.z; bd[3] = vb.w;
                cd[0] = vc.x; cd[1] = vc.y; cd[2] = vc.z; cd[3] = vc.w;
            }
        } else {
            for (int idx = tid; idx < rows * N; idx += kThreads) {
                const int i = idx / N, n = idx % N;
                const int64_t g = (tok(t0 + i / R) * R + i % R) * N + n;
                Bs[i * NS + n] = ldv(a.B, g, nBC, kSiteRows);
                Cs[i * NS + n] = ldv(a.C, g, nBC, kSiteRows);
            }
        }
        for (int s = tid; s < L; s += kThreads) {
            const int64_t t = t0 + s;
            const float d = ldv(a.dt, tok(t), nTok, kSiteScalars), l = ldv(a.lam, tok(t), nTok, kSiteScalars);
            dts[s] = d;
            cA[s] = d * (a.a_tok ? ldv(a.A, tok(t), nTok, kSiteScalars) : Ah);
            gam[s] = l * d;
            float nxt = 0.f;  // (1 - lam_{t+1}) dt_{t+1}; absent after the last token
            if (t + 1 < T) {
                const float d1 = ldv(a.dt, tok(t + 1), nTok, kSiteScalars);
                const float l1 = ldv(a.lam, tok(t + 1), nTok, kSiteScalars);
                nxt = (1.f - l1) * d1;
            }
            ghat[s] = l * d + nxt;
        }
        __syncthreads();
        if (a.wB) {  // BC-norm prologue: one warp per (token, rank) row of B, then of C
            const int warp = tid >> 5, lane = tid & 31;
            for (int row = warp; row < 2 * rows; row += kThreads / 32) {
                const bool isB = row < rows;
                float *v = isB ? Bs + row * NS : Cs + (row - rows) * NS;
                const int r = (isB ? row : row - rows) % R;
                const float *w = isB ? a.wB : a.wC;
                const float *bias = isB ? a.bB : a.bC;
                const float sc = bcn_row_scale_warp([&](int n) { return v[n]; }, N, a.eps);
                for (int n = lane; n < N; n += 32)
                    v[n] = fmaf(v[n] * sc, ldv(w, n, N, kSiteNorm), ldv(bias, (h * R + r) * N + n, H * R * N, kSiteNorm));
            }
            __syncthreads();
        }
        if (tid == 0) {  // chunk-local inclusive prefix of dt*A
            float run = 0.f;
            for (int s = 0; s < L; ++s) { run += cA[s]; cA[s] = run; }
        }
        // ---- rotate B and C by the chunk-local cumulative angle: the angle
        //      increments dt_s theta_s[k], their running sum over the chunk's
        //      tokens (one thread per pair, in token order), then every (row,
        //      pair) rotated by its token's angle in parallel
#pragma unroll 4
        for (int idx = tid; idx < L * K2; idx += kThreads) {
            const int s = idx / K2, k = idx % K2;
            phis[idx] = dts[s] * ldv(a.theta, (a.th_head ? (int64_t)h : tok(t0 + s)) * K2 + k,
                                     (a.th_head ? H : nTok) * K2, kSiteTheta);
        }
        __syncthreads();
        for (int k = tid; k < K2; k += kThreads) {
            float phi = 0.f;
            for (int s = 0; s < L; ++s) {
                phi += phis[s * K2 + k];
                phis[s * K2 + k] = phi;
            }
            phiE[k] = phi;
            float sn, cs;
            sincosf(phi, &sn, &cs);
            cosE[k] = cs;
            sinE[k] = sn;
        }
        __syncthreads();
        for (int idx = tid; idx < rows * K2; idx += kThreads) {
            const int i = idx / K2, k = idx % K2;
            float sn, cs;
            sincosf(phis[(i / R) * K2 + k], &sn, &cs);
            float u = Bs[i * NS + 2 * k], v = Bs[i * NS + 2 * k + 1];
            Bs[i * NS + 2 * k] = u * cs - v * sn;
            Bs[i * NS + 2 * k + 1] = u * sn + v * cs;
            u = Cs[i * NS + 2 * k];
            v = Cs[i * NS + 2 * k + 1];
            Cs[i * NS + 2 * k] = u * cs - v * sn;
            Cs[i * NS + 2 * k + 1] = u * sn + v * cs;
        }
        __syncthreads();
        const float cAe = cA[L - 1];
        for (int s = tid; s < L; s += kThreads) {
            // weight of token s in the chunk-end state; the sequence's very
            // last token has no successor, so only its own lam*dt applies.
            const float g = (last_chunk && s == L - 1) ? gam[s] : ghat[s];
            wst[s] = expf(cAe - cA[s]) * g;
        }
        // ---- (i) masked decay-weighted scores: mask applied before exp.  Each
        //      thread owns a 4 x 4 tile of rows i = it + TI a, columns
        //      j = jt + TI b (a, b < 4): 16 products per 8 shared-memory loads
        const int TI = (rows + 3) / 4;
        for (int tt = tid; tt < TI * TI; tt += kThreads) {
            const int it = tt / TI, jt = tt % TI;
            float acc[4][4] = {};
            for (int n = 0; n < N; ++n) {
                float c[4], bv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i = it + TI * q, j = jt + TI * q;
                    c[q] = i < rows ? Cs[i * NS + n] : 0.f;
                    bv[q] = j < rows ? Bs[j * NS + n] : 0.f;
                }
#pragma unroll
                for (int qa = 0; qa < 4; ++qa)
#pragma unroll
                    for (int qb = 0; qb < 4; ++qb) acc[qa][qb] = fmaf(c[qa], bv[qb], acc[qa][qb]);
            }
#pragma unroll
            for (int qa = 0; qa < 4; ++qa)
#pragma unroll
                for (int qb = 0; qb < 4; ++qb) {
                    const int i = it + TI * qa, j = jt + TI * qb;
                    if (i >= rows || j >= rows) continue;
                    const int ti = i / R, tj = j / R;
                    float v = 0.f;
                    if (tj <= ti) {
                        const float coef = (ti == tj) ? gam[ti] : ghat[tj];
                        v = acc[qa][qb] * expf(cA[ti] - cA[tj]) * coef;
                    }
                    Pm[i * rows + j] = v;
                }
        }
        __syncthreads();
        // ---- outputs: (i) diagonal block + (iv) carried-state readout + skip,
        //      4 x 4 tiles of rows i = it + TI a and columns p = pt + TP b
        const int TP = (P + 3) / 4;
        for (int tt = tid; tt < TI * TP; tt += kThreads) {
            const int it = tt / TP, pt = tt % TP;
            float dg[4][4] = {}, of[4][4] = {};
            for (int j = 0; j < rows; ++j) {
                float pm[4], xv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i = it + TI * q, p = pt + TP * q;
                    pm[q] = i < rows ? Pm[i * rows + j] : 0.f;
                    xv[q] = p < P ? Xs[j * P + p] : 0.f;
                }
#pragma unroll
                for (int qa = 0; qa < 4; ++qa)
#pragma unroll
                    for (int qb = 0; qb < 4; ++qb) dg[qa][qb] = fmaf(pm[qa], xv[qb], dg[qa][qb]);
            }
            for (int n = 0; n < N; ++n) {
                float c[4], hv[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i = it + TI * q, p = pt + TP * q;
                    c[q] = i < rows ? Cs[i * NS + n] : 0.f;
                    hv[q] = p < P ? hs[n * P + p] : 0.f;
                }
#pragma unroll
                for (int qa = 0; qa < 4; ++qa)
#pragma unroll
                    for (int qb = 0; qb < 4; ++qb) of[qa][qb] = fmaf(c[qa], hv[qb], of[qa][qb]);
            }
#pragma unroll
            for (int qa = 0; qa < 4; ++qa) {
                const int i = it + TI * qa;
                if (i >= rows) continue;
                const float ei = expf(cA[i / R]);
#pragma unroll
                for (int qb = 0; qb < 4; ++qb) {
                    const int p = pt + TP * qb;
                    if (p >= P) continue;
                    const float yv = dg[qa][qb] + ei * of[qa][qb] + Dh * Xs[i * P + p];
                    stv(a.y, (tok(t0 + i / R) * R + i % R) * P + p, nX, kSiteY, yv);
                }
            }
        }
        __syncthreads();
        // ---- (ii)+(iii): h* <- Rot(-Phi)(exp(cA_end) h* + G), tiles of 2 pairs
        //      k = kt + TK a (a < 2) by 4 columns p = pt + TP b
        const float eA = expf(cAe);
        const int TK = (K2 + 1) / 2;
        for (int tt = tid; tt < TK * TP; tt += kThreads) {
            const int kt = tt / TP, pt = tt % TP;
            float g[2][2][4] = {};  // [pair][row of the pair][column]
            for (int j = 0; j < rows; ++j) {
                const float w = wst[j / R];
                float wx[4], bu[2], bv[2];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int p = pt + TP * q;
                    wx[q] = p < P ? w * Xs[j * P + p] : 0.f;
                }
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int k = kt + TK * q;
                    bu[q] = k < K2 ? Bs[j * NS + 2 * k] : 0.f;
                    bv[q] = k < K2 ? Bs[j * NS + 2 * k + 1] : 0.f;
                }
#pragma unroll
                for (int qa = 0; qa < 2; ++qa)
#pragma unroll
                    for (int qb = 0; qb < 4; ++qb) {
                        g[qa][0][qb] = fmaf(bu[qa], wx[qb], g[qa][0][qb]);
                        g[qa][1][qb] = fmaf(bv[qa], wx[qb], g[qa][1][qb]);
                    }
            }
#pragma unroll
            for (int qa = 0; qa < 2; ++qa) {
                const int k = kt + TK * qa;
                if (k >= K2) continue;
                const float cs = cosE[k], sn = sinE[k];
#pragma unroll
                for (int qb = 0; qb < 4; ++qb) {
                    const int p = pt + TP * qb;
                    if (p >= P) continue;
                    const float u = eA * hs[(2 * k) * P + p] + g[qa][0][qb];
                    const float v = eA * hs[(2 * k + 1) * P + p] + g[qa][1][qb];
                    hs[(2 * k) * P + p] = u * cs + v * sn;
                    hs[(2 * k + 1) * P + p] = -u * sn + v * cs;
                }
            }
        }
        __syncthreads();
    }

    // ---- final state: plain-frame h_{T-1} and the raw last token as pending
    if (a.hT) {
        for (int idx = tid; idx < N * P; idx += kThreads) {
            float v = hs[idx];
            if (T == 0) v = a.h0 ? ldv(a.h0, bh * N * P + idx, nSt, kSiteInit) : 0.f;
            stv(a.hT, bh * N * P + idx, nSt, kSiteFinal, v);
        }
    }
    if (a.bpT && a.wB && T > 0) {  // the last token's normalised B, one warp per rank row
        const int warp = tid >> 5, lane = tid & 31;
        for (int r = warp; r < R; r += kThreads / 32) {
            const int64_t src = tok(T - 1) * R * N + r * N;
            const float sc = bcn_row_scale_warp([&](int n) { return ldv(a.B, src + n, nBC, kSiteFinal); }, N, a.eps);
            for (int n = lane; n < N; n += 32)
                stv(a.bpT, (bh * R + r) * N + n, BH * R * N, kSiteFinal,
                    fmaf(ldv(a.B, src + n, nBC, kSiteFinal) * sc, ldv(a.wB, n, N, kSiteNorm),
                         ldv(a.bB, (h * R + r) * N + n, H * R * N, kSiteNorm)));
        }
    } else if (a.bpT) {
        for (int idx = tid; idx < R * N; idx += kThreads)
            stv(a.bpT, bh * R * N + idx, BH * R * N, kSiteFinal,
                T > 0 ? ldv(a.B, tok(T - 1) * R * N + idx, nBC, kSiteFinal)
                      : (a.bp0 ? ldv(a.bp0, bh * R * N + idx, BH * R * N, kSiteInit) : 0.f));
    }
    if (a.xpT) {
        for (int idx = tid; idx < R * P; idx += kThreads)
            stv(a.xpT, bh * R * P + idx, BH * R * P, kSiteFinal,
                T > 0 ? ldv(a.x, tok(T - 1) * R * P + idx, nX, kSiteFinal)
                      : (a.xp0 ? ldv(a.xp0, bh * R * P + idx, BH * R * P, kSiteInit) : 0.f));
    }
}

template <typename IO>
cudaError_t launch_typed(const Problem &p, const char **why) {
    SimtArgs<IO> a;
    a.Bt = p.Bt; a.T = p.T; a.H = p.H;
    a.P = (int)p.P; a.N = (int)p.N; a.R = (int)p.R;
    a.x = (const IO *)p.x; a.B = (const IO *)p.B; a.C = (const IO *)p.C;
    a.dt = (const IO *)p.dt; a.lam = (const IO *)p.lam; a.theta = (const IO *)p.theta;
    a.A = p.A; a.D = p.D; a.h0 = p.h0; a.bp0 = p.bp0; a.xp0 = p.xp0;
    a.a_tok = p.a_tok;
    a.th_head = p.th_head;
    a.wB = p.wB; a.wC = p.wC; a.bB = p.bB; a.bC = p.bC; a.eps = p.eps;
    a.y = (IO *)p.y; a.hT = p.hT; a.bpT = p.bpT; a.xpT = p.xpT;
    // largest chunk (<= 64 rows) whose working set fits in shared memory
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int maxsm = 0;
    e = cudaDeviceGetAttribute(&maxsm, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    int Q = 64 / a.R > 0 ? 64 / a.R : 1;
    while (Q > 1 && simt_smem_floats(a.P, a.N, a.R, Q) * sizeof(float) > (size_t)maxsm) Q /= 2;
    const size_t smem = simt_smem_floats(a.P, a.N, a.R, Q) * sizeof(float);
    if (smem > (size_t)maxsm) {
        *why = "prefill (SIMT): state too large for shared memory";
        return cudaErrorNotSupported;
    }
    a.Q = Q;
    e = cudaFuncSetAttribute(prefill_simt_kernel<IO>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = p.Bt * p.H;
    if (grid == 0) return cudaSuccess;
    prefill_simt_kernel<IO><<<(unsigned)grid, kThreads, smem, p.stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_simt(const Problem &p, const char **why) {
    return p.bf16 ? launch_typed<__nv_bfloat16>(p, why) : launch_typed<float>(p, why);
}

M3_DCHECK_READER(read_dcheck_simt)

}  // namespace m3
