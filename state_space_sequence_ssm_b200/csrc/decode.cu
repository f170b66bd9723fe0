// decode.cu -- single-token decode step against a resident fp32 state.
//
// The recurrent form of the method, one token per (batch, head):
//   h <- h + (1 - lam) dt * b_prev x_prev^T          (trapezoid, previous token)
//   h <- exp(dt A) Rot(-dt theta) h                  (decay + pair rotation)
//   h <- h + lam dt * B x^T                          (trapezoid, current token)
//   y  = h^T C + D x ;   b_prev <- B, x_prev <- x
// ("Знакомство с Mamba-3", sections 1-3: three-term recurrence, complex state
// as 2x2 rotations, rank-R MIMO write and readout).
//
// The step is HBM-bound: the N x P fp32 state is read and written exactly
// once with 128-bit streaming accesses; everything else (rotation, both
// trapezoid writes, readout) is fused into that single pass.  One CTA owns
// one (batch, head) slice.  Thread (kk, cg) holds column group cg (4
// consecutive p) of pairs kk, kk + K2/PT, ... so that both rows of a pair
// live in one thread (the rotation needs no exchange); the readout's sum over
// N is a warp shuffle plus one shared-memory pass.
#include <cuda_bf16.h>

#include "bcnorm.cuh"
#include "dcheck.cuh"
#include "m3_internal.h"
#include "tc_primitives.cuh"

namespace m3 {

// Device-side failure word of the decode kernels (bounded waits that gave up).
__device__ unsigned g_decode_error;

namespace {

// Index-check sites of this file (bounds build).
enum : unsigned {
    kSiteScalars = 0x401,  // dt, lam, A, D
    kSiteTheta = 0x402,    // angle rates
    kSiteVec = 0x403,      // x, B, C of the step
    kSiteNorm = 0x404,     // BC-norm weights and biases
    kSiteState = 0x405,    // the state h
    kSitePend = 0x406,     // b_prev, x_prev
    kSiteY = 0x407,        // output
    kSiteProj = 0x408,     // MIMO projection weights
};

// Element i of a buffer of n elements (the bounds build checks i and reads 0
// outside; `site` names the access).
template <typename T>
__device__ __forceinline__ float ldv(const T *p, int64_t i, int64_t n, unsigned site);
template <>
__device__ __forceinline__ float ldv<float>(const float *p, int64_t i, int64_t n, unsigned site) {
    return dchk::in(site, i, 1, n) ? __ldg(p + i) : 0.f;
}
template <>
__device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i, int64_t n, unsigned site) {
    return dchk::in(site, i, 1, n) ? __bfloat162float(p[i]) : 0.f;
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
// Plain fp32 element (state side buffers, per-head parameters), checked like ldv.
__device__ __forceinline__ float ldf(const float *p, int64_t i, int64_t n, unsigned site) {
    return dchk::in(site, i, 1, n) ? p[i] : 0.f;
}
template <typename IO>
struct StepArgs {
    int64_t BH, H;
    int P, N, R;
    const IO *x, *B, *C, *dt, *lam, *theta;
    const float *A, *D;
    float *h, *bp, *xp;
    IO *y;
};

// The optional features, a kernel argument of their own: growing StepArgs
// changed the plain kernel's code generation (and cost it 7 % of its
// bandwidth), a second argument does not.
struct StepFeat {
    int a_tok;    // A is [Bt, H] (per token-head) instead of [H]
    int th_head;  // theta is [H, N/2] (fixed per head)
    const float *wB, *wC, *bB, *bC;  // BC-norm prologue (wB == nullptr: off)
    float eps;
    // MIMO projections (pwx == nullptr: off): x, B, C, y hold one row per
    // slice; wx, wy [H, R, P] and wB, wC [H, R, N] widen them to rank R
    const float *pwx, *pwB, *pwC, *pwy;
};

// Register-tiled kernel for the common sizes.  Each thread owns PT pairs x 4
// columns of the state (both rows of each pair, so the rotation is local);
// the slice's small per-token vectors (b_prev, x_prev, B, C, x and the
// decay-scaled cos/sin of each pair's angle) are staged once in shared memory
// with coalesced loads while the state loads are in flight.
template <int N, int P, int R, typename IO>
struct StepCfg {
    static constexpr int K2 = N / 2;
    static constexpr int CG = P / 4;        // column groups (float4)
    static constexpr int PT = 4;            // pairs per thread
    static constexpr int KK = K2 / PT;      // pair groups
    static constexpr int THREADS = KK * CG;
    static constexpr int WARPS = THREADS / 32;
    static_assert(K2 % PT == 0, "pairs must split evenly");
    static_assert(THREADS % 32 == 0 && THREADS <= 1024, "bad block size");
    static_assert(32 % CG == 0 || CG % 32 == 0, "column groups must tile a warp");
};

// GEN = false: the plain method (A per head, theta per token, no BC-norm),
// compiled without the optional features' branches; GEN = true reads them
// from the arguments.
template <int N, int P, int R, typename IO, bool GEN>
__global__ void __launch_bounds__(StepCfg<N, P, R, IO>::THREADS)
step_kernel(const StepArgs<IO> a, const StepFeat f) {
    using Cfg = StepCfg<N, P, R, IO>;
    constexpr int K2 = Cfg::K2, CG = Cfg::CG, PT = Cfg::PT, KK = Cfg::KK, NT = Cfg::THREADS;
    __shared__ __align__(16) float sBp[R][N], sB[R][N], sC[R][N];
    __shared__ __align__(16) float sXp[R][P], sX[R][P];
    __shared__ __align__(16) float sAc[K2], sAs[K2];  // alpha cos, alpha sin of each pair's angle
    __shared__ float ypart[Cfg::WARPS][R][P];

    const int tid = threadIdx.x;
    const int cg = tid % CG, kk = tid / CG;
    const int64_t bh = blockIdx.x;
    const int h = (int)(bh % a.H);
    const int p0 = cg * 4;

    // buffer extents in elements, for the bounds build's index checks
    const int64_t nSt = a.BH * N * P, nBN = a.BH * R * N, nBP = a.BH * R * P;
    float4 *hst = reinterpret_cast<float4 *>(a.h + bh * N * P);
    // ---- issue the state loads first (the bulk of the bytes)
    float4 hu[PT], hv[PT];
#pragma unroll
    for (int j = 0; j < PT; ++j) {
        const int k = kk + j * KK;
        const bool in = dchk::in(kSiteState, bh * N * P + (2 * k) * P + p0, P + 4, nSt);
        hu[j] = in ? __ldcs(hst + ((2 * k) * P + p0) / 4) : make_float4(0.f, 0.f, 0.f, 0.f);
        hv[j] = in ? __ldcs(hst + ((2 * k + 1) * P + p0) / 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float dtv = ldv(a.dt, bh, a.BH, kSiteScalars), lamv = ldv(a.lam, bh, a.BH, kSiteScalars);
    const float alpha = __expf(dtv * ldf(a.A, (GEN && f.a_tok) ? bh : h, (GEN && f.a_tok) ? a.BH : a.H, kSiteScalars));
    const float gam = lamv * dtv, betap = (1.f - lamv) * dtv;
    // ---- stage the slice's small vectors (with the MIMO projections: the
    //      slice's one row of B, C and x, widened to its R rows)
    const bool proj = GEN && f.pwx;
    for (int i = tid; i < R * N; i += NT) {
        (&sBp[0][0])[i] = ldf(a.bp, bh * R * N + i, nBN, kSitePend);
        if (proj) {
            const int64_t w = h * R * N + i, v = bh * N + i % N;
            (&sB[0][0])[i] = ldf(f.pwB, w, a.H * R * N, kSiteProj) * ldv(a.B, v, a.BH * N, kSiteVec);
            (&sC[0][0])[i] = ldf(f.pwC, w, a.H * R * N, kSiteProj) * ldv(a.C, v, a.BH * N, kSiteVec);
        } else {
            (&sB[0][0])[i] = ldv(a.B, bh * R * N + i, nBN, kSiteVec);
            (&sC[0][0])[i] = ldv(a.C, bh * R * N + i, nBN, kSiteVec);
        }
    }
    for (int i = tid; i < R * P; i += NT) {
        (&sXp[0][0])[i] = ldf(a.xp, bh * R * P + i, nBP, kSitePend);
        (&sX[0][0])[i] = proj ? ldf(f.pwx, h * R * P + i, a.H * R * P, kSiteProj) *
                                    ldv(a.x, bh * P + i % P, a.BH * P, kSiteVec)
                              : ldv(a.x, bh * R * P + i, nBP, kSiteVec);
    }
    for (int k = tid; k < K2; k += NT) {
        float sn, cs;
        sincosf(dtv * ldv(a.theta, ((GEN && f.th_head) ? (int64_t)h : bh) * K2 + k,
                          ((GEN && f.th_head) ? a.H : a.BH) * K2, kSiteTheta),
                &sn, &cs);
        sAc[k] = alpha * cs;
        sAs[k] = alpha * sn;
    }
    __syncthreads();
    if (GEN && f.wB) {  // BC-norm prologue on the staged rows: one warp per row of B, then of C
        const int warp = tid / 32, lane = tid % 32;
        for (int row = warp; row < 2 * R; row += Cfg::WARPS) {
            const bool isB = row < R;
            const int r = isB ? row : row - R;
            float *v = isB ? sB[r] : sC[r];
            const float *w = isB ? f.wB : f.wC;
            const float *bias = isB ? f.bB : f.bC;
            const float sc = bcn_row_scale_warp([&](int n) { return v[n]; }, N, f.eps);
            for (int n = lane; n < N; n += 32)
                v[n] = fmaf(v[n] * sc, ldf(w, n, N, kSiteNorm), ldf(bias, (h * R + r) * N + n, a.H * R * N, kSiteNorm));
        }
        __syncthreads();
    }

    float4 yacc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) yacc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < PT; ++j) {
        const int k = kk + j * KK;
        float4 u = hu[j], v = hv[j];
        // previous-token trapezoid write
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float2 bpk = *reinterpret_cast<const float2 *>(&sBp[r][2 * k]);
            const float4 xp = *reinterpret_cast<const float4 *>(&sXp[r][p0]);
            const float cu = betap * bpk.x, cv = betap * bpk.y;
            u.x = fmaf(cu, xp.x, u.x); u.y = fmaf(cu, xp.y, u.y); u.z = fmaf(cu, xp.z, u.z); u.w = fmaf(cu, xp.w, u.w);
            v.x = fmaf(cv, xp.x, v.x); v.y = fmaf(cv, xp.y, v.y); v.z = fmaf(cv, xp.z, v.z); v.w = fmaf(cv, xp.w, v.w);
        }
        // decay + rotation by -dt*theta_k
        const float ac = sAc[k], as = sAs[k];
        float4 nu, nv;
        nu.x = ac * u.x + as * v.x; nv.x = ac * v.x - as * u.x;
        nu.y = ac * u.y + as * v.y; nv.y = ac * v.y - as * u.y;
        nu.z = ac * u.z + as * v.z; nv.z = ac * v.z - as * u.z;
        nu.w = ac * u.w + as * v.w; nv.w = ac * v.w - as * u.w;
        // current-token write and readout
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float2 bk = *reinterpret_cast<const float2 *>(&sB[r][2 * k]);
            const float4 xv = *reinterpret_cast<const float4 *>(&sX[r][p0]);
            const float cu = gam * bk.x, cv = gam * bk.y;
            nu.x = fmaf(cu, xv.x, nu.x); nu.y = fmaf(cu, xv.y, nu.y); nu.z = fmaf(cu, xv.z, nu.z); nu.w = fmaf(cu, xv.w, nu.w);
            nv.x = fmaf(cv, xv.x, nv.x); nv.y = fmaf(cv, xv.y, nv.y); nv.z = fmaf(cv, xv.z, nv.z); nv.w = fmaf(cv, xv.w, nv.w);
        }
        if (dchk::in(kSiteState, bh * N * P + (2 * k) * P + p0, P + 4, nSt)) {
            __stcs(hst + ((2 * k) * P + p0) / 4, nu);
            __stcs(hst + ((2 * k + 1) * P + p0) / 4, nv);
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float2 ck = *reinterpret_cast<const float2 *>(&sC[r][2 * k]);
            yacc[r].x = fmaf(nu.x, ck.x, fmaf(nv.x, ck.y, yacc[r].x));
            yacc[r].y = fmaf(nu.y, ck.x, fmaf(nv.y, ck.y, yacc[r].y));
            yacc[r].z = fmaf(nu.z, ck.x, fmaf(nv.z, ck.y, yacc[r].z));
            yacc[r].w = fmaf(nu.w, ck.x, fmaf(nv.w, ck.y, yacc[r].w));
        }
    }
    // ---- readout: sum over pair groups (same cg) -- shuffle within the warp
#pragma unroll
    for (int off = CG; off < 32; off *= 2) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            yacc[r].x += __shfl_xor_sync(0xffffffffu, yacc[r].x, off);
            yacc[r].y += __shfl_xor_sync(0xffffffffu, yacc[r].y, off);
            yacc[r].z += __shfl_xor_sync(0xffffffffu, yacc[r].z, off);
            yacc[r].w += __shfl_xor_sync(0xffffffffu, yacc[r].w, off);
        }
    }
    const int warp = tid / 32, lane = tid % 32;
    if (lane < CG || CG >= 32) {
#pragma unroll
        for (int r = 0; r < R; ++r) *reinterpret_cast<float4 *>(&ypart[warp][r][p0]) = yacc[r];
    }
    __syncthreads();
    const float Dh = ldf(a.D, h, a.H, kSiteScalars);
    if (proj) {  // y = sum over the R rows of wy_r times the row
        for (int p = tid; p < P; p += NT) {
            float acc = 0.f;
            for (int r = 0; r < R; ++r) {
                float s = 0.f;
#pragma unroll
                for (int w = 0; w < Cfg::WARPS; ++w) s += ypart[w][r][p];
                acc = fmaf(ldf(f.pwy, (h * R + r) * P + p, a.H * R * P, kSiteProj), s + Dh * sX[r][p], acc);
            }
            stv(a.y, bh * P + p, a.BH * P, kSiteY, acc);
        }
        for (int idx = tid; idx < R * P; idx += NT) stv(a.xp, bh * R * P + idx, nBP, kSitePend, (&sX[0][0])[idx]);
    } else {
        for (int idx = tid; idx < R * P; idx += NT) {
            const int r = idx / P, p = idx % P;
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < Cfg::WARPS; ++w) s += ypart[w][r][p];
            const float xval = sX[r][p];
            stv(a.y, (bh * R + r) * P + p, nBP, kSiteY, s + Dh * xval);
            stv(a.xp, (bh * R + r) * P + p, nBP, kSitePend, xval);
        }
    }
    for (int i = tid; i < R * N; i += NT) stv(a.bp, bh * R * N + i, nBN, kSitePend, (&sB[0][0])[i]);
}

// Generic kernel for any even N and any P: one thread per (pair, column),
// shared-memory atomics for the readout.  Same arithmetic, no tiling.
template <typename IO>
__global__ void __launch_bounds__(256) step_generic_kernel(const StepArgs<IO> a, const StepFeat f) {
    extern __shared__ float ysum[];  // [R][P], then (BC-norm) normalised B and C [R][N] each
    const int N = a.N, P = a.P, R = a.R, K2 = N / 2;
    const int64_t bh = blockIdx.x;
    const int h = (int)(bh % a.H);
    // buffer extents in elements, for the bounds build's index checks
    const int64_t nSt = a.BH * N * P, nBN = a.BH * R * N, nBP = a.BH * R * P;
    float *nB = ysum + R * P, *nC = nB + R * N;
    for (int i = threadIdx.x; i < R * P; i += blockDim.x) ysum[i] = 0.f;
    if (f.wB) {  // BC-norm prologue: one warp per row of B, then of C
        const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
        for (int row = warp; row < 2 * R; row += blockDim.x / 32) {
            const bool isB = row < R;
            const int r = isB ? row : row - R;
            const IO *src = isB ? a.B : a.C;
            const int64_t o = (bh * R + r) * N;
            const float *w = isB ? f.wB : f.wC;
            const float *bias = isB ? f.bB : f.bC;
            float *dst = (isB ? nB : nC) + r * N;
            const float sc = bcn_row_scale_warp([&](int n) { return ldv(src, o + n, nBN, kSiteVec); }, N, f.eps);
            for (int n = lane; n < N; n += 32)
                dst[n] = fmaf(ldv(src, o + n, nBN, kSiteVec) * sc, ldf(w, n, N, kSiteNorm),
                              ldf(bias, (h * R + r) * N + n, a.H * R * N, kSiteNorm));
        }
    }
    __syncthreads();
    auto Bv = [&](int i) { return f.wB ? nB[i] : ldv(a.B, bh * R * N + i, nBN, kSiteVec); };  // i = r * N + n
    auto Cv = [&](int i) { return f.wB ? nC[i] : ldv(a.C, bh * R * N + i, nBN, kSiteVec); };
    const float dtv = ldv(a.dt, bh, a.BH, kSiteScalars), lamv = ldv(a.lam, bh, a.BH, kSiteScalars);
    const float alpha = expf(dtv * ldf(a.A, f.a_tok ? bh : h, f.a_tok ? a.BH : a.H, kSiteScalars));
    const float gam = lamv * dtv, betap = (1.f - lamv) * dtv;
    float *hs = a.h + bh * N * P;
    for (int idx = threadIdx.x; idx < K2 * P; idx += blockDim.x) {
        const int k = idx / P, p = idx % P;
        const int64_t iu = bh * N * P + (2 * k) * P + p, iv = iu + P;
        float u = ldf(a.h, iu, nSt, kSiteState), v = ldf(a.h, iv, nSt, kSiteState);
        for (int r = 0; r < R; ++r) {
            const float xpp = ldf(a.xp, (bh * R + r) * P + p, nBP, kSitePend);
            u += betap * ldf(a.bp, (bh * R + r) * N + 2 * k, nBN, kSitePend) * xpp;
            v += betap * ldf(a.bp, (bh * R + r) * N + 2 * k + 1, nBN, kSitePend) * xpp;
        }
        float sn, cs;
        sincosf(dtv * ldv(a.theta, (f.th_head ? (int64_t)h : bh) * K2 + k, (f.th_head ? a.H : a.BH) * K2, kSiteTheta),
                &sn, &cs);
        float nu = alpha * (u * cs + v * sn), nv = alpha * (-u * sn + v * cs);
        for (int r = 0; r < R; ++r) {
            const float xx = ldv(a.x, (bh * R + r) * P + p, nBP, kSiteVec);
            nu += gam * Bv(r * N + 2 * k) * xx;
            nv += gam * Bv(r * N + 2 * k + 1) * xx;
        }
        stv(a.h, iu, nSt, kSiteState, nu);
        stv(a.h, iv, nSt, kSiteState, nv);
        for (int r = 0; r < R; ++r)
            atomicAdd(&ysum[r * P + p], nu * Cv(r * N + 2 * k) + nv * Cv(r * N + 2 * k + 1));
    }
    __syncthreads();
    const float Dh = ldf(a.D, h, a.H, kSiteScalars);
    for (int idx = threadIdx.x; idx < R * P; idx += blockDim.x) {
        const float xval = ldv(a.x, bh * R * P + idx, nBP, kSiteVec);
        stv(a.y, bh * R * P + idx, nBP, kSiteY, ysum[idx] + Dh * xval);
        stv(a.xp, bh * R * P + idx, nBP, kSitePend, xval);
    }
    for (int idx = threadIdx.x; idx < R * N; idx += blockDim.x) stv(a.bp, bh * R * N + idx, nBN, kSitePend, Bv(idx));
}

// Persistent streaming variant: each CTA walks slices bh = blockIdx.x,
// blockIdx.x + gridDim.x, ...; a bulk asynchronous copy brings the next-but-one
// slice's state and small vectors into a 2-stage shared-memory ring while the
// current slice is computed, so every SM keeps state bytes in flight all the
// time instead of alternating load, compute and store per CTA.
template <int N, int P, int R, typename IO>
struct StreamCfg {
    static constexpr int K2 = N / 2;
    static constexpr int CG = P / 4;
    static constexpr int PT = 4;
    static constexpr int KK = K2 / PT;
    static constexpr int THREADS = KK * CG;
    static constexpr int WARPS = THREADS / 32;
    // one stage: state, b_prev, x_prev (fp32); B, C, x, theta (io)
    static constexpr uint32_t B_H = N * P * 4;
    static constexpr uint32_t B_BP = R * N * 4, B_XP = R * P * 4;
    static constexpr uint32_t B_B = R * N * sizeof(IO), B_X = R * P * sizeof(IO), B_TH = K2 * sizeof(IO);
    static constexpr uint32_t O_BP = B_H, O_XP = O_BP + B_BP, O_B = O_XP + B_XP, O_C = O_B + B_B,
                              O_X = O_C + B_B, O_TH = O_X + B_X;
    static constexpr uint32_t STAGE = ((O_TH + B_TH + 127) / 128) * 128;
    static constexpr uint32_t TX = B_H + B_BP + B_XP + 2 * B_B + B_X + B_TH;
    static constexpr uint32_t O_YP = 2 * STAGE;                       // ypart [WARPS][R][P]
    static constexpr uint32_t O_AC = O_YP + WARPS * R * P * 4;        // alpha cos [K2], alpha sin [K2]
    // the slice's vectors, scaled and in fp32 once per slice: beta' b_prev,
    // gamma B and C, each [R][N]
    static constexpr uint32_t O_VEC = O_AC + 2 * K2 * 4;
    static constexpr uint32_t O_BAR = O_VEC + 3 * R * N * 4;
    static constexpr uint32_t SMEM = O_BAR + 16;
    static constexpr int CTAS_PER_SM = (3 * (SMEM + 1024) <= 232448) ? 3 : 2;  // as many as shared memory allows
    static_assert(B_BP % 16 == 0 && B_XP % 16 == 0 && B_B % 16 == 0 && B_X % 16 == 0 && B_TH % 16 == 0,
                  "bulk copies move multiples of 16 bytes");
    static_assert(THREADS % 32 == 0 && THREADS <= 1024, "bad block size");
};

template <typename T>
__device__ __forceinline__ float sv(const T *p, int i);
template <>
__device__ __forceinline__ float sv<float>(const float *p, int i) { return p[i]; }
template <>
__device__ __forceinline__ float sv<__nv_bfloat16>(const __nv_bfloat16 *p, int i) { return __bfloat162float(p[i]); }
template <typename T>
__device__ __forceinline__ float4 sv4(const T *p, int i);
template <>
__device__ __forceinline__ float4 sv4<float>(const float *p, int i) { return *reinterpret_cast<const float4 *>(p + i); }
template <>
__device__ __forceinline__ float4 sv4<__nv_bfloat16>(const __nv_bfloat16 *p, int i) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p + i);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

template <int N, int P, int R, typename IO, bool GEN>
__global__ void __launch_bounds__(StreamCfg<N, P, R, IO>::THREADS, StreamCfg<N, P, R, IO>::CTAS_PER_SM)
step_stream_kernel(const StepArgs<IO> a, const StepFeat f) {
    using Cfg = StreamCfg<N, P, R, IO>;
    constexpr int K2 = Cfg::K2, CG = Cfg::CG, PT = Cfg::PT, KK = Cfg::KK, NT = Cfg::THREADS;
    extern __shared__ __align__(128) uint8_t sm[];
    float *ypart = reinterpret_cast<float *>(sm + Cfg::O_YP);
    float *sAc = reinterpret_cast<float *>(sm + Cfg::O_AC);
    float *sAs = sAc + K2;
    float *vBp = reinterpret_cast<float *>(sm + Cfg::O_VEC), *vB = vBp + R * N, *vC = vB + R * N;
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + Cfg::O_BAR);
    __shared__ int abort_flag;
    const int tid = threadIdx.x;
    const int cg = tid % CG, kk = tid / CG, p0 = cg * 4;
    const int warp = tid / 32, lane = tid % 32;
    const int64_t BH = a.BH, step = gridDim.x;
    // buffer extents in elements, for the bounds build's index checks
    const int64_t nSt = BH * N * P, nBN = BH * R * N, nBP = BH * R * P;

    // MIMO projections: B, C and x hold one row per slice (the copies move
    // 1/R of the bytes), widened with the head's weights when staged
    const bool proj = GEN && f.pwx;
    const int RIO = proj ? 1 : R;
    const uint32_t cB = proj ? Cfg::B_B / R : Cfg::B_B, cX = proj ? Cfg::B_X / R : Cfg::B_X;
    // the slice's copies; the bounds build checks each source range and
    // copies from the buffer's start instead of outside it (so that the
    // expected bytes still arrive)
    auto issue = [&](int64_t bh, int st) {
        uint8_t *s = sm + st * Cfg::STAGE;
        const int64_t th = ((GEN && f.th_head) ? bh % a.H : bh) * K2;
        const int64_t nth = ((GEN && f.th_head) ? a.H : BH) * K2;
        const bool ist = dchk::in(kSiteState, bh * N * P, N * P, nSt);
        const bool ibn = dchk::in(kSitePend, bh * R * N, R * N, nBN) &&
                         dchk::in(kSiteVec, bh * RIO * N, RIO * N, BH * RIO * N);
        const bool ibp = dchk::in(kSitePend, bh * R * P, R * P, nBP) &&
                         dchk::in(kSiteVec, bh * RIO * P, RIO * P, BH * RIO * P);
        const bool ith = dchk::in(kSiteTheta, th, K2, nth);
        tc::mbar_arrive_expect_tx(&full[st], Cfg::TX - 2 * (Cfg::B_B - cB) - (Cfg::B_X - cX));
        tc::bulk_g2s(s, a.h + (ist ? bh * N * P : 0), Cfg::B_H, &full[st]);
        tc::bulk_g2s(s + Cfg::O_BP, a.bp + (ibn ? bh * R * N : 0), Cfg::B_BP, &full[st]);
        tc::bulk_g2s(s + Cfg::O_XP, a.xp + (ibp ? bh * R * P : 0), Cfg::B_XP, &full[st]);
        tc::bulk_g2s(s + Cfg::O_B, a.B + (ibn ? bh * RIO * N : 0), cB, &full[st]);
        tc::bulk_g2s(s + Cfg::O_C, a.C + (ibn ? bh * RIO * N : 0), cB, &full[st]);
        tc::bulk_g2s(s + Cfg::O_X, a.x + (ibp ? bh * RIO * P : 0), cX, &full[st]);
        tc::bulk_g2s(s + Cfg::O_TH, a.theta + (ith ? th : 0), Cfg::B_TH, &full[st]);
    };
    if (tid == 0) {
        tc::mbar_init(&full[0], 1);
        tc::mbar_init(&full[1], 1);
        abort_flag = 0;
        tc::fence_mbar_init();
    }
    __syncthreads();
    // With fewer slices than resident CTAs the kernel is launched as a
    // programmatic dependent of the previous kernel on the stream: its CTAs are
    // scheduled while that kernel still runs, nothing is read before that
    // kernel has completed (the wait below), and the next step may launch as
    // soon as every CTA here has started.  Without the launch attribute both
    // instructions do nothing.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (tid == 0) {
        if ((int64_t)blockIdx.x < BH) issue(blockIdx.x, 0);
        if ((int64_t)blockIdx.x + step < BH) issue(blockIdx.x + step, 1);
    }
    int it = 0;
    for (int64_t bh = blockIdx.x; bh < BH; bh += step, ++it) {
        const int st = it & 1;
        const uint8_t *s = sm + st * Cfg::STAGE;
        const float *sh = reinterpret_cast<const float *>(s);
        const float *sBp = reinterpret_cast<const float *>(s + Cfg::O_BP);
        const float *sXp = reinterpret_cast<const float *>(s + Cfg::O_XP);
        const IO *sB = reinterpret_cast<const IO *>(s + Cfg::O_B);
        const IO *sC = reinterpret_cast<const IO *>(s + Cfg::O_C);
        const IO *sX = reinterpret_cast<const IO *>(s + Cfg::O_X);
        const IO *sTh = reinterpret_cast<const IO *>(s + Cfg::O_TH);
        const int h = (int)(bh % a.H);
        const float dtv = ldv(a.dt, bh, BH, kSiteScalars), lamv = ldv(a.lam, bh, BH, kSiteScalars);
        const float gam = lamv * dtv, betap = (1.f - lamv) * dtv;
        const bool ok = tc::mbar_wait(&full[st], (it >> 1) & 1, &abort_flag, &g_decode_error, tc::kErrWaitTma);
        if (__syncthreads_or(!ok)) break;
        if (tid < K2) {
            const float alpha =
                __expf(dtv * ldf(a.A, (GEN && f.a_tok) ? bh : h, (GEN && f.a_tok) ? BH : a.H, kSiteScalars));
            float sn, cs;
            sincosf(dtv * sv(sTh, tid), &sn, &cs);
            sAc[tid] = alpha * cs;
            sAs[tid] = alpha * sn;
        }
        for (int i = tid; i < R * N; i += NT) {
            vBp[i] = betap * sBp[i];
            if (proj) {
                const int64_t w = (int64_t)h * R * N + i;
                vB[i] = gam * ldf(f.pwB, w, a.H * R * N, kSiteProj) * sv(sB, i % N);
                vC[i] = ldf(f.pwC, w, a.H * R * N, kSiteProj) * sv(sC, i % N);
            } else {
                vB[i] = gam * sv(sB, i);
                vC[i] = sv(sC, i);
            }
        }
        __syncthreads();
        float4 xp[R], xv[R], yacc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            xp[r] = *reinterpret_cast<const float4 *>(sXp + r * P + p0);
            if (proj) {
                const float4 x4 = sv4(sX, p0);
                const int64_t w = ((int64_t)h * R + r) * P + p0;
                const int64_t nw = a.H * R * P;
                xv[r] = make_float4(ldf(f.pwx, w, nw, kSiteProj) * x4.x, ldf(f.pwx, w + 1, nw, kSiteProj) * x4.y,
                                    ldf(f.pwx, w + 2, nw, kSiteProj) * x4.z, ldf(f.pwx, w + 3, nw, kSiteProj) * x4.w);
            } else {
                xv[r] = sv4(sX, r * P + p0);
            }
            yacc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float4 *hg = reinterpret_cast<float4 *>(a.h + bh * N * P);
#pragma unroll
        for (int j = 0; j < PT; ++j) {
            const int k = kk + j * KK;
            float4 u = *reinterpret_cast<const float4 *>(sh + (2 * k) * P + p0);
            float4 v = *reinterpret_cast<const float4 *>(sh + (2 * k + 1) * P + p0);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float2 bpk = *reinterpret_cast<const float2 *>(vBp + r * N + 2 * k);
                const float cu = bpk.x, cv = bpk.y;
                u.x = fmaf(cu, xp[r].x, u.x); u.y = fmaf(cu, xp[r].y, u.y);
                u.z = fmaf(cu, xp[r].z, u.z); u.w = fmaf(cu, xp[r].w, u.w);
                v.x = fmaf(cv, xp[r].x, v.x); v.y = fmaf(cv, xp[r].y, v.y);
                v.z = fmaf(cv, xp[r].z, v.z); v.w = fmaf(cv, xp[r].w, v.w);
            }
            const float ac = sAc[k], as = sAs[k];
            float4 nu, nv;
            nu.x = ac * u.x + as * v.x; nv.x = ac * v.x - as * u.x;
            nu.y = ac * u.y + as * v.y; nv.y = ac * v.y - as * u.y;
            nu.z = ac * u.z + as * v.z; nv.z = ac * v.z - as * u.z;
            nu.w = ac * u.w + as * v.w; nv.w = ac * v.w - as * u.w;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float2 bk = *reinterpret_cast<const float2 *>(vB + r * N + 2 * k);
                const float cu = bk.x, cv = bk.y;
                nu.x = fmaf(cu, xv[r].x, nu.x); nu.y = fmaf(cu, xv[r].y, nu.y);
                nu.z = fmaf(cu, xv[r].z, nu.z); nu.w = fmaf(cu, xv[r].w, nu.w);
                nv.x = fmaf(cv, xv[r].x, nv.x); nv.y = fmaf(cv, xv[r].y, nv.y);
                nv.z = fmaf(cv, xv[r].z, nv.z); nv.w = fmaf(cv, xv[r].w, nv.w);
            }
            if (dchk::in(kSiteState, bh * N * P + (2 * k) * P + p0, P + 4, nSt)) {
                __stcs(hg + ((2 * k) * P + p0) / 4, nu);
                __stcs(hg + ((2 * k + 1) * P + p0) / 4, nv);
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float2 ck = *reinterpret_cast<const float2 *>(vC + r * N + 2 * k);
                yacc[r].x = fmaf(nu.x, ck.x, fmaf(nv.x, ck.y, yacc[r].x));
                yacc[r].y = fmaf(nu.y, ck.x, fmaf(nv.y, ck.y, yacc[r].y));
                yacc[r].z = fmaf(nu.z, ck.x, fmaf(nv.z, ck.y, yacc[r].z));
                yacc[r].w = fmaf(nu.w, ck.x, fmaf(nv.w, ck.y, yacc[r].w));
            }
        }
#pragma unroll
        for (int off = CG; off < 32; off *= 2) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                yacc[r].x += __shfl_xor_sync(0xffffffffu, yacc[r].x, off);
                yacc[r].y += __shfl_xor_sync(0xffffffffu, yacc[r].y, off);
                yacc[r].z += __shfl_xor_sync(0xffffffffu, yacc[r].z, off);
                yacc[r].w += __shfl_xor_sync(0xffffffffu, yacc[r].w, off);
            }
        }
        if (lane < CG || CG >= 32) {
#pragma unroll
            for (int r = 0; r < R; ++r)
                *reinterpret_cast<float4 *>(ypart + (warp * R + r) * P + p0) = yacc[r];
        }
        __syncthreads();
        const float Dh = ldf(a.D, h, a.H, kSiteScalars);
        if (proj) {  // y = sum over the R rows of wy_r times the row; the pending rows widened
            const int64_t nw = a.H * R * P;
            for (int p = tid; p < P; p += NT) {
                float acc = 0.f;
                for (int r = 0; r < R; ++r) {
                    float sum = 0.f;
#pragma unroll
                    for (int w = 0; w < Cfg::WARPS; ++w) sum += ypart[w * R * P + r * P + p];
                    const int64_t wi = ((int64_t)h * R + r) * P + p;
                    const float xval = ldf(f.pwx, wi, nw, kSiteProj) * sv(sX, p);
                    acc = fmaf(ldf(f.pwy, wi, nw, kSiteProj), sum + Dh * xval, acc);
                }
                stv(a.y, bh * P + p, BH * P, kSiteY, acc);
            }
            for (int idx = tid; idx < R * P; idx += NT)
                stv(a.xp, bh * R * P + idx, nBP, kSitePend,
                    ldf(f.pwx, (int64_t)h * R * P + idx, nw, kSiteProj) * sv(sX, idx % P));
            for (int i = tid; i < R * N; i += NT)
                stv(a.bp, bh * R * N + i, nBN, kSitePend,
                    ldf(f.pwB, (int64_t)h * R * N + i, a.H * R * N, kSiteProj) * sv(sB, i % N));
        } else {
            for (int idx = tid; idx < R * P; idx += NT) {
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < Cfg::WARPS; ++w) sum += ypart[w * R * P + idx];
                const float xval = sv(sX, idx);
                stv(a.y, bh * R * P + idx, nBP, kSiteY, sum + Dh * xval);
                stv(a.xp, bh * R * P + idx, nBP, kSitePend, xval);
            }
            for (int i = tid; i < R * N; i += NT) stv(a.bp, bh * R * N + i, nBN, kSitePend, sv(sB, i));
        }
        __syncthreads();  // every read of this stage is done: refill it
        if (tid == 0 && bh + 2 * step < BH) issue(bh + 2 * step, st);
    }
    // let any copy still in flight land before the CTA exits (only after an abort)
    if (tid == 0 && abort_flag) {
        for (int q = 0; q < 2; ++q) tc::mbar_wait(&full[q], 0, nullptr, &g_decode_error, 0, 400000000LL);
    }
}

template <int N, int P, int R, typename IO, bool GEN>
cudaError_t launch_stream(const StepArgs<IO> &a, const StepFeat &f, cudaStream_t s) {
    using Cfg = StreamCfg<N, P, R, IO>;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(step_stream_kernel<N, P, R, IO, GEN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)Cfg::SMEM);
    if (e != cudaSuccess) return e;
    int64_t grid = (int64_t)sms * Cfg::CTAS_PER_SM;
    // programmatic dependent launch only where the grid leaves SMs free (few
    // slices: it hides the launch gap of a latency-bound step; measured: the
    // long-context decode's 64 slices 3.44 -> 3.27 us per step, while a grid
    // that fills every SM ran 1.6 % slower with it)
    const bool pdl = grid > a.BH;
    if (grid > a.BH) grid = a.BH;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = Cfg::SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, step_stream_kernel<N, P, R, IO, GEN>, a, f);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int N, int P, int R, typename IO, bool GEN>
cudaError_t launch_tiled(const StepArgs<IO> &a, const StepFeat &f, cudaStream_t s) {
    step_kernel<N, P, R, IO, GEN><<<(unsigned)a.BH, StepCfg<N, P, R, IO>::THREADS, 0, s>>>(a, f);
    return cudaGetLastError();
}

template <typename IO, int R, bool GEN>
cudaError_t dispatch_np(const StepArgs<IO> &a, const StepFeat &f, cudaStream_t s, bool *done) {
    *done = true;
    // rank 1: one CTA per slice (measured faster); rank >= 2: the persistent
    // streaming kernel (its heavier per-element work overlaps the next slice's load)
    // (BC-norm: the tiled kernel, which normalises its staged rows in place)
    const bool tiled = R == 1 || f.wB;
    if (a.N == 128 && a.P == 64)
        return tiled ? launch_tiled<128, 64, R, IO, GEN>(a, f, s) : launch_stream<128, 64, R, IO, GEN>(a, f, s);
    if (a.N == 64 && a.P == 64)
        return tiled ? launch_tiled<64, 64, R, IO, GEN>(a, f, s) : launch_stream<64, 64, R, IO, GEN>(a, f, s);
    if (a.N == 128 && a.P == 128) return launch_tiled<128, 128, R, IO, GEN>(a, f, s);
    if (a.N == 64 && a.P == 128) return launch_tiled<64, 128, R, IO, GEN>(a, f, s);
    if (a.N == 256 && a.P == 64) return launch_tiled<256, 64, R, IO, GEN>(a, f, s);
    *done = false;
    return cudaSuccess;
}

template <typename IO>
cudaError_t launch_typed(const Problem &p) {
    StepArgs<IO> a;
    a.BH = p.Bt * p.H; a.H = p.H;
    a.P = (int)p.P; a.N = (int)p.N; a.R = (int)p.R;
    a.x = (const IO *)p.x; a.B = (const IO *)p.B; a.C = (const IO *)p.C;
    a.dt = (const IO *)p.dt; a.lam = (const IO *)p.lam; a.theta = (const IO *)p.theta;
    a.A = p.A; a.D = p.D;
    StepFeat f{};
    f.a_tok = p.a_tok;
    f.th_head = p.th_head;
    f.wB = p.wB; f.wC = p.wC; f.bB = p.bB; f.bC = p.bC; f.eps = p.eps;
    f.pwx = p.pwx; f.pwB = p.pwB; f.pwC = p.pwC; f.pwy = p.pwy;
    a.h = p.hT; a.bp = p.bpT; a.xp = p.xpT;
    a.y = (IO *)p.y;
    if (a.BH == 0) return cudaSuccess;
    bool done = false;
    cudaError_t e = cudaSuccess;
    const bool gen = f.a_tok || f.th_head || f.wB || f.pwx;  // any optional feature on
    if (a.R == 1) e = gen ? dispatch_np<IO, 1, true>(a, f, p.stream, &done) : dispatch_np<IO, 1, false>(a, f, p.stream, &done);
    else if (a.R == 2) e = gen ? dispatch_np<IO, 2, true>(a, f, p.stream, &done) : dispatch_np<IO, 2, false>(a, f, p.stream, &done);
    else if (a.R == 4) e = gen ? dispatch_np<IO, 4, true>(a, f, p.stream, &done) : dispatch_np<IO, 4, false>(a, f, p.stream, &done);
    if (done) return e;
    if (f.pwx) return cudaErrorNotSupported;  // the MIMO projections: the tiled sizes only
    const size_t smem = sizeof(float) * ((size_t)a.R * a.P + (f.wB ? 2 * (size_t)a.R * a.N : 0));
    step_generic_kernel<IO><<<(unsigned)a.BH, 256, smem, p.stream>>>(a, f);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step(const Problem &p, const char **why) {
    const cudaError_t e = p.bf16 ? launch_typed<__nv_bfloat16>(p) : launch_typed<float>(p);
    if (e == cudaErrorNotSupported)
        *why = "decode step with the MIMO projections: (dstate, headdim) in {(64|128, 64|128), (256, 64)} and "
               "rank 1, 2 or 4 only";
    return e;
}

cudaError_t read_decode_error(unsigned *code) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_decode_error, sizeof v);
    if (e != cudaSuccess) return e;
    if (v) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_decode_error, &zero, sizeof zero);
    }
    *code = v;
    return e;
}

M3_DCHECK_READER(read_dcheck_decode)

}  // namespace m3
