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

#include "m3_internal.h"

namespace m3 {
namespace {

template <typename T>
__device__ __forceinline__ float ldv(const T *p, int64_t i);
template <>
__device__ __forceinline__ float ldv<float>(const float *p, int64_t i) { return __ldg(p + i); }
template <>
__device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i) {
    return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ void stv(T *p, int64_t i, float v);
template <>
__device__ __forceinline__ void stv<float>(float *p, int64_t i, float v) { p[i] = v; }
template <>
__device__ __forceinline__ void stv<__nv_bfloat16>(__nv_bfloat16 *p, int64_t i, float v) {
    p[i] = __float2bfloat16_rn(v);
}
// 4 consecutive io values starting at element i (i multiple of 4)
template <typename T>
__device__ __forceinline__ float4 ld4(const T *p, int64_t i);
template <>
__device__ __forceinline__ float4 ld4<float>(const float *p, int64_t i) {
    return __ldg(reinterpret_cast<const float4 *>(p + i));
}
template <>
__device__ __forceinline__ float4 ld4<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i) {
    const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p + i));
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&raw.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&raw.y);
    const float2 a = __bfloat1622float2(lo), b = __bfloat1622float2(hi);
    return make_float4(a.x, a.y, b.x, b.y);
}
// 2 consecutive io values starting at element i (i even)
template <typename T>
__device__ __forceinline__ float2 ld2(const T *p, int64_t i);
template <>
__device__ __forceinline__ float2 ld2<float>(const float *p, int64_t i) {
    return __ldg(reinterpret_cast<const float2 *>(p + i));
}
template <>
__device__ __forceinline__ float2 ld2<__nv_bfloat16>(const __nv_bfloat16 *p, int64_t i) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162 *>(p + i);
    return __bfloat1622float2(v);
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

// Register-tiled kernel for the common sizes.  PT pairs per thread.
template <int N, int P, int R, typename IO>
struct StepCfg {
    static constexpr int K2 = N / 2;
    static constexpr int CG = P / 4;                      // column groups (float4)
    static constexpr int PT = (K2 * CG >= 1024) ? 8 : 4;  // pairs per thread
    static constexpr int KK = K2 / PT;                    // pair groups
    static constexpr int THREADS = KK * CG;
    static constexpr int WARPS = THREADS / 32;
    static_assert(K2 % PT == 0, "pairs must split evenly");
    static_assert(THREADS % 32 == 0 && THREADS <= 1024, "bad block size");
    static_assert(32 % CG == 0 || CG % 32 == 0, "column groups must tile a warp");
};

template <int N, int P, int R, typename IO>
__global__ void __launch_bounds__(StepCfg<N, P, R, IO>::THREADS)
step_kernel(const StepArgs<IO> a) {
    using Cfg = StepCfg<N, P, R, IO>;
    constexpr int K2 = Cfg::K2, CG = Cfg::CG, PT = Cfg::PT, KK = Cfg::KK;
    __shared__ float ypart[Cfg::WARPS][R][P];

    const int tid = threadIdx.x;
    const int cg = tid % CG, kk = tid / CG;
    const int64_t bh = blockIdx.x;
    const int h = (int)(bh % a.H);
    const int p0 = cg * 4;

    float4 *hst = reinterpret_cast<float4 *>(a.h + bh * N * P);
    // ---- issue the state loads first (the bulk of the bytes)
    float4 hu[PT], hv[PT];
#pragma unroll
    for (int j = 0; j < PT; ++j) {
        const int k = kk + j * KK;
        hu[j] = __ldcs(hst + ((2 * k) * P + p0) / 4);
        hv[j] = __ldcs(hst + ((2 * k + 1) * P + p0) / 4);
    }
    const float dtv = ldv(a.dt, bh), lamv = ldv(a.lam, bh);
    const float alpha = __expf(dtv * a.A[h]);
    const float gam = lamv * dtv, betap = (1.f - lamv) * dtv;
    float4 xpv[R], xv[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        xpv[r] = __ldg(reinterpret_cast<const float4 *>(a.xp + (bh * R + r) * P + p0));
        xv[r] = ld4(a.x, (bh * R + r) * P + p0);
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
            const float2 bpk = __ldg(reinterpret_cast<const float2 *>(a.bp + (bh * R + r) * N + 2 * k));
            const float cu = betap * bpk.x, cv = betap * bpk.y;
            u.x += cu * xpv[r].x; u.y += cu * xpv[r].y; u.z += cu * xpv[r].z; u.w += cu * xpv[r].w;
            v.x += cv * xpv[r].x; v.y += cv * xpv[r].y; v.z += cv * xpv[r].z; v.w += cv * xpv[r].w;
        }
        // decay + rotation by -dt*theta_k
        float sn, cs;
        sincosf(dtv * ldv(a.theta, bh * K2 + k), &sn, &cs);
        const float ac = alpha * cs, as = alpha * sn;
        float4 nu, nv;
        nu.x = ac * u.x + as * v.x; nv.x = ac * v.x - as * u.x;
        nu.y = ac * u.y + as * v.y; nv.y = ac * v.y - as * u.y;
        nu.z = ac * u.z + as * v.z; nv.z = ac * v.z - as * u.z;
        nu.w = ac * u.w + as * v.w; nv.w = ac * v.w - as * u.w;
        // current-token write and readout
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float2 bk = ld2(a.B, (bh * R + r) * N + 2 * k);
            const float cu = gam * bk.x, cv = gam * bk.y;
            nu.x += cu * xv[r].x; nu.y += cu * xv[r].y; nu.z += cu * xv[r].z; nu.w += cu * xv[r].w;
            nv.x += cv * xv[r].x; nv.y += cv * xv[r].y; nv.z += cv * xv[r].z; nv.w += cv * xv[r].w;
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const float2 ck = ld2(a.C, (bh * R + r) * N + 2 * k);
            yacc[r].x += nu.x * ck.x + nv.x * ck.y;
            yacc[r].y += nu.y * ck.x + nv.y * ck.y;
            yacc[r].z += nu.z * ck.x + nv.z * ck.y;
            yacc[r].w += nu.w * ck.x + nv.w * ck.y;
        }
        __stcs(hst + ((2 * k) * P + p0) / 4, nu);
        __stcs(hst + ((2 * k + 1) * P + p0) / 4, nv);
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
        for (int r = 0; r < R; ++r) {
            ypart[warp][r][p0 + 0] = yacc[r].x;
            ypart[warp][r][p0 + 1] = yacc[r].y;
            ypart[warp][r][p0 + 2] = yacc[r].z;
            ypart[warp][r][p0 + 3] = yacc[r].w;
        }
    }
    __syncthreads();  // also orders every read of b_prev/x_prev before the writes below
    const float Dh = a.D[h];
    for (int idx = tid; idx < R * P; idx += Cfg::THREADS) {
        const int r = idx / P, p = idx % P;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < Cfg::WARPS; ++w) s += ypart[w][r][p];
        const float xval = ldv(a.x, (bh * R + r) * P + p);
        stv(a.y, (bh * R + r) * P + p, s + Dh * xval);
        a.xp[(bh * R + r) * P + p] = xval;
    }
    for (int idx = tid; idx < R * N; idx += Cfg::THREADS)
        a.bp[bh * R * N + idx] = ldv(a.B, bh * R * N + idx);
}

// Generic kernel for any even N and any P: one thread per (pair, column),
// shared-memory atomics for the readout.  Same arithmetic, no tiling.
template <typename IO>
__global__ void __launch_bounds__(256) step_generic_kernel(const StepArgs<IO> a) {
    extern __shared__ float ysum[];  // [R][P]
    const int N = a.N, P = a.P, R = a.R, K2 = N / 2;
    const int64_t bh = blockIdx.x;
    const int h = (int)(bh % a.H);
    for (int i = threadIdx.x; i < R * P; i += blockDim.x) ysum[i] = 0.f;
    __syncthreads();
    const float dtv = ldv(a.dt, bh), lamv = ldv(a.lam, bh);
    const float alpha = expf(dtv * a.A[h]);
    const float gam = lamv * dtv, betap = (1.f - lamv) * dtv;
    float *hs = a.h + bh * N * P;
    for (int idx = threadIdx.x; idx < K2 * P; idx += blockDim.x) {
        const int k = idx / P, p = idx % P;
        float u = hs[(2 * k) * P + p], v = hs[(2 * k + 1) * P + p];
        for (int r = 0; r < R; ++r) {
            const float xpp = a.xp[(bh * R + r) * P + p];
            u += betap * a.bp[(bh * R + r) * N + 2 * k] * xpp;
            v += betap * a.bp[(bh * R + r) * N + 2 * k + 1] * xpp;
        }
        float sn, cs;
        sincosf(dtv * ldv(a.theta, bh * K2 + k), &sn, &cs);
        float nu = alpha * (u * cs + v * sn), nv = alpha * (-u * sn + v * cs);
        for (int r = 0; r < R; ++r) {
            const float xx = ldv(a.x, (bh * R + r) * P + p);
            nu += gam * ldv(a.B, (bh * R + r) * N + 2 * k) * xx;
            nv += gam * ldv(a.B, (bh * R + r) * N + 2 * k + 1) * xx;
        }
        hs[(2 * k) * P + p] = nu;
        hs[(2 * k + 1) * P + p] = nv;
        for (int r = 0; r < R; ++r)
            atomicAdd(&ysum[r * P + p], nu * ldv(a.C, (bh * R + r) * N + 2 * k) +
                                            nv * ldv(a.C, (bh * R + r) * N + 2 * k + 1));
    }
    __syncthreads();
    const float Dh = a.D[h];
    for (int idx = threadIdx.x; idx < R * P; idx += blockDim.x) {
        const float xval = ldv(a.x, bh * R * P + idx);
        stv(a.y, bh * R * P + idx, ysum[idx] + Dh * xval);
        a.xp[bh * R * P + idx] = xval;
    }
    for (int idx = threadIdx.x; idx < R * N; idx += blockDim.x)
        a.bp[bh * R * N + idx] = ldv(a.B, bh * R * N + idx);
}

template <int N, int P, int R, typename IO>
cudaError_t launch_tiled(const StepArgs<IO> &a, cudaStream_t s) {
    step_kernel<N, P, R, IO><<<(unsigned)a.BH, StepCfg<N, P, R, IO>::THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename IO, int R>
cudaError_t dispatch_np(const StepArgs<IO> &a, cudaStream_t s, bool *done) {
    *done = true;
    if (a.N == 128 && a.P == 64) return launch_tiled<128, 64, R, IO>(a, s);
    if (a.N == 64 && a.P == 64) return launch_tiled<64, 64, R, IO>(a, s);
    if (a.N == 128 && a.P == 128) return launch_tiled<128, 128, R, IO>(a, s);
    if (a.N == 64 && a.P == 128) return launch_tiled<64, 128, R, IO>(a, s);
    if (a.N == 256 && a.P == 64) return launch_tiled<256, 64, R, IO>(a, s);
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
    a.h = p.hT; a.bp = p.bpT; a.xp = p.xpT;
    a.y = (IO *)p.y;
    if (a.BH == 0) return cudaSuccess;
    bool done = false;
    cudaError_t e = cudaSuccess;
    if (a.R == 1) e = dispatch_np<IO, 1>(a, p.stream, &done);
    else if (a.R == 2) e = dispatch_np<IO, 2>(a, p.stream, &done);
    else if (a.R == 4) e = dispatch_np<IO, 4>(a, p.stream, &done);
    if (done) return e;
    const size_t smem = sizeof(float) * (size_t)a.R * a.P;
    step_generic_kernel<IO><<<(unsigned)a.BH, 256, smem, p.stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_step(const Problem &p, const char **) {
    return p.bf16 ? launch_typed<__nv_bfloat16>(p) : launch_typed<float>(p);
}

}  // namespace m3
