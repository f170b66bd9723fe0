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
#include "m3_internal.h"

namespace m3 {
namespace {

template <typename T>
__device__ __forceinline__ float ldv(const T *p, int64_t i);
template <>
__device__ __forceinline__ float ldv<float>(const float *p, int64_t i) { return p[i]; }
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

__host__ __device__ inline size_t simt_smem_floats(int P, int N, int R, int Q) {
    const size_t rows = (size_t)Q * R;
    return rows * P + 2 * rows * N + rows * rows + (size_t)N * P + 6 * (size_t)Q + 3 * (size_t)(N / 2);
}

template <typename IO>
__global__ void __launch_bounds__(kThreads) prefill_simt_kernel(const SimtArgs<IO> a) {
    extern __shared__ float smem[];
    const int P = a.P, N = a.N, R = a.R, Q = a.Q, K2 = N / 2;
    const int rowsmax = Q * R;
    float *Xs = smem;                       // [rows][P]
    float *Bs = Xs + rowsmax * P;           // [rows][N]  (rotated in place)
    float *Cs = Bs + rowsmax * N;           // [rows][N]  (rotated in place)
    float *Pm = Cs + rowsmax * N;           // [rows][rows] masked scores
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

    const int tid = threadIdx.x;
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / a.H, h = bh % a.H;
    const int64_t T = a.T, H = a.H;
    const float Ah = a.a_tok ? 0.f : a.A[h], Dh = a.D[h];
    auto tok = [&](int64_t t) { return (b * T + t) * H + h; };  // token-head index

    // ---- initial state: h0 + beta'_0 * b_prev x_prev^T (pending write of token -1)
    float betap0 = 0.f;
    if (T > 0) {
        const float d0 = ldv(a.dt, tok(0)), l0 = ldv(a.lam, tok(0));
        betap0 = (1.f - l0) * d0;
    }
    for (int idx = tid; idx < N * P; idx += kThreads) {
        const int n = idx / P, p = idx % P;
        float v = a.h0 ? a.h0[bh * N * P + idx] : 0.f;
        if (a.bp0 && a.xp0 && T > 0) {
            float acc = 0.f;
            for (int r = 0; r < R; ++r) acc += a.bp0[(bh * R + r) * N + n] * a.xp0[(bh * R + r) * P + p];
            v += betap0 * acc;
        }
        hs[idx] = v;
    }
    __syncthreads();

    for (int64_t t0 = 0; t0 < T; t0 += Q) {
        const int L = (int)((T - t0) < Q ? (T - t0) : Q);
        const int rows = L * R;
        const bool last_chunk = (t0 + L == T);

        // ---- load the chunk (rows = (token, rank))
        for (int idx = tid; idx < rows * P; idx += kThreads) {
            const int i = idx / P, p = idx % P;
            Xs[idx] = ldv(a.x, (tok(t0 + i / R) * R + i % R) * P + p);
        }
        for (int idx = tid; idx < rows * N; idx += kThreads) {
            const int i = idx / N, n = idx % N;
            const int64_t g = (tok(t0 + i / R) * R + i % R) * N + n;
            Bs[idx] = ldv(a.B, g);
            Cs[idx] = ldv(a.C, g);
        }
        for (int s = tid; s < L; s += kThreads) {
            const int64_t t = t0 + s;
            const float d = ldv(a.dt, tok(t)), l = ldv(a.lam, tok(t));
            dts[s] = d;
            cA[s] = d * (a.a_tok ? a.A[tok(t)] : Ah);
            gam[s] = l * d;
            float nxt = 0.f;  // (1 - lam_{t+1}) dt_{t+1}; absent after the last token
            if (t + 1 < T) {
                const float d1 = ldv(a.dt, tok(t + 1)), l1 = ldv(a.lam, tok(t + 1));
                nxt = (1.f - l1) * d1;
            }
            ghat[s] = l * d + nxt;
        }
        __syncthreads();
        if (a.wB) {  // BC-norm prologue: one warp per (token, rank) row of B, then of C
            const int warp = tid >> 5, lane = tid & 31;
            for (int row = warp; row < 2 * rows; row += kThreads / 32) {
                const bool isB = row < rows;
                float *v = isB ? Bs + row * N : Cs + (row - rows) * N;
                const int r = (isB ? row : row - rows) % R;
                const float *w = isB ? a.wB : a.wC;
                const float *bias = (isB ? a.bB : a.bC) + (h * R + r) * N;
                const float sc = bcn_row_scale_warp([&](int n) { return v[n]; }, N, a.eps);
                for (int n = lane; n < N; n += 32) v[n] = fmaf(v[n] * sc, w[n], bias[n]);
            }
            __syncthreads();
        }
        if (tid == 0) {  // chunk-local inclusive prefix of dt*A
            float run = 0.f;
            for (int s = 0; s < L; ++s) { run += cA[s]; cA[s] = run; }
        }
        // ---- rotate B and C by the chunk-local cumulative angle (one thread per pair)
        for (int k = tid; k < K2; k += kThreads) {
            float phi = 0.f;
            for (int s = 0; s < L; ++s) {
                phi += dts[s] * ldv(a.theta, (a.th_head ? (int64_t)h : tok(t0 + s)) * K2 + k);
                float sn, cs;
                sincosf(phi, &sn, &cs);
                for (int r = 0; r < R; ++r) {
                    const int i = s * R + r;
                    float u = Bs[i * N + 2 * k], v = Bs[i * N + 2 * k + 1];
                    Bs[i * N + 2 * k] = u * cs - v * sn;
                    Bs[i * N + 2 * k + 1] = u * sn + v * cs;
                    u = Cs[i * N + 2 * k];
                    v = Cs[i * N + 2 * k + 1];
                    Cs[i * N + 2 * k] = u * cs - v * sn;
                    Cs[i * N + 2 * k + 1] = u * sn + v * cs;
                }
            }
            phiE[k] = phi;
            float sn, cs;
            sincosf(phi, &sn, &cs);
            cosE[k] = cs;
            sinE[k] = sn;
        }
        __syncthreads();
        const float cAe = cA[L - 1];
        for (int s = tid; s < L; s += kThreads) {
            // weight of token s in the chunk-end state; the sequence's very
            // last token has no successor, so only its own lam*dt applies.
            const float g = (last_chunk && s == L - 1) ? gam[s] : ghat[s];
            wst[s] = expf(cAe - cA[s]) * g;
        }
        // ---- (i) masked decay-weighted scores: mask applied before exp
        for (int idx = tid; idx < rows * rows; idx += kThreads) {
            const int i = idx / rows, j = idx % rows;
            const int ti = i / R, tj = j / R;
            float v = 0.f;
            if (tj <= ti) {
                float dot = 0.f;
                for (int n = 0; n < N; ++n) dot += Cs[i * N + n] * Bs[j * N + n];
                const float coef = (ti == tj) ? gam[ti] : ghat[tj];
                v = dot * expf(cA[ti] - cA[tj]) * coef;
            }
            Pm[idx] = v;
        }
        __syncthreads();
        // ---- outputs: (i) diagonal block + (iv) carried-state readout + skip
        for (int idx = tid; idx < rows * P; idx += kThreads) {
            const int i = idx / P, p = idx % P;
            float acc = 0.f;
            for (int j = 0; j < rows; ++j) acc += Pm[i * rows + j] * Xs[j * P + p];
            float off = 0.f;
            for (int n = 0; n < N; ++n) off += Cs[i * N + n] * hs[n * P + p];
            const float yv = acc + expf(cA[i / R]) * off + Dh * Xs[idx];
            stv(a.y, (tok(t0 + i / R) * R + i % R) * P + p, yv);
        }
        __syncthreads();
        // ---- (ii)+(iii): h* <- Rot(-Phi)(exp(cA_end) h* + G)
        const float eA = expf(cAe);
        for (int idx = tid; idx < K2 * P; idx += kThreads) {
            const int k = idx / P, p = idx % P;
            float g0 = 0.f, g1 = 0.f;
            for (int j = 0; j < rows; ++j) {
                const float wx = wst[j / R] * Xs[j * P + p];
                g0 += Bs[j * N + 2 * k] * wx;
                g1 += Bs[j * N + 2 * k + 1] * wx;
            }
            const float u = eA * hs[(2 * k) * P + p] + g0;
            const float v = eA * hs[(2 * k + 1) * P + p] + g1;
            const float cs = cosE[k], sn = sinE[k];
            hs[(2 * k) * P + p] = u * cs + v * sn;
            hs[(2 * k + 1) * P + p] = -u * sn + v * cs;
        }
        __syncthreads();
    }

    // ---- final state: plain-frame h_{T-1} and the raw last token as pending
    if (a.hT) {
        for (int idx = tid; idx < N * P; idx += kThreads) {
            float v = hs[idx];
            if (T == 0) v = a.h0 ? a.h0[bh * N * P + idx] : 0.f;
            a.hT[bh * N * P + idx] = v;
        }
    }
    if (a.bpT && a.wB && T > 0) {  // the last token's normalised B, one warp per rank row
        const int warp = tid >> 5, lane = tid & 31;
        for (int r = warp; r < R; r += kThreads / 32) {
            const int64_t src = tok(T - 1) * R * N + r * N;
            const float sc = bcn_row_scale_warp([&](int n) { return ldv(a.B, src + n); }, N, a.eps);
            for (int n = lane; n < N; n += 32)
                a.bpT[(bh * R + r) * N + n] = fmaf(ldv(a.B, src + n) * sc, a.wB[n], a.bB[(h * R + r) * N + n]);
        }
    } else if (a.bpT) {
        for (int idx = tid; idx < R * N; idx += kThreads)
            a.bpT[bh * R * N + idx] = T > 0 ? ldv(a.B, tok(T - 1) * R * N + idx)
                                            : (a.bp0 ? a.bp0[bh * R * N + idx] : 0.f);
    }
    if (a.xpT) {
        for (int idx = tid; idx < R * P; idx += kThreads)
            a.xpT[bh * R * P + idx] = T > 0 ? ldv(a.x, tok(T - 1) * R * P + idx)
                                            : (a.xp0 ? a.xp0[bh * R * P + idx] : 0.f);
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

}  // namespace m3
