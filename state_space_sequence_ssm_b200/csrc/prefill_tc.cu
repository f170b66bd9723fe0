// prefill_tc.cu -- tcgen05/TMEM/TMA chunked prefill (bf16 I/O, fp32 state).
//
// The chunked algorithm of "La dualità: Mamba-2 e Mamba-3" (section "Perché
// conviene: i tensor core": a masked block inside each chunk, chunk states,
// a recurrence between chunks, and the state read out through the decay),
// extended with the Mamba-3 pieces of "Знакомство с Mamba-3" (sections 1-3):
// the trapezoid's previous-token write folded into the off-diagonal weight
// gamma_hat_s = lam_s dt_s + (1 - lam_{s+1}) dt_{s+1}, the pair rotations
// of B and C by the chunk-local cumulative angle, and rank-R MIMO rows.
//
// One CTA per (batch, head) walks its sequence in chunks of 128 rows
// (Q = 128 / R tokens x R ranks), which is the M = 128 shape of one tcgen05
// MMA.  Roles (192 threads):
//   warps 0-3  compute warpgroup: per-token scalars, angles, in-place
//              rotation of the B/C tiles, the decay mask S -> P, the fp32
//              carried state (in registers), and the output epilogue;
//   warp 4     TMA producer: x, B, C tiles (128B-swizzled) into a 2-stage ring;
//   warp 5     TMEM owner and single-thread MMA issuer.
// Per chunk c (tensor cores, bf16 operands from shared memory, fp32 in TMEM):
//   S  = C~ B~^T               (128 x 128, K = N)      -> masked into P (bf16)
//   G  = B~^T (w o X)          (N x 64,  K = 128 rows) chunk state
//   Yo = C~ h*_{c-1}           (128 x 64, K = N)       carried-state readout
//   Yd = P X                   (128 x 64, K = 128 rows) diagonal block
// and on CUDA cores: y = Yd + exp(cA_t) Yo + D x;
// h*_c = Rot(-Phi_c)(exp(cA_end) h*_{c-1} + G) kept in fp32 registers (the
// plain frame, so no angle ever exceeds one chunk's sum).
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "m3_internal.h"
#include "tc_primitives.cuh"

namespace m3 {

// Device-side failure word (bounded waits that gave up); read and cleared by
// read_device_error() on the host.
__device__ unsigned g_device_error;

namespace {
using namespace tc;

constexpr int kP = 64;           // head dim this kernel is built for
constexpr int kRows = 128;       // rows per chunk = MMA M
constexpr int kCompute = 128;    // compute warpgroup threads (warps 0-3)
constexpr int kWarpTma = 4;
constexpr int kWarpMma = 5;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColG = 128, kColYo = 192, kColYd = 256;
constexpr float kLog2e = 1.4426950408889634f;

template <int N, int R>
struct Cfg {
    static constexpr int Q = kRows / R;      // tokens per chunk
    static constexpr int K2 = N / 2;         // state pairs
    static constexpr int KB = N / 64;        // 64-wide blocks of the state dim
    static constexpr int TPP = kCompute / K2;  // threads per pair (angle pass)
    static constexpr int TPT = Q / TPP;      // tokens per thread (angle pass)
    static constexpr uint32_t X_BYTES = kRows * 128;         // 16 KB
    static constexpr uint32_t BC_BYTES = KB * kRows * 128;   // one B or C tile
    static constexpr uint32_t STAGE_BYTES = X_BYTES + 2 * BC_BYTES;
    static constexpr bool P_IN_C = (N >= 128);  // P reuses the chunk's C~ tile
    static constexpr uint32_t OFF_XW = 2 * STAGE_BYTES;
    static constexpr uint32_t OFF_HB = OFF_XW + X_BYTES;
    static constexpr uint32_t HB_BYTES = N * 128;
    static constexpr uint32_t OFF_P = OFF_HB + HB_BYTES;
    static constexpr uint32_t P_BYTES = P_IN_C ? 0u : 2u * kRows * 128u;
    static constexpr uint32_t OFF_SCAL = OFF_P + P_BYTES;
    static constexpr uint32_t SCAL_FLOATS = 5 * Q + 2 * K2 + TPP * K2 + 8;
    static constexpr uint32_t OFF_BAR = OFF_SCAL + ((SCAL_FLOATS * 4 + 15) / 16) * 16;
    static constexpr uint32_t NBARS = 9;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024 alignment
    static_assert(K2 <= kCompute && kCompute % K2 == 0, "pairs must tile the warpgroup");
    static_assert(Q % TPP == 0, "tokens must split across a pair's threads");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct TcArgs {
    int64_t T, H;
    int nchunks;
    const __nv_bfloat16 *x, *B, *dt, *lam, *theta;
    const float *A, *D, *h0, *bp0, *xp0;
    __nv_bfloat16 *y;
    float *hT, *bpT, *xpT;
};

__device__ __forceinline__ float bf(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }

// OR-reduction over the compute warpgroup that doubles as its barrier: every
// thread gets the same answer, so control flow stays uniform on failure.
__device__ __forceinline__ bool bar_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 1, 128, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void cbar() { named_bar(1, kCompute); }

// bf16 copy of the 64 fp32 values of state row n into the 128B-swizzled
// MN-major operand tile (row n = K index of the readout MMA).
__device__ __forceinline__ void store_state_row(uint8_t *hb, int n, const float (&h)[64]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint4 v;
        v.x = pack_bf16(h[8 * j + 0], h[8 * j + 1]);
        v.y = pack_bf16(h[8 * j + 2], h[8 * j + 3]);
        v.z = pack_bf16(h[8 * j + 4], h[8 * j + 5]);
        v.w = pack_bf16(h[8 * j + 6], h[8 * j + 7]);
        *reinterpret_cast<uint4 *>(hb + sw128(n, j)) = v;
    }
}

template <int N, int R>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const TcArgs a) {
    using C = Cfg<N, R>;
    constexpr int Q = C::Q, K2 = C::K2, KB = C::KB, TPP = C::TPP, TPT = C::TPT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *cAl2 = reinterpret_cast<float *>(smem + C::OFF_SCAL);  // chunk-local cumsum of dt*A, log2 units
    float *gam = cAl2 + Q;      // lam dt           (diagonal weight)
    float *ghat = gam + Q;      // lam dt + (1-lam') dt'  (off-diagonal weight)
    float *wst = ghat + Q;      // exp(cA_end - cA_s) * ghat_s  (chunk-state weight)
    float *dts = wst + Q;       // dt
    float *cosE = dts + Q;      // cos/sin of the chunk's total angle per pair
    float *sinE = cosE + K2;
    float *phis = sinE + K2;    // partial angle sums [TPP][K2]
    float *wtot = phis + TPP * K2;  // per-warp totals of the dt*A scan
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *full = bars, *empty = bars + 2, *ops_ready = bars + 4, *sgo_done = bars + 5, *p_ready = bars + 6,
             *yd_done = bars + 7, *drain = bars + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    unsigned *err = &g_device_error;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bh = blockIdx.x;
    const int64_t T = a.T, H = a.H;
    const int64_t b = bh / H, h = bh % H;
    auto tok = [&](int64_t t) { return (b * T + t) * H + h; };

    if (tid == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(&empty[0], 1);
        mbar_init(&empty[1], 1);
        mbar_init(ops_ready, 1);
        mbar_init(sgo_done, 1);
        mbar_init(p_ready, 1);
        mbar_init(yd_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kWarpTma && lane == 0) {
        prefetch_tmap(&tmX);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmC);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const int nchunks = a.nchunks;

    if (warp == kWarpTma) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                if (c >= 2 && !mbar_wait(&empty[s], ((c >> 1) - 1) & 1, abort_flag, err, kErrWaitCompute)) break;
                uint8_t *st = smem + s * C::STAGE_BYTES;
                const int t0 = c * Q;
                mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
                tma_load_5d(st, &tmX, &full[s], 0, 0, (int)h, t0, (int)b);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_5d(st + C::X_BYTES + kb * 16384, &tmB, &full[s], kb * 64, 0, (int)h, t0, (int)b);
                    tma_load_5d(st + C::X_BYTES + C::BC_BYTES + kb * 16384, &tmC, &full[s], kb * 64, 0, (int)h, t0,
                                (int)b);
                }
                issued = c + 1;
            }
            if (*abort_flag) {  // let the copies already in flight land before the CTA exits
                for (int c = issued - 2 > 0 ? issued - 2 : 0; c < issued; ++c)
                    mbar_wait(&full[c & 1], (c >> 1) & 1, nullptr, err, 0, 400000000LL);
            }
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idG = idesc_bf16(N, 64, 1, 1);
            constexpr uint32_t idY = idesc_bf16(128, 64, 0, 1);
            const uint32_t xw = smem_u32(smem + C::OFF_XW);
            const uint32_t hb = smem_u32(smem + C::OFF_HB);
            bool any = false;
            for (int c = 0; c < nchunks; ++c) {
                const int s = c & 1;
                const uint32_t xs = smem_u32(smem + s * C::STAGE_BYTES);
                const uint32_t bs = xs + C::X_BYTES;
                const uint32_t cs = bs + C::BC_BYTES;
                const uint32_t pb = C::P_IN_C ? cs : smem_u32(smem + C::OFF_P);
                if (!mbar_wait(ops_ready, c & 1, abort_flag, err, kErrWaitCompute)) break;
                tc_fence_after();
                any = true;
                // S = C~ B~^T  (both K-major over the state dim)
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tbase + kColS, sdesc_sw128(cs + kb * 16384 + kk * 32, 16, 1024),
                                 sdesc_sw128(bs + kb * 16384 + kk * 32, 16, 1024), idS, (kb | kk) != 0);
                // G = B~^T (w o X)  (both MN-major, K = the chunk's 128 rows)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tbase + kColG, sdesc_sw128(bs + ks * 2048, 16384, 1024),
                             sdesc_sw128(xw + ks * 2048, 16384, 1024), idG, ks != 0);
                // Yo = C~ h*  (C~ K-major; h* MN-major, K = state rows)
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tbase + kColYo, sdesc_sw128(cs + kb * 16384 + kk * 32, 16, 1024),
                                 sdesc_sw128(hb + (kb * 4 + kk) * 2048, 16384, 1024), idY, (kb | kk) != 0);
                mma_commit(sgo_done);
                if (!mbar_wait(p_ready, c & 1, abort_flag, err, kErrWaitCompute)) break;
                tc_fence_after();
                // Yd = P X  (P K-major over the chunk's rows; X MN-major)
#pragma unroll
                for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tbase + kColYd, sdesc_sw128(pb + kb * 16384 + kk * 32, 16, 1024),
                                 sdesc_sw128(xs + (kb * 4 + kk) * 2048, 16384, 1024), idY, (kb | kk) != 0);
                mma_commit(yd_done);
            }
            if (*abort_flag && any) {  // no MMA may still run when TMEM is released
                mma_commit(drain);
                mbar_wait(drain, 0, nullptr, err, 0, 400000000LL);
            }
        }
    } else {
        // ------------------------------------------------------------ compute warpgroup
        const bool own_state = (N == 128) || (lane < 16);
        const int srow = (N == 128) ? tid : (warp * 16 + lane);  // TMEM lane layout of G
        uint8_t *hbuf = smem + C::OFF_HB;
        const float Ah2 = a.A[h] * kLog2e;
        const float Dh = a.D[h];
        float hreg[64];
        // initial state h0 + beta'_0 b_prev x_prev^T (pending write of token -1)
        {
            float betap0 = 0.f;
            if (T > 0) betap0 = (1.f - bf(a.lam, tok(0))) * bf(a.dt, tok(0));
#pragma unroll
            for (int p = 0; p < 64; ++p) hreg[p] = 0.f;
            if (own_state) {
                if (a.h0) {
#pragma unroll
                    for (int p = 0; p < 64; ++p) hreg[p] = a.h0[(bh * N + srow) * kP + p];
                }
                if (a.bp0 && a.xp0) {
                    for (int r = 0; r < R; ++r) {
                        const float cb = betap0 * a.bp0[(bh * R + r) * N + srow];
#pragma unroll
                        for (int p = 0; p < 64; ++p) hreg[p] = fmaf(cb, a.xp0[(bh * R + r) * kP + p], hreg[p]);
                    }
                }
                store_state_row(hbuf, srow, hreg);
            }
        }
        bool ok = true;
        for (int c = 0; c < nchunks && ok; ++c) {
            const int s = c & 1;
            const int64_t t0 = (int64_t)c * Q;
            uint8_t *st = smem + s * C::STAGE_BYTES;
            uint8_t *xst = st;
            uint8_t *bst = st + C::X_BYTES;
            uint8_t *cst = bst + C::BC_BYTES;
            uint8_t *pbuf = C::P_IN_C ? cst : smem + C::OFF_P;

            // ---- A. per-token scalars and the chunk-local scan of dt*A
            float acc = 0.f;
            if (tid < Q) {
                const int64_t t = t0 + tid;
                float d = 0.f, l = 0.f, nx = 0.f;
                if (t < T) {
                    d = bf(a.dt, tok(t));
                    l = bf(a.lam, tok(t));
                }
                if (t + 1 < T) nx = (1.f - bf(a.lam, tok(t + 1))) * bf(a.dt, tok(t + 1));
                dts[tid] = d;
                gam[tid] = l * d;
                ghat[tid] = l * d + nx;
                acc = d * Ah2;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const float v = __shfl_up_sync(0xffffffffu, acc, off);
                    if (lane >= off) acc += v;
                }
                if (lane == 31 || tid == Q - 1) wtot[warp] = acc;
            }
            cbar();
            if (tid < Q) {
                float off = 0.f, tot = 0.f;
#pragma unroll
                for (int w = 0; w < (Q + 31) / 32; ++w) {
                    const float v = wtot[w];
                    if (w < warp) off += v;
                    tot += v;
                }
                const float ca = acc + off;
                cAl2[tid] = ca;
                wst[tid] = ex2(tot - ca) * ghat[tid];
            }
            // ---- wait for this chunk's tiles
            ok = !bar_any(!mbar_wait(&full[s], (c >> 1) & 1, abort_flag, err, kErrWaitTma));
            if (!ok) break;

            // ---- B. cumulative angles per pair and in-place rotation of B and C
            {
                const int k = tid % K2, part = tid / K2;
                const int64_t thb = (int64_t)k;
                float loc = 0.f;
#pragma unroll 4
                for (int j = 0; j < TPT; ++j) {
                    const int i = part * TPT + j;
                    const int64_t t = t0 + i;
                    const float th = t < T ? bf(a.theta, tok(t) * K2 + thb) : 0.f;
                    loc = fmaf(dts[i], th, loc);
                }
                phis[part * K2 + k] = loc;
                cbar();
                float phi = 0.f;
                for (int q = 0; q < part; ++q) phi += phis[q * K2 + k];
                const uint32_t cofs = (uint32_t)(k >> 5) * 16384u;       // 64-wide K block
                const uint32_t chunkj = (uint32_t)((k & 31) >> 2);        // 16-byte chunk in the row
                const uint32_t within = (uint32_t)(k & 3) * 4u;           // byte offset of the pair
#pragma unroll 2
                for (int j = 0; j < TPT; ++j) {
                    const int i = part * TPT + j;
                    const int64_t t = t0 + i;
                    const float th = t < T ? bf(a.theta, tok(t) * K2 + thb) : 0.f;
                    phi = fmaf(dts[i], th, phi);
                    float sn, cs;
                    sincos_reduced(phi, &sn, &cs);
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const uint32_t row = (uint32_t)(i * R + r);
                        const uint32_t off = cofs + sw128(row, chunkj) + within;
                        uint32_t *pb = reinterpret_cast<uint32_t *>(bst + off);
                        uint32_t *pc = reinterpret_cast<uint32_t *>(cst + off);
                        const float2 vb = unpack_bf16(*pb);
                        const float2 vc = unpack_bf16(*pc);
                        *pb = pack_bf16(vb.x * cs - vb.y * sn, vb.x * sn + vb.y * cs);
                        *pc = pack_bf16(vc.x * cs - vc.y * sn, vc.x * sn + vc.y * cs);
                    }
                }
                if (part == TPP - 1) {
                    float sn, cs;
                    sincos_reduced(phi, &sn, &cs);
                    cosE[k] = cs;
                    sinE[k] = sn;
                }
            }
            // ---- C. w o X (chunk-state weights on the value rows)
            {
                const int row = tid;
                const float wv = wst[row / R];
                uint8_t *xw = smem + C::OFF_XW;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t off = sw128(row, j);
                    uint4 v = *reinterpret_cast<const uint4 *>(xst + off);
                    float2 f;
                    f = unpack_bf16(v.x); v.x = pack_bf16(f.x * wv, f.y * wv);
                    f = unpack_bf16(v.y); v.y = pack_bf16(f.x * wv, f.y * wv);
                    f = unpack_bf16(v.z); v.z = pack_bf16(f.x * wv, f.y * wv);
                    f = unpack_bf16(v.w); v.w = pack_bf16(f.x * wv, f.y * wv);
                    *reinterpret_cast<uint4 *>(xw + off) = v;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            cbar();
            if (tid == 0) mbar_arrive(ops_ready);

            // ---- D. decay mask: P = S o L, L(t,s) = exp(cA_t - cA_s) * (s < t ? ghat_s : gam_t), s <= t
            ok = !bar_any(!mbar_wait(sgo_done, c & 1, abort_flag, err, kErrWaitMma));
            if (!ok) break;
            tc_fence_after();
            {
                const int row = tid;
                const int ti = row / R;
                const float cai = cAl2[ti], gi = gam[ti];
                const uint32_t tl = tbase + ((uint32_t)(32 * warp) << 16);
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint8_t *dst = pbuf + (cb >> 1) * 16384;
                    if (cb <= warp) {  // warp-uniform: blocks right of the diagonal are all zero
                        float v[32];
                        tmem_ld32(tl + kColS + 32 * cb, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t pk[4];
#pragma unroll
                            for (int e = 0; e < 8; e += 2) {
                                float pv[2];
#pragma unroll
                                for (int u = 0; u < 2; ++u) {
                                    const int jcol = 32 * cb + 8 * q + e + u;
                                    const int tj = jcol / R;
                                    float val = 0.f;
                                    if (tj < ti) val = v[8 * q + e + u] * ex2(cai - cAl2[tj]) * ghat[tj];
                                    else if (tj == ti) val = v[8 * q + e + u] * gi;
                                    pv[u] = val;
                                }
                                pk[e >> 1] = pack_bf16(pv[0], pv[1]);
                            }
                            const uint32_t jj = (uint32_t)((cb & 1) * 4 + q);
                            *reinterpret_cast<uint4 *>(dst + sw128(row, jj)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint32_t jj = (uint32_t)((cb & 1) * 4 + q);
                            *reinterpret_cast<uint4 *>(dst + sw128(row, jj)) = make_uint4(0u, 0u, 0u, 0u);
                        }
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            cbar();
            if (tid == 0) mbar_arrive(p_ready);

            // ---- E. carried state: h* <- Rot(-Phi)(exp(cA_end) h* + G), fp32 in registers
            {
                const uint32_t tl = tbase + ((uint32_t)(32 * warp) << 16);
                float g[64];
                {
                    float g0[32], g1[32];
                    tmem_ld32(tl + kColG, g0);
                    tmem_ld32(tl + kColG + 32, g1);
                    tmem_wait_ld();
#pragma unroll
                    for (int p = 0; p < 32; ++p) {
                        g[p] = g0[p];
                        g[32 + p] = g1[p];
                    }
                }
                const float eA = ex2(cAl2[Q - 1]);
                const int kp = (own_state ? srow : 0) >> 1;
                const float cs = cosE[kp], sn = sinE[kp];
                const float sgn = (srow & 1) ? -sn : sn;
#pragma unroll
                for (int p = 0; p < 64; ++p) {
                    const float u = fmaf(eA, hreg[p], g[p]);
                    const float o = __shfl_xor_sync(0xffffffffu, u, 1);
                    hreg[p] = fmaf(u, cs, o * sgn);
                }
                if (own_state) store_state_row(hbuf, srow, hreg);
            }

            // ---- F. epilogue: y = Yd + exp(cA_t) Yo + D x
            ok = !bar_any(!mbar_wait(yd_done, c & 1, abort_flag, err, kErrWaitMma));
            if (!ok) break;
            tc_fence_after();
            {
                const int row = tid;
                const int ti = row / R, r = row % R;
                const int64_t t = t0 + ti;
                const float sc = ex2(cAl2[ti]);
                const uint32_t tl = tbase + ((uint32_t)(32 * warp) << 16);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float yd[32], yo[32];
                    tmem_ld32(tl + kColYd + 32 * half, yd);
                    tmem_ld32(tl + kColYo + 32 * half, yo);
                    tmem_wait_ld();
                    if (t < T) {
                        __nv_bfloat16 *yrow = a.y + (tok(t) * R + r) * kP + 32 * half;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint4 xv = *reinterpret_cast<const uint4 *>(xst + sw128(row, 4 * half + q));
                            const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
                            uint32_t o[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 xf = unpack_bf16(xs[e]);
                                const int p = 8 * q + 2 * e;
                                const float y0 = fmaf(Dh, xf.x, fmaf(sc, yo[p], yd[p]));
                                const float y1 = fmaf(Dh, xf.y, fmaf(sc, yo[p + 1], yd[p + 1]));
                                o[e] = pack_bf16(y0, y1);
                            }
                            *reinterpret_cast<uint4 *>(yrow + 8 * q) = make_uint4(o[0], o[1], o[2], o[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            cbar();
            if (tid == 0) mbar_arrive(&empty[s]);
        }
        // ---- final state: plain-frame h_{T-1}, raw last token as the pending term
        if (ok) {
            if (a.hT && own_state) {
                float4 *dst = reinterpret_cast<float4 *>(a.hT + (bh * N + srow) * kP);
#pragma unroll
                for (int p = 0; p < 16; ++p)
                    dst[p] = make_float4(hreg[4 * p], hreg[4 * p + 1], hreg[4 * p + 2], hreg[4 * p + 3]);
            }
            if (a.bpT)
                for (int i = tid; i < R * N; i += kCompute)
                    a.bpT[bh * R * N + i] = bf(a.B, tok(T - 1) * R * N + i);
            if (a.xpT)
                for (int i = tid; i < R * kP; i += kCompute)
                    a.xpT[bh * R * kP + i] = bf(a.x, tok(T - 1) * R * kP + i);
        }
    }

    __syncwarp();  // reconverge the single-lane roles before the block barrier
    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [Bt, T, H, R, inner] bf16, box = {64 of inner, R, 1 head, Q tokens, 1 batch}, 128B swizzle.
bool make_map(CUtensorMap *m, const void *base, int64_t inner, int64_t R, int64_t H, int64_t T, int64_t Bt, int Q) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[5] = {(cuuint64_t)inner, (cuuint64_t)R, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)Bt};
    const cuuint64_t strides[4] = {(cuuint64_t)(inner * 2), (cuuint64_t)(R * inner * 2),
                                   (cuuint64_t)(H * R * inner * 2), (cuuint64_t)(T * H * R * inner * 2)};
    const cuuint32_t box[5] = {64, (cuuint32_t)R, 1, (cuuint32_t)Q, 1};
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int N, int R>
cudaError_t launch_nr(const Problem &p, const char **why) {
    using C = Cfg<N, R>;
    CUtensorMap mx, mb, mc;
    if (!make_map(&mx, p.x, kP, R, p.H, p.T, p.Bt, C::Q) || !make_map(&mb, p.B, N, R, p.H, p.T, p.Bt, C::Q) ||
        !make_map(&mc, p.C, N, R, p.H, p.T, p.Bt, C::Q)) {
        *why = "tensor-core prefill: TMA descriptor encoding failed";
        return cudaErrorNotSupported;
    }
    TcArgs a;
    a.T = p.T;
    a.H = p.H;
    a.nchunks = (int)((p.T + C::Q - 1) / C::Q);
    a.x = (const __nv_bfloat16 *)p.x;
    a.B = (const __nv_bfloat16 *)p.B;
    a.dt = (const __nv_bfloat16 *)p.dt;
    a.lam = (const __nv_bfloat16 *)p.lam;
    a.theta = (const __nv_bfloat16 *)p.theta;
    a.A = p.A;
    a.D = p.D;
    a.h0 = p.h0;
    a.bp0 = p.bp0;
    a.xp0 = p.xp0;
    a.y = (__nv_bfloat16 *)p.y;
    a.hT = p.hT;
    a.bpT = p.bpT;
    a.xpT = p.xpT;
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<N, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    prefill_tc_kernel<N, R><<<(unsigned)(p.Bt * p.H), kThreads, C::SMEM_BYTES, p.stream>>>(mx, mb, mc, a);
    return cudaGetLastError();
}

bool device_is_sm100() {
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
    return major == 10 && minor == 0;
}

}  // namespace

bool prefill_tc_supported(const Problem &p, const char **why) {
    if (!p.bf16) { *why = "tensor-core prefill: bf16 I/O only"; return false; }
    if (p.P != kP) { *why = "tensor-core prefill: headdim 64 only"; return false; }
    if (p.N != 64 && p.N != 128) { *why = "tensor-core prefill: dstate 64 or 128 only"; return false; }
    if (p.R != 1 && p.R != 2 && p.R != 4) { *why = "tensor-core prefill: rank 1, 2 or 4 only"; return false; }
    if (p.T < 1 || p.Bt < 1) { *why = "tensor-core prefill: empty problem"; return false; }
    if (p.T > (int64_t)1 << 30) { *why = "tensor-core prefill: seqlen too long"; return false; }
    if (!device_is_sm100()) { *why = "tensor-core prefill: needs an sm_100 device"; return false; }
    return true;
}

size_t prefill_tc_workspace(const Problem &) { return 0; }

cudaError_t launch_prefill_tc(const Problem &p, const char **why) {
    if (p.N == 128) {
        if (p.R == 1) return launch_nr<128, 1>(p, why);
        if (p.R == 2) return launch_nr<128, 2>(p, why);
        return launch_nr<128, 4>(p, why);
    }
    if (p.R == 1) return launch_nr<64, 1>(p, why);
    if (p.R == 2) return launch_nr<64, 2>(p, why);
    return launch_nr<64, 4>(p, why);
}

cudaError_t read_device_error(unsigned *code, cudaStream_t stream) {
    *code = 0;
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    unsigned v = 0;
    e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof v);
    if (e != cudaSuccess) return e;
    if (v) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
    }
    *code = v;
    return e;
}

}  // namespace m3
