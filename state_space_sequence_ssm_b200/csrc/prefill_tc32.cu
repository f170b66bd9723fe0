// prefill_tc32.cu -- tcgen05 chunked prefill for fp32 I/O at the fp32 bar.
//
// The chunked algorithm of "La dualità: Mamba-2 e Mamba-3" (section "Perché
// conviene: i tensor core": the masked block inside a chunk, the chunk state,
// the recurrence between chunks and the carried state read out through the
// decay), with the Mamba-3 pieces of "Знакомство с Mamba-3" (sections 1-3):
// the trapezoid's previous-token write folded into the off-diagonal weight
// gamma_hat_s = lam_s dt_s + (1 - lam_{s+1}) dt_{s+1}, the pair rotations of
// B and C by the chunk-local cumulative angle, and rank-R MIMO rows -- the
// same algebra as the bf16 tensor-core kernel, for fp32 inputs and outputs.
//
// The page's case for moving this work onto tensor cores is their throughput
// over generic fp32 units (same page, same section).  To keep fp32 accuracy on
// bf16 tensor cores every operand v of the four chunk products is split into
// two bf16 values, hi = bf16(v) and lo = bf16(v - hi) (v - hi - lo is below
// 2^-17 of v), and every product A B is taken as hi.hi + hi.lo + lo.hi in the
// fp32 accumulators: three MMAs where the bf16 kernel takes one, the dropped
// lo.lo term and the splits' rounding about 2^-16 of the product.  Angles,
// decays, the decay mask, the carried state and the epilogue stay fp32.
//
// One CTA of 512 threads per (batch, head) walks its sequence in chunks of
// 128 rows (Q = 128 / R tokens x R ranks), in synchronous phases per chunk:
//   1. per-token scalars, the chunk-local scan of dt*A, the angle table
//      (for chunk c + 1, while the tensor cores run step 3 of chunk c);
//   2. B, C (BC-normed first when the prologue is on) rotated in fp32 and
//      split into 128B-swizzled bf16 hi/lo tiles (K-major), x and w o x
//      split likewise (MN-major);
//   3. one thread issues S = C~ B~^T, G = B~^T (w o X) and Yo = C~ h* (three
//      terms each);
//   4. the decay mask S -> P in fp32, written back to TMEM as hi and lo bf16;
//      Yd = P X (three terms, P read from TMEM);
//   5. the carried state h* <- Rot(-Phi)(exp(cA_end) h* + G) in fp32
//      registers, its hi/lo tiles for the next chunk's Yo;
//   6. y = Yd + exp(cA_t) Yo + D x, stored in fp32.
// Built for headdim 64 and dstate 64 (the hi/lo tiles of one chunk take
// 144 KB of shared memory, 173 KB with the angle table and the scalars; all
// 512 TMEM columns); other fp32 sizes run the SIMT kernel.  Every wait is
// bounded and reports through this kernel's device error word, which
// m3_stream_status reads.
#include <cuda_bf16.h>

#include "bcnorm.cuh"
#include "dcheck.cuh"
#include "m3_internal.h"
#include "tc_primitives.cuh"

namespace m3 {

// This kernel's failure word (an MMA wait that gave up: kErrWaitMma), read and
// cleared by read_tc32_error() on the host.
__device__ unsigned g_tc32_error;

namespace {
using namespace tc;

constexpr int kP = 64, kN = 64, kK2 = kN / 2;
constexpr int kRows = 128;   // rows per chunk = MMA M
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
// Thread roles on TMEM: warp w reads lanes 32 (w % 4) .. +31 (one chunk row per
// thread) and takes column quarter w / 4 of each accumulator.
constexpr int kCQ = kWarps / 4;    // column quarters
constexpr int kTC = kP / kCQ;      // state / output columns per thread (16)
constexpr int kSC = kRows / kCQ;   // S columns per thread in the mask (32)
constexpr uint32_t kTile = kRows * 128;  // one bf16 tile of 128 rows x 64 columns (16 KB)
// TMEM columns: S [0,128), G [128,192), Yo [192,256), Yd [256,320),
// P hi [320,384), P lo [384,448) (P as packed bf16 pairs)
constexpr uint32_t kColS = 0, kColG = 128, kColYo = 192, kColYd = 256, kColPh = 320, kColPl = 384;
constexpr uint32_t kTmemCols = 512;

// shared memory: tiles (hi, lo) of C~, B~, X, w o X (each 128 x 64 bf16),
// h* (64 x 64 bf16), the angle table, the per-token scalars, barriers
constexpr uint32_t OFF_C = 0, OFF_B = OFF_C + 2 * kTile, OFF_X = OFF_B + 2 * kTile, OFF_XW = OFF_X + 2 * kTile;
constexpr uint32_t H_TILE = kN * 128;
constexpr uint32_t OFF_H = OFF_XW + 2 * kTile;
constexpr uint32_t OFF_PHI = OFF_H + 2 * H_TILE;                  // phi [128][K2] fp32
constexpr uint32_t OFF_SCAL = OFF_PHI + kRows * kK2 * 4;
// two buffers (chunk c and c + 1) of {gam, ghat, cA, wst, colf}[128] + {cos, sin}[K2];
// then wtot [8], segment angle totals [kWarps][K2], cA_0
constexpr uint32_t SB32 = 5 * kRows + 2 * kK2;
constexpr uint32_t OFF_BAR = OFF_SCAL + (2 * SB32 + 8 + kWarps * kK2 + 8) * 4;
constexpr uint32_t OFF_MISC = OFF_BAR + 4 * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// Index-check sites of this file (bounds build).
enum : unsigned {
    kSiteScalars = 0x201,  // dt, lam, A
    kSiteTheta = 0x202,    // angle rates
    kSiteRows = 0x203,     // B, C and x rows
    kSiteNorm = 0x204,     // BC-norm weights and biases
    kSiteHead = 0x205,     // D
    kSiteInit = 0x206,     // initial state h0, b_prev, x_prev
    kSiteY = 0x207,        // output rows
    kSiteFinal = 0x208,    // final state and the last token's B and x
};

struct Tc32Args {
    int64_t T, H;
    const float *x, *B, *C, *dt, *lam, *theta, *A, *D;
    int a_tok, th_head;
    const float *h0, *bp0, *xp0;
    const float *wB, *wC, *bB, *bC;  // BC-norm prologue (wB == nullptr: off)
    float eps;
    float *y, *hT, *bpT, *xpT;
};

// v = hi + lo, both bf16: the pair for 8 consecutive values (two uint4 of packed pairs)
__device__ __forceinline__ void split8(const float (&v)[8], uint4 &hi, uint4 &lo) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 hh = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
        const float2 hf = __bfloat1622float2(hh);
        const __nv_bfloat162 ll = __floats2bfloat162_rn(v[2 * e] - hf.x, v[2 * e + 1] - hf.y);
        h[e] = *reinterpret_cast<const uint32_t *>(&hh);
        l[e] = *reinterpret_cast<const uint32_t *>(&ll);
    }
    hi = make_uint4(h[0], h[1], h[2], h[3]);
    lo = make_uint4(l[0], l[1], l[2], l[3]);
}

// sin and cos of a chunk-local angle (|x| < 2^16 * 2 pi): Cody and Waite's
// reduction by 2 pi in two parts (the first, 6.28125, has 8 significant bits,
// so n times it is exact; the second is the rest of 2 pi in fp32), then the
// hardware approximation on [-pi, pi], whose absolute error there is about
// 4e-7.  Used where each angle rotates one chunk's B and C rows only; the
// chunk's total angle, which rotates the carried state once per chunk (so its
// error would compound), takes the full-accuracy sincosf.
__device__ __forceinline__ void sincos_reduced(float x, float *s, float *c) {
    constexpr float kInv2Pi = 0.15915494309189535f;
    constexpr float k2PiHi = 6.28125f;
    constexpr float k2PiLo = 1.9353071795864769e-3f;  // 2 pi - 6.28125
    const float n = rintf(x * kInv2Pi);
    const float r = fmaf(-n, k2PiLo, fmaf(-n, k2PiHi, x));
    __sincosf(r, s, c);
}

// hi and lo of a pair, packed (low half = first value)
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __nv_bfloat162 hh = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(hh);
    const __nv_bfloat162 ll = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&hh);
    lo = *reinterpret_cast<const uint32_t *>(&ll);
}

// hi/lo of this thread's kTC state values (row n, columns c0 ..) into the
// MN-major h* tiles
__device__ __forceinline__ void store_state(uint8_t *hhi, uint8_t *hlo, int n, int c0, const float (&h)[kTC]) {
#pragma unroll
    for (int j = 0; j < kTC / 8; ++j) {
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = h[8 * j + e];
        uint4 hi, lo;
        split8(v, hi, lo);
        *reinterpret_cast<uint4 *>(hhi + sw128(n, c0 / 8 + j)) = hi;
        *reinterpret_cast<uint4 *>(hlo + sw128(n, c0 / 8 + j)) = lo;
    }
}

template <int R>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc32_kernel(const Tc32Args a) {
    constexpr int Q = kRows / R;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *Chi = smem + OFF_C, *Clo = Chi + kTile, *Bhi = smem + OFF_B, *Blo = Bhi + kTile;
    uint8_t *Xhi = smem + OFF_X, *Xlo = Xhi + kTile, *XWhi = smem + OFF_XW, *XWlo = XWhi + kTile;
    uint8_t *Hhi = smem + OFF_H, *Hlo = Hhi + H_TILE;
    float *phi = reinterpret_cast<float *>(smem + OFF_PHI);
    float *sbuf = reinterpret_cast<float *>(smem + OFF_SCAL);  // two chunks' scalars, SB32 floats each
    float *wtot = sbuf + 2 * SB32, *segtot = wtot + 8, *cA0 = segtot + kWarps * kK2;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);  // [0] S/G/Yo, [1] Yd, [2] drain
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
    unsigned *err = &g_tc32_error;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, cq = warp >> 2;  // TMEM lane quarter, column quarter
    const int lq = 32 * wq + lane;            // TMEM lane = chunk row
    const int c0 = kTC * cq;                  // first of this thread's state / output columns
    const bool own_state = lane < 16;         // G (M = 64): lanes 0-15 of each quarter
    const int srow = wq * 16 + lane;          // its state row
    const int64_t bh = blockIdx.x, T = a.T, H = a.H;
    const int64_t b = bh / H, h = bh % H;
    auto tok = [&](int64_t t) { return (b * T + t) * H + h; };
    // buffer extents in elements, for the bounds build's index checks
    const int64_t BH = gridDim.x, nTok = BH * T, nSt = BH * kN * kP;
    const float Dh = dchk::in(kSiteHead, h, 1, H) ? a.D[h] : 0.f;

    if (tid == 0) {
        for (int i = 0; i < 3; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tl = tbase + ((uint32_t)(32 * wq) << 16);

    // carried state (plain frame, pending-inclusive): h0 + beta'_0 b_prev x_prev^T
    float hreg[kTC];
#pragma unroll
    for (int p = 0; p < kTC; ++p) hreg[p] = 0.f;
    if (own_state && T > 0) {
        const float betap0 =
            dchk::in(kSiteScalars, tok(0), 1, nTok) ? (1.f - a.lam[tok(0)]) * a.dt[tok(0)] : 0.f;
        if (a.h0 && dchk::in(kSiteInit, (bh * kN + srow) * kP + c0, kTC, nSt)) {
#pragma unroll
            for (int p = 0; p < kTC; ++p) hreg[p] = a.h0[(bh * kN + srow) * kP + c0 + p];
        }
        if (a.bp0 && a.xp0) {
            for (int r = 0; r < R; ++r) {
                if (!dchk::in(kSiteInit, (bh * R + r) * kN + srow, 1, BH * R * kN) ||
                    !dchk::in(kSiteInit, (bh * R + r) * kP + c0, kTC, BH * R * kP))
                    continue;
                const float cw = betap0 * a.bp0[(bh * R + r) * kN + srow];
#pragma unroll
                for (int p = 0; p < kTC; ++p) hreg[p] = fmaf(cw, a.xp0[(bh * R + r) * kP + c0 + p], hreg[p]);
            }
        }
    }
    if (own_state) store_state(Hhi, Hlo, srow, c0, hreg);

    constexpr uint32_t idS = idesc_bf16(kRows, kRows, 0, 0);
    constexpr uint32_t idG = idesc_bf16(kN, kP, 1, 1);
    constexpr uint32_t idY = idesc_bf16(kRows, kP, 0, 1);
    // ---- 1. per-token scalars of the chunk starting at token t0 into the scalar
    //      buffer sb, the chunk-local scan of dt*A and the angle table.  Every
    //      thread also takes one state pair k and one of kWarps segments of TPS
    //      tokens: the angle increments dt_s theta_s[k], their running sum in
    //      registers, then the earlier segments' totals added.  Two CTA barriers.
    auto phase1 = [&](const int64_t t0, float *sb) {
        float *gam = sb, *ghat = sb + kRows, *cA = sb + 2 * kRows, *wst = sb + 3 * kRows, *colf = sb + 4 * kRows;
        float *cosE = sb + 5 * kRows, *sinE = cosE + kK2;
        constexpr int TPS = Q / kWarps;
        const int kq = tid & 31, sg = tid >> 5;
        float dtv[TPS], thv[TPS];
#pragma unroll
        for (int u = 0; u < TPS; ++u) {
            const int64_t t = t0 + sg * TPS + u;
            const int64_t ti = (a.th_head ? (int64_t)h : tok(t)) * kK2 + kq;
            dtv[u] = (t < T && dchk::in(kSiteScalars, tok(t), 1, nTok)) ? a.dt[tok(t)] : 0.f;
            thv[u] = (t < T && dchk::in(kSiteTheta, ti, 1, (a.th_head ? H : nTok) * kK2)) ? a.theta[ti] : 0.f;
        }
        float acc = 0.f, gh = 0.f;
        if (tid < Q) {
            const int64_t t = t0 + tid;
            float d = 0.f, l = 0.f, nx = 0.f, av = 0.f;
            if (t < T && dchk::in(kSiteScalars, tok(t), 1, nTok) &&
                dchk::in(kSiteScalars, a.a_tok ? tok(t) : h, 1, a.a_tok ? nTok : H)) {
                d = a.dt[tok(t)];
                l = a.lam[tok(t)];
                av = a.a_tok ? a.A[tok(t)] : a.A[h];
                if (t + 1 < T && dchk::in(kSiteScalars, tok(t + 1), 1, nTok))
                    nx = (1.f - a.lam[tok(t + 1)]) * a.dt[tok(t + 1)];
            }
            gam[tid] = l * d;
            gh = l * d + nx;
            ghat[tid] = gh;
            acc = d * av;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, acc, off);
                if (lane >= off) acc += v;
            }
            if (lane == 31) wtot[warp] = acc;
            if (tid == 0) *cA0 = acc;
        }
        float pre[TPS];
        {
            float run = 0.f;
#pragma unroll
            for (int u = 0; u < TPS; ++u) {
                run = fmaf(dtv[u], thv[u], run);
                pre[u] = run;
            }
            segtot[sg * kK2 + kq] = run;
        }
        __syncthreads();
        if (tid < Q) {  // cA_t, the chunk-state weight exp(cA_end - cA_t) ghat_t, the column factor
            constexpr int NW = Q / 32;
            float off = 0.f, offl = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                if (w < warp) off += wtot[w];
                if (w < NW - 1) offl += wtot[w];
            }
            const float ca = acc + off, cend = wtot[NW - 1] + offl;  // cend: the same sum as cA_{Q-1}
            cA[tid] = ca;
            wst[tid] = expf(cend - ca) * gh;
            colf[tid] = expf(*cA0 - ca) * gh;
        }
        {
            float off = 0.f;  // the earlier segments' totals: independent loads, no serial chain
#pragma unroll
            for (int s2 = 0; s2 < kWarps - 1; ++s2)
                if (s2 < sg) off += segtot[s2 * kK2 + kq];
#pragma unroll
            for (int u = 0; u < TPS; ++u) phi[(sg * TPS + u) * kK2 + kq] = pre[u] + off;
            if (sg == kWarps - 1) {  // the chunk's total angle of pair kq
                float sn, cs;
                sincosf(pre[TPS - 1] + off, &sn, &cs);
                cosE[kq] = cs;
                sinE[kq] = sn;
            }
        }
        __syncthreads();
    };
    const int nch = (int)((T + Q - 1) / Q);
    bool ok = true;
    bool issued = false;  // MMAs may be in flight
    phase1(0, sbuf);
    for (int c = 0; c < nch && ok; ++c) {
        const int64_t t0 = (int64_t)c * Q;
        // this chunk's scalars (phase 1 of chunk c + 1 fills the other buffer
        // while the tensor cores run S, G and Yo of chunk c)
        float *sb = sbuf + (c & 1) * SB32;
        float *gam = sb, *ghat = sb + kRows, *cA = sb + 2 * kRows, *wst = sb + 3 * kRows, *colf = sb + 4 * kRows;
        float *cosE = sb + 5 * kRows, *sinE = cosE + kK2;
        // ---- 2. rotated B, C and the value rows as hi/lo tiles: thread (row i,
        //      16-byte chunk j) for rows i = tid / 8 + 64 u, u = 0, 1, the loads
        //      of both rows issued together
        const int j = tid & 7;
        {
            float4 ld[2][6];
            bool valid[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = (tid >> 3) + 64 * u;
                const int64_t t = t0 + i / R;
                const int64_t row = tok(t) * R + i % R;
                valid[u] = t < T && dchk::in(kSiteRows, row * kN + 8 * j, 8, nTok * R * kN) &&
                           dchk::in(kSiteRows, row * kP + 8 * j, 8, nTok * R * kP);
                if (valid[u]) {
                    const float4 *pb = reinterpret_cast<const float4 *>(a.B + row * kN + 8 * j);
                    const float4 *pc = reinterpret_cast<const float4 *>(a.C + row * kN + 8 * j);
                    const float4 *px = reinterpret_cast<const float4 *>(a.x + row * kP + 8 * j);
                    ld[u][0] = pb[0];
                    ld[u][1] = pb[1];
                    ld[u][2] = pc[0];
                    ld[u][3] = pc[1];
                    ld[u][4] = px[0];
                    ld[u][5] = px[1];
                } else {
#pragma unroll
                    for (int e = 0; e < 6; ++e) ld[u][e] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int i = (tid >> 3) + 64 * u;
                const int si = i / R, r = i % R;
                float bb[8] = {ld[u][0].x, ld[u][0].y, ld[u][0].z, ld[u][0].w,
                               ld[u][1].x, ld[u][1].y, ld[u][1].z, ld[u][1].w};
                float cc[8] = {ld[u][2].x, ld[u][2].y, ld[u][2].z, ld[u][2].w,
                               ld[u][3].x, ld[u][3].y, ld[u][3].z, ld[u][3].w};
                const float xx[8] = {ld[u][4].x, ld[u][4].y, ld[u][4].z, ld[u][4].w,
                                     ld[u][5].x, ld[u][5].y, ld[u][5].z, ld[u][5].w};
                if (a.wB && valid[u] && dchk::in(kSiteNorm, (h * R + r) * kN + 8 * j, 8, H * R * kN) &&
                    dchk::in(kSiteNorm, 8 * j, 8, kN)) {  // BC-norm: the row's RMS over its 8 lanes, weight and bias
                    const unsigned grp = 0xffu << (lane & 24);
                    float sb = 0.f, sq = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        sb = fmaf(bb[e], bb[e], sb);
                        sq = fmaf(cc[e], cc[e], sq);
                    }
#pragma unroll
                    for (int o = 1; o < 8; o <<= 1) {
                        sb += __shfl_xor_sync(grp, sb, o);
                        sq += __shfl_xor_sync(grp, sq, o);
                    }
                    const float kb = rsqrtf(sb / (float)kN + a.eps), kc = rsqrtf(sq / (float)kN + a.eps);
                    const float *biB = a.bB + (h * R + r) * kN + 8 * j, *biC = a.bC + (h * R + r) * kN + 8 * j;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        bb[e] = fmaf(bb[e] * kb, a.wB[8 * j + e], biB[e]);
                        cc[e] = fmaf(cc[e] * kc, a.wC[8 * j + e], biC[e]);
                    }
                }
                float vb[8], vc[8], vw[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {  // pair k = 4 j + e: rotate by +phi_s[k]
                    float sn, cs;
                    sincos_reduced(phi[si * kK2 + 4 * j + e], &sn, &cs);
                    vb[2 * e] = bb[2 * e] * cs - bb[2 * e + 1] * sn;
                    vb[2 * e + 1] = bb[2 * e] * sn + bb[2 * e + 1] * cs;
                    vc[2 * e] = cc[2 * e] * cs - cc[2 * e + 1] * sn;
                    vc[2 * e + 1] = cc[2 * e] * sn + cc[2 * e + 1] * cs;
                }
                const float w = wst[si];
#pragma unroll
                for (int e = 0; e < 8; ++e) vw[e] = w * xx[e];
                const uint32_t off = sw128((uint32_t)i, (uint32_t)j);
                uint4 hi, lo;
                split8(vb, hi, lo);
                *reinterpret_cast<uint4 *>(Bhi + off) = hi;
                *reinterpret_cast<uint4 *>(Blo + off) = lo;
                split8(vc, hi, lo);
                *reinterpret_cast<uint4 *>(Chi + off) = hi;
                *reinterpret_cast<uint4 *>(Clo + off) = lo;
                split8(xx, hi, lo);
                *reinterpret_cast<uint4 *>(Xhi + off) = hi;
                *reinterpret_cast<uint4 *>(Xlo + off) = lo;
                split8(vw, hi, lo);
                *reinterpret_cast<uint4 *>(XWhi + off) = hi;
                *reinterpret_cast<uint4 *>(XWlo + off) = lo;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- 3. S = C~ B~^T, G = B~^T (w o X), Yo = C~ h*: hi.hi + hi.lo + lo.hi
        if (tid == 0) {
            tc_fence_after();
            const uint32_t ch[2] = {smem_u32(Chi), smem_u32(Clo)}, bv[2] = {smem_u32(Bhi), smem_u32(Blo)};
            const uint32_t xw[2] = {smem_u32(XWhi), smem_u32(XWlo)}, hh[2] = {smem_u32(Hhi), smem_u32(Hlo)};
            const int ta[3] = {0, 0, 1}, tb[3] = {0, 1, 0};  // (a, b) halves of the three terms
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const uint64_t dCk = sdesc_sw128(ch[ta[q]], 16, 1024), dBk = sdesc_sw128(bv[tb[q]], 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tbase + kColS, dCk + (uint64_t)((kk * 32) >> 4), dBk + (uint64_t)((kk * 32) >> 4), idS,
                             (q | kk) != 0);
            }
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const uint64_t dBm = sdesc_sw128(bv[ta[q]], 16384, 1024), dXw = sdesc_sw128(xw[tb[q]], 16384, 1024);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_bf16(tbase + kColG, dBm + (uint64_t)((ks * 2048) >> 4), dXw + (uint64_t)((ks * 2048) >> 4),
                             idG, (q | ks) != 0);
            }
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const uint64_t dCk = sdesc_sw128(ch[ta[q]], 16, 1024), dH = sdesc_sw128(hh[tb[q]], 16384, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tbase + kColYo, dCk + (uint64_t)((kk * 32) >> 4), dH + (uint64_t)((kk * 2048) >> 4), idY,
                             (q | kk) != 0);
            }
            mma_commit(&bars[0]);
        }
        issued = true;
        // phase 1 of the next chunk while the MMAs run: the angle table is free
        // (phase 2 above was its last reader) and the other scalar buffer was
        // last read by the previous chunk's epilogue
        if (c + 1 < nch) phase1(t0 + Q, sbuf + ((c + 1) & 1) * SB32);
        ok = !__syncthreads_or(!mbar_wait(&bars[0], c & 1, abort_flag, err, kErrWaitMma));
        if (!ok) break;
        tc_fence_after();

        // ---- 4. decay mask S -> P (fp32), written to TMEM as hi and lo bf16:
        //      P(t,s) = S(t,s) exp(cA_t - cA_s) (s < t ? ghat_s : gam_t), 0 for s > t.
        //      While the chunk's decay stays within e^60 the exponential is a row
        //      factor exp(cA_t - cA_0) times the column factor exp(cA_0 - cA_s)
        //      ghat_s (both in fp32 range); deeper chunks take one exp per element.
        {
            const int ti = lq / R;
            const float cai = cA[ti], gi = gam[ti];
            const bool fact = (cA[0] - cA[Q - 1]) < 60.f;  // uniform across the CTA
            const float rowf = expf(cai - cA[0]);
#pragma unroll 1
            for (int g = 0; g < kSC / 16; ++g) {  // this thread's kSC columns, 16 at a time
                const int j0 = kSC * cq + 16 * g;
                float v[16];
                tmem_ld16(tl + kColS + j0, v);
                tmem_wait_ld();
                uint32_t ph[8], pl[8];
#pragma unroll
                for (int e = 0; e < 16; e += 2) {
                    float pv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int tj = (j0 + e + u) / R;
                        const float f = tj < ti ? (fact ? rowf * colf[tj] : expf(cai - cA[tj]) * ghat[tj])
                                                : (tj == ti ? gi : 0.f);
                        pv[u] = v[e + u] * f;
                    }
                    split2(pv[0], pv[1], ph[e >> 1], pl[e >> 1]);
                }
                tmem_st8(tl + kColPh + (uint32_t)(j0 >> 1), ph);
                tmem_st8(tl + kColPl + (uint32_t)(j0 >> 1), pl);
            }
            tmem_wait_st();
        }
        tc_fence_before();
        __syncthreads();
        // Yd = P X: P hi.X hi + P hi.X lo + P lo.X hi, P read from TMEM
        if (tid == 0) {
            tc_fence_after();
            const uint32_t pa[3] = {kColPh, kColPh, kColPl};
            const uint32_t xb[3] = {smem_u32(Xhi), smem_u32(Xlo), smem_u32(Xhi)};
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                const uint64_t dX = sdesc_sw128(xb[q], 16384, 1024);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tbase + kColYd, tbase + pa[q] + (uint32_t)kk * 8u, dX + (uint64_t)((kk * 2048) >> 4),
                                idY, (q | kk) != 0);
            }
            mma_commit(&bars[1]);
        }
        // this thread's x row segment for the epilogue, loaded while the state update runs
        const int ty = lq / R, ry = lq % R;
        const int64_t t_y = t0 + ty;
        float4 xv[kTC / 4];
        if (t_y < T && dchk::in(kSiteRows, (tok(t_y) * R + ry) * kP + c0, kTC, nTok * R * kP)) {
            const float4 *xr = reinterpret_cast<const float4 *>(a.x + (tok(t_y) * R + ry) * kP + c0);
#pragma unroll
            for (int e = 0; e < kTC / 4; ++e) xv[e] = xr[e];
        } else {
#pragma unroll
            for (int e = 0; e < kTC / 4; ++e) xv[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        }

        // ---- 5. carried state: h* <- Rot(-Phi)(exp(cA_end) h* + G), fp32 in registers
        //      (Yo, the last reader of the h* tiles, completed before the mask)
        {
            const float eA = expf(cA[Q - 1]);
            const int kp = (own_state ? srow : 0) >> 1;
            const float cs = cosE[kp], sn = sinE[kp];
            const float sgn = (srow & 1) ? -sn : sn;
            float gv[kTC];
            tmem_ld16(tl + kColG + c0, gv);
            tmem_wait_ld();
#pragma unroll
            for (int p = 0; p < kTC; ++p) {
                const float u = fmaf(eA, hreg[p], gv[p]);
                const float o = __shfl_xor_sync(0xffffffffu, u, 1);
                hreg[p] = fmaf(u, cs, o * sgn);
            }
            if (own_state) store_state(Hhi, Hlo, srow, c0, hreg);
        }

        // ---- 6. y = Yd + exp(cA_t) Yo + D x
        ok = !__syncthreads_or(!mbar_wait(&bars[1], c & 1, abort_flag, err, kErrWaitMma));
        if (!ok) break;
        tc_fence_after();
        {
            const float sc = expf(cA[ty]);
#pragma unroll
            for (int qq = 0; qq < kTC / 16; ++qq) {
                float yd[16], yo[16];
                tmem_ld16(tl + kColYd + c0 + 16 * qq, yd);
                tmem_ld16(tl + kColYo + c0 + 16 * qq, yo);
                tmem_wait_ld();
                if (t_y < T && dchk::in(kSiteY, (tok(t_y) * R + ry) * kP + c0 + 16 * qq, 16, nTok * R * kP)) {
                    float4 *yr = reinterpret_cast<float4 *>(a.y + (tok(t_y) * R + ry) * kP + c0 + 16 * qq);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float4 x4 = xv[4 * qq + e];
                        yr[e] = make_float4(fmaf(Dh, x4.x, fmaf(sc, yo[4 * e], yd[4 * e])),
                                            fmaf(Dh, x4.y, fmaf(sc, yo[4 * e + 1], yd[4 * e + 1])),
                                            fmaf(Dh, x4.z, fmaf(sc, yo[4 * e + 2], yd[4 * e + 2])),
                                            fmaf(Dh, x4.w, fmaf(sc, yo[4 * e + 3], yd[4 * e + 3])));
                    }
                }
            }
        }
        issued = false;  // both batches of MMAs have completed
        fence_proxy_async_smem();  // the new h* tiles, before the next chunk's MMAs
        tc_fence_before();
        __syncthreads();
    }

    if (ok) {  // final state: plain-frame h_{T-1}, the raw last token as the pending term
        if (a.hT && own_state && dchk::in(kSiteFinal, (bh * kN + srow) * kP + c0, kTC, nSt)) {
            float4 *dst = reinterpret_cast<float4 *>(a.hT + (bh * kN + srow) * kP + c0);
#pragma unroll
            for (int p = 0; p < kTC / 4; ++p)
                dst[p] = make_float4(hreg[4 * p], hreg[4 * p + 1], hreg[4 * p + 2], hreg[4 * p + 3]);
        }
        const int64_t last = tok(T - 1);
        if (T > 0 && dchk::in(kSiteFinal, last * R * kN, R * kN, nTok * R * kN) &&
            dchk::in(kSiteFinal, last * R * kP, R * kP, nTok * R * kP) &&
            dchk::in(kSiteFinal, bh * R * kN, R * kN, BH * R * kN) && dchk::in(kSiteFinal, bh * R * kP, R * kP, BH * R * kP) &&
            (!a.wB || (dchk::in(kSiteNorm, h * R * kN, R * kN, H * R * kN)))) {
            if (a.bpT && a.wB) {  // the last token's normalised B, one warp per rank row
                for (int r = warp; r < R; r += kThreads / 32) {
                    const float *src = a.B + (last * R + r) * kN;
                    const float sc = bcn_row_scale_warp([&](int n) { return src[n]; }, kN, a.eps);
                    for (int n = lane; n < kN; n += 32)
                        a.bpT[(bh * R + r) * kN + n] = fmaf(src[n] * sc, a.wB[n], a.bB[(h * R + r) * kN + n]);
                }
            } else if (a.bpT) {
                for (int i = tid; i < R * kN; i += kThreads) a.bpT[bh * R * kN + i] = a.B[last * R * kN + i];
            }
            if (a.xpT)
                for (int i = tid; i < R * kP; i += kThreads) a.xpT[bh * R * kP + i] = a.x[last * R * kP + i];
        }
    } else if (issued && tid == 0) {  // no MMA may still run when TMEM is released
        mma_commit(&bars[2]);
        mbar_wait(&bars[2], 0, nullptr, err, 0, 400000000LL);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
}

template <int R>
cudaError_t launch_r(const Tc32Args &a, int64_t grid, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(prefill_tc32_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    prefill_tc32_kernel<R><<<(unsigned)grid, kThreads, SMEM_BYTES, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

bool prefill_tc32_supported(const Problem &p, const char **why) {
    if (p.bf16) { *why = "fp32 tensor-core prefill: fp32 I/O only"; return false; }
    if (p.P != kP || p.N != kN) { *why = "fp32 tensor-core prefill: headdim 64 and dstate 64 only"; return false; }
    if (p.R != 1 && p.R != 2 && p.R != 4) { *why = "fp32 tensor-core prefill: rank 1, 2 or 4 only"; return false; }
    if (p.segments > 0) { *why = "fp32 tensor-core prefill: sequences are not split"; return false; }
    if (p.T < 1 || p.Bt < 1) { *why = "fp32 tensor-core prefill: empty problem"; return false; }
    if (p.T > (int64_t)1 << 30) { *why = "fp32 tensor-core prefill: seqlen too long"; return false; }
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess || major != 10 ||
        minor != 0) {
        *why = "fp32 tensor-core prefill: needs an sm_100 device";
        return false;
    }
    return true;
}

cudaError_t launch_prefill_tc32(const Problem &p, const char **) {
    Tc32Args a{};
    a.T = p.T;
    a.H = p.H;
    a.x = static_cast<const float *>(p.x);
    a.B = static_cast<const float *>(p.B);
    a.C = static_cast<const float *>(p.C);
    a.dt = static_cast<const float *>(p.dt);
    a.lam = static_cast<const float *>(p.lam);
    a.theta = static_cast<const float *>(p.theta);
    a.A = p.A;
    a.D = p.D;
    a.a_tok = p.a_tok;
    a.th_head = p.th_head;
    a.h0 = p.h0;
    a.bp0 = p.bp0;
    a.xp0 = p.xp0;
    a.wB = p.wB;
    a.wC = p.wC;
    a.bB = p.bB;
    a.bC = p.bC;
    a.eps = p.eps;
    a.y = static_cast<float *>(p.y);
    a.hT = p.hT;
    a.bpT = p.bpT;
    a.xpT = p.xpT;
    const int64_t grid = p.Bt * p.H;
    if (grid == 0) return cudaSuccess;
    if (p.R == 1) return launch_r<1>(a, grid, p.stream);
    if (p.R == 2) return launch_r<2>(a, grid, p.stream);
    return launch_r<4>(a, grid, p.stream);
}

cudaError_t read_tc32_error(unsigned *code) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tc32_error, sizeof v);
    if (e != cudaSuccess) return e;
    if (v) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_tc32_error, &zero, sizeof zero);
    }
    *code = v;
    return e;
}

M3_DCHECK_READER(read_dcheck_tc32)

}  // namespace m3
