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
// (Q = 128 / R tokens x R ranks), the M = 128 shape of one tcgen05 MMA.
// Per chunk c the tensor cores compute (bf16 operands in shared memory,
// fp32 accumulators in TMEM)
//   S  = C~ B~^T          (128 x 128, K = N)        masked into P (bf16)
//   G  = B~^T (w o X)     (N x 64,  K = 128 rows)   chunk state
//   Yo = C~ h*_{c-1}      (128 x 64, K = N)         carried-state readout
//   Yd = P X              (128 x 64, K = 128 rows)  diagonal block
// and the CUDA cores y = Yd + exp(cA_t) Yo + D x and
// h*_c = Rot(-Phi_c)(exp(cA_end) h*_{c-1} + G), the carried state kept in
// fp32 registers in the plain frame (no angle exceeds one chunk's sum).
//
// Warp roles (576 threads: 18 warps of 96 registers), pipelined across chunks:
//   warps 0-7   prologue: per-token scalars and the chunk-local scan of dt*A,
//               cumulative angles, the in-place rotation of the B and C
//               tiles, and w o X;
//   warps 8-15  state: the carried state update, the decay mask S -> P
//               (written to TMEM, the A operand of Yd) and the epilogue
//               (about one chunk behind the prologue); each thread owns one
//               TMEM lane (row) and one 32-column half;
//   warp 16     TMA producers: lane 0 fills a 2-stage ring of B and C tiles
//               (freed as soon as S, G and Yo have read them), lane 1 a
//               3-stage ring of x tiles (freed after the epilogue), both
//               128B-swizzled (for N = 64 also L2 prefetches of the chunks
//               ahead);
//   warp 17     TMEM owner and single-thread MMA issuer.
// A sequence too long for the grid to fill the GPU is split into segments
// (a summary pass, then this pass per segment, which first scans the
// summaries of the segments before its own: the MODE template argument).
// Every wait is bounded; a wait that gives up records a code that the host
// reads back with m3_stream_status() and the CTA drains and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "dcheck.cuh"
#include "m3_internal.h"
#include "tc_primitives.cuh"

namespace m3 {

// Device-side failure word (bounded waits that gave up); read and cleared by
// read_device_error() on the host.
__device__ unsigned g_device_error;

// Scratch of m3_scan_fwd_static (per-segment states of split sequences), so
// that entry point needs no caller workspace.  24 MiB covers the split of a
// 64-sequence, 65,536-token, N = 128 problem (about 19 MiB).
constexpr size_t kStaticScratchBytes = size_t(24) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {
using namespace tc;

constexpr int kP = 64;           // head dim this kernel is built for
constexpr int kRows = 128;       // rows per chunk = MMA M
constexpr int kPro = 256;        // prologue threads (warps 0-7)
constexpr int kSt = 256;         // state / epilogue threads (warps 8-15)
constexpr int kWarpTma = 16;
constexpr int kWarpMma = 17;
constexpr int kThreads = 576;
constexpr uint32_t kTmemCols = 512;
// TMEM columns: S [0,128), G [128,192), Yo double-buffered [192,320), Yd [320,384),
// P (bf16 pairs) [384,448)
constexpr uint32_t kColS = 0, kColG = 128, kColYo = 192, kColYd = 320, kColP = 384;
constexpr int kNX = 3;   // x tile stages (also the number of per-chunk scalar buffers)
constexpr uint32_t kBarPro = 1, kBarState = 2;  // named barriers of the two warpgroups
constexpr float kLog2e = 1.4426950408889634f;
// Sequence splitting (host policy): at most kMaxSegments segments of at least
// kMinSegChunks chunks; a summary-pass chunk costs about kSumCost of a
// main-pass chunk, and every CTA about kCtaCost chunk-times of its own
// (launch, set-up, pipeline fill and drain).
constexpr int64_t kMaxSegments = 64, kMinSegChunks = 8;
// Clock cycles a split sequence's main pass waits for a flag (about 1 s):
// half the pipeline waits' budget, so that a summary that is never published
// is reported as such (code 0x8) rather than as a stalled pipeline wait.
// Summaries are published within the time of one segment's summary pass
// (milliseconds for any problem that fits in device memory).
constexpr long long kFlagBudget = 2000000000LL;
constexpr double kSumCost = 0.55, kCtaCost = 2.0;

// SEP: the MIMO projections' token rows land in staging tiles of their own
// (N = 64, R > 1, where shared memory has room) instead of in the first rows
// of the rank-row tiles, so that widening them needs no barrier.
template <int N, int R, bool SEP = false>
struct Cfg {
    static constexpr int Q = kRows / R;      // tokens per chunk
    static constexpr int K2 = N / 2;         // state pairs
    static constexpr int KB = N / 64;        // 64-wide blocks of the state dim
    static constexpr int G4 = K2 / 4;        // groups of 4 pairs = one 16-byte chunk of a row
    static constexpr int NPART = kPro / G4;  // token parts of the angle pass
    static constexpr int TPT = Q / NPART;    // tokens per thread in the angle pass
    static constexpr int TB = (2 / R) < 1 ? 1 : ((2 / R) < TPT ? (2 / R) : TPT);  // tokens per rotation batch
    // chunks of tiles prefetched into L2 ahead of their load.  Measured: for
    // N = 128 any prefetch distance over-fetches (lines evicted before their
    // load) and costs time, so none; for N = 64 (half the bytes per chunk)
    // three chunks are as good as or better than fewer.
    static constexpr int PREFETCH = N == 128 ? 0 : 3;
    static constexpr uint32_t X_BYTES = kRows * 128;         // 16 KB
    static constexpr uint32_t BC_BYTES = KB * kRows * 128;   // one B or C tile
    static constexpr uint32_t BCS_BYTES = 2 * BC_BYTES;      // one stage of the B/C ring
    static constexpr uint32_t OFF_BC = 0;                    // 2 stages of {B, C}
    static constexpr uint32_t OFF_X = OFF_BC + 2 * BCS_BYTES;  // kNX stages of x
    static constexpr uint32_t OFF_XW = OFF_X + kNX * X_BYTES;
    static constexpr uint32_t OFF_HB = OFF_XW + X_BYTES;
    static constexpr uint32_t HB_BYTES = N * 128;
    static constexpr uint32_t OFF_SCAL = OFF_HB + HB_BYTES;
    // kNX buffers of {cAl2, gam, ghat, colf}[Q] + {cos, sin}[K2] (read by the
    // state warpgroup a chunk later) + {wst, dts}[Q] + phis[NPART][K2] + wtot[16]
    static constexpr uint32_t SB = 4 * Q + 2 * K2;
    // + the BC-norm biases of this head as bf16 pairs [2][R][K2] (with the
    // MIMO projections: the B and C weights) and the row scales of the chunk's
    // B and C tiles [2][128], + the MIMO projections' x weights as bf16 pairs
    // [R][P/2] and y weights [R][P]
    static constexpr uint32_t SCAL_FLOATS =
        kNX * SB + 2 * Q + NPART * K2 + 16 + 2 * R * K2 + 2 * kRows + R * kP / 2 + R * kP;
    static constexpr uint32_t OFF_BAR = OFF_SCAL + ((SCAL_FLOATS * 4 + 15) / 16) * 16;
    static constexpr uint32_t NBARS = 20;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
    // staging (SEP): 2 stages of {B, C} token-row tiles, then kNX x token-row tiles
    static constexpr uint32_t STG_ROWS = SEP ? (uint32_t)Q * 128u : 0u;  // one 64-column block of token rows
    static constexpr uint32_t STG_BC = KB * STG_ROWS;
    static constexpr uint32_t OFF_STG = ((OFF_MISC + 16 + 1023) / 1024) * 1024;
    static constexpr uint32_t OFF_STGX = OFF_STG + 4 * STG_BC;
    static constexpr uint32_t SMEM_BYTES =
        (SEP ? OFF_STGX + kNX * STG_ROWS : OFF_MISC + 16) + 1024;  // + slack for 1024 alignment
    static_assert(K2 % 4 == 0 && kPro % G4 == 0, "pair groups must tile the prologue threads");
    static_assert(Q % NPART == 0 && TPT % TB == 0, "tokens must split across the angle-pass parts");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

struct TcArgs {
    int64_t T, H, BH;  // BH = batch * heads
    int nchunks;
    int cpseg;         // chunks per segment (nchunks when the sequence is not split)
    int nseg;          // segments per sequence
    const __nv_bfloat16 *x, *B, *dt, *lam, *theta;
    const float *A, *D, *h0, *bp0, *xp0;
    const float *A_tok;  // non-null: A per token-head [Bt, T, H] (A unused)
    int th_head;         // theta fixed per head, [H, N/2]
    const float *wB, *wC, *bB, *bC;  // BC-norm prologue (BCN instantiations)
    float eps;
    // MIMO projections (PROJ instantiations): x, B, C and y hold one row per
    // token-head; wx, wy [H, R, P] and wB, wC [H, R, N] widen them to rank R
    const float *pwx, *pwB, *pwC, *pwy;
    __nv_bfloat16 *y;
    float *hT, *bpT, *xpT;
    // Split sequences: ws_h [nseg][BH][N][P] fp32 holds in slot j + 1 the
    // summary pass's local end state of segment j; ws_m [nseg][BH][N] holds
    // segment j's transition exp(cA) Rot(-Phi) as (e cos, e sin) per pair;
    // flags [nseg][BH] (zeroed before the summary pass): [j][bh] for j <
    // nseg - 1 is set to 1 once segment j's summary is published (2 if that
    // CTA gave up), [nseg - 1][bh] once the main pass has read the caller's
    // initial state (the last segment overwrites it when resumed in place).
    float *ws_h, *ws_m;
    unsigned *flags;
};

__device__ __forceinline__ float bf(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float bf16_bits(unsigned short u) { return __uint_as_float((uint32_t)u << 16); }

// OR-reduction over one role's threads that doubles as its barrier: every
// thread gets the same answer, so control flow stays uniform on failure.
template <uint32_t ID, uint32_t COUNT>
__device__ __forceinline__ bool bar_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "n"(ID), "n"(COUNT)
        : "memory");
    return r != 0;
}
// The same over one warp (no barrier between warps): a role whose warps signal
// the MMA issuer one arrival each lets its warps drift apart within a chunk.
__device__ __forceinline__ bool warp_any(bool pred) { return __any_sync(0xffffffffu, pred) != 0; }

// bf16 copy of 32 fp32 values (columns 32*half ..) of state row n into the
// 128B-swizzled MN-major operand tile (row n = K index of the readout MMA).
__device__ __forceinline__ void store_state_half(uint8_t *hb, int n, int half, const float (&h)[32]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        uint4 v;
        v.x = pack_bf16(h[8 * j + 0], h[8 * j + 1]);
        v.y = pack_bf16(h[8 * j + 2], h[8 * j + 3]);
        v.z = pack_bf16(h[8 * j + 4], h[8 * j + 5]);
        v.w = pack_bf16(h[8 * j + 6], h[8 * j + 7]);
        *reinterpret_cast<uint4 *>(hb + sw128(n, 4 * half + j)) = v;
    }
}

// Rotate the pair (u, v) packed in `uv` (u in the low half) by the angle whose
// cosine is packed twice in `cc` and whose sine is packed as (-s, s) in `nss`:
// (u c - v s, u s + v c), in packed bf16x2 arithmetic.
__device__ __forceinline__ uint32_t rot_pair(uint32_t uv, uint32_t cc, uint32_t nss) {
    const uint32_t vu = __byte_perm(uv, 0u, 0x1032u);  // (v, u)
    __nv_bfloat162 t = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&vu),
                               *reinterpret_cast<const __nv_bfloat162 *>(&nss));
    __nv_bfloat162 o = __hfma2(*reinterpret_cast<const __nv_bfloat162 *>(&uv),
                               *reinterpret_cast<const __nv_bfloat162 *>(&cc), t);
    return *reinterpret_cast<uint32_t *>(&o);
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    __nv_bfloat162 o = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&a),
                               *reinterpret_cast<const __nv_bfloat162 *>(&b));
    return *reinterpret_cast<uint32_t *>(&o);
}

// BC-norm row scale 1 / sqrt(mean_n v^2 + eps) of row `row` of a 128B-swizzled
// K-major tile of KB 64-column blocks (one thread per row).
// The squares are formed by the mixed-precision multiply-add (bf16 operands,
// fp32 addend and result: the bf16 product is exact in fp32), two running
// sums for the two halves of each bf16 pair.
template <int KB>
__device__ __forceinline__ float bc_row_scale(const uint8_t *tile, uint32_t row, float inv_n, float eps) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
        for (uint32_t j = 0; j < 8; ++j) {
            const uint4 v = *reinterpret_cast<const uint4 *>(tile + kb * 16384 + sw128(row, j));
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                unsigned short lo, hi;
                asm("mov.b32 {%0, %1}, %2;" : "=h"(lo), "=h"(hi) : "r"(u[e]));
                asm("fma.rn.f32.bf16 %0, %1, %1, %0;" : "+f"(s0) : "h"(lo));
                asm("fma.rn.f32.bf16 %0, %1, %1, %0;" : "+f"(s1) : "h"(hi));
            }
        }
    return rsqrtf(fmaf(s0 + s1, inv_n, eps));
}

// The BC-norm affine map of this thread's 4 pairs of one row: b * sc * w + bias
// in packed bf16x2 arithmetic (w: the thread's four weight pairs; bias: its
// four bias pairs of this head and rank; sc: the row's scale).
__device__ __forceinline__ uint4 bc_norm_row(uint4 v, const uint32_t (&w2)[4], uint4 b2, float sc) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    const uint32_t s2 = pack_bf16(sc, sc);
    const uint32_t bb[4] = {b2.x, b2.y, b2.z, b2.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint32_t sw = mul_bf16x2(s2, w2[e]);
        __nv_bfloat162 r = __hfma2(*reinterpret_cast<const __nv_bfloat162 *>(&u[e]),
                                   *reinterpret_cast<const __nv_bfloat162 *>(&sw),
                                   *reinterpret_cast<const __nv_bfloat162 *>(&bb[e]));
        o[e] = *reinterpret_cast<uint32_t *>(&r);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// Decay mask of S (from TMEM) into P (bf16 pairs, written back to TMEM as the
// A operand of Yd = P X): P(t,s) = S(t,s) exp(cA_t - cA_s) (s < t ? ghat_s :
// gam_t) for s <= t, else 0.  `row` is the thread's row (its TMEM lane), `wq`
// its lane quarter; 32-column blocks strictly right of the quarter's diagonal
// are all zero (warp-uniform), blocks strictly left need no causal test.
// When the chunk's whole decay stays within 2^-100 the exponential factorises
// into a row factor exp(cA_t - cA_0) and a column factor
// colf_s = exp(cA_0 - cA_s) ghat_s (both in fp32 range), so each element
// costs two multiplies; otherwise every element takes its own exp.
template <int R, int Q>
__device__ __forceinline__ void mask_to_tmem(int cbA, int cbB, int wq, int row, uint32_t tl, const float *cAl2,
                                             const float *gam, const float *ghat, const float *colf) {
    constexpr int NT = 16 / R;  // tokens per 16-column half block
    const int ti = row / R;
    const float cai = cAl2[ti], gi = gam[ti];
    const float ca0 = cAl2[0];
    const bool fact = (ca0 - cAl2[Q - 1]) < 100.f;  // uniform across the CTA
    const float rowf = ex2(cai - ca0);
#pragma unroll 1
    for (int bi = 0; bi < 2; ++bi) {
        const int cb = bi == 0 ? cbA : cbB;  // this thread's two 32-column blocks
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
            uint32_t pk[8];
            if (cb <= wq) {
                float v[16];
                tmem_ld16(tl + kColS + 32 * cb + 16 * hf, v);
                const int tb = (32 * cb + 16 * hf) / R;
                if (fact) {
                    float cf[NT];
#pragma unroll
                    for (int k = 0; k < NT; ++k) cf[k] = colf[tb + k];
                    tmem_wait_ld();
                    if (cb < wq) {
#pragma unroll
                        for (int k = 0; k < 16; k += 2)
                            pk[k >> 1] = pack_bf16(v[k] * cf[k / R] * rowf, v[k + 1] * cf[(k + 1) / R] * rowf);
                    } else {
#pragma unroll
                        for (int k = 0; k < 16; k += 2) {
                            float pv[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const int tj = tb + (k + u) / R;
                                const float f = tj < ti ? cf[(k + u) / R] * rowf : (tj == ti ? gi : 0.f);
                                pv[u] = v[k + u] * f;
                            }
                            pk[k >> 1] = pack_bf16(pv[0], pv[1]);
                        }
                    }
                } else {
                    float ca[NT], gh[NT];
#pragma unroll
                    for (int k = 0; k < NT; ++k) {
                        ca[k] = cAl2[tb + k];
                        gh[k] = ghat[tb + k];
                    }
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; k += 2) {
                        float pv[2];
#pragma unroll
                        for (int u = 0; u < 2; ++u) {
                            const int tj = tb + (k + u) / R;
                            const float coef = tj < ti ? gh[(k + u) / R] : (tj == ti ? gi : 0.f);
                            pv[u] = v[k + u] * ex2(fminf(cai - ca[(k + u) / R], 0.f)) * coef;
                        }
                        pk[k >> 1] = pack_bf16(pv[0], pv[1]);
                    }
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) pk[k] = 0u;
            }
            tmem_st8(tl + kColP + 16 * cb + 8 * hf, pk);
        }
    }
    tmem_wait_st();
}

struct Bars {
    uint64_t *full_bc, *empty_bc, *full_x, *empty_x, *ops, *sg, *hrdy, *p, *yd, *drain, *sc;
    uint64_t *sd;  // S of the chunk done (the plain kernel's mask starts on it, before G and Yo)
};

// Pass kinds.  kWhole: the full forward pass, one CTA per sequence.
// kSummary: the summary pass of a split sequence -- only the chunk states and
// the carried-state chain over one segment, from a zero state (segment 0: the
// caller's initial state), ending in the segment's local end state and its
// transition, published for the main pass.  kSegment: the full forward pass
// over one segment, from the scan of the summaries before it (look-back).
constexpr int kWhole = 0, kSummary = 1, kSegment = 2;

// Index-check sites of this file (bounds build).
enum : unsigned {
    kSiteScalars = 0x101,  // dt, lam, per-token A
    kSiteHead = 0x102,     // A, D per head
    kSiteNorm = 0x103,     // BC-norm weights and biases
    kSiteTheta = 0x104,    // angle rates
    kSiteFlags = 0x105,    // split sequences: segment flags
    kSiteWsH = 0x106,      // split sequences: segment end states
    kSiteWsM = 0x107,      // split sequences: segment transitions
    kSiteInit = 0x108,     // initial state h0, b_prev, x_prev
    kSiteY = 0x109,        // output rows
    kSiteFinal = 0x10a,    // final state and the last token's B and x
    kSiteProj = 0x10b,     // MIMO projection weights
};

// FEAT: which optional input layouts the instantiation reads from the
// arguments -- bit 0: A per token-head (A_tok), bit 1: theta fixed per head
// (th_head); 0 is the plain method, compiled without those branches, and
// each layout alone has an instantiation of its own.  BCN: the BC-norm
// prologue (with FEAT = 3).  PROJ: the
// MIMO projections (not with BCN): the tile loads bring one
// row per token, the prologue widens B, C and x to the R rows of each token
// in shared memory, and the epilogue sums each token's R output rows with
// the y weights into one row.
template <int N, int R, int MODE, int FEAT, bool BCN, bool PROJ = false>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmT,
                  const TcArgs a) {
    constexpr bool kSep = PROJ && N == 64 && R > 1;  // the projections' token rows in staging tiles
    using C = Cfg<N, R, kSep>;
    constexpr int Q = C::Q, K2 = C::K2, KB = C::KB, G4 = C::G4, NPART = C::NPART, TPT = C::TPT, TB = C::TB;
    constexpr bool SUM = MODE == kSummary, SEGD = MODE != kWhole;
    constexpr bool GEN = FEAT != 0;                               // some optional layout compiled in
    // The state warps signal the MMA issuer one arrival per warp (and agree on
    // a failed wait within the warp), instead of a barrier of all 256 threads
    // and one arrival, where that measured faster: the split passes and the
    // per-head-theta instantiation (the plain, per-token-A, BC-norm and
    // projection ones measured the same or slower that way).
    constexpr bool kWarpSig = SEGD || FEAT == 2;
    constexpr uint32_t kStArrivals = kWarpSig ? kSt / 32 : 1;
    const float *const A_tok = (FEAT & 1) ? a.A_tok : nullptr;  // A per token-head, or none
    const bool th_head = (FEAT & 2) && a.th_head;               // theta fixed per head
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *scal = reinterpret_cast<float *>(smem + C::OFF_SCAL);
    // kNX per-chunk buffers (index c % kNX) of cAl2 (chunk-local cumsum of
    // dt*A, log2 units), gam = lam dt (diagonal weight), ghat = lam dt +
    // (1-lam') dt' (off-diagonal weight), colf (column factor of the mask) and
    // cos/sin of each pair's total angle over the chunk
    float *sbuf = scal;
    float *wst = scal + kNX * C::SB;  // exp(cA_end - cA_s) ghat_s (chunk-state weight)
    float *dts = wst + Q;             // dt
    float *phis = dts + Q;            // partial angle sums [NPART][K2]
    // per-warp totals of the dt*A scan ([0, 4)); [4] = cA of token 0; [8, 12):
    // per-warp totals of the dt scan (angle rates fixed per head)
    float *wtot = phis + NPART * K2;
    uint32_t *sbias = reinterpret_cast<uint32_t *>(wtot + 16);  // BC-norm biases [B, C][R][K2] (bf16 pairs)
    float *rsc = reinterpret_cast<float *>(sbias + 2 * R * C::K2);  // BC-norm row scales [B, C][128]
    uint32_t *sxw = reinterpret_cast<uint32_t *>(rsc + 2 * kRows);  // projections: x weights [R][P/2] (bf16 pairs)
    float *swy = reinterpret_cast<float *>(sxw + R * kP / 2);        // projections: y weights [R][P]
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    Bars bb{bars, bars + 2, bars + 4, bars + 7, bars + 10, bars + 11, bars + 12, bars + 13, bars + 14, bars + 15,
            bars + 16, bars + 19};
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    // first chunk of this CTA's segment, re-read where needed (a register
    // held across the prologue warps' loop would spill)
    volatile int *chunk0 = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);
    unsigned *err = &g_device_error;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // segment-major CTA order: CTAs of neighbouring heads share dt/lam sectors
    const uint32_t BH = SEGD ? (uint32_t)a.BH : gridDim.x;
    const int seg = SEGD ? (int)(blockIdx.x / BH) : 0;
    const int64_t bh = SEGD ? blockIdx.x % BH : blockIdx.x;
    const int64_t T = a.T, H = a.H;
    const int64_t b = bh / H, h = bh % H;
    auto tok = [&](int64_t t) { return (b * T + t) * H + h; };
    // buffer extents in elements, for the bounds build's index checks
    const int64_t nTok = (int64_t)a.BH * T, nSt = (int64_t)a.BH * N * kP, nSeg = SEGD ? (int64_t)a.nseg : 1;

    // the main pass is launched as a programmatic dependent of the summary
    // pass: its CTAs take SMs as summary CTAs leave them, and all summary CTAs
    // are resident (or done) before any of them starts, so its bounded waits
    // on their flags always wait on running CTAs
    if (SUM && tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bb.full_bc[i], 1);
            mbar_init(&bb.empty_bc[i], 1);
        }
        for (int i = 0; i < kNX; ++i) {
            mbar_init(&bb.full_x[i], 1);
            mbar_init(&bb.empty_x[i], kStArrivals);
            mbar_init(&bb.sc[i], 1);  // per-chunk scalars published to the state warpgroup
        }
        mbar_init(bb.ops, 1);
        mbar_init(bb.sg, 1);
        mbar_init(bb.hrdy, kStArrivals);
        mbar_init(bb.p, kStArrivals);
        mbar_init(bb.yd, 1);
        mbar_init(bb.drain, 1);
        mbar_init(bb.sd, 1);
        *abort_flag = 0;
        *chunk0 = SEGD ? (int)(blockIdx.x / (uint32_t)a.BH) * a.cpseg : 0;
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
        prefetch_tmap(&tmT);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    // this CTA's chunks [cb, cb + nloc); ring stages and mbarrier phases
    // count from the segment's first chunk (local index i)
    const int cb = SEGD ? seg * a.cpseg : 0;
    const int nloc = SEGD ? ((a.nchunks - cb < a.cpseg) ? a.nchunks - cb : a.cpseg) : a.nchunks;
    auto first_chunk = [&]() { return SEGD ? *chunk0 : 0; };

    if (warp == kWarpTma) {
        // ============================================================ TMA producers
        if (lane == 0) {
            // B/C ring (2 stages), plus L2 prefetches of everything a chunk needs
            auto prefetch_chunk = [&](int c) {
                const int t0 = c * Q;
                tma_prefetch_5d(&tmX, 0, 0, (int)h, t0, (int)b);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    tma_prefetch_5d(&tmB, kb * 64, 0, (int)h, t0, (int)b);
                    if (!SUM) tma_prefetch_5d(&tmC, kb * 64, 0, (int)h, t0, (int)b);
                }
                if (!th_head) tma_prefetch_4d(&tmT, 0, (int)h, t0, (int)b);  // read straight into registers
            };
            int issued = 0;
            for (int i = 0; i < C::PREFETCH && i < nloc; ++i) prefetch_chunk(cb + i);
            for (int i = 0; i < nloc; ++i) {
                if (i + C::PREFETCH < nloc) prefetch_chunk(cb + i + C::PREFETCH);
                const int s = i & 1;
                if (i >= 2 && !mbar_wait(&bb.empty_bc[s], ((i >> 1) - 1) & 1, abort_flag, err, kErrWaitMma)) break;
                uint8_t *st = smem + C::OFF_BC + s * C::BCS_BYTES;
                const int t0 = (cb + i) * Q;
                // (with the projections a tile load brings one row per token)
                mbar_arrive_expect_tx(&bb.full_bc[s], (SUM ? C::BC_BYTES : C::BCS_BYTES) / (PROJ ? R : 1));
                uint8_t *sb = kSep ? smem + C::OFF_STG + s * 2 * C::STG_BC : st;
                const uint32_t blk = kSep ? C::STG_ROWS : 16384u, ctile = kSep ? C::STG_BC : C::BC_BYTES;
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_5d(sb + kb * blk, &tmB, &bb.full_bc[s], kb * 64, 0, (int)h, t0, (int)b);
                    if (!SUM)
                        tma_load_5d(sb + ctile + kb * blk, &tmC, &bb.full_bc[s], kb * 64, 0, (int)h, t0, (int)b);
                }
                issued = i + 1;
            }
            if (*abort_flag) {  // let the copies already in flight land before the CTA exits
                for (int i = issued - 2 > 0 ? issued - 2 : 0; i < issued; ++i)
                    mbar_wait(&bb.full_bc[i & 1], (i >> 1) & 1, nullptr, err, 0, 400000000LL);
            }
        } else if (lane == 1) {
            // x ring (kNX stages), freed by the epilogue (the summary pass: by the
            // state update, once w o X has been formed from it)
            int issued = 0;
            for (int i = 0; i < nloc; ++i) {
                const int s = i % kNX;
                if (i >= kNX && !mbar_wait(&bb.empty_x[s], ((i / kNX) - 1) & 1, abort_flag, err, kErrWaitCompute))
                    break;
                mbar_arrive_expect_tx(&bb.full_x[s], C::X_BYTES / (PROJ ? R : 1));
                tma_load_5d(kSep ? smem + C::OFF_STGX + s * C::STG_ROWS : smem + C::OFF_X + s * C::X_BYTES, &tmX,
                            &bb.full_x[s], 0, 0, (int)h, (cb + i) * Q, (int)b);
                issued = i + 1;
            }
            if (*abort_flag) {
                for (int i = issued - kNX > 0 ? issued - kNX : 0; i < issued; ++i)
                    mbar_wait(&bb.full_x[i % kNX], (i / kNX) & 1, nullptr, err, 0, 400000000LL);
            }
        }
    } else if (warp == kWarpMma) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idG = idesc_bf16(N, 64, 1, 1);
            constexpr uint32_t idY = idesc_bf16(128, 64, 0, 1);
            // Operand descriptors per tile; an offset inside a tile is added to the
            // 14-bit start-address field (address >> 4), which cannot carry because
            // shared-memory addresses stay below 256 KB.
            const uint64_t dXw = sdesc_sw128(smem_u32(smem + C::OFF_XW), 16384, 1024);
            const uint64_t dHb = sdesc_sw128(smem_u32(smem + C::OFF_HB), 16384, 1024);
            const uint32_t bc0 = smem_u32(smem + C::OFF_BC);
            const uint32_t x0 = smem_u32(smem + C::OFF_X);
            bool any = false;
            for (int i = 0; i < nloc; ++i) {
                const int s = i & 1, sx = i % kNX;
                const uint32_t bs = bc0 + (uint32_t)s * C::BCS_BYTES;
                const uint32_t cs = bs + C::BC_BYTES;
                const uint64_t dX = sdesc_sw128(x0 + (uint32_t)sx * C::X_BYTES, 16384, 1024);  // X, MN-major
                const uint64_t dBk = sdesc_sw128(bs, 16, 1024);     // B~, K-major
                const uint64_t dBm = sdesc_sw128(bs, 16384, 1024);  // B~^T, MN-major
                const uint64_t dCk = sdesc_sw128(cs, 16, 1024);     // C~, K-major
                // S(i) as soon as the rotated tiles and w o X are in place
                if (!mbar_wait(bb.ops, i & 1, abort_flag, err, kErrWaitCompute)) break;
                tc_fence_after();
                any = true;
                if (!SUM) {
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t o = (uint64_t)((kb * 16384 + kk * 32) >> 4);
                            mma_bf16(tbase + kColS, dCk + o, dBk + o, idS, (kb | kk) != 0);
                        }
                    mma_commit(bb.sd);
                }
                // G(i) and Yo(i) once the state warpgroup has consumed G(i-1) and
                // published h*_{i-1} (completion i of hrdy; the first is the initial state)
                if (!mbar_wait(bb.hrdy, i & 1, abort_flag, err, kErrWaitCompute)) break;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint64_t o = (uint64_t)((ks * 2048) >> 4);
                    mma_bf16(tbase + kColG, dBm + o, dXw + o, idG, ks != 0);
                }
                if (!SUM) {
                    const uint32_t yo = tbase + kColYo + (uint32_t)(i & 1) * 64u;
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16(yo, dCk + (uint64_t)((kb * 16384 + kk * 32) >> 4),
                                     dHb + (uint64_t)(((kb * 4 + kk) * 2048) >> 4), idY, (kb | kk) != 0);
                }
                mma_commit(bb.sg);
                mma_commit(&bb.empty_bc[s]);  // the B/C stage is free once these MMAs are done
                if (SUM) continue;
                // Yd(i) = P X once P is in TMEM and the epilogue of i-1 has read Yd
                if (!mbar_wait(bb.p, i & 1, abort_flag, err, kErrWaitCompute)) break;
                if (i >= 1 && !mbar_wait(&bb.empty_x[(i - 1) % kNX], ((i - 1) / kNX) & 1, abort_flag, err,
                                         kErrWaitCompute))
                    break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tbase + kColYd, tbase + kColP + (uint32_t)kk * 8u,
                                dX + (uint64_t)((kk * 2048) >> 4), idY, kk != 0);
                mma_commit(bb.yd);
            }
            if (*abort_flag && any) {  // no MMA may still run when TMEM is released
                mma_commit(bb.drain);
                mbar_wait(bb.drain, 0, nullptr, err, 0, 400000000LL);
            }
        }
    } else if (warp < 8) {
        // ============================================================ prologue warps (0-7)
        const float Ah2 = (A_tok || !dchk::in(kSiteHead, h, 1, H)) ? 0.f : a.A[h] * kLog2e;
        uint8_t *xw = smem + C::OFF_XW;
        const unsigned short *dtr = reinterpret_cast<const unsigned short *>(a.dt);
        const unsigned short *lmr = reinterpret_cast<const unsigned short *>(a.lam);
        const int g = tid % G4, part = tid / G4;  // angle pass: 4 pairs x TPT tokens per thread
        // raw bf16 bits of dt, lam for this thread's token and the one after it,
        // loaded one chunk ahead and converted only when used
        unsigned short pd = 0, pl = 0, pd1 = 0, pl1 = 0;
        float pa = 0.f;  // A of this thread's token (per-token A only)
        auto prefetch_scalars = [&](int64_t t0s) {
            const int64_t t = t0s + tid;
            pd = pl = pd1 = pl1 = 0;
            if (tid < Q && t < T && dchk::in(kSiteScalars, tok(t), 1, nTok)) {
                pd = __ldg(dtr + tok(t));
                pl = __ldg(lmr + tok(t));
                if (A_tok) pa = __ldg(A_tok + tok(t));
                if (t + 1 < T && dchk::in(kSiteScalars, tok(t + 1), 1, nTok)) {
                    pd1 = __ldg(dtr + tok(t + 1));
                    pl1 = __ldg(lmr + tok(t + 1));
                }
            }
        };
        // theta of this thread's 4 pairs for its TPT tokens, read straight from
        // global memory into registers one chunk ahead of use
        uint2 thr[TPT];
        // BC-norm: this thread's 4 weight pairs of B and C; the head's biases in
        // shared memory (visible after the first barrier of the chunk loop)
        uint32_t wB2[4] = {0u, 0u, 0u, 0u}, wC2[4] = {0u, 0u, 0u, 0u};
        if (BCN) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int n = 8 * g + 2 * e;
                if (!dchk::in(kSiteNorm, n, 2, N)) continue;
                wB2[e] = pack_bf16(a.wB[n], a.wB[n + 1]);
                wC2[e] = pack_bf16(a.wC[n], a.wC[n + 1]);
            }
            for (int i = tid; i < 2 * R * K2; i += kPro) {
                const int which = i / (R * K2), rk = i % (R * K2);
                const int64_t o = (h * R + rk / K2) * N + 2 * (rk % K2);
                const float *src = (which ? a.bC : a.bB) + o;
                sbias[i] = dchk::in(kSiteNorm, o, 2, H * R * N) ? pack_bf16(src[0], src[1]) : 0u;
            }
        }
        if (PROJ) {  // the head's projection weights: B, C and x as bf16 pairs, y in fp32
            for (int i = tid; i < 2 * R * K2; i += kPro) {
                const int which = i / (R * K2), rk = i % (R * K2);
                const int64_t o = (h * R + rk / K2) * N + 2 * (rk % K2);
                const float *src = (which ? a.pwC : a.pwB) + o;
                sbias[i] = dchk::in(kSiteProj, o, 2, H * R * N) ? pack_bf16(src[0], src[1]) : 0u;
            }
            for (int i = tid; i < R * kP / 2; i += kPro) {
                const int64_t o = h * R * kP + 2 * i;
                sxw[i] = dchk::in(kSiteProj, o, 2, H * R * kP) ? pack_bf16(a.pwx[o], a.pwx[o + 1]) : 0u;
            }
            for (int i = tid; i < R * kP; i += kPro)
                swy[i] = dchk::in(kSiteProj, h * R * kP + i, 1, H * R * kP) ? a.pwy[h * R * kP + i] : 0.f;
        }
        // angle rates fixed per head: the thread's 4 pairs, for the whole sequence
        float thh[4] = {0.f, 0.f, 0.f, 0.f};
        if (th_head) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                thh[e] = dchk::in(kSiteTheta, h * K2 + 4 * g + e, 1, H * K2) ? bf(a.theta, h * K2 + 4 * g + e) : 0.f;
        }
        auto prefetch_theta = [&](int64_t t0s) {
            if (th_head) return;
#pragma unroll
            for (int j = 0; j < TPT; ++j) {
                const int64_t t = t0s + part * TPT + j;
                thr[j] = (t < T && dchk::in(kSiteTheta, tok(t) * K2 + 4 * g, 4, nTok * K2))
                             ? __ldg(reinterpret_cast<const uint2 *>(a.theta + tok(t) * K2 + 4 * g))
                             : make_uint2(0u, 0u);
            }
        };
        prefetch_scalars((int64_t)cb * Q);
        prefetch_theta((int64_t)cb * Q);
        for (int lc = 0; lc < nloc; ++lc) {
            const int s = lc & 1, sx = lc % kNX;
            float *cAl2 = sbuf + sx * C::SB;
            float *gam = cAl2 + Q;
            float *ghat = gam + Q;
            float *colf = ghat + Q;
            float *cosE = colf + Q;
            float *sinE = cosE + K2;
            uint8_t *bst = smem + C::OFF_BC + s * C::BCS_BYTES;
            uint8_t *cst = bst + C::BC_BYTES;
            uint8_t *xst = smem + C::OFF_X + sx * C::X_BYTES;
            // the scalar buffer lc % kNX is free once the epilogue of lc - kNX is done
            if (lc >= kNX && bar_any<kBarPro, kPro>(!mbar_wait(&bb.empty_x[sx], ((lc / kNX) - 1) & 1, abort_flag,
                                                              err, kErrWaitCompute)))
                break;

            // ---- A. per-token scalars and the chunk-local scan of dt*A
            float acc = 0.f, acd = 0.f;
            {
                const float d = bf16_bits(pd), l = bf16_bits(pl);
                const float nx = (1.f - bf16_bits(pl1)) * bf16_bits(pd1);  // 0 past the sequence end
                const float a2 = A_tok ? pa * kLog2e : Ah2;                // A_t in log2 units
                if (lc + 1 < nloc) prefetch_scalars((int64_t)(first_chunk() + lc + 1) * Q);
                if (tid < Q) {
                    dts[tid] = d;
                    gam[tid] = l * d;
                    ghat[tid] = l * d + nx;
                    acc = d * a2;
                    if (tid == 0) wtot[4] = acc;  // cA of the chunk's first token
#pragma unroll
                    for (int off = 1; off < 32; off <<= 1) {
                        const float v = __shfl_up_sync(0xffffffffu, acc, off);
                        if (lane >= off) acc += v;
                    }
                    if (lane == 31) wtot[warp] = acc;
                    if (th_head) {  // chunk-local cumulative dt: the angle is theta_k times it
                        acd = d;
#pragma unroll
                        for (int off = 1; off < 32; off <<= 1) {
                            const float v = __shfl_up_sync(0xffffffffu, acd, off);
                            if (lane >= off) acd += v;
                        }
                        if (lane == 31) wtot[8 + warp] = acd;
                    }
                }
            }
            named_bar(kBarPro, kPro);
            if (tid < Q) {
                float off = 0.f, tot = 0.f;
#pragma unroll
                for (int w = 0; w < Q / 32; ++w) {
                    const float v = wtot[w];
                    if (w < warp) off += v;
                    tot += v;
                }
                const float ca = acc + off;
                cAl2[tid] = ca;
                wst[tid] = ex2(tot - ca) * ghat[tid];
                // column factor of the decay mask, relative to the chunk's first token
                colf[tid] = ex2(wtot[4] - ca) * ghat[tid];
                if (th_head) {  // dts becomes the cumulative dt (read after the next barrier)
                    float offd = 0.f;
#pragma unroll
                    for (int w = 0; w < Q / 32; ++w)
                        if (w < warp) offd += wtot[8 + w];
                    dts[tid] = acd + offd;
                }
            }

            // ---- B. cumulative angles of 4 pairs per thread, in-place rotation
            //      of B and C
            {
                float loc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < TPT; ++j) {
                    if (th_head) break;
                    const float di = dts[part * TPT + j];
                    const float2 t01 = unpack_bf16(thr[j].x), t23 = unpack_bf16(thr[j].y);
                    loc[0] = fmaf(di, t01.x, loc[0]);
                    loc[1] = fmaf(di, t01.y, loc[1]);
                    loc[2] = fmaf(di, t23.x, loc[2]);
                    loc[3] = fmaf(di, t23.y, loc[3]);
                }
                *reinterpret_cast<float4 *>(phis + part * K2 + 4 * g) = make_float4(loc[0], loc[1], loc[2], loc[3]);
                // the B/C tiles of this chunk
                if (bar_any<kBarPro, kPro>(!mbar_wait(&bb.full_bc[s], (lc >> 1) & 1, abort_flag, err, kErrWaitTma)))
                    break;
                if (BCN) {  // one row scale per thread: B rows (tid < 128), then C rows
                    if (!SUM || tid < kRows)
                        rsc[tid] = bc_row_scale<KB>(tid < kRows ? bst : cst, (uint32_t)(tid % kRows), 1.f / N, a.eps);
                    named_bar(kBarPro, kPro);
                }
                float phi[4] = {0.f, 0.f, 0.f, 0.f};
                for (int q = 0; q < (th_head ? 0 : part); ++q) {
                    const float4 v = *reinterpret_cast<const float4 *>(phis + q * K2 + 4 * g);
                    phi[0] += v.x;
                    phi[1] += v.y;
                    phi[2] += v.z;
                    phi[3] += v.w;
                }
                const uint32_t kbo = (uint32_t)(g >> 3) * 16384u;
                const uint32_t jchunk = (uint32_t)(g & 7);
                // MIMO projections: the tiles hold one row per token (row i);
                // for R > 1 every thread first takes its tokens' rows into
                // registers, since the widened rows i R + r overwrite rows of
                // other threads' tokens
                constexpr bool kStage = PROJ && R > 1 && !kSep;
                // where the token rows are: the staging tiles (kSep) or the tiles' first rows
                const uint8_t *bsrc = kSep ? smem + C::OFF_STG + s * 2 * C::STG_BC : bst;
                const uint8_t *csrc = kSep ? bsrc + C::STG_BC : cst;
                const uint32_t kbs = kSep ? (uint32_t)(g >> 3) * C::STG_ROWS : kbo;
                uint4 pb[kStage ? TPT : 1], pc[kStage ? TPT : 1];
                if (kStage) {
#pragma unroll
                    for (int j = 0; j < TPT; ++j) {
                        const uint32_t off = kbo + sw128((uint32_t)(part * TPT + j), jchunk);
                        pb[j] = *reinterpret_cast<const uint4 *>(bst + off);
                        if (!SUM) pc[j] = *reinterpret_cast<const uint4 *>(cst + off);
                    }
                    named_bar(kBarPro, kPro);
                }
#pragma unroll
                for (int j0 = 0; j0 < TPT; j0 += TB) {
                    // all loads of the batch first (the stores below go to the same
                    // tiles, so the compiler could not hoist them itself)
                    uint4 vb[TB][R], vc[TB][R];
#pragma unroll
                    for (int jj = 0; jj < TB; ++jj) {
                        const int i = part * TPT + j0 + jj;
#pragma unroll
                        for (int r = 0; r < R; ++r) {
                            if (PROJ) {  // widen: this rank's weights times the token's row
                                const uint4 src = kStage ? pb[j0 + jj]
                                                         : *reinterpret_cast<const uint4 *>(
                                                               bsrc + kbs + sw128((uint32_t)i, jchunk));
                                const uint4 w = *reinterpret_cast<const uint4 *>(sbias + r * K2 + 4 * g);
                                vb[jj][r] = make_uint4(mul_bf16x2(src.x, w.x), mul_bf16x2(src.y, w.y),
                                                       mul_bf16x2(src.z, w.z), mul_bf16x2(src.w, w.w));
                                if (!SUM) {
                                    const uint4 srcc = kStage ? pc[j0 + jj]
                                                              : *reinterpret_cast<const uint4 *>(
                                                                    csrc + kbs + sw128((uint32_t)i, jchunk));
                                    const uint4 wc = *reinterpret_cast<const uint4 *>(sbias + (R + r) * K2 + 4 * g);
                                    vc[jj][r] = make_uint4(mul_bf16x2(srcc.x, wc.x), mul_bf16x2(srcc.y, wc.y),
                                                           mul_bf16x2(srcc.z, wc.z), mul_bf16x2(srcc.w, wc.w));
                                }
                                continue;
                            }
                            const uint32_t off = kbo + sw128((uint32_t)(i * R + r), jchunk);
                            vb[jj][r] = *reinterpret_cast<const uint4 *>(bst + off);
                            if (!SUM) vc[jj][r] = *reinterpret_cast<const uint4 *>(cst + off);
                        }
                    }
                    if (BCN) {
#pragma unroll
                        for (int jj = 0; jj < TB; ++jj)
#pragma unroll
                            for (int r = 0; r < R; ++r) {
                                const int row = (part * TPT + j0 + jj) * R + r;
                                vb[jj][r] = bc_norm_row(vb[jj][r], wB2,
                                                        *reinterpret_cast<const uint4 *>(sbias + r * K2 + 4 * g),
                                                        rsc[row]);
                                if (!SUM)
                                    vc[jj][r] = bc_norm_row(
                                        vc[jj][r], wC2, *reinterpret_cast<const uint4 *>(sbias + (R + r) * K2 + 4 * g),
                                        rsc[kRows + row]);
                            }
                    }
#pragma unroll
                    for (int jj = 0; jj < TB; ++jj) {
                        const int i = part * TPT + j0 + jj;
                        const float di = dts[i];
                        if (th_head) {  // di is the cumulative dt of token i
#pragma unroll
                            for (int e = 0; e < 4; ++e) phi[e] = di * thh[e];
                        } else {
                            const float2 t01 = unpack_bf16(thr[j0 + jj].x), t23 = unpack_bf16(thr[j0 + jj].y);
                            phi[0] = fmaf(di, t01.x, phi[0]);
                            phi[1] = fmaf(di, t01.y, phi[1]);
                            phi[2] = fmaf(di, t23.x, phi[2]);
                            phi[3] = fmaf(di, t23.y, phi[3]);
                        }
                        uint32_t cc[4], nss[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            float sn, cs;
                            __sincosf(phi[e], &sn, &cs);
                            cc[e] = pack_bf16(cs, cs);
                            nss[e] = pack_bf16(-sn, sn);
                        }
#pragma unroll
                        for (int r = 0; r < R; ++r) {
                            const uint32_t off = kbo + sw128((uint32_t)(i * R + r), jchunk);
                            uint4 b4 = vb[jj][r];
                            b4.x = rot_pair(b4.x, cc[0], nss[0]);
                            b4.y = rot_pair(b4.y, cc[1], nss[1]);
                            b4.z = rot_pair(b4.z, cc[2], nss[2]);
                            b4.w = rot_pair(b4.w, cc[3], nss[3]);
                            *reinterpret_cast<uint4 *>(bst + off) = b4;
                            if (!SUM) {
                                uint4 c4 = vc[jj][r];
                                c4.x = rot_pair(c4.x, cc[0], nss[0]);
                                c4.y = rot_pair(c4.y, cc[1], nss[1]);
                                c4.z = rot_pair(c4.z, cc[2], nss[2]);
                                c4.w = rot_pair(c4.w, cc[3], nss[3]);
                                *reinterpret_cast<uint4 *>(cst + off) = c4;
                            }
                        }
                    }
                }
                if (part == NPART - 1) {  // phi now holds each pair's total angle over the chunk
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float sn, cs;
                        __sincosf(phi[e], &sn, &cs);
                        cosE[4 * g + e] = cs;
                        sinE[4 * g + e] = sn;
                    }
                }
                if (lc + 1 < nloc) prefetch_theta((int64_t)(first_chunk() + lc + 1) * Q);
            }
            // ---- C. w o X (chunk-state weights on the value rows), once G(c-1)
            //      has finished reading the previous w o X and x of chunk c is in
            if (bar_any<kBarPro, kPro>((lc >= 1 && !mbar_wait(bb.sg, (lc - 1) & 1, abort_flag, err, kErrWaitMma)) ||
                                       !mbar_wait(&bb.full_x[sx], (lc / kNX) & 1, abort_flag, err, kErrWaitTma)))
                break;
            {
                const int row = tid >> 1, j0 = (tid & 1) * 4;  // half a row per thread
                const float wv = wst[row / R];
                const uint32_t ww = pack_bf16(wv, wv);
                uint4 v[4];
                if (PROJ) {  // one row per token (staging tile, or the x tile's first rows): widen into rows i R + r
                    const uint8_t *xsrc = kSep ? smem + C::OFF_STGX + sx * C::STG_ROWS : xst;
#pragma unroll
                    for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4 *>(xsrc + sw128(row / R, j0 + j));
                    if (R > 1 && !kSep) named_bar(kBarPro, kPro);  // every token's row read before any is overwritten
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(sxw + (row % R) * (kP / 2) + 4 * (j0 + j));
                        v[j] = make_uint4(mul_bf16x2(v[j].x, w.x), mul_bf16x2(v[j].y, w.y), mul_bf16x2(v[j].z, w.z),
                                          mul_bf16x2(v[j].w, w.w));
                        *reinterpret_cast<uint4 *>(xst + sw128(row, j0 + j)) = v[j];
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j) v[j] = *reinterpret_cast<const uint4 *>(xst + sw128(row, j0 + j));
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    v[j].x = mul_bf16x2(v[j].x, ww);
                    v[j].y = mul_bf16x2(v[j].y, ww);
                    v[j].z = mul_bf16x2(v[j].z, ww);
                    v[j].w = mul_bf16x2(v[j].w, ww);
                    *reinterpret_cast<uint4 *>(xw + sw128(row, j0 + j)) = v[j];
                }
            }
            fence_proxy_async_smem();
            named_bar(kBarPro, kPro);
            if (tid == 0) {
                mbar_arrive(bb.ops);
                mbar_arrive(&bb.sc[sx]);
            }
        }
    } else {
        // ============================================================ state warps (8-15)
        // Thread (wq, lane, hf): TMEM lane quarter wq, state row / output row of
        // that lane, and half hf of the 64 columns.
        const int lt = tid - kPro;         // 0..255
        const int hf = lt >> 7;            // column half
        const int lq = lt & 127;           // TMEM lane = row
        const int wq = warp & 3;           // TMEM lane quarter
        const bool own_state = (N == 128) || (lane < 16);
        const int srow = (N == 128) ? lq : (wq * 16 + lane);  // TMEM lane layout of G (M = N)
        uint8_t *hbuf = smem + C::OFF_HB;
        const float Dh = dchk::in(kSiteHead, h, 1, H) ? a.D[h] : 0.f;
        const uint32_t tl = tbase + ((uint32_t)(32 * wq) << 16);
        const int c0 = 32 * hf;            // first column of this thread's half
        float hreg[32];
        // a failed wait anywhere in the role (or the warp); the role's (or the
        // warp's) signal to the MMA issuer once all its threads are done
        auto role_any = [&](bool pred) { return kWarpSig ? warp_any(pred) : bar_any<kBarState, kSt>(pred); };
        auto role_done = [&]() {
            if (kWarpSig) {
                __syncwarp();
                return lane == 0;
            }
            named_bar(kBarState, kSt);
            return lt == 0;
        };
        // Pending-inclusive state entering the segment.  The whole sequence and
        // segment 0 of either pass: the caller's h0 + beta'_0 b_prev x_prev^T
        // (pending write of token -1); later summary segments: zero (their
        // local state); later segments of the main pass: the scan of the
        // published summaries of the segments before it (look-back).
        bool ok = true;
        {
#pragma unroll
            for (int p = 0; p < 32; ++p) hreg[p] = 0.f;
            if (MODE == kSegment && seg > 0) {
                // Every earlier segment's summary (bounded waits; the summary
                // CTAs are all resident or done), then S_1 = L_0 and S_{j+1} =
                // M_j S_j + L_j, with L_j in slot j + 1 and M_j acting on row pairs
                // exactly like the chunk-to-chunk update.
                if (bar_any<kBarState, kSt>(lt == 0 && [&] {
                        for (int j = 0; j < seg; ++j)
                            if (!dchk::in(kSiteFlags, (int64_t)j * BH + bh, 1, nSeg * BH) ||
                                !flag_wait(a.flags + (int64_t)j * BH + bh, abort_flag, err, kErrWaitSegment,
                                           kFlagBudget))
                                return true;
                        return false;
                    }())) {
                    ok = false;
                } else {
                    const int rr = own_state ? srow : 0;
                    const int64_t slot = (int64_t)BH * N * kP;
                    const int64_t ho = slot + bh * N * kP + rr * kP + c0;
                    const float *hs = a.ws_h + ho;
                    const bool in1 = dchk::in(kSiteWsH, ho, 32, nSeg * slot);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 v =
                            in1 ? __ldcg(reinterpret_cast<const float4 *>(hs) + q) : make_float4(0.f, 0.f, 0.f, 0.f);
                        hreg[4 * q] = v.x;
                        hreg[4 * q + 1] = v.y;
                        hreg[4 * q + 2] = v.z;
                        hreg[4 * q + 3] = v.w;
                    }
                    for (int j = 1; j < seg; ++j) {
                        const int64_t mo = ((int64_t)j * BH + bh) * N + (rr & ~1);
                        const float2 m = dchk::in(kSiteWsM, mo, 2, nSeg * BH * N)
                                             ? __ldcg(reinterpret_cast<const float2 *>(a.ws_m + mo))
                                             : make_float2(0.f, 0.f);
                        const float ms = (rr & 1) ? -m.y : m.y;
                        const bool inj = dchk::in(kSiteWsH, ho + (int64_t)j * slot, 32, nSeg * slot);
                        float4 l[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            l[q] = inj ? __ldcg(reinterpret_cast<const float4 *>(hs + (int64_t)j * slot) + q)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float lv[4] = {l[q].x, l[q].y, l[q].z, l[q].w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float u = hreg[4 * q + e];
                                const float o = __shfl_xor_sync(0xffffffffu, u, 1);
                                hreg[4 * q + e] = fmaf(m.x, u, fmaf(ms, o, lv[e]));
                            }
                        }
                    }
                }
            } else if (seg == 0) {
                const float betap0 = dchk::in(kSiteScalars, tok(0), 1, nTok)
                                         ? (1.f - bf(a.lam, tok(0))) * bf(a.dt, tok(0)) : 0.f;
                if (own_state) {
                    if (a.h0 && dchk::in(kSiteInit, (bh * N + srow) * kP + c0, 32, nSt)) {
#pragma unroll
                        for (int p = 0; p < 32; ++p) hreg[p] = a.h0[(bh * N + srow) * kP + c0 + p];
                    }
                    if (a.bp0 && a.xp0) {
                        for (int r = 0; r < R; ++r) {
                            if (!dchk::in(kSiteInit, (bh * R + r) * N + srow, 1, (int64_t)a.BH * R * N) ||
                                !dchk::in(kSiteInit, (bh * R + r) * kP + c0, 32, (int64_t)a.BH * R * kP))
                                continue;
                            const float cw = betap0 * a.bp0[(bh * R + r) * N + srow];
#pragma unroll
                            for (int p = 0; p < 32; ++p)
                                hreg[p] = fmaf(cw, a.xp0[(bh * R + r) * kP + c0 + p], hreg[p]);
                        }
                    }
                }
            }
            if (!SUM && own_state) store_state_half(hbuf, srow, hf, hreg);
        }
        // summary pass: the segment's transition exp(cA) Rot(-Phi) on this row's pair
        float m_l2 = 0.f, m_cs = 1.f, m_sn = 0.f;
        fence_proxy_async_smem();
        named_bar(kBarState, kSt);
        if (kWarpSig ? lane == 0 : lt == 0) mbar_arrive(bb.hrdy);
        if (lt == 0) {
            // the caller's initial state is read (the last segment may now overwrite it)
            if (MODE == kSegment && seg == 0 && dchk::in(kSiteFlags, (int64_t)(a.nseg - 1) * BH + bh, 1, nSeg * BH))
                flag_release(a.flags + (int64_t)(a.nseg - 1) * BH + bh, 1u);
        }
        for (int lc = 0; ok && lc < nloc; ++lc) {
            const int sx = lc % kNX;
            const float *cAl2 = sbuf + sx * C::SB;
            const float *gam = cAl2 + Q;
            const float *ghat = gam + Q;
            const float *colf = ghat + Q;
            const float *cosE = colf + Q;
            const float *sinE = cosE + K2;
            const uint8_t *xst = smem + C::OFF_X + sx * C::X_BYTES;
            // ---- D. decay mask S -> P (TMEM): half 0 takes column blocks 0 and 3,
            //      half 1 blocks 1 and 2 (balances the lower triangle).  The plain
            //      kernel takes it before the carried-state update, so that Yd runs
            //      under the update; for N = 64 it starts as soon as S is done (G
            //      and Yo finish meanwhile; for N = 128 that measured slower).  So
            //      does the per-head-theta instantiation (2 % faster that way); the
            //      per-token-A, general and BC-norm ones measured slower with the
            //      mask first (register allocation) and take it after the update.
            constexpr bool kMaskFirst = (FEAT == 0 || FEAT == 2) && !BCN && !SUM;
            constexpr bool kMaskOnS = kMaskFirst && N == 64;
            // scalars of chunk c (release/acquire through sc), its x tile, and
            // S(c) (mask on S alone) or S, G and Yo of chunk c
            if (role_any(!mbar_wait(&bb.sc[sx], (lc / kNX) & 1, abort_flag, err, kErrWaitCompute) ||
                         !mbar_wait(&bb.full_x[sx], (lc / kNX) & 1, abort_flag, err, kErrWaitTma) ||
                         !mbar_wait(kMaskOnS ? bb.sd : bb.sg, lc & 1, abort_flag, err, kErrWaitMma))) {
                ok = false;
                break;
            }
            tc_fence_after();
            auto decay_mask = [&]() {
                mask_to_tmem<R, Q>(hf == 0 ? 0 : 1, hf == 0 ? 3 : 2, wq, lq, tl, cAl2, gam, ghat, colf);
                tc_fence_before();
                if (role_done()) mbar_arrive(bb.p);
            };
            if (kMaskFirst) decay_mask();
            if (kMaskOnS) {  // G(c) and Yo(c), for the update below and the epilogue
                if (role_any(!mbar_wait(bb.sg, lc & 1, abort_flag, err, kErrWaitMma))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            // ---- E. carried state: h* <- Rot(-Phi)(exp(cA_end) h* + G), fp32 in registers
            {
                const float eA = ex2(cAl2[Q - 1]);
                const int kp = (own_state ? srow : 0) >> 1;
                const float cs = cosE[kp], sn = sinE[kp];
                const float sgn = (srow & 1) ? -sn : sn;
                float gv[32];
                tmem_ld32(tl + kColG + c0, gv);
                tmem_wait_ld();
#pragma unroll
                for (int p = 0; p < 32; ++p) {
                    const float u = fmaf(eA, hreg[p], gv[p]);
                    const float o = __shfl_xor_sync(0xffffffffu, u, 1);
                    hreg[p] = fmaf(u, cs, o * sgn);
                }
                if (SUM) {
                    m_l2 += cAl2[Q - 1];
                    const float ncs = m_cs * cs - m_sn * sn;
                    m_sn = fmaf(m_sn, cs, m_cs * sn);
                    m_cs = ncs;
                } else if (own_state) {
                    store_state_half(hbuf, srow, hf, hreg);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (role_done()) {
                mbar_arrive(bb.hrdy);
                if (SUM) mbar_arrive(&bb.empty_x[sx]);  // x tile and scalars consumed
            }
            if (SUM) continue;
            if (!kMaskFirst) decay_mask();

            // ---- F. epilogue: y = Yd + exp(cA_t) Yo + D x, this thread's 32 columns
            if (role_any(!mbar_wait(bb.yd, lc & 1, abort_flag, err, kErrWaitMma))) {
                ok = false;
                break;
            }
            tc_fence_after();
            {
                const int row = lq;
                const int ti = row / R, r = row % R;
                const int64_t t = (int64_t)(first_chunk() + lc) * Q + ti;
                const float sc = ex2(cAl2[ti]);
                const uint32_t yo = kColYo + (uint32_t)(lc & 1) * 64u;
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                    float yd[16], yv[16];
                    tmem_ld16(tl + kColYd + c0 + 16 * qq, yd);
                    tmem_ld16(tl + yo + c0 + 16 * qq, yv);
                    tmem_wait_ld();
                    if (PROJ) {  // y of the token = sum over its R rows (R neighbouring lanes) of wy_r times the row
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const uint4 xv =
                                *reinterpret_cast<const uint4 *>(xst + sw128(row, (c0 >> 3) + 2 * qq + q));
                            const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
                            const float4 w0 = *reinterpret_cast<const float4 *>(swy + r * kP + c0 + 16 * qq + 8 * q);
                            const float4 w1 =
                                *reinterpret_cast<const float4 *>(swy + r * kP + c0 + 16 * qq + 8 * q + 4);
                            const float w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 xf = unpack_bf16(xs[e]);
                                const int p = 8 * q + 2 * e;
                                yd[p] = w[2 * e] * fmaf(Dh, xf.x, fmaf(sc, yv[p], yd[p]));
                                yd[p + 1] = w[2 * e + 1] * fmaf(Dh, xf.y, fmaf(sc, yv[p + 1], yd[p + 1]));
                            }
                        }
                        // reduce-scatter over the R lanes of the token: at each
                        // halving step a lane keeps half of its columns and adds
                        // the partner's copy of them; lane r ends with the sums
                        // of 16 / R columns, at offset cofs
                        int cofs = 0;
#pragma unroll
                        for (int half = 8, bit = R / 2; bit >= 1; half >>= 1, bit >>= 1) {
                            const bool up = (r & bit) != 0;
#pragma unroll
                            for (int k = 0; k < half; ++k) {
                                const float mine = up ? yd[k + half] : yd[k];
                                const float other = __shfl_xor_sync(0xffffffffu, up ? yd[k] : yd[k + half], bit);
                                yd[k] = mine + other;
                            }
                            cofs += up ? half : 0;
                        }
                        constexpr int kOut = 16 / R;  // columns stored by each lane
                        if (t < T && dchk::in(kSiteY, tok(t) * kP + c0 + 16 * qq + cofs, kOut, nTok * kP)) {
                            __nv_bfloat16 *yp = a.y + tok(t) * kP + c0 + 16 * qq + cofs;
                            if (kOut == 16) {
#pragma unroll
                                for (int q = 0; q < 2; ++q)
                                    *reinterpret_cast<uint4 *>(yp + 8 * q) = make_uint4(
                                        pack_bf16(yd[8 * q], yd[8 * q + 1]), pack_bf16(yd[8 * q + 2], yd[8 * q + 3]),
                                        pack_bf16(yd[8 * q + 4], yd[8 * q + 5]), pack_bf16(yd[8 * q + 6], yd[8 * q + 7]));
                            } else if (kOut == 8) {
                                *reinterpret_cast<uint4 *>(yp) =
                                    make_uint4(pack_bf16(yd[0], yd[1]), pack_bf16(yd[2], yd[3]), pack_bf16(yd[4], yd[5]),
                                               pack_bf16(yd[6], yd[7]));
                            } else {
                                *reinterpret_cast<uint2 *>(yp) = make_uint2(pack_bf16(yd[0], yd[1]), pack_bf16(yd[2], yd[3]));
                            }
                        }
                        continue;
                    }
                    if (t < T && dchk::in(kSiteY, (tok(t) * R + r) * kP + c0 + 16 * qq, 16, nTok * R * kP)) {
                        __nv_bfloat16 *yrow = a.y + (tok(t) * R + r) * kP + c0 + 16 * qq;
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const uint4 xv =
                                *reinterpret_cast<const uint4 *>(xst + sw128(row, (c0 >> 3) + 2 * qq + q));
                            const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
                            uint32_t o[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const float2 xf = unpack_bf16(xs[e]);
                                const int p = 8 * q + 2 * e;
                                const float y0 = fmaf(Dh, xf.x, fmaf(sc, yv[p], yd[p]));
                                const float y1 = fmaf(Dh, xf.y, fmaf(sc, yv[p + 1], yd[p + 1]));
                                o[e] = pack_bf16(y0, y1);
                            }
                            *reinterpret_cast<uint4 *>(yrow + 8 * q) = make_uint4(o[0], o[1], o[2], o[3]);
                        }
                    }
                }
            }
            tc_fence_before();
            if (role_done()) mbar_arrive(&bb.empty_x[sx]);
        }
        // a warp that gave up left the loop on its own: agree before the barriers below
        if (kWarpSig) ok = !bar_any<kBarState, kSt>(!ok);
        if (SUM) {
            // ---- summary: the segment's local end state (pending-inclusive) into
            //      slot seg + 1, its transition exp(cA) Rot(-Phi) per pair
            const int64_t ho = (((int64_t)seg + 1) * BH + bh) * N * kP + srow * kP + c0;
            if (ok && own_state && dchk::in(kSiteWsH, ho, 32, nSeg * nSt)) {
                float4 *dst = reinterpret_cast<float4 *>(a.ws_h + ho);
#pragma unroll
                for (int p = 0; p < 8; ++p)
                    dst[p] = make_float4(hreg[4 * p], hreg[4 * p + 1], hreg[4 * p + 2], hreg[4 * p + 3]);
                if (hf == 0 && (srow & 1) == 0 &&
                    dchk::in(kSiteWsM, ((int64_t)seg * BH + bh) * N + srow, 2, nSeg * BH * N)) {
                    const float e = ex2(m_l2);
                    *reinterpret_cast<float2 *>(a.ws_m + ((int64_t)seg * BH + bh) * N + srow) =
                        make_float2(e * m_cs, e * m_sn);
                }
            }
            __threadfence();  // before the flag release below
        } else if (ok && (!SEGD || seg == a.nseg - 1) &&
                   !(MODE == kSegment &&
                     bar_any<kBarState, kSt>(lt == 0 &&
                                             (!dchk::in(kSiteFlags, (int64_t)(a.nseg - 1) * BH + bh, 1, nSeg * BH) ||
                                              !flag_wait(a.flags + (int64_t)(a.nseg - 1) * BH + bh, abort_flag, err,
                                                         kErrWaitSegment, kFlagBudget))))) {
            // ---- final state: plain-frame h_{T-1}, raw last token as the pending term
            //      (the last segment of a split sequence: once segment 0 has read
            //      the initial state, which this may overwrite)
            if (a.hT && own_state && dchk::in(kSiteFinal, (bh * N + srow) * kP + c0, 32, nSt)) {
                float4 *dst = reinterpret_cast<float4 *>(a.hT + (bh * N + srow) * kP + c0);
#pragma unroll
                for (int p = 0; p < 8; ++p)
                    dst[p] = make_float4(hreg[4 * p], hreg[4 * p + 1], hreg[4 * p + 2], hreg[4 * p + 3]);
            }
            if (a.bpT && BCN) {  // the last token's normalised B, one state warp per rank row
                const int wl = lt >> 5;
                if (wl < R && dchk::in(kSiteFinal, tok(T - 1) * R * N + wl * N, N, nTok * R * N) &&
                    dchk::in(kSiteFinal, (bh * R + wl) * N, N, (int64_t)a.BH * R * N) &&
                    dchk::in(kSiteNorm, (h * R + wl) * N, N, H * R * N)) {
                    const int64_t src = tok(T - 1) * R * N + wl * N;
                    float ss = 0.f;
                    for (int n = lane; n < N; n += 32) ss = fmaf(bf(a.B, src + n), bf(a.B, src + n), ss);
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                    const float sc = rsqrtf(ss / N + a.eps);
                    for (int n = lane; n < N; n += 32)
                        a.bpT[(bh * R + wl) * N + n] = fmaf(bf(a.B, src + n) * sc, a.wB[n], a.bB[(h * R + wl) * N + n]);
                }
            } else if (PROJ) {  // the last token's B and x, widened to rank R
                if (a.bpT && dchk::in(kSiteFinal, tok(T - 1) * N, N, nTok * N) &&
                    dchk::in(kSiteFinal, bh * R * N, R * N, (int64_t)a.BH * R * N) &&
                    dchk::in(kSiteProj, h * R * N, R * N, H * R * N))
                    for (int i = lt; i < R * N; i += kSt)
                        a.bpT[bh * R * N + i] = a.pwB[h * R * N + i] * bf(a.B, tok(T - 1) * N + i % N);
            } else if (a.bpT && dchk::in(kSiteFinal, tok(T - 1) * R * N, R * N, nTok * R * N) &&
                       dchk::in(kSiteFinal, bh * R * N, R * N, (int64_t)a.BH * R * N)) {
                for (int i = lt; i < R * N; i += kSt) a.bpT[bh * R * N + i] = bf(a.B, tok(T - 1) * R * N + i);
            }
            if (PROJ) {
                if (a.xpT && dchk::in(kSiteFinal, tok(T - 1) * kP, kP, nTok * kP) &&
                    dchk::in(kSiteFinal, bh * R * kP, R * kP, (int64_t)a.BH * R * kP) &&
                    dchk::in(kSiteProj, h * R * kP, R * kP, H * R * kP))
                    for (int i = lt; i < R * kP; i += kSt)
                        a.xpT[bh * R * kP + i] = a.pwx[h * R * kP + i] * bf(a.x, tok(T - 1) * kP + i % kP);
            } else if (a.xpT && dchk::in(kSiteFinal, tok(T - 1) * R * kP, R * kP, nTok * R * kP) &&
                       dchk::in(kSiteFinal, bh * R * kP, R * kP, (int64_t)a.BH * R * kP)) {
                for (int i = lt; i < R * kP; i += kSt) a.xpT[bh * R * kP + i] = bf(a.x, tok(T - 1) * R * kP + i);
            }
        }
    }
    __syncwarp();  // reconverge the single-lane roles before the block barrier
    tc_fence_before();
    __syncthreads();
    if (SUM && tid == 0 && dchk::in(kSiteFlags, (int64_t)seg * BH + bh, 1, nSeg * BH))
        flag_release(a.flags + (int64_t)seg * BH + bh, *abort_flag ? 2u : 1u);
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tbase, kTmemCols);
    }
    // the main pass completes only after the summary pass (so that later work
    // on the stream finds both done)
    if (MODE == kSegment && tid == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
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

// theta [Bt, T, H, N/2] bf16, box = {N/2, 1 head, Q tokens, 1 batch}, no swizzle.
bool make_theta_map(CUtensorMap *m, const void *base, int64_t K2, int64_t H, int64_t T, int64_t Bt, int Q) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)K2, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)Bt};
    const cuuint64_t strides[3] = {(cuuint64_t)(K2 * 2), (cuuint64_t)(H * K2 * 2), (cuuint64_t)(T * H * K2 * 2)};
    const cuuint32_t box[4] = {(cuuint32_t)K2, 1, (cuuint32_t)Q, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// `dependent`: launched as a programmatic dependent of the previous kernel on
// the stream (the main pass of a split sequence after its summary pass).
template <int N, int R, int MODE, int FEAT, bool BCN, bool PROJ>
cudaError_t launch_pass(const CUtensorMap &mx, const CUtensorMap &mb, const CUtensorMap &mc, const CUtensorMap &mt,
                        const TcArgs &a, int64_t ctas, cudaStream_t stream, bool dependent = false) {
    using C = Cfg<N, R, (PROJ && N == 64 && R > 1)>;
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel<N, R, MODE, FEAT, BCN, PROJ>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, prefill_tc_kernel<N, R, MODE, FEAT, BCN, PROJ>, mx, mb, mc, mt, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int N, int R, int FEAT, bool BCN, bool PROJ = false>
cudaError_t launch_nr(const Problem &p, const TcPlan &plan, const char **why) {
    using C = Cfg<N, R>;
    CUtensorMap mx, mb, mc, mt;
    // (theta fixed per head: a valid map over [H, N/2] that the kernel never loads from;
    // with the MIMO projections x, B, C have one row per token-head)
    constexpr int RIO = PROJ ? 1 : R;
    if (!make_map(&mx, p.x, kP, RIO, p.H, p.T, p.Bt, C::Q) || !make_map(&mb, p.B, N, RIO, p.H, p.T, p.Bt, C::Q) ||
        !make_map(&mc, p.C, N, RIO, p.H, p.T, p.Bt, C::Q) ||
        !make_theta_map(&mt, p.theta, N / 2, p.H, p.th_head ? 1 : p.T, p.th_head ? 1 : p.Bt, p.th_head ? 1 : C::Q)) {
        *why = "tensor-core prefill: TMA descriptor encoding failed";
        return cudaErrorNotSupported;
    }
    const int64_t BH = p.Bt * p.H;
    TcArgs a{};
    a.T = p.T;
    a.H = p.H;
    a.BH = BH;
    a.nchunks = plan.nchunks;
    a.cpseg = plan.cpseg;
    a.nseg = plan.nseg;
    a.x = (const __nv_bfloat16 *)p.x;
    a.B = (const __nv_bfloat16 *)p.B;
    a.dt = (const __nv_bfloat16 *)p.dt;
    a.lam = (const __nv_bfloat16 *)p.lam;
    a.theta = (const __nv_bfloat16 *)p.theta;
    a.A = p.A;
    a.A_tok = p.a_tok ? p.A : nullptr;
    a.th_head = p.th_head;
    a.wB = p.wB;
    a.wC = p.wC;
    a.bB = p.bB;
    a.bC = p.bC;
    a.eps = p.eps;
    a.pwx = p.pwx;
    a.pwB = p.pwB;
    a.pwC = p.pwC;
    a.pwy = p.pwy;
    a.D = p.D;
    a.h0 = p.h0;
    a.bp0 = p.bp0;
    a.xp0 = p.xp0;
    if (plan.nseg == 1) {
        a.y = (__nv_bfloat16 *)p.y;
        a.hT = p.hT;
        a.bpT = p.bpT;
        a.xpT = p.xpT;
        return launch_pass<N, R, kWhole, FEAT, BCN, PROJ>(mx, mb, mc, mt, a, BH, p.stream);
    }
    // split sequences: the summary pass over segments 0 .. nseg-2 publishes
    // each segment's local end state and transition; the main pass over all
    // segments, launched as its programmatic dependent, scans the published
    // summaries of the segments before its own (look-back)
    a.ws_h = static_cast<float *>(p.ws);
    a.ws_m = a.ws_h + (size_t)plan.nseg * BH * N * kP;
    a.flags = reinterpret_cast<unsigned *>(a.ws_m + (size_t)plan.nseg * BH * N);
    cudaError_t e = cudaMemsetAsync(a.flags, 0, (size_t)plan.nseg * BH * sizeof(unsigned), p.stream);
    if (e != cudaSuccess) return e;
    // (the failure-path self-test leaves the summary pass out: its flags are
    // never published and the look-back waits give up)
    if (!p.skip_summary) {
        e = launch_pass<N, R, kSummary, FEAT, BCN, PROJ>(mx, mb, mc, mt, a, BH * (plan.nseg - 1), p.stream);
        if (e != cudaSuccess) return e;
    }
    a.y = (__nv_bfloat16 *)p.y;
    a.hT = p.hT;
    a.bpT = p.bpT;
    a.xpT = p.xpT;
    return launch_pass<N, R, kSegment, FEAT, BCN, PROJ>(mx, mb, mc, mt, a, BH * plan.nseg, p.stream,
                                                       !p.skip_summary);
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

// workspace of a split call: the local end states, the transitions and the flags
static size_t split_ws_bytes(int64_t S, int64_t BH, int64_t N, int64_t P) {
    return (size_t)S * BH * (N * (P + 1) * sizeof(float) + sizeof(unsigned));
}

TcPlan prefill_tc_plan(const Problem &p) {
    TcPlan plan{};
    const int64_t Q = kRows / p.R;
    const int64_t nch = (p.T + Q - 1) / Q;
    const int64_t BH = p.Bt * p.H;
    int64_t S = 1;
    if (p.segments > 0) {
        S = p.segments;
    } else {
        // Split a sequence only when it shortens the estimated time: one CTA
        // per SM taken in launch order, the BH (S - 1) summary CTAs first, then
        // the BH S main-pass CTAs as SMs come free; segments of at least
        // kMinSegChunks chunks.
        int dev = 0, nsm = 148;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
        if (nsm < 1) nsm = 1;
        // finishing time of n1 CTAs of length t1 followed by n2 of length t2:
        // after the first kind the SMs form two groups (the last, partial wave
        // of summary CTAs and the rest) that stay in lock step
        auto makespan = [&](int64_t n1, double t1, int64_t n2, double t2) {
            const int64_t w1 = n1 / nsm, r1 = n1 % nsm;
            double ta = (double)w1 * t1, tb = (double)(w1 + 1) * t1, end = r1 ? tb : ta;
            int64_t ca = nsm - r1, cb = r1, rem = n2;
            while (rem > 0) {
                if (cb == 0 || (ca > 0 && ta <= tb)) {
                    rem -= ca < rem ? ca : rem;
                    ta += t2;
                    end = end > ta ? end : ta;
                } else {
                    rem -= cb < rem ? cb : rem;
                    tb += t2;
                    end = end > tb ? end : tb;
                }
            }
            return end;
        };
        double best = makespan(0, 0.0, BH, (double)nch + kCtaCost);
        for (int64_t s = 2; s <= kMaxSegments && s * kMinSegChunks <= nch; ++s) {
            const int64_t L = (nch + s - 1) / s, Se = (nch + L - 1) / L;
            if (Se != s) continue;
            if (p.ws_cap && split_ws_bytes(Se, BH, p.N, p.P) > p.ws_cap) break;
            const double cost = makespan(BH * (Se - 1), L * kSumCost + kCtaCost, BH * Se, (double)L + kCtaCost);
            if (cost < best * 0.97) {
                best = cost;
                S = s;
            }
        }
    }
    if (S > nch) S = nch;
    if (S < 1) S = 1;
    const int64_t L = (nch + S - 1) / S;
    S = (nch + L - 1) / L;  // no empty segment
    plan.nchunks = (int)nch;
    plan.cpseg = (int)L;
    plan.nseg = (int)S;
    plan.launches = S > 1 ? 2 : 1;
    plan.ctas = BH * S;
    plan.ws_bytes = S > 1 ? split_ws_bytes(S, BH, p.N, p.P) : 0;
    return plan;
}

size_t prefill_tc_workspace(const Problem &p) { return prefill_tc_plan(p).ws_bytes; }

template <int FEAT, bool BCN, bool PROJ>
cudaError_t dispatch_nr(const Problem &p, const TcPlan &plan, const char **why) {
    if (p.N == 128) {
        if (p.R == 1) return launch_nr<128, 1, FEAT, BCN, PROJ>(p, plan, why);
        if (p.R == 2) return launch_nr<128, 2, FEAT, BCN, PROJ>(p, plan, why);
        return launch_nr<128, 4, FEAT, BCN, PROJ>(p, plan, why);
    }
    if (p.R == 1) return launch_nr<64, 1, FEAT, BCN, PROJ>(p, plan, why);
    if (p.R == 2) return launch_nr<64, 2, FEAT, BCN, PROJ>(p, plan, why);
    return launch_nr<64, 4, FEAT, BCN, PROJ>(p, plan, why);
}

cudaError_t launch_prefill_tc(const Problem &p, const char **why) {
    const TcPlan plan = prefill_tc_plan(p);
    if (plan.nseg > 1 && (!p.ws || p.ws_bytes < plan.ws_bytes)) {
        *why = "tensor-core prefill: workspace too small for the split sequence";
        return cudaErrorNotSupported;
    }
    // the instantiation for (N, R) with feature mask FEAT (bit 0 A per token,
    // bit 1 theta per head), BC-norm and the MIMO projections
    const int feat = (p.a_tok ? 1 : 0) | (p.th_head ? 2 : 0);
    if (p.pwx) {  // MIMO projections (never with the BC-norm prologue); plain unless A_t or theta per head
        return feat ? dispatch_nr<3, false, true>(p, plan, why) : dispatch_nr<0, false, true>(p, plan, why);
    }
    if (p.wB) return dispatch_nr<3, true, false>(p, plan, why);
    switch (feat) {
        case 1: return dispatch_nr<1, false, false>(p, plan, why);
        case 2: return dispatch_nr<2, false, false>(p, plan, why);
        case 3: return dispatch_nr<3, false, false>(p, plan, why);
        default: return dispatch_nr<0, false, false>(p, plan, why);
    }
}

// Failure-path self-test: one thread waits, with a bounded wait, on an
// mbarrier phase that nothing ever completes; the wait gives up after
// `budget` cycles and records kErrWaitSelftest, exactly as a stuck wait in the
// prefill kernel would.  No trap, no fault: the context stays usable.
__global__ void __launch_bounds__(32) wait_selftest_kernel(long long budget) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        tc::fence_mbar_init();
        tc::mbar_wait(&bar, 0, nullptr, &g_device_error, tc::kErrWaitSelftest, budget);
    }
}

cudaError_t launch_wait_selftest(cudaStream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>(2000000LL);  // about 1 ms
    return cudaGetLastError();
}

size_t static_scratch_bytes() { return kStaticScratchBytes; }

cudaError_t static_scratch(void **ptr, size_t *bytes) {
    static std::mutex mu;
    static void *addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *ptr = addr[dev];
    *bytes = kStaticScratchBytes;
    return cudaSuccess;
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

M3_DCHECK_READER(read_dcheck_tc)

}  // namespace m3
