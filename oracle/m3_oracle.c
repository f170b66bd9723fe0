/*
 * m3_oracle.c -- plain, sequential fp64 CPU oracle for the Mamba-3 SSM
 * sequence-mixer forward.  TEST INFRASTRUCTURE ONLY: only the tests, the
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares no
 * code, header or table with the CUDA library.
 *
 * What it computes (per batch b, head h; tokens t = 0..T-1), in fp64:
 *
 *   Three-term exponential-trapezoidal recurrence, as displayed in
 *   "Знакомство с Mamba-3" (chernovdev.ru), section 1 "Экспоненциально-
 *   трапецеидальная дискретизация":
 *       h_t = e^{D_t A} h_{t-1} + (1-l_t) D_t e^{D_t A} B_{t-1} x_{t-1}^T
 *             + l_t D_t B_t x_t^T
 *   (D_t = step, l_t = trapezoid weight, A = per-head negative scalar).
 *
 *   Complex-valued state realised as 2x2 rotation blocks ("RoPE trick"):
 *   same page, section 2; "La dualità: Mamba-2 e Mamba-3"
 *   (book.paithon.it), section "Mamba-3", paragraph on complex transitions:
 *   a complex state of size N/2 equals a real state of size N whose
 *   transition is a block of 2x2 rotations scaled by the decay.  Pair k holds
 *   state rows (2k, 2k+1); its angle per token is w_t[k] = D_t * theta_t[k].
 *   Transition on pair k: decay * Rot(-w_t[k]), i.e. the complex eigenvalue
 *   exp(D_t (A - i theta_t[k])) acting on z = h[2k] + i h[2k+1].  This is the
 *   plain-frame form of rotating B and C by +phi_t = +sum_{s<=t} w_s.
 *
 *   MIMO rank R: "La dualità", section "Mamba-3", MIMO paragraph, and
 *   "Знакомство с Mamba-3" section 3: x_t is P x R, B_t and C_t are N x R,
 *   the write B_t x_t^T is a sum of R outer products, the state stays N x P,
 *   and the readout y_t = H_t^T C_t is P x R.  D * x_t is added (skip).
 *
 * Readings where the pages are silent (each one stated, not inferred):
 *   - the t-1 term of the first token uses (b_prev, x_prev) from the initial
 *     state when one is supplied, else zero;
 *   - the state returned at the end is h_{T-1} plus (b_prev, x_prev) =
 *     (B_{T-1}, x_{T-1}), which makes prefill -> decode resume exact;
 *   - pairs are interleaved (2k, 2k+1); theta_t has N/2 entries per token-head;
 *   - B and C are per head (no sharing across heads); D per head.
 *
 * A per head or per token.  The displayed recurrence carries A_t: in Mamba-3
 * the transition scalar is itself produced from the input at every token
 * ("La dualità: Mamba-2 e Mamba-3", section "Mamba-3", paragraph on the
 * exponential-trapezoidal rule), where Mamba-2 held it fixed per head.  Both
 * layouts are accepted: A [H] (fixed per head) or A [Bt, T, H] (one value per
 * token-head; [Bt, H] for a decode step); the token update is the same with
 * A read at the token.
 *
 * theta per token or per head.  The angle rates may also be fixed per head,
 * theta [H, N/2] (a time-constant rotation, as in the complex-diagonal SSMs
 * where the eigenvalue's phase is a learned constant): the token's angle is
 * then D_t * theta[h][k], everything else unchanged.
 *
 * BC-norm prologue (optional).  Mamba-3 normalises the B and C projections
 * with an RMS norm, as QKNorm does for queries and keys, and adds learnable
 * head-specific biases after the norm ("Знакомство с Mamba-3", section
 * "Архитектура и нормализация"; "Mamba-3, parte 1", paragraphs on the
 * normalisations and on dropping the short convolution).  Reading taken here:
 * every (token, head, rank) row of B (and of C) over its N entries becomes
 *   B^ = B / sqrt(mean_n B^2 + eps) * w_B + b_B[h, r],
 * w_B [N] shared by heads and ranks, b_B [H, R, N]; the recurrence then uses
 * B^ and C^ wherever it used B and C (rotation included), and b_prev holds
 * the last token's B^.
 *
 * Layouts (row-major, last index fastest), all fp64 here:
 *   x, y  [Bt, T, H, R, P]     B, C [Bt, T, H, R, N]
 *   dt, lam [Bt, T, H]         theta [Bt, T, H, N/2]      D [H]
 *   A [H] or [Bt, T, H]
 *   h [Bt, H, N, P]   b_prev [Bt, H, R, N]   x_prev [Bt, H, R, P]
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    int64_t Bt, T, H, P, N, R;
    const double *x, *B, *C, *dt, *lam, *theta, *A, *D;
    const double *h0, *bp0, *xp0; /* nullable: zero initial state */
    double *y, *hT, *bpT, *xpT;   /* y required; final-state outputs nullable */
    int a_per_token;              /* A is [Bt, T, H] instead of [H] */
    int theta_per_head;           /* theta is [H, N/2] instead of [Bt, T, H, N/2] */
    const double *wB, *wC, *bB, *bC; /* BC-norm (all or none) */
    double eps;
    int64_t next;                 /* next (b,h) slice to claim */
    pthread_mutex_t lock;
} job_t;

/* One token of the recurrence on one (b,h) slice, in place on (h, bp, xp).
 * Order of operations follows the displayed formula factored as
 *   h <- decay * Rot(-w) (h + (1-l) D B_{t-1} x_{t-1}^T) + l D B_t x_t^T,
 * which is the same expression with e^{D A} (a scalar) and the rotation
 * (orthogonal, acting on the state's row pairs) applied to both old terms. */
static void token_update(int64_t N, int64_t P, int64_t R,
                         double *h, double *bp, double *xp,
                         const double *xt, const double *Bt, const double *Ct,
                         double dt, double lam, const double *th,
                         double A, double D, double *yt)
{
    const double decay = exp(dt * A);
    const double gam = lam * dt;          /* weight of the current write   */
    const double betap = (1.0 - lam) * dt; /* weight of the previous write */

    /* pending write of the previous token */
    for (int64_t n = 0; n < N; ++n)
        for (int64_t p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int64_t r = 0; r < R; ++r) acc += bp[r * N + n] * xp[r * P + p];
            h[n * P + p] += betap * acc;
        }
    /* decay and rotate each state pair by -w */
    for (int64_t k = 0; k < N / 2; ++k) {
        const double w = dt * th[k];
        const double c = cos(w), s = sin(w);
        double *u = h + (2 * k) * P, *v = h + (2 * k + 1) * P;
        for (int64_t p = 0; p < P; ++p) {
            const double uu = u[p], vv = v[p];
            u[p] = decay * (uu * c + vv * s);
            v[p] = decay * (-uu * s + vv * c);
        }
    }
    /* current write */
    for (int64_t n = 0; n < N; ++n)
        for (int64_t p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int64_t r = 0; r < R; ++r) acc += Bt[r * N + n] * xt[r * P + p];
            h[n * P + p] += gam * acc;
        }
    /* readout y = h^T C + D x, one column per rank */
    for (int64_t r = 0; r < R; ++r)
        for (int64_t p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) acc += h[n * P + p] * Ct[r * N + n];
            yt[r * P + p] = acc + D * xt[r * P + p];
        }
    /* the current token becomes the pending one */
    memcpy(bp, Bt, sizeof(double) * (size_t)(R * N));
    memcpy(xp, xt, sizeof(double) * (size_t)(R * P));
}

/* The BC-norm of one token's R rows of N entries, out of place. */
static void bc_norm(int64_t N, int64_t R, const double *in, const double *w, const double *bias,
                    double eps, double *out)
{
    for (int64_t r = 0; r < R; ++r) {
        double ss = 0.0;
        for (int64_t n = 0; n < N; ++n) ss += in[r * N + n] * in[r * N + n];
        const double inv = 1.0 / sqrt(ss / (double)N + eps);
        for (int64_t n = 0; n < N; ++n) out[r * N + n] = in[r * N + n] * inv * w[n] + bias[r * N + n];
    }
}

static void run_slice(job_t *j, int64_t bh)
{
    const int64_t H = j->H, T = j->T, N = j->N, P = j->P, R = j->R;
    const int64_t b = bh / H, hd = bh % H;
    double *h = (double *)calloc((size_t)(N * P), sizeof(double));
    double *bp = (double *)calloc((size_t)(R * N), sizeof(double));
    double *xp = (double *)calloc((size_t)(R * P), sizeof(double));
    if (j->h0) memcpy(h, j->h0 + bh * N * P, sizeof(double) * (size_t)(N * P));
    if (j->bp0) memcpy(bp, j->bp0 + bh * R * N, sizeof(double) * (size_t)(R * N));
    if (j->xp0) memcpy(xp, j->xp0 + bh * R * P, sizeof(double) * (size_t)(R * P));
    double *Bn = (double *)malloc(sizeof(double) * (size_t)(R * N));
    double *Cn = (double *)malloc(sizeof(double) * (size_t)(R * N));
    for (int64_t t = 0; t < T; ++t) {
        const int64_t th_ = (b * T + t) * H + hd; /* token-head index */
        const double *Bt = j->B + th_ * R * N, *Ct = j->C + th_ * R * N;
        if (j->wB) {
            bc_norm(N, R, Bt, j->wB, j->bB + hd * R * N, j->eps, Bn);
            bc_norm(N, R, Ct, j->wC, j->bC + hd * R * N, j->eps, Cn);
            Bt = Bn;
            Ct = Cn;
        }
        token_update(N, P, R, h, bp, xp, j->x + th_ * R * P, Bt,
                     Ct, j->dt[th_], j->lam[th_],
                     j->theta + (j->theta_per_head ? hd : th_) * (N / 2), j->A[j->a_per_token ? th_ : hd], j->D[hd],
                     j->y + th_ * R * P);
    }
    if (j->hT) memcpy(j->hT + bh * N * P, h, sizeof(double) * (size_t)(N * P));
    if (j->bpT) memcpy(j->bpT + bh * R * N, bp, sizeof(double) * (size_t)(R * N));
    if (j->xpT) memcpy(j->xpT + bh * R * P, xp, sizeof(double) * (size_t)(R * P));
    free(Bn);
    free(Cn);
    free(h);
    free(bp);
    free(xp);
}

static void *worker(void *arg)
{
    job_t *j = (job_t *)arg;
    for (;;) {
        pthread_mutex_lock(&j->lock);
        const int64_t bh = j->next++;
        pthread_mutex_unlock(&j->lock);
        if (bh >= j->Bt * j->H) break;
        run_slice(j, bh);
    }
    return NULL;
}

int m3o_num_cores(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/* Full sequence scan.  Returns 0 on success, -1 on bad arguments.
 * nthreads <= 0 means one thread per online core; a_per_token != 0 means A is
 * [Bt, T, H] (else [H]); theta_per_head != 0 means theta is [H, N/2]. */
int m3o_scan(int64_t Bt, int64_t T, int64_t H, int64_t P, int64_t N, int64_t R,
             const double *x, const double *B, const double *C,
             const double *dt, const double *lam, const double *theta,
             const double *A, const double *D,
             const double *h0, const double *bp0, const double *xp0,
             double *y, double *hT, double *bpT, double *xpT, int nthreads, int a_per_token,
             int theta_per_head, const double *wB, const double *wC, const double *bB,
             const double *bC, double eps)
{
    if (Bt < 0 || T < 0 || H <= 0 || P <= 0 || N <= 0 || (N & 1) || R <= 0) return -1;
    if (!y && T > 0) return -1;
    job_t j;
    memset(&j, 0, sizeof j);
    j.Bt = Bt; j.T = T; j.H = H; j.P = P; j.N = N; j.R = R;
    j.x = x; j.B = B; j.C = C; j.dt = dt; j.lam = lam; j.theta = theta;
    j.A = A; j.D = D; j.h0 = h0; j.bp0 = bp0; j.xp0 = xp0;
    j.y = y; j.hT = hT; j.bpT = bpT; j.xpT = xpT;
    j.a_per_token = a_per_token;
    j.theta_per_head = theta_per_head;
    if ((wB != NULL) != (wC != NULL) || (wB != NULL) != (bB != NULL) || (wB != NULL) != (bC != NULL)) return -1;
    j.wB = wB; j.wC = wC; j.bB = bB; j.bC = bC; j.eps = eps;
    pthread_mutex_init(&j.lock, NULL);
    int nt = nthreads > 0 ? nthreads : m3o_num_cores();
    if (nt > Bt * H) nt = (int)(Bt * H);
    if (nt <= 1) {
        worker(&j);
    } else {
        pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
        for (int i = 0; i < nt; ++i) pthread_create(&tid[i], NULL, worker, &j);
        for (int i = 0; i < nt; ++i) pthread_join(tid[i], NULL);
        free(tid);
    }
    pthread_mutex_destroy(&j.lock);
    return 0;
}

/* One decode step for every (b,h) slice, in place on (h, b_prev, x_prev).
 * Inputs are one token per slice: x [Bt,H,R,P], B/C [Bt,H,R,N], dt/lam [Bt,H],
 * theta [Bt,H,N/2] or (theta_per_head) [H,N/2], A [H] or (a_per_token)
 * [Bt,H]; y [Bt,H,R,P].  It is the
 * same token update as the scan. */
int m3o_step(int64_t Bt, int64_t H, int64_t P, int64_t N, int64_t R,
             const double *x, const double *B, const double *C,
             const double *dt, const double *lam, const double *theta,
             const double *A, const double *D,
             double *h, double *bp, double *xp, double *y, int a_per_token, int theta_per_head,
             const double *wB, const double *wC, const double *bB, const double *bC, double eps)
{
    if ((wB != NULL) != (wC != NULL) || (wB != NULL) != (bB != NULL) || (wB != NULL) != (bC != NULL)) return -1;
    if (Bt < 0 || H <= 0 || P <= 0 || N <= 0 || (N & 1) || R <= 0) return -1;
    double *Bn = (double *)malloc(sizeof(double) * (size_t)(R * N));
    double *Cn = (double *)malloc(sizeof(double) * (size_t)(R * N));
    for (int64_t bh = 0; bh < Bt * H; ++bh) {
        const int64_t hd = bh % H;
        const double *Bt_ = B + bh * R * N, *Ct_ = C + bh * R * N;
        if (wB) {
            bc_norm(N, R, Bt_, wB, bB + hd * R * N, eps, Bn);
            bc_norm(N, R, Ct_, wC, bC + hd * R * N, eps, Cn);
            Bt_ = Bn;
            Ct_ = Cn;
        }
        token_update(N, P, R, h + bh * N * P, bp + bh * R * N, xp + bh * R * P,
                     x + bh * R * P, Bt_, Ct_, dt[bh], lam[bh],
                     theta + (theta_per_head ? hd : bh) * (N / 2), A[a_per_token ? bh : hd], D[hd],
                     y + bh * R * P);
    }
    free(Bn);
    free(Cn);
    return 0;
}
