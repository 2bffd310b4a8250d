/*
 * mru_oracle.c -- plain, slow, fp64 CPU oracle for the Matrix Recurrent Unit
 * (MRU) prefix-product scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load this library.  It shares no code, header,
 * table or helper with the CUDA library; it reads the same input bytes and
 * nothing else.
 *
 * What it computes (sources are the web pages the method is described on):
 *
 *   "MRU Update: An independent developer's alternative to Attention is now
 *    running successfully", section "What MRU Actually Does":
 *     1. each token's embedding is reshaped into an input state matrix X_t;
 *     2. the matrices are multiplied together along the sequence, the state
 *        being multiplied by the new input matrix at every step, i.e.
 *        S_t = S_{t-1} . X_t with S_0 = I (right multiplication);
 *     3. the state matrix is mapped back to a vector.
 *   "Improving Matrix Recurrent Units as an Attention Alternative", section
 *   "Key Points" and "Technical Deep Dive": two construction variants,
 *     - determinant correction: a scalar keeps det(X) at unit magnitude;
 *       read here as X = Xr / |det Xr|^(1/n) (sign of det kept);
 *     - LDU factor filling: X = L . D . U with L unit lower, U unit upper,
 *       D diagonal; read here as L = I + a*strict_lower(M),
 *       U = I + a*strict_upper(M), D = diag(exp(d*tanh(M_ii)));
 *     - orthogonal constructions, the Cayley map and the matrix exponential
 *       of a skew-symmetric matrix; read here with A = alpha (M - M^T) / 2
 *       (the skew-symmetric part of alpha M) as X = (I - A)^-1 (I + A) and
 *       X = exp(A).
 *
 * The oracle is the plain definition written out: every X_t is built in fp64
 * from the widened input, and S_t is the serial left-to-right product with a
 * textbook triple loop.  No blocking, no reordering, no library BLAS.  The
 * determinant uses textbook LU with partial pivoting.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t B, H, L;
    int32_t n;
    int32_t x_dtype;      /* 0: float32, 1: bfloat16 (raw 16-bit patterns) */
    int32_t mode;         /* 0: reshape, 1: determinant-corrected, 2: LDU fill,
                             3: Cayley map, 4: matrix exponential */
    float alpha;          /* Xr = add_identity*I + alpha*M (modes 0 and 1);
                             A = alpha (M - M^T) / 2 (modes 3 and 4) */
    int32_t add_identity;
    float ldu_offdiag;    /* a in L = I + a*strict_lower(M), U = I + a*strict_upper(M) */
    float ldu_diag;       /* d in D = diag(exp(d*tanh(M_ii))) */
} mro_problem;

enum { MRO_OK = 0, MRO_ERR_ARG = 1, MRO_ERR_SINGULAR = 5 };

/* ---- input widening -------------------------------------------------- */

/* bfloat16 is the top half of an IEEE binary32 pattern: widening is exact. */
double mro_bf16_to_double(uint16_t bits)
{
    uint32_t w = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

static double widen(const mro_problem* p, const void* x, int64_t idx)
{
    if (p->x_dtype == 1)
        return mro_bf16_to_double(((const uint16_t*)x)[idx]);
    return (double)((const float*)x)[idx];
}

/* ---- textbook dense helpers (row-major n x n) ------------------------ */

static void matmul(int n, const double* A, const double* Bm, double* C)
{
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) {
            double s = 0.0;
            for (int k = 0; k < n; ++k)
                s += A[i * n + k] * Bm[k * n + j];
            C[i * n + j] = s;
        }
}

static void set_identity(int n, double* A)
{
    for (int i = 0; i < n * n; ++i) A[i] = 0.0;
    for (int i = 0; i < n; ++i) A[i * n + i] = 1.0;
}

/* log|det A| and sign(det A) by LU with partial pivoting (A is destroyed).
 * Returns 0 when det A == 0 (an exact zero pivot). */
static int log_abs_det(int n, double* A, double* logabs, int* sign)
{
    double acc = 0.0;
    int sg = 1;
    for (int k = 0; k < n; ++k) {
        int piv = k;
        double best = fabs(A[k * n + k]);
        for (int i = k + 1; i < n; ++i)
            if (fabs(A[i * n + k]) > best) { best = fabs(A[i * n + k]); piv = i; }
        if (best == 0.0) return 0;
        if (piv != k) {
            for (int j = 0; j < n; ++j) {
                double t = A[k * n + j]; A[k * n + j] = A[piv * n + j]; A[piv * n + j] = t;
            }
            sg = -sg;
        }
        double pk = A[k * n + k];
        if (pk < 0) sg = -sg;
        acc += log(fabs(pk));
        for (int i = k + 1; i < n; ++i) {
            double l = A[i * n + k] / pk;
            for (int j = k + 1; j < n; ++j)
                A[i * n + j] -= l * A[k * n + j];
        }
    }
    *logabs = acc;
    *sign = sg;
    return 1;
}

static void transpose(int n, const double* A, double* T)
{
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) T[j * n + i] = A[i * n + j];
}

/* A^-1 into Ai by Gauss-Jordan elimination with partial pivoting on [A | I]
 * (A is destroyed).  Returns 0 when A is singular. */
static int invert(int n, double* A, double* Ai)
{
    set_identity(n, Ai);
    for (int k = 0; k < n; ++k) {
        int piv = k;
        double best = fabs(A[k * n + k]);
        for (int i = k + 1; i < n; ++i)
            if (fabs(A[i * n + k]) > best) { best = fabs(A[i * n + k]); piv = i; }
        if (best == 0.0) return 0;
        if (piv != k)
            for (int j = 0; j < n; ++j) {
                double t = A[k * n + j]; A[k * n + j] = A[piv * n + j]; A[piv * n + j] = t;
                t = Ai[k * n + j]; Ai[k * n + j] = Ai[piv * n + j]; Ai[piv * n + j] = t;
            }
        const double pk = A[k * n + k];
        for (int j = 0; j < n; ++j) { A[k * n + j] /= pk; Ai[k * n + j] /= pk; }
        for (int i = 0; i < n; ++i) {
            if (i == k) continue;
            const double f = A[i * n + k];
            if (f == 0.0) continue;
            for (int j = 0; j < n; ++j) { A[i * n + j] -= f * A[k * n + j]; Ai[i * n + j] -= f * Ai[k * n + j]; }
        }
    }
    return 1;
}

/* X = exp(A) by scaling and squaring (Moler and Van Loan, "Nineteen dubious
 * ways to compute the exponential of a matrix", 1978): with B = A / 2^s and
 * ||B||_1 <= 1/2, exp(B) is its power series summed until the terms vanish
 * in fp64, and exp(A) = exp(B)^(2^s).  A is overwritten by B; term and tmp
 * are n x n scratch.  Returns 0 for a non-finite A. */
static int expm_inplace(int n, double* A, double* X, double* term, double* tmp)
{
    const int64_t nn = (int64_t)n * n;
    double norm = 0.0;
    for (int j = 0; j < n; ++j) {
        double c = 0.0;
        for (int i = 0; i < n; ++i) c += fabs(A[i * n + j]);
        if (c > norm) norm = c;
    }
    if (!isfinite(norm)) return 0;
    int sq = 0;
    double scale = 1.0;
    while (norm * scale > 0.5) { scale *= 0.5; ++sq; }
    for (int64_t e = 0; e < nn; ++e) A[e] *= scale;
    set_identity(n, X);
    set_identity(n, term);
    for (int k = 1; k <= 60; ++k) {
        matmul(n, term, A, tmp);                       /* term <- term B / k */
        double big = 0.0, xbig = 0.0;
        for (int64_t e = 0; e < nn; ++e) {
            term[e] = tmp[e] / k;
            X[e] += term[e];
            if (fabs(term[e]) > big) big = fabs(term[e]);
            if (fabs(X[e]) > xbig) xbig = fabs(X[e]);
        }
        if (big <= 1e-18 * xbig) break;
    }
    for (int r = 0; r < sq; ++r) {
        matmul(n, X, X, tmp);
        memcpy(X, tmp, sizeof(double) * (size_t)nn);
    }
    return 1;
}

/* ---- step 1: lift one token-head embedding slice to X_t ----------------
 * The slice of head h is x[b, t, h*n*n : (h+1)*n*n], viewed row-major as
 * n x n: M[i][j] = x[... + i*n + j].  work must hold 3*n*n doubles. */
int mro_lift(const mro_problem* p, const void* x, int64_t b, int64_t t, int64_t h,
             double* X, double* work)
{
    const int n = p->n;
    const int64_t nn = (int64_t)n * n;
    const int64_t base = ((b * p->L + t) * p->H + h) * nn;
    double* M = work;
    for (int64_t e = 0; e < nn; ++e) M[e] = widen(p, x, base + e);

    if (p->mode == 0 || p->mode == 1) {
        const double a = (double)p->alpha;
        for (int64_t e = 0; e < nn; ++e) X[e] = a * M[e];
        if (p->add_identity)
            for (int i = 0; i < n; ++i) X[i * n + i] += 1.0;
        if (p->mode == 1) {
            double* A = work + nn;
            memcpy(A, X, (size_t)nn * sizeof(double));
            double la; int sg;
            if (!log_abs_det(n, A, &la, &sg) || !isfinite(la)) return MRO_ERR_SINGULAR;
            const double c = exp(-la / n);   /* |det X|^(-1/n) */
            for (int64_t e = 0; e < nn; ++e) X[e] *= c;
        }
        return MRO_OK;
    }
    if (p->mode == 2) {
        const double a = (double)p->ldu_offdiag, d = (double)p->ldu_diag;
        double* Lm = work + nn;
        double* DU = work + 2 * nn;
        set_identity(n, Lm);
        set_identity(n, DU);
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) {
                if (i > j) Lm[i * n + j] = a * M[i * n + j];
                if (i < j) DU[i * n + j] = a * M[i * n + j];
            }
        /* DU = D . U (row i of U scaled by D_i), then X = L . DU */
        for (int i = 0; i < n; ++i) {
            const double Di = exp(d * tanh(M[i * n + i]));
            for (int j = 0; j < n; ++j) DU[i * n + j] *= Di;
        }
        matmul(n, Lm, DU, X);
        return MRO_OK;
    }
    if (p->mode == 3 || p->mode == 4) {
        const double a = (double)p->alpha;
        double* A = work + nn;                     /* skew-symmetric part of alpha M */
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) A[i * n + j] = 0.5 * a * (M[i * n + j] - M[j * n + i]);
        if (p->mode == 3) {
            /* Cayley map: X = (I - A)^-1 (I + A).  I - A is never singular
             * for a real skew-symmetric A (its eigenvalues are 1 - i lambda). */
            double* W = work;                      /* M is no longer needed */
            double* Wi = work + 2 * nn;
            for (int64_t e = 0; e < nn; ++e) W[e] = -A[e];
            for (int i = 0; i < n; ++i) W[i * n + i] += 1.0;
            if (!invert(n, W, Wi)) return MRO_ERR_SINGULAR;
            for (int64_t e = 0; e < nn; ++e) W[e] = A[e];
            for (int i = 0; i < n; ++i) W[i * n + i] += 1.0;
            matmul(n, Wi, W, X);
            return MRO_OK;
        }
        /* matrix exponential */
        if (!expm_inplace(n, A, X, work + 2 * nn, work)) return MRO_ERR_ARG;   /* M is no longer needed */
        return MRO_OK;
    }
    return MRO_ERR_ARG;
}

/* ---- step 2: the serial left-to-right product ------------------------- */

typedef struct {
    const mro_problem* p;
    const void* x;
    const double* S0;        /* [B,H,n,n] or NULL (identity) */
    double* S_all;           /* [B,L,H,n,n] or NULL */
    /* comparison targets (all optional) */
    const float* S_gpu;      /* [B,L,H,n,n] */
    const double* u;         /* readout query columns U: [n,q], or [H,n,q] per head */
    int q;                   /* columns of U */
    int u_per_head;
    const float* o_gpu;      /* [B,L,H,n,q] */
    double* o_all;           /* [B,L,H,n,q] oracle readout, optional */
    int64_t snap_every;      /* 0: none */
    const float* snap_gpu;   /* [B,L/snap_every,H,n,n] */
    double* snap_all;        /* oracle snapshots, optional */
    double* dS;              /* [B,L,H] squared Frobenius norm of the difference */
    double* rS;              /* [B,L,H] squared Frobenius norm of the oracle S_t */
    double* dO;              /* [B,L,H] */
    double* rO;
    double* dP;              /* [B,L/snap_every,H] */
    double* rP;
    int64_t t_end;           /* process t in [0, t_end) */
    const int64_t* bh;       /* list of (b*H + h) */
    int64_t n_bh;
    int64_t next;            /* work counter (under lock) */
    pthread_mutex_t lock;
    int status;
} job_t;

static void run_sequence(job_t* J, int64_t bh_idx)
{
    const mro_problem* p = J->p;
    const int n = p->n;
    const int64_t nn = (int64_t)n * n;
    const int64_t b = bh_idx / p->H, h = bh_idx % p->H;
    double* S = malloc(sizeof(double) * nn);
    double* Sn = malloc(sizeof(double) * nn);
    double* X = malloc(sizeof(double) * nn);
    double* work = malloc(sizeof(double) * 3 * nn);
    if (!S || !Sn || !X || !work) { J->status = MRO_ERR_ARG; goto done; }

    if (J->S0) memcpy(S, J->S0 + (b * p->H + h) * nn, sizeof(double) * nn);
    else set_identity(n, S);

    for (int64_t t = 0; t < J->t_end; ++t) {
        int rc = mro_lift(p, J->x, b, t, h, X, work);
        if (rc != MRO_OK) { J->status = rc; goto done; }
        matmul(n, S, X, Sn);                       /* S_t = S_{t-1} . X_t */
        double* sw = S; S = Sn; Sn = sw;

        const int64_t row = (b * p->L + t) * p->H + h;   /* index of (b,t,h) */
        if (J->S_all) memcpy(J->S_all + row * nn, S, sizeof(double) * nn);
        if (J->S_gpu) {
            double d2 = 0.0, r2 = 0.0;
            const float* g = J->S_gpu + row * nn;
            for (int64_t e = 0; e < nn; ++e) {
                double df = (double)g[e] - S[e];
                d2 += df * df;
                r2 += S[e] * S[e];
            }
            J->dS[row] = d2;
            J->rS[row] = r2;
        }
        if (J->u && (J->o_gpu || J->o_all)) {
            const int q = J->q;
            const double* U = J->u + (J->u_per_head ? h * n * q : 0);
            const int64_t base = row * n * q;
            double d2 = 0.0, r2 = 0.0;
            for (int i = 0; i < n; ++i)
                for (int c = 0; c < q; ++c) {
                    double o = 0.0;                /* o_t = S_t . U */
                    for (int j = 0; j < n; ++j) o += S[i * n + j] * U[j * q + c];
                    if (J->o_all) J->o_all[base + i * q + c] = o;
                    if (J->o_gpu) {
                        double df = (double)J->o_gpu[base + i * q + c] - o;
                        d2 += df * df;
                        r2 += o * o;
                    }
                }
            if (J->o_gpu) { J->dO[row] = d2; J->rO[row] = r2; }
        }
        if (J->snap_every > 0 && ((t + 1) % J->snap_every) == 0) {
            const int64_t k = (t + 1) / J->snap_every - 1;     /* 1-based t = (k+1)*every */
            const int64_t L_s = p->L / J->snap_every;
            const int64_t srow = (b * L_s + k) * p->H + h;
            if (J->snap_all) memcpy(J->snap_all + srow * nn, S, sizeof(double) * nn);
            if (J->snap_gpu) {
                double d2 = 0.0, r2 = 0.0;
                const float* g = J->snap_gpu + srow * nn;
                for (int64_t e = 0; e < nn; ++e) {
                    double df = (double)g[e] - S[e];
                    d2 += df * df;
                    r2 += S[e] * S[e];
                }
                J->dP[srow] = d2;
                J->rP[srow] = r2;
            }
        }
    }
done:
    free(S); free(Sn); free(X); free(work);
}

static void* worker(void* arg)
{
    job_t* J = (job_t*)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t i = J->next++;
        int st = J->status;
        pthread_mutex_unlock(&J->lock);
        if (i >= J->n_bh || st != MRO_OK) break;
        run_sequence(J, J->bh[i]);
    }
    return NULL;
}

static int run_job(job_t* J, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > J->n_bh) nthreads = (int)(J->n_bh > 0 ? J->n_bh : 1);
    pthread_mutex_init(&J->lock, NULL);
    J->next = 0;
    J->status = MRO_OK;
    pthread_t* th = malloc(sizeof(pthread_t) * nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->lock);
    return J->status;
}

static int check_problem(const mro_problem* p)
{
    if (!p || p->B < 0 || p->H < 0 || p->L < 0 || p->n < 1) return MRO_ERR_ARG;
    if (p->x_dtype != 0 && p->x_dtype != 1) return MRO_ERR_ARG;
    if (p->mode < 0 || p->mode > 4) return MRO_ERR_ARG;
    return MRO_OK;
}

/* All states S_t (fp64) for every (b, t, h): S_all is [B, L, H, n, n]. */
int mro_scan(const mro_problem* p, const void* x, const double* S0, double* S_all,
             int nthreads)
{
    if (check_problem(p) != MRO_OK) return MRO_ERR_ARG;
    const int64_t nbh = p->B * p->H;
    int64_t* bh = malloc(sizeof(int64_t) * (nbh > 0 ? nbh : 1));
    for (int64_t i = 0; i < nbh; ++i) bh[i] = i;
    job_t J;
    memset(&J, 0, sizeof J);
    J.p = p; J.x = x; J.S0 = S0; J.S_all = S_all;
    J.t_end = p->L; J.bh = bh; J.n_bh = nbh;
    int rc = run_job(&J, nthreads);
    free(bh);
    return rc;
}

/* Readout o_t = S_t . U for every (b,t,h) ([B,L,H,n,q]; U is [n,q], or
 * [H,n,q] when u_per_head) and snapshots S_t at 1-based t = every, 2*every,
 * ... ([B, L/every, H, n, n]); either output may be NULL. */
int mro_readout(const mro_problem* p, const void* x, const double* S0, const double* u,
                int q, int u_per_head, double* o_all, int64_t snap_every, double* snap_all,
                int nthreads)
{
    if (check_problem(p) != MRO_OK || !u || q < 1) return MRO_ERR_ARG;
    const int64_t nbh = p->B * p->H;
    int64_t* bh = malloc(sizeof(int64_t) * (nbh > 0 ? nbh : 1));
    for (int64_t i = 0; i < nbh; ++i) bh[i] = i;
    job_t J;
    memset(&J, 0, sizeof J);
    J.p = p; J.x = x; J.S0 = S0; J.u = u; J.q = q; J.u_per_head = u_per_head; J.o_all = o_all;
    J.snap_every = snap_every; J.snap_all = snap_all;
    J.t_end = p->L; J.bh = bh; J.n_bh = nbh;
    int rc = run_job(&J, nthreads);
    free(bh);
    return rc;
}

/* Streaming comparison for sizes too large to hold in fp64: for each listed
 * sequence (b*H + h), recompute S_t for t < t_end and accumulate, per
 * (b,t,h), the squared Frobenius norm of (gpu - oracle) and of the oracle.
 * Any of the gpu arrays may be NULL; with all of them NULL the call only
 * runs the product (used to time the oracle). */
int mro_compare(const mro_problem* p, const void* x, const double* S0,
                const int64_t* bh, int64_t n_bh, int64_t t_end,
                const float* S_gpu, double* dS, double* rS,
                const double* u, int q, int u_per_head, const float* o_gpu, double* dO, double* rO,
                int64_t snap_every, const float* snap_gpu, double* dP, double* rP,
                int nthreads)
{
    if (check_problem(p) != MRO_OK) return MRO_ERR_ARG;
    if (t_end < 0 || t_end > p->L) return MRO_ERR_ARG;
    if (S_gpu && (!dS || !rS)) return MRO_ERR_ARG;
    if (o_gpu && (!u || q < 1 || !dO || !rO)) return MRO_ERR_ARG;
    if (snap_gpu && (snap_every <= 0 || !dP || !rP)) return MRO_ERR_ARG;
    for (int64_t i = 0; i < n_bh; ++i)
        if (bh[i] < 0 || bh[i] >= p->B * p->H) return MRO_ERR_ARG;
    job_t J;
    memset(&J, 0, sizeof J);
    J.p = p; J.x = x; J.S0 = S0;
    J.S_gpu = S_gpu; J.dS = dS; J.rS = rS;
    J.u = u; J.q = q; J.u_per_head = u_per_head; J.o_gpu = o_gpu; J.dO = dO; J.rO = rO;
    J.snap_every = snap_gpu ? snap_every : 0; J.snap_gpu = snap_gpu; J.dP = dP; J.rP = rP;
    J.t_end = t_end; J.bh = bh; J.n_bh = n_bh;
    return run_job(&J, nthreads);
}

/* ---- backward: the vector-Jacobian product of the scan ------------------
 *
 * Not described on the pages (they train the MRU but print no gradient); this
 * is the chain rule of the forward definition above, written out plainly.
 * With G_t = dL/dS_t (all later states included) and upstream gradients dS_t:
 *     G_L = dS_L,   G_{t-1} = dS_{t-1} + G_t X_t^T,
 *     dL/dX_t = S_{t-1}^T G_t (S_0 = S0 or I),   dL/dS0 = G_1 X_1^T.
 * Through the construction of X_t from the embedding slice M:
 *   reshape:   X = add_identity I + alpha M          dM = alpha dX
 *   det-corr.: X = c Xr, c = |det Xr|^(-1/n)         dXr = c (dX - <dX, Xr> Xr^-T / n)
 *              (d log|det Xr| = tr(Xr^-1 dXr)),      dM = alpha dXr
 *   LDU:       X = L D U                             dL = dX (D U)^T, d(DU) = L^T dX,
 *              dU = D d(DU), dD_i = sum_j d(DU)_ij U_ij;
 *              dM_ij = a dL_ij (i > j), a dU_ij (i < j),
 *              dM_ii = dD_i D_i d (1 - tanh^2 M_ii).
 * The inverse is textbook Gauss-Jordan with partial pivoting. */

/* dM from dX for one token-head (the construction's chain rule above).
 * work holds 7 n*n doubles. */
static int lift_vjp(const mro_problem* p, const void* x, int64_t b, int64_t t, int64_t h,
                    const double* dX, double* dM, double* work)
{
    const int n = p->n;
    const int64_t nn = (int64_t)n * n;
    const int64_t base = ((b * p->L + t) * p->H + h) * nn;
    double* M = work;
    for (int64_t e = 0; e < nn; ++e) M[e] = widen(p, x, base + e);
    if (p->mode == 0) {
        for (int64_t e = 0; e < nn; ++e) dM[e] = (double)p->alpha * dX[e];
        return MRO_OK;
    }
    if (p->mode == 1) {
        const double a = (double)p->alpha;
        double* Xr = work + nn;
        double* A = work + 2 * nn;
        double* Ai = work + 3 * nn;
        for (int64_t e = 0; e < nn; ++e) Xr[e] = a * M[e];
        if (p->add_identity)
            for (int i = 0; i < n; ++i) Xr[i * n + i] += 1.0;
        memcpy(A, Xr, (size_t)nn * sizeof(double));
        double la; int sg;
        if (!log_abs_det(n, A, &la, &sg) || !isfinite(la)) return MRO_ERR_SINGULAR;
        const double c = exp(-la / n);
        memcpy(A, Xr, (size_t)nn * sizeof(double));
        if (!invert(n, A, Ai)) return MRO_ERR_SINGULAR;
        double inner = 0.0;                       /* <dX, Xr> */
        for (int64_t e = 0; e < nn; ++e) inner += dX[e] * Xr[e];
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) {
                const double dXr = c * (dX[i * n + j] - inner * Ai[j * n + i] / n);   /* Xr^-T */
                dM[i * n + j] = a * dXr;
            }
        return MRO_OK;
    }
    if (p->mode == 3 || p->mode == 4) {
        const double a = (double)p->alpha;
        double* A = work + nn;
        double* Ab = work + 2 * nn;                /* dL/dA */
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) A[i * n + j] = 0.5 * a * (M[i * n + j] - M[j * n + i]);
        if (p->mode == 3) {
            /* X = 2 W^-1 - I with W = I - A, so dX = 2 W^-1 dA W^-1 and
             * dA = 2 W^-T dX W^-T */
            double* W = work + 3 * nn;
            double* Wi = work + 4 * nn;
            double* WiT = work + 5 * nn;
            double* T = work + 6 * nn;
            for (int64_t e = 0; e < nn; ++e) W[e] = -A[e];
            for (int i = 0; i < n; ++i) W[i * n + i] += 1.0;
            if (!invert(n, W, Wi)) return MRO_ERR_SINGULAR;
            transpose(n, Wi, WiT);
            matmul(n, WiT, dX, T);
            matmul(n, T, WiT, Ab);
            for (int64_t e = 0; e < nn; ++e) Ab[e] *= 2.0;
        } else {
            /* The adjoint of the Frechet derivative of exp at A is the
             * derivative at A^T: dA = L(A^T, dX), the upper right block of
             * exp([[A^T, dX], [0, A^T]]) (Van Loan, "Computing integrals
             * involving the matrix exponential", 1978). */
            const int m = 2 * n;
            const int64_t mm = (int64_t)m * m;
            double* Z = malloc(sizeof(double) * 4 * mm);
            if (!Z) return MRO_ERR_ARG;
            double* EZ = Z + mm;
            for (int64_t e = 0; e < mm; ++e) Z[e] = 0.0;
            for (int i = 0; i < n; ++i)
                for (int j = 0; j < n; ++j) {
                    Z[i * m + j] = A[j * n + i];
                    Z[(i + n) * m + (j + n)] = A[j * n + i];
                    Z[i * m + (j + n)] = dX[i * n + j];
                }
            const int ok = expm_inplace(m, Z, EZ, Z + 2 * mm, Z + 3 * mm);
            for (int i = 0; i < n; ++i)
                for (int j = 0; j < n; ++j) Ab[i * n + j] = EZ[i * m + (j + n)];
            free(Z);
            if (!ok) return MRO_ERR_ARG;
        }
        /* A = alpha (M - M^T) / 2 */
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) dM[i * n + j] = 0.5 * a * (Ab[i * n + j] - Ab[j * n + i]);
        return MRO_OK;
    }
    if (p->mode == 2) {
        const double a = (double)p->ldu_offdiag, d = (double)p->ldu_diag;
        double* Lm = work + nn;
        double* U = work + 2 * nn;
        double* DU = work + 3 * nn;
        double* T = work + 4 * nn;
        double* T2 = work + 5 * nn;
        double D[64 * 8];                          /* n <= 512 */
        set_identity(n, Lm);
        set_identity(n, U);
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) {
                if (i > j) Lm[i * n + j] = a * M[i * n + j];
                if (i < j) U[i * n + j] = a * M[i * n + j];
            }
        for (int i = 0; i < n; ++i) D[i] = exp(d * tanh(M[i * n + i]));
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) DU[i * n + j] = D[i] * U[i * n + j];
        /* dL = dX (DU)^T */
        transpose(n, DU, T);
        double* dL = T2;
        matmul(n, dX, T, dL);
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < i; ++j) dM[i * n + j] = a * dL[i * n + j];
        /* d(DU) = L^T dX */
        transpose(n, Lm, T);
        double* dDU = T2;
        matmul(n, T, dX, dDU);
        for (int i = 0; i < n; ++i) {
            double dD = 0.0;
            for (int j = 0; j < n; ++j) dD += dDU[i * n + j] * U[i * n + j];
            const double th = tanh(M[i * n + i]);
            dM[i * n + i] = dD * D[i] * d * (1.0 - th * th);
            for (int j = i + 1; j < n; ++j) dM[i * n + j] = a * D[i] * dDU[i * n + j];
        }
        return MRO_OK;
    }
    return MRO_ERR_ARG;
}

/* Upstream gradient of the readout form: o_t = S_t U (and the snapshots
 * S_t at 1-based t = k * every) are the outputs, so
 *   dL/dS_t = do_t U^T  (+ dP_k when t = k * every),
 * with U the head's [n, q] query columns.  Written for position t (0-based)
 * of sequence (b, h) into G. */
typedef struct {
    const double* u;        /* [n, q], or [H, n, q] with u_per_head */
    int q, u_per_head;
    const double* d_o;      /* [B, L, H, n, q] */
    int64_t snap_every;     /* 0: no snapshots */
    const double* d_snap;   /* [B, L/every, H, n, n] or NULL */
} readout_grad_t;

static void readout_dS(const mro_problem* p, const readout_grad_t* R, int64_t b, int64_t t, int64_t h,
                       double* G)
{
    const int n = p->n, q = R->q;
    const double* U = R->u + (R->u_per_head ? h * n * q : 0);
    const double* dO = R->d_o + ((b * p->L + t) * p->H + h) * (int64_t)n * q;
    for (int i = 0; i < n; ++i)
        for (int j = 0; j < n; ++j) {
            double a = 0.0;                       /* (do_t U^T)_ij = sum_c do_t[i][c] U[j][c] */
            for (int c = 0; c < q; ++c) a += dO[i * q + c] * U[j * q + c];
            G[i * n + j] = a;
        }
    if (R->snap_every > 0 && R->d_snap && (t + 1) % R->snap_every == 0) {
        const int64_t L_s = p->L / R->snap_every, k = (t + 1) / R->snap_every - 1;
        const double* dP = R->d_snap + ((b * L_s + k) * p->H + h) * (int64_t)n * n;
        for (int e = 0; e < n * n; ++e) G[e] += dP[e];
    }
}

/* dL/dS_t for position t: from the dense array dS, or from the readout's
 * gradients. */
static void upstream(const mro_problem* p, const double* dS, const readout_grad_t* R, int64_t b, int64_t t,
                     int64_t h, double* G)
{
    const int64_t nn = (int64_t)p->n * p->n;
    if (R) readout_dS(p, R, b, t, h, G);
    else memcpy(G, dS + ((b * p->L + t) * p->H + h) * nn, (size_t)nn * sizeof(double));
}

/* Backward of one (b, h) sequence.  dS: [B,L,H,n,n] (or, with R, the
 * readout's gradients); dx: [B,L,H*n*n]; dS0: [B,H,n,n] or NULL.  Holds
 * every X_t and S_t of the sequence. */
static int backward_sequence(const mro_problem* p, const void* x, const double* S0, const double* dS,
                             const readout_grad_t* R, double* dx, double* dS0, int64_t bh)
{
    const int n = p->n;
    const int64_t nn = (int64_t)n * n, L = p->L;
    const int64_t b = bh / p->H, h = bh % p->H;
    double* X = malloc(sizeof(double) * (size_t)(L * nn + 1));
    double* S = malloc(sizeof(double) * (size_t)((L + 1) * nn));
    double* work = malloc(sizeof(double) * (size_t)(13 * nn));    /* 6 n*n here + 7 n*n for lift_vjp */
    int rc = MRO_OK;
    if (!X || !S || !work) { rc = MRO_ERR_ARG; goto done; }
    /* forward: S[0] = S0 (or I), S[t+1] = S[t] X_{t+1} */
    if (S0) memcpy(S, S0 + bh * nn, (size_t)nn * sizeof(double));
    else set_identity(n, S);
    for (int64_t t = 0; t < L; ++t) {
        if ((rc = mro_lift(p, x, b, t, h, X + t * nn, work)) != MRO_OK) goto done;
        matmul(n, S + t * nn, X + t * nn, S + (t + 1) * nn);
    }
    /* reverse */
    double* G = work;              /* G_t */
    double* Gn = work + nn;
    double* Xt = work + 2 * nn;
    double* dX = work + 3 * nn;
    double* St = work + 4 * nn;
    double* ds = work + 5 * nn;
    if (L > 0) upstream(p, dS, R, b, L - 1, h, G);
    for (int64_t t = L - 1; t >= 0; --t) {
        transpose(n, S + t * nn, St);                 /* S_{t-1}^T (position t holds X_{t+1}) */
        matmul(n, St, G, dX);
        if ((rc = lift_vjp(p, x, b, t, h, dX, dx + ((b * L + t) * p->H + h) * nn, work + 6 * nn)) != MRO_OK)
            goto done;
        transpose(n, X + t * nn, Xt);
        matmul(n, G, Xt, Gn);                         /* G_t X_t^T */
        if (t > 0) {
            upstream(p, dS, R, b, t - 1, h, ds);
            for (int64_t e = 0; e < nn; ++e) G[e] = ds[e] + Gn[e];
        } else if (dS0) {
            memcpy(dS0 + bh * nn, Gn, (size_t)nn * sizeof(double));
        }
    }
    if (L == 0 && dS0) memset(dS0 + bh * nn, 0, (size_t)nn * sizeof(double));
done:
    free(X);
    free(S);
    free(work);
    return rc;
}

typedef struct {
    const mro_problem* p;
    const void* x;
    const double* S0;
    const double* dS;
    const readout_grad_t* R;
    double* dx;
    double* dS0;
    int64_t next;
    pthread_mutex_t lock;
    int status;
} bwd_job_t;

static void* bwd_worker(void* arg)
{
    bwd_job_t* J = arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t i = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (i >= J->p->B * J->p->H) break;
        const int rc = backward_sequence(J->p, J->x, J->S0, J->dS, J->R, J->dx, J->dS0, i);
        if (rc != MRO_OK) {
            pthread_mutex_lock(&J->lock);
            J->status = rc;
            pthread_mutex_unlock(&J->lock);
        }
    }
    return NULL;
}

/* dx [B,L,H*n*n] (gradient with respect to the widened embedding values) and
 * dS0 [B,H,n,n] (may be NULL) from upstream gradients dS [B,L,H,n,n]. */
int mro_backward(const mro_problem* p, const void* x, const double* S0, const double* dS,
                 double* dx, double* dS0, int nthreads)
{
    if (check_problem(p) != MRO_OK || !dS || !dx) return MRO_ERR_ARG;
    if (p->mode == 2 && p->n > 512) return MRO_ERR_ARG;
    bwd_job_t J;
    memset(&J, 0, sizeof J);
    J.p = p; J.x = x; J.S0 = S0; J.dS = dS; J.dx = dx; J.dS0 = dS0;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    pthread_t th[256];
    if (nthreads > 256) nthreads = 256;
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, bwd_worker, &J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&J.lock);
    return J.status;
}

/* Backward of the readout form: dx [B,L,H*n*n] and dS0 [B,H,n,n] (may be
 * NULL) from the gradients of the readout outputs, d_o [B,L,H,n,q] (with o_t
 * = S_t U, U [n,q] or [H,n,q] when u_per_head) and d_snap [B,L/every,H,n,n]
 * of the snapshots S_t at 1-based t = k * every (NULL or every == 0: none).
 * The chain rule of o_t = S_t U gives dL/dS_t = do_t U^T, then the scan's
 * backward as in mro_backward. */
int mro_backward_readout(const mro_problem* p, const void* x, const double* S0, const double* u, int q,
                         int u_per_head, const double* d_o, int64_t snap_every, const double* d_snap,
                         double* dx, double* dS0, int nthreads)
{
    if (check_problem(p) != MRO_OK || !u || q < 1 || !d_o || !dx || snap_every < 0) return MRO_ERR_ARG;
    if (p->mode == 2 && p->n > 512) return MRO_ERR_ARG;
    readout_grad_t R;
    R.u = u; R.q = q; R.u_per_head = u_per_head; R.d_o = d_o; R.snap_every = snap_every; R.d_snap = d_snap;
    bwd_job_t J;
    memset(&J, 0, sizeof J);
    J.p = p; J.x = x; J.S0 = S0; J.R = &R; J.dx = dx; J.dS0 = dS0;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    pthread_t th[256];
    if (nthreads > 256) nthreads = 256;
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, bwd_worker, &J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&J.lock);
    return J.status;
}
