/*
 * muon_oracle.c -- plain fp64 CPU oracle for the Muon / MONA optimizer step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file or the library built from it: only the tests, the smoke
 * check and the CPU-baseline leg of the benchmark use it.  It shares no code,
 * header, table or constant with the CUDA library; it is written from the
 * method's published description:
 *
 *   [MONA]  "MONA - Muon-optimizer met Nesterov-versnelling" (gist.science,
 *           paper 2605.26842), section 2 "Methodologie: MONA", Kernalgoritme
 *           steps 1-4: gradient difference, acceleration EMA, curvature-aware
 *           gradient, momentum, Newton-Schulz orthogonalisation, weight update
 *           with decoupled decay.
 *   [POLAR] Telegram review "quant_prune_distill" post 677 (tgviewer.app),
 *           opening paragraph: the Muon step replaces the momentum by its
 *           polar factor polar(X) = U V^T for X = U S V^T; paragraphs on the
 *           Gram route: polar(X) = X (X^T X)^{-1/2} with the matrix power also
 *           found by Newton-Schulz on the small Gram matrix, restarts, and a
 *           division by 1.02-1.05 to keep the eigenvalues inside [0, 1].
 *
 * Every floating-point operation is done in IEEE double precision, in the
 * order the definitions state, with full (unblocked) matrix products.  The
 * only parallelism is OpenMP over independent output rows of a product and
 * over disjoint column pairs of one Jacobi round; neither changes any
 * arithmetic.
 *
 * Readings taken where the pages are silent (each is also listed in the
 * design notes of the repository):
 *   - Newton-Schulz form: the quintic step X <- a X + (b A + c A A) X with
 *     A = X X^T on the wide view (short side first); coefficients are inputs.
 *   - Normalisation before the iteration: X0 = M / ((||M||_F + eps) * f).
 *   - Gram route restarts: at a restart step k > 0 the accumulated factor is
 *     applied (Xb <- Q Xb), divided by f, the Gram matrix is recomputed and
 *     Q is reset to the identity.
 *   - Heavy-ball momentum exactly as written on the MONA page (no extra
 *     look-ahead), decay uses the pre-update weights.
 *
 * parity pins: see the CPU tests (closed form through an SVD, invariants of
 * the polar factor, hand-worked MONA examples, Gram == direct route).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Rounding of a double to the 16-bit and 32-bit floating formats           */
/* (round to nearest, ties to even), written from the formats' definitions:  */
/* p significant bits, smallest normal exponent emin, subnormals with the    */
/* fixed quantum 2^(emin-p+1), overflow to infinity.                         */
/* ------------------------------------------------------------------------ */
static double round_to_format(double x, int p, int emin, double maxval)
{
    if (isnan(x) || isinf(x) || x == 0.0) return x;
    int e;
    (void)frexp(x, &e);            /* x = m 2^e with 0.5 <= |m| < 1 */
    int q = e - p;                 /* weight of the last kept bit    */
    int qmin = emin - p + 1;       /* subnormal quantum              */
    if (q < qmin) q = qmin;
    double scaled = ldexp(x, -q);  /* exact                           */
    double r = nearbyint(scaled);  /* default mode: ties to even      */
    double y = ldexp(r, q);
    if (fabs(y) > maxval) return x > 0 ? INFINITY : -INFINITY;
    return y;
}

double oracle_round_bf16(double x) { return round_to_format(x, 8, -126, 0x1.fep127); }
double oracle_round_fp16(double x) { return round_to_format(x, 11, -14, 65504.0); }
double oracle_round_fp32(double x) { return round_to_format(x, 24, -126, 0x1.fffffep127); }

/* kind: 0 = keep, 1 = bf16, 2 = fp16, 3 = fp32 */
void oracle_round_array(double* x, long long n, int kind)
{
    if (kind == 0) return;
    for (long long i = 0; i < n; ++i) {
        if (kind == 1) x[i] = oracle_round_bf16(x[i]);
        else if (kind == 2) x[i] = oracle_round_fp16(x[i]);
        else x[i] = oracle_round_fp32(x[i]);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------------ */
/* Dense helpers (row-major).                                                */
/* ------------------------------------------------------------------------ */

/* C[m x n] = A[m x k] * B[k x n] */
static void mat_mul(const double* A, const double* B, double* C, int m, int k, int n)
{
    #pragma omp parallel for schedule(static)
    for (int i = 0; i < m; ++i) {
        double* c = C + (size_t)i * n;
        for (int j = 0; j < n; ++j) c[j] = 0.0;
        for (int p = 0; p < k; ++p) {
            double a = A[(size_t)i * k + p];
            const double* b = B + (size_t)p * n;
            for (int j = 0; j < n; ++j) c[j] += a * b[j];
        }
    }
}

/* C[m x m] = A[m x k] * A^T */
static void mat_mul_aat(const double* A, double* C, int m, int k)
{
    #pragma omp parallel for schedule(dynamic, 4)
    for (int i = 0; i < m; ++i) {
        const double* ai = A + (size_t)i * k;
        for (int j = 0; j < m; ++j) {
            const double* aj = A + (size_t)j * k;
            double s = 0.0;
            for (int p = 0; p < k; ++p) s += ai[p] * aj[p];
            C[(size_t)i * m + j] = s;
        }
    }
}

static void transpose(const double* X, double* Y, int rows, int cols)
{
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c)
            Y[(size_t)c * rows + r] = X[(size_t)r * cols + c];
}

double oracle_frobenius(const double* X, long long n)
{
    double s = 0.0;
    for (long long i = 0; i < n; ++i) s += X[i] * X[i];
    return sqrt(s);
}

/* ------------------------------------------------------------------------ */
/* [MONA] section 2, steps 1-4 (elementwise part).                           */
/*   D   = G - Gp                 (step 1, gradient difference)              */
/*   A'  = beta_a A + (1-beta_a) D (step 2, acceleration EMA)                */
/*   Gt  = G + alpha A'            (step 3, curvature-aware gradient)        */
/*   M'  = mu M + Gt               (step 4, momentum)                        */
/*   Gp' = G                       (the previous gradient for the next step) */
/* ------------------------------------------------------------------------ */
void oracle_mona(long long n, const double* G, double* Gp, double* A, double* M,
                 double beta_a, double alpha, double mu)
{
    for (long long i = 0; i < n; ++i) {
        double D = G[i] - Gp[i];
        double An = beta_a * A[i] + (1.0 - beta_a) * D;
        double Gt = G[i] + alpha * An;
        double Mn = mu * M[i] + Gt;
        A[i] = An;
        M[i] = Mn;
        Gp[i] = G[i];
    }
}

/* [MONA] section 2, step 4, last equation: W' = W - eta (gamma O + lambda W) */
void oracle_weight_update(long long n, double* W, const double* O,
                          double eta, double gamma, double lambda)
{
    for (long long i = 0; i < n; ++i)
        W[i] = W[i] - eta * (gamma * O[i] + lambda * W[i]);
}

/* ------------------------------------------------------------------------ */
/* Quintic Newton-Schulz iteration on the wide view X (s x l, s <= l).       */
/* For k = 0..K-1:  X *= prescale[k] (if given);  A = X X^T;                 */
/*                  B = b_k A + c_k A A;  X = a_k X + B X.                   */
/* coeffs holds (a_k, b_k, c_k) for each step.  No normalisation is done     */
/* here.  X is updated in place.                                             */
/* ------------------------------------------------------------------------ */
void oracle_ns_poly(double* X, int s, int l, int n_steps, const double* coeffs,
                    const double* prescale)
{
    double* A = (double*)malloc(sizeof(double) * (size_t)s * s);
    double* AA = (double*)malloc(sizeof(double) * (size_t)s * s);
    double* B = (double*)malloc(sizeof(double) * (size_t)s * s);
    double* BX = (double*)malloc(sizeof(double) * (size_t)s * l);
    for (int k = 0; k < n_steps; ++k) {
        double a = coeffs[3 * k + 0], b = coeffs[3 * k + 1], c = coeffs[3 * k + 2];
        if (prescale) {
            double f = prescale[k];
            for (size_t i = 0; i < (size_t)s * l; ++i) X[i] *= f;
        }
        mat_mul_aat(X, A, s, l);          /* A = X X^T      */
        mat_mul(A, A, AA, s, s, s);       /* A A            */
        for (size_t i = 0; i < (size_t)s * s; ++i) B[i] = b * A[i] + c * AA[i];
        mat_mul(B, X, BX, s, s, l);       /* B X            */
        for (size_t i = 0; i < (size_t)s * l; ++i) X[i] = a * X[i] + BX[i];
    }
    free(A); free(AA); free(B); free(BX);
}

/* ------------------------------------------------------------------------ */
/* [POLAR] Gram route: polar(X) = X (X^T X)^{-1/2}, written on the wide      */
/* view with the short side first, R = X X^T (s x s).  The same polynomial   */
/* h_k(R) = a_k I + b_k R + c_k R^2 as the direct iteration is applied       */
/* through the Gram matrix: with X_k = Q Xb,                                 */
/*      X_{k+1} = h_k X_k   =>   Q <- h_k Q,   R <- h_k R h_k.               */
/* Restarts (steps listed in `restarts`, k > 0): Xb <- Q Xb, Xb /= f,        */
/* R <- Xb Xb^T, Q <- I.  Finally X = Q Xb.  The input X must already hold   */
/* the normalised start (including the first division by f).  In place.      */
/* ------------------------------------------------------------------------ */
void oracle_gram_poly(double* X, int s, int l, int n_steps, const double* coeffs,
                      const int* restarts, int n_restarts, double f)
{
    size_t ss = (size_t)s * s;
    double* R = (double*)malloc(sizeof(double) * ss);
    double* R2 = (double*)malloc(sizeof(double) * ss);
    double* Q = (double*)malloc(sizeof(double) * ss);
    double* H = (double*)malloc(sizeof(double) * ss);
    double* T = (double*)malloc(sizeof(double) * ss);
    double* Xn = (double*)malloc(sizeof(double) * (size_t)s * l);

    mat_mul_aat(X, R, s, l);
    memset(Q, 0, sizeof(double) * ss);
    for (int i = 0; i < s; ++i) Q[(size_t)i * s + i] = 1.0;

    for (int k = 0; k < n_steps; ++k) {
        int is_restart = 0;
        for (int r = 0; r < n_restarts; ++r)
            if (restarts[r] == k && k > 0) is_restart = 1;
        if (is_restart) {
            mat_mul(Q, X, Xn, s, s, l);                     /* Xb <- Q Xb */
            for (size_t i = 0; i < (size_t)s * l; ++i) X[i] = Xn[i] / f;
            mat_mul_aat(X, R, s, l);                        /* R <- Xb Xb^T */
            memset(Q, 0, sizeof(double) * ss);
            for (int i = 0; i < s; ++i) Q[(size_t)i * s + i] = 1.0;
        }
        double a = coeffs[3 * k + 0], b = coeffs[3 * k + 1], c = coeffs[3 * k + 2];
        mat_mul(R, R, R2, s, s, s);                         /* R^2 */
        for (size_t i = 0; i < ss; ++i) H[i] = b * R[i] + c * R2[i];
        for (int i = 0; i < s; ++i) H[(size_t)i * s + i] += a;  /* h = aI + bR + cR^2 */
        mat_mul(H, Q, T, s, s, s);                          /* Q <- h Q */
        memcpy(Q, T, sizeof(double) * ss);
        mat_mul(H, R, T, s, s, s);                          /* R <- h R h */
        mat_mul(T, H, R, s, s, s);
    }
    mat_mul(Q, X, Xn, s, s, l);                             /* X = Q Xb */
    memcpy(X, Xn, sizeof(double) * (size_t)s * l);
    free(R); free(R2); free(Q); free(H); free(T); free(Xn);
}

/* ------------------------------------------------------------------------ */
/* Exact polar factor by one-sided (Hestenes) Jacobi.  X is s x l with       */
/* s <= l (wide view); the rows of X play the role of the columns of the     */
/* tall matrix Y = X^T.  Rotations of row pairs (p, q) make the rows         */
/* mutually orthogonal: X_f = V^T X with orthogonal V (s x s).  Then         */
/* X = V Sigma U^T with sigma_j = ||row j of X_f|| and                       */
/* polar(X) = V U^T = V diag(1/sigma) X_f.  Rows with sigma below            */
/* 1e-14 * sigma_max are dropped (partial isometry on the range).            */
/* Rotation (textbook): alpha = |x_p|^2, beta = |x_q|^2, gamma = x_p . x_q,  */
/* zeta = (beta - alpha) / (2 gamma), t = sign(zeta)/(|zeta| + sqrt(1+z^2)), */
/* c = 1/sqrt(1 + t^2), s = c t, x_p <- c x_p - s x_q, x_q <- s x_p + c x_q. */
/* Pairs are visited in round-robin (tournament) order so that the pairs of  */
/* one round are disjoint; a sweep is s-1 (or s) rounds.  Converged when no  */
/* pair in a sweep has |gamma| > 1e-15 sqrt(alpha beta).                     */
/* Returns the number of sweeps, or -1 if 60 sweeps did not converge.        */
/* ------------------------------------------------------------------------ */
int oracle_polar_jacobi(const double* Xin, int s, int l, double* P)
{
    size_t sl = (size_t)s * l;
    double* X = (double*)malloc(sizeof(double) * sl);
    double* V = (double*)malloc(sizeof(double) * (size_t)s * s);
    memcpy(X, Xin, sizeof(double) * sl);
    memset(V, 0, sizeof(double) * (size_t)s * s);
    for (int i = 0; i < s; ++i) V[(size_t)i * s + i] = 1.0;

    int n = s + (s & 1);              /* even number of players (one dummy) */
    int* slot = (int*)malloc(sizeof(int) * n);
    for (int i = 0; i < n; ++i) slot[i] = i;
    int sweeps = -1;

    for (int sweep = 0; sweep < 60; ++sweep) {
        int rotated = 0;
        for (int round = 0; round < n - 1; ++round) {
            #pragma omp parallel for schedule(dynamic, 1) reduction(|:rotated)
            for (int m = 0; m < n / 2; ++m) {
                int p = slot[m], q = slot[n - 1 - m];
                if (p >= s || q >= s) continue;
                if (p > q) { int t = p; p = q; q = t; }
                double* xp = X + (size_t)p * l;
                double* xq = X + (size_t)q * l;
                double al = 0.0, be = 0.0, ga = 0.0;
                for (int j = 0; j < l; ++j) {
                    al += xp[j] * xp[j];
                    be += xq[j] * xq[j];
                    ga += xp[j] * xq[j];
                }
                if (ga == 0.0 || fabs(ga) <= 1e-15 * sqrt(al * be)) continue;
                rotated = 1;
                double zeta = (be - al) / (2.0 * ga);
                double t = (zeta >= 0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
                double c = 1.0 / sqrt(1.0 + t * t);
                double sn = c * t;
                for (int j = 0; j < l; ++j) {
                    double a = xp[j], b = xq[j];
                    xp[j] = c * a - sn * b;
                    xq[j] = sn * a + c * b;
                }
                for (int i = 0; i < s; ++i) {
                    double a = V[(size_t)i * s + p], b = V[(size_t)i * s + q];
                    V[(size_t)i * s + p] = c * a - sn * b;
                    V[(size_t)i * s + q] = sn * a + c * b;
                }
            }
            /* rotate the tournament: slot[0] fixed, the rest shift by one */
            int last = slot[n - 1];
            for (int i = n - 1; i > 1; --i) slot[i] = slot[i - 1];
            slot[1] = last;
        }
        if (!rotated) { sweeps = sweep + 1; break; }
    }

    double* sig = (double*)malloc(sizeof(double) * s);
    double smax = 0.0;
    for (int i = 0; i < s; ++i) {
        sig[i] = oracle_frobenius(X + (size_t)i * l, l);
        if (sig[i] > smax) smax = sig[i];
    }
    for (int i = 0; i < s; ++i) {
        double inv = (sig[i] > 1e-14 * smax && sig[i] > 0.0) ? 1.0 / sig[i] : 0.0;
        for (int j = 0; j < l; ++j) X[(size_t)i * l + j] *= inv;   /* U^T rows */
    }
    mat_mul(V, X, P, s, s, l);        /* polar = V U^T */
    free(sig); free(slot); free(X); free(V);
    return sweeps;
}

/* Polar factor of an arbitrary rows x cols matrix: transposes tall input.  */
int oracle_polar(const double* Xin, int rows, int cols, double* P)
{
    if (rows <= cols) return oracle_polar_jacobi(Xin, rows, cols, P);
    double* Xt = (double*)malloc(sizeof(double) * (size_t)rows * cols);
    double* Pt = (double*)malloc(sizeof(double) * (size_t)rows * cols);
    transpose(Xin, Xt, rows, cols);
    int r = oracle_polar_jacobi(Xt, cols, rows, Pt);
    transpose(Pt, P, cols, rows);
    free(Xt); free(Pt);
    return r;
}

/* ------------------------------------------------------------------------ */
/* Orthogonalisation of one rows x cols matrix as the Muon step uses it.     */
/*   n  = ||M||_F;  view X = M (rows <= cols) or M^T (rows > cols);          */
/*   X  = round(X) to the 16-bit format the iteration runs in (kind, see     */
/*        oracle_round_array; 0 = none);  X /= (n + eps) f;                  */
/*   route 0: quintic iteration, X /= f again before each step in restarts;  */
/*   route 1: Gram route with the same schedule and restarts;                */
/*   O  = X (transposed back).                                               */
/* ------------------------------------------------------------------------ */
void oracle_orthogonalise(const double* M, int rows, int cols, double* O,
                          int route, int n_steps, const double* coeffs,
                          const int* restarts, int n_restarts, double f,
                          double eps, int round_kind)
{
    int s = rows <= cols ? rows : cols;
    int l = rows <= cols ? cols : rows;
    size_t sl = (size_t)s * l;
    double nrm = oracle_frobenius(M, (long long)sl);
    double* X = (double*)malloc(sizeof(double) * sl);
    if (rows <= cols) memcpy(X, M, sizeof(double) * sl);
    else transpose(M, X, rows, cols);
    oracle_round_array(X, (long long)sl, round_kind);
    double scale = 1.0 / ((nrm + eps) * f);
    for (size_t i = 0; i < sl; ++i) X[i] *= scale;

    if (route == 0) {
        double* pre = (double*)malloc(sizeof(double) * (n_steps > 0 ? n_steps : 1));
        for (int k = 0; k < n_steps; ++k) {
            pre[k] = 1.0;
            for (int r = 0; r < n_restarts; ++r)
                if (restarts[r] == k && k > 0) pre[k] = 1.0 / f;
        }
        oracle_ns_poly(X, s, l, n_steps, coeffs, pre);
        free(pre);
    } else {
        oracle_gram_poly(X, s, l, n_steps, coeffs, restarts, n_restarts, f);
    }
    if (rows <= cols) memcpy(O, X, sizeof(double) * sl);
    else transpose(X, O, cols, rows);
    free(X);
}

/* ------------------------------------------------------------------------ */
/* MONA-Lite, [MONA] section "Efficientie en Implementatie": the auxiliary   */
/* state is kept in bfloat16 and the gradient difference is formed in place  */
/* instead of from a stored previous gradient.  Reading taken (the page     */
/* gives no formulas): step 2 rewritten with the one buffer                 */
/*   B_{k-1} = beta_a A_{k-1} - (1-beta_a) G_{k-1}                           */
/* so that                                                                   */
/*   A_k  = B_{k-1} + (1-beta_a) G_k          (= step 2 exactly)             */
/*   Gt   = G_k + alpha A_k                   (step 3)                       */
/*   M_k  = mu M_{k-1} + Gt                   (step 4)                       */
/*   B_k  = beta_a A_k - (1-beta_a) G_k       (for the next step)            */
/* B starts at 0 (A_0 = G_prev = 0).  round_b != 0 stores B rounded to       */
/* bfloat16 (RNE), the page's precision for the auxiliary state; with      */
/* round_b == 0 the sequence of M equals oracle_mona's exactly (algebra).   */
/* ------------------------------------------------------------------------ */
void oracle_mona_lite(long long n, const double* G, double* B, double* M,
                      double beta_a, double alpha, double mu, int round_b)
{
    for (long long i = 0; i < n; ++i) {
        double An = B[i] + (1.0 - beta_a) * G[i];
        double Gt = G[i] + alpha * An;
        double Mn = mu * M[i] + Gt;
        double Bn = beta_a * An - (1.0 - beta_a) * G[i];
        M[i] = Mn;
        B[i] = round_b ? oracle_round_bf16(Bn) : Bn;
    }
}

/* ------------------------------------------------------------------------ */
/* One full MONA/Muon step for one matrix parameter, [MONA] section 2:       */
/* elementwise pre-pass, orthogonalisation of M', decoupled weight update.   */
/* W, Gp, A, M are updated in place; O (rows x cols) receives the            */
/* orthogonalised momentum.  round_kind applies to the start of the          */
/* iteration only (see oracle_orthogonalise).                                */
/* ------------------------------------------------------------------------ */
void oracle_muon_step(int rows, int cols, double* W, const double* G, double* Gp,
                      double* A, double* M, double* O,
                      double mu, double eta, double lambda, double gamma,
                      double beta_a, double alpha,
                      int n_steps, const double* coeffs, double eps, double f,
                      int round_kind)
{
    long long n = (long long)rows * cols;
    oracle_mona(n, G, Gp, A, M, beta_a, alpha, mu);
    oracle_orthogonalise(M, rows, cols, O, 0, n_steps, coeffs, NULL, 0, f, eps, round_kind);
    oracle_weight_update(n, W, O, eta, gamma, lambda);
}

/* ------------------------------------------------------------------------ */
/* One MONA-Lite step for one matrix parameter: oracle_mona_lite (B in      */
/* bfloat16 when round_b), then the same orthogonalisation and update as     */
/* oracle_muon_step.                                                         */
/* ------------------------------------------------------------------------ */
void oracle_muon_lite_step(int rows, int cols, double* W, const double* G, double* B,
                           double* M, double* O,
                           double mu, double eta, double lambda, double gamma,
                           double beta_a, double alpha,
                           int n_steps, const double* coeffs, double eps, double f,
                           int round_kind, int round_b)
{
    long long n = (long long)rows * cols;
    oracle_mona_lite(n, G, B, M, beta_a, alpha, mu, round_b);
    oracle_orthogonalise(M, rows, cols, O, 0, n_steps, coeffs, NULL, 0, f, eps, round_kind);
    oracle_weight_update(n, W, O, eta, gamma, lambda);
}

/* ------------------------------------------------------------------------ */
/* AdamW for vector-valued parameters (embeddings, biases): the MONA page,  */
/* section 2 ("Ontwerprichtlijnen"), keeps Muon's convention of standard    */
/* AdamW for them and prints no formulas.  Reading: Adam with bias          */
/* correction and decoupled weight decay (Loshchilov and Hutter), step t>=1:*/
/*   m' = b1 m + (1-b1) g        v' = b2 v + (1-b2) g^2                      */
/*   W' = W - lr ( (m'/(1-b1^t)) / (sqrt(v'/(1-b2^t)) + eps) + wd W )        */
/* ------------------------------------------------------------------------ */
void oracle_adamw(long long n, double* W, const double* G, double* m, double* v,
                  double lr, double b1, double b2, double eps, double wd, int t)
{
    const double c1 = 1.0 - pow(b1, (double)t);
    const double c2 = 1.0 - pow(b2, (double)t);
    for (long long i = 0; i < n; ++i) {
        const double mn = b1 * m[i] + (1.0 - b1) * G[i];
        const double vn = b2 * v[i] + (1.0 - b2) * G[i] * G[i];
        const double upd = (mn / c1) / (sqrt(vn / c2) + eps);
        W[i] = W[i] - lr * (upd + wd * W[i]);
        m[i] = mn;
        v[i] = vn;
    }
}
