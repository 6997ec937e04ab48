/*
 * sketchssm_oracle.c -- plain fp64 CPU oracle of the SketchSSM windowed decode.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's CPU
 * baseline leg load this library; the product path never does.  It shares no
 * code, header or constant with the CUDA library, and it does not include it.
 *
 * What it computes (method: "SketchSSM: Write to the Full State, Read from a
 * Compact Sketch", arXiv 2609.33051v1, Abstract; agihunt digest of the same
 * paper, bullets "Core idea", "Mechanism details" and "Error control"):
 *   - the per-token recurrence of the three linear-attention families the
 *     abstract names (Mamba-2 scalar decay, Gated DeltaNet, Kimi-Delta KDA);
 *   - the exact full read o = S^T q after each token (the full-read baseline);
 *   - the windowed update: the buffered tokens applied exactly, in order, once
 *     per window, followed by the sketch refresh P = S^T U (the abstract: one
 *     full-state read per state update precomputes the outputs of the basis
 *     vectors; the digest: the same kernel updates the state and refreshes the
 *     sketch, and approximation error never enters S);
 *   - the sketch read of one decode step: the query carried back to the
 *     window-start state through the buffered tokens, the exact contribution of
 *     those tokens, and the state part reconstructed as P (R q~) (the digest:
 *     a query that is a combination of basis vectors has as output the same
 *     combination of the stored basis outputs).
 *
 * Logical layout used here (and only here): per head, S is dk x dv row-major,
 * S[i*dv + c], i a key channel, c a value channel.  Token arrays are
 * time-major, [t][head][channel].  Everything is double; the build uses
 * -O2 -ffp-contract=off so that no multiply-add is fused behind our back.
 *
 * Readings where the pages give no formula (the workload definitions fix the
 * GDN rule; the rest is the plainest reading):
 *   Mamba-2: S <- a S + k v^T          (no dt scaling, no skip term, no gate)
 *   GDN:     S <- a (I - b k k^T) S + b k v^T
 *   KDA:     S <- (I - b k k^T) diag(a) S + b k v^T   (decay, then delta)
 *   read:    o_t = S_t^T q_t, after token t has been applied.
 * Parity status: pinned by the tests in tests/test_oracle_*.py (closed forms,
 * brute force on tiny heads, invariants); the choice of basis U is a reading
 * and is pinned only through its optimality, not by the pages.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_MAMBA2 = 0, ORC_GDN = 1, ORC_KDA = 2 };

/* bf16 storage of a state value: round to float (nearest-even), then keep the
 * top 16 bits of the float with round-to-nearest-even on the dropped 16. */
static double to_bf16(double x)
{
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) return (double)f; /* inf / nan unchanged */
    uint32_t lsb = (u >> 16) & 1u;
    u = (u + 0x7fffu + lsb) & 0xffff0000u;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* One token of the recurrence, applied in place to one head's S (dk x dv).
 * alpha points at 1 value (Mamba-2, GDN) or dk values (KDA). */
static void token_update(int kind, int dk, int dv, double *S, const double *k,
                         const double *v, const double *alpha, double beta)
{
    if (kind == ORC_MAMBA2) {
        double a = alpha[0];
        for (int i = 0; i < dk; ++i)
            for (int c = 0; c < dv; ++c)
                S[i * dv + c] = a * S[i * dv + c] + k[i] * v[c];
        return;
    }
    for (int c = 0; c < dv; ++c) {
        if (kind == ORC_KDA)
            for (int i = 0; i < dk; ++i) S[i * dv + c] = alpha[i] * S[i * dv + c];
        double x = 0.0; /* x_c = sum_i k_i S_ic, i ascending */
        for (int i = 0; i < dk; ++i) x += k[i] * S[i * dv + c];
        for (int i = 0; i < dk; ++i) {
            double bk = beta * k[i];
            if (kind == ORC_GDN)
                S[i * dv + c] = alpha[0] * (S[i * dv + c] - bk * x) + bk * v[c];
            else
                S[i * dv + c] = S[i * dv + c] - bk * x + bk * v[c];
        }
    }
}

/* o = S^T q for one head. */
static void read_state(int dk, int dv, const double *S, const double *q, double *o)
{
    for (int c = 0; c < dv; ++c) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += S[i * dv + c] * q[i];
        o[c] = acc;
    }
}

static int valid(int kind, int N, int dk, int dv)
{
    return (kind == ORC_MAMBA2 || kind == ORC_GDN || kind == ORC_KDA) && N >= 0 && dk > 0 && dv > 0;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads the following calls use (n >= 1); a timing control only, no effect on results:
 * every head is computed by one thread, in the same order, whatever the count. */
int orc_set_num_threads(int n)
{
    if (n < 1) return -1;
#ifdef _OPENMP
    omp_set_num_threads(n);
#endif
    return 0;
}

/* Per-step exact recurrence over T tokens for N heads (the full-read path):
 * for t = 0..T-1: S <- token t; if Q: O[t] = S^T Q[t].  With bf16_state the
 * state is rounded to bf16 after every token (after that token's read, which
 * sees the unrounded update), as a path that stores S in bf16 and writes it
 * back every step.
 *   S [N][dk][dv] in/out;  K [T][N][dk];  V [T][N][dv];  A [T][N][na]
 *   (na = dk for KDA, else 1);  Bt [T][N] (ignored for Mamba-2, may be NULL);
 *   Q [T][N][dk] or NULL;  O [T][N][dv] or NULL. */
int orc_exact_steps(int kind, int N, int dk, int dv, int T, double *S, const double *K,
                    const double *V, const double *A, const double *Bt, const double *Q,
                    double *O, int bf16_state)
{
    if (!valid(kind, N, dk, dv) || T < 0 || !S || !K || !V || !A) return -1;
    if (kind != ORC_MAMBA2 && !Bt) return -1;
    const int na = kind == ORC_KDA ? dk : 1;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        double *Sn = S + (size_t)n * dk * dv;
        for (int t = 0; t < T; ++t) {
            size_t tn = (size_t)t * N + n;
            double beta = kind == ORC_MAMBA2 ? 1.0 : Bt[tn];
            token_update(kind, dk, dv, Sn, K + tn * dk, V + tn * dv, A + tn * na, beta);
            if (Q && O) read_state(dk, dv, Sn, Q + tn * dk, O + tn * dv);
            if (bf16_state)
                for (int e = 0; e < dk * dv; ++e) Sn[e] = to_bf16(Sn[e]);
        }
    }
    return 0;
}

/* Exact read o = S^T q for N heads: S [N][dk][dv], Q [N][dk], O [N][dv]. */
int orc_read(int N, int dk, int dv, const double *S, const double *Q, double *O)
{
    if (N < 0 || dk <= 0 || dv <= 0 || !S || !Q || !O) return -1;
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n)
        read_state(dk, dv, S + (size_t)n * dk * dv, Q + (size_t)n * dk, O + (size_t)n * dv);
    return 0;
}

/* Windowed update of N heads: apply buffered tokens 0..n-1 in order (n = 0 is a
 * sketch refresh only), round the stored state to bf16 if bf16_state, then
 * refresh the sketch of the stored state, P = S^T U.
 *   S [N][dk][dv] in/out;  K [n][N][dk];  V [n][N][dv];  A [n][N][na];
 *   Bt [n][N];  U [N][dk][r] (the head's basis);  P [N][dv][r] out. */
int orc_update_window(int kind, int N, int dk, int dv, int r, int n, double *S,
                      const double *K, const double *V, const double *A, const double *Bt,
                      const double *U, double *P, int bf16_state)
{
    if (!valid(kind, N, dk, dv) || r <= 0 || n < 0 || !S || !U || !P) return -1;
    if (n > 0 && (!K || !V || !A || (kind != ORC_MAMBA2 && !Bt))) return -1;
    const int na = kind == ORC_KDA ? dk : 1;
#pragma omp parallel for schedule(static)
    for (int h = 0; h < N; ++h) {
        double *Sh = S + (size_t)h * dk * dv;
        for (int t = 0; t < n; ++t) {
            size_t th = (size_t)t * N + h;
            double beta = kind == ORC_MAMBA2 ? 1.0 : Bt[th];
            token_update(kind, dk, dv, Sh, K + th * dk, V + th * dv, A + th * na, beta);
        }
        if (bf16_state)
            for (int e = 0; e < dk * dv; ++e) Sh[e] = to_bf16(Sh[e]);
        const double *Uh = U + (size_t)h * dk * r;
        double *Ph = P + (size_t)h * dv * r;
        for (int c = 0; c < dv; ++c)
            for (int m = 0; m < r; ++m) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += Sh[i * dv + c] * Uh[i * r + m];
                Ph[c * r + m] = acc;
            }
    }
    return 0;
}

/* Sketch read of decode step j (1 <= j): buffered tokens 0..j-1 are not yet in
 * the window-start state S0, whose sketch is P = S0^T U; token j-1 is the
 * current step's own token.  Backward over the buffered tokens:
 *     w <- q;  o_buf <- 0
 *     for t = j-1 .. 0:
 *         x = k_t . w;  s = b_t x  (b = 1 for Mamba-2);  o_buf += s v_t
 *         w <- M_t^T w:  Mamba-2 a_t w;  GDN a_t (w - b_t x k_t);
 *                        KDA a_t (.) (w - b_t x k_t)   (elementwise decay)
 *     q~ = w;  c = R q~;  o = P c + o_buf
 * In exact arithmetic S_j^T q = S0^T q~ + o_buf, so the only approximation is
 * S0^T q~ ~= S0^T U R q~ = P R q~.
 *   P [N][dv][r];  R [N][r][dk];  q [N][dk];  K [j][N][dk];  V [j][N][dv];
 *   A [j][N][na];  Bt [j][N];  o [N][dv] out;  qt [N][dk], ob [N][dv] optional. */
int orc_sketch_read(int kind, int N, int dk, int dv, int r, int j, const double *P,
                    const double *R, const double *q, const double *K, const double *V,
                    const double *A, const double *Bt, double *o, double *qt, double *ob)
{
    if (!valid(kind, N, dk, dv) || r <= 0 || j < 0 || !P || !R || !q || !o) return -1;
    if (j > 0 && (!K || !V || !A || (kind != ORC_MAMBA2 && !Bt))) return -1;
    const int na = kind == ORC_KDA ? dk : 1;
#pragma omp parallel for schedule(static)
    for (int h = 0; h < N; ++h) {
        double *w = (double *)malloc(sizeof(double) * (size_t)(dk + dv + r));
        double *obuf = w + dk, *coef = w + dk + dv;
        for (int i = 0; i < dk; ++i) w[i] = q[(size_t)h * dk + i];
        for (int c = 0; c < dv; ++c) obuf[c] = 0.0;
        for (int t = j - 1; t >= 0; --t) {
            size_t th = (size_t)t * N + h;
            const double *k = K + th * dk, *v = V + th * dv, *a = A + th * na;
            double b = kind == ORC_MAMBA2 ? 1.0 : Bt[th];
            double x = 0.0;
            for (int i = 0; i < dk; ++i) x += k[i] * w[i];
            double s = b * x;
            for (int c = 0; c < dv; ++c) obuf[c] += s * v[c];
            for (int i = 0; i < dk; ++i) {
                if (kind == ORC_MAMBA2) w[i] = a[0] * w[i];
                else if (kind == ORC_GDN) w[i] = a[0] * (w[i] - s * k[i]);
                else w[i] = a[i] * (w[i] - s * k[i]);
            }
        }
        const double *Rh = R + (size_t)h * r * dk;
        for (int m = 0; m < r; ++m) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += Rh[m * dk + i] * w[i];
            coef[m] = acc;
        }
        const double *Ph = P + (size_t)h * dv * r;
        for (int c = 0; c < dv; ++c) {
            double acc = 0.0;
            for (int m = 0; m < r; ++m) acc += Ph[c * r + m] * coef[m];
            o[(size_t)h * dv + c] = acc + obuf[c];
        }
        if (qt)
            for (int i = 0; i < dk; ++i) qt[(size_t)h * dk + i] = w[i];
        if (ob)
            for (int c = 0; c < dv; ++c) ob[(size_t)h * dv + c] = obuf[c];
        free(w);
    }
    return 0;
}

/* bf16 rounding of an array, exposed so that tests can mirror bf16 storage. */
int orc_round_bf16(size_t n, double *x)
{
    if (!x) return -1;
    for (size_t e = 0; e < n; ++e) x[e] = to_bf16(x[e]);
    return 0;
}
