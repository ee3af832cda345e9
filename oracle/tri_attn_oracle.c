/*
 * tri_attn_oracle.c -- plain, slow, FP64 CPU oracle for triangle attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header, table or helper with the
 * CUDA kernels.
 *
 * Pages this follows:
 *   (A) "16张H100，训练步提速1.73倍：TurboPairFormer为什么不是'装个包就能加速AlphaFold3'"
 *       (biocloudservice.com blog), section "它优化了什么，而不是只'少存一点张量'":
 *       the backward produces gradients for query, key, value and the pair
 *       bias that is shared by all rows; section "先看清'1.73倍'对应什么":
 *       the cost is cubic in the crop size.
 *   (B) "TurboPairFormer: более быстрое, стабильное и точное дообучение OpenFold3"
 *       (dev48.org), section "Точность": accuracy is judged against an FP64
 *       reference fed the identical BF16 inputs.
 *
 * Definition (triangle attention around the starting node, AlphaFold3
 * Pairformer; the pages do not print it, so this is the plain textbook form):
 * for every batch b, pair row i, head h and query j,
 *   s_k    = scale * sum_c q[b,i,j,h,c] k[b,i,k,h,c] + bias[b,h,j,k] + mask[b,i,k]
 *   p_k    = exp(s_k - m) / sum_k' exp(s_k' - m),   m = max_k s_k
 *   out    = sum_k p_k v[b,i,k,h,:]
 *   lse    = m + log sum_k exp(s_k - m)
 * and for an upstream gradient dout:
 *   dv[k]  = sum_j p_jk dout_j
 *   dp_jk  = dout_j . v_k ;  D_j = dout_j . out_j ;  ds_jk = p_jk (dp_jk - D_j)
 *   dq_j   = scale sum_k ds_jk k_k ;  dk_k = scale sum_j ds_jk q_j
 *   dbias[b,h,j,k] = sum_i ds[b,i,j,h,k]     (the bias is shared across rows i)
 *
 * Layouts (all contiguous, row-major, FP64):
 *   q,k,v,dout,out,dq,dk,dv : [B,N,N,H,d]     (b,i,j,h,c)
 *   bias, dbias             : [B,H,N,N]       (b,h,j,k)
 *   mask                    : [B,N,N] (b,i,k) or NULL (no mask)
 *   lse                     : [B,H,N,N]       (b,h,i,j)
 *
 * Every sum runs serially in ascending index order, so the oracle is itself
 * deterministic.  Parallelism (OpenMP) is only across independent rows.
 *
 * `planted` is 0 in normal use.  Non-zero values plant one deliberate mistake
 * so that the test suite can show that its pins detect it:
 *   1 drop the bias term          2 drop the scale
 *   3 softmax over the query axis instead of keys (transposed index)
 *   4 D_j without dout (uses sum of out)   5 wrong sign in ds
 *   6 dbias summed over j instead of i      7 mask applied per query not key
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARGS 1
#define ORC_ERR_FULLY_MASKED 2
#define ORC_ERR_NOMEM 3

/* A key whose additive mask is at or below this value counts as masked when
 * checking that every row keeps at least one key (rows with no key left are
 * outside the contract). */
#define ORC_MASKED_AT (-1.0e8)

static size_t ix5(int b, int i, int j, int h, int c, int N, int H, int d)
{
    return ((((size_t)b * N + i) * N + j) * H + h) * (size_t)d + c;
}
static size_t ix_bias(int b, int h, int j, int k, int N, int H)
{
    return (((size_t)b * H + h) * N + j) * (size_t)N + k;
}

/* scores s[k] for one (b,i,h,j), k = 0..N-1 */
static void scores(int B, int N, int H, int d, double scale,
                   const double *q, const double *k, const double *bias,
                   const double *mask, int b, int i, int h, int j,
                   double *s, int planted)
{
    (void)B;
    for (int kk = 0; kk < N; ++kk) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c)
            dot += q[ix5(b, i, j, h, c, N, H, d)] * k[ix5(b, i, kk, h, c, N, H, d)];
        double v = (planted == 2) ? dot : scale * dot;
        if (planted != 1) v += bias[ix_bias(b, h, j, kk, N, H)];
        if (mask) {
            if (planted == 7) v += mask[((size_t)b * N + i) * N + j];
            else v += mask[((size_t)b * N + i) * N + kk];
        }
        s[kk] = v;
    }
}

/* softmax row: p[k] = exp(s_k - m)/Z, returns lse = m + log Z */
static double softmax_row(int N, const double *s, double *p)
{
    double m = -INFINITY;
    for (int kk = 0; kk < N; ++kk) if (s[kk] > m) m = s[kk];
    double z = 0.0;
    for (int kk = 0; kk < N; ++kk) { p[kk] = exp(s[kk] - m); z += p[kk]; }
    for (int kk = 0; kk < N; ++kk) p[kk] /= z;
    return m + log(z);
}

/* probabilities P[j][k] of one problem (b,i,h), all queries j */
static double *problem_probs(int B, int N, int H, int d, double scale,
                             const double *q, const double *k, const double *bias,
                             const double *mask, int b, int i, int h,
                             double *lse_row, int planted)
{
    double *P = (double *)malloc(sizeof(double) * (size_t)N * N);
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    if (!P || !s) { free(P); free(s); return NULL; }
    for (int j = 0; j < N; ++j) {
        scores(B, N, H, d, scale, q, k, bias, mask, b, i, h, j, s, planted);
        double l = softmax_row(N, s, P + (size_t)j * N);
        if (lse_row) lse_row[j] = l;
    }
    if (planted == 3) { /* normalise over queries instead of keys */
        for (int j = 0; j < N; ++j)
            scores(B, N, H, d, scale, q, k, bias, mask, b, i, h, j, P + (size_t)j * N, 0);
        for (int kk = 0; kk < N; ++kk) {
            double m = -INFINITY, z = 0.0;
            for (int j = 0; j < N; ++j) if (P[(size_t)j * N + kk] > m) m = P[(size_t)j * N + kk];
            for (int j = 0; j < N; ++j) { P[(size_t)j * N + kk] = exp(P[(size_t)j * N + kk] - m); z += P[(size_t)j * N + kk]; }
            for (int j = 0; j < N; ++j) P[(size_t)j * N + kk] /= z;
        }
    }
    free(s);
    return P;
}

static int check_rows_have_keys(int B, int N, const double *mask)
{
    if (!mask) return ORC_OK;
    for (int b = 0; b < B; ++b)
        for (int i = 0; i < N; ++i) {
            int any = 0;
            for (int kk = 0; kk < N; ++kk)
                if (mask[((size_t)b * N + i) * N + kk] > ORC_MASKED_AT) { any = 1; break; }
            if (!any) return ORC_ERR_FULLY_MASKED;
        }
    return ORC_OK;
}

/*
 * Forward for a list of pair rows (b,i): rows[2*r] = b, rows[2*r+1] = i.
 * out is written at the full-size positions of those rows only; lse too.
 * nrows < 0 means every row.
 */
int tri_attn_oracle_fwd(int B, int N, int H, int d, double scale,
                        const double *q, const double *k, const double *v,
                        const double *bias, const double *mask,
                        const int *rows, int nrows,
                        double *out, double *lse, int planted)
{
    if (B <= 0 || N <= 0 || H <= 0 || d <= 0 || !q || !k || !v || !bias || !out || !lse)
        return ORC_ERR_ARGS;
    int st = check_rows_have_keys(B, N, mask);
    if (st) return st;
    int total = (nrows < 0) ? B * N : nrows;
    int err = 0;
    #pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int r = 0; r < total; ++r) {
        for (int h = 0; h < H; ++h) {
            int b = (nrows < 0) ? r / N : rows[2 * r];
            int i = (nrows < 0) ? r % N : rows[2 * r + 1];
            double *lrow = lse + (((size_t)b * H + h) * N + i) * (size_t)N;
            double *P = problem_probs(B, N, H, d, scale, q, k, bias, mask, b, i, h, lrow, planted);
            if (!P) {
                #pragma omp atomic write
                err = ORC_ERR_NOMEM;
                continue;
            }
            for (int j = 0; j < N; ++j)
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int kk = 0; kk < N; ++kk)
                        acc += P[(size_t)j * N + kk] * v[ix5(b, i, kk, h, c, N, H, d)];
                    out[ix5(b, i, j, h, c, N, H, d)] = acc;
                }
            free(P);
        }
    }
    return err;
}

/* ds[j][k] of one problem, given its probabilities P; needs out_j recomputed */
static void problem_ds(int N, int H, int d, const double *P,
                       const double *v, const double *dout,
                       int b, int i, int h, double *ds, int planted)
{
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    for (int j = 0; j < N; ++j) {
        /* out_j = sum_k p_jk v_k (recomputed from the definition) */
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int kk = 0; kk < N; ++kk)
                acc += P[(size_t)j * N + kk] * v[ix5(b, i, kk, h, c, N, H, d)];
            o[c] = acc;
        }
        double Dj = 0.0;
        for (int c = 0; c < d; ++c)
            Dj += ((planted == 4) ? 1.0 : dout[ix5(b, i, j, h, c, N, H, d)]) * o[c];
        for (int kk = 0; kk < N; ++kk) {
            double dp = 0.0;
            for (int c = 0; c < d; ++c)
                dp += dout[ix5(b, i, j, h, c, N, H, d)] * v[ix5(b, i, kk, h, c, N, H, d)];
            double p = P[(size_t)j * N + kk];
            ds[(size_t)j * N + kk] = (planted == 5) ? p * (Dj - dp) : p * (dp - Dj);
        }
    }
    free(o);
}

/*
 * Backward for a list of pair rows: dq, dk, dv at those rows' positions.
 * nrows < 0 means every row.  dbias is not produced here (it sums over all
 * rows i); see tri_attn_oracle_dbias.
 */
int tri_attn_oracle_bwd_rows(int B, int N, int H, int d, double scale,
                             const double *q, const double *k, const double *v,
                             const double *bias, const double *mask,
                             const double *dout, const int *rows, int nrows,
                             double *dq, double *dk, double *dv, int planted)
{
    if (B <= 0 || N <= 0 || H <= 0 || d <= 0 || !q || !k || !v || !bias || !dout ||
        !dq || !dk || !dv)
        return ORC_ERR_ARGS;
    int st = check_rows_have_keys(B, N, mask);
    if (st) return st;
    int total = (nrows < 0) ? B * N : nrows;
    int err = 0;
    #pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int r = 0; r < total; ++r) {
        for (int h = 0; h < H; ++h) {
            int b = (nrows < 0) ? r / N : rows[2 * r];
            int i = (nrows < 0) ? r % N : rows[2 * r + 1];
            double *P = problem_probs(B, N, H, d, scale, q, k, bias, mask, b, i, h, NULL, planted);
            double *ds = (double *)malloc(sizeof(double) * (size_t)N * N);
            if (!P || !ds) {
                free(P); free(ds);
                #pragma omp atomic write
                err = ORC_ERR_NOMEM;
                continue;
            }
            problem_ds(N, H, d, P, v, dout, b, i, h, ds, planted);
            for (int kk = 0; kk < N; ++kk)
                for (int c = 0; c < d; ++c) {
                    double av = 0.0, ak = 0.0;
                    for (int j = 0; j < N; ++j) {
                        av += P[(size_t)j * N + kk] * dout[ix5(b, i, j, h, c, N, H, d)];
                        ak += ds[(size_t)j * N + kk] * q[ix5(b, i, j, h, c, N, H, d)];
                    }
                    dv[ix5(b, i, kk, h, c, N, H, d)] = av;
                    dk[ix5(b, i, kk, h, c, N, H, d)] = scale * ak;
                }
            for (int j = 0; j < N; ++j)
                for (int c = 0; c < d; ++c) {
                    double aq = 0.0;
                    for (int kk = 0; kk < N; ++kk)
                        aq += ds[(size_t)j * N + kk] * k[ix5(b, i, kk, h, c, N, H, d)];
                    dq[ix5(b, i, j, h, c, N, H, d)] = scale * aq;
                }
            free(P);
            free(ds);
        }
    }
    return err;
}

/*
 * dbias[b,h,j,:] for a list of (b,h,j) triples (sel[3r..3r+2]); nsel < 0
 * means every (b,h,j).  Each entry is the sum over all rows i (ascending) of
 * ds[b,i,j,h,:], recomputed from the definition for that query row only.
 */
int tri_attn_oracle_dbias(int B, int N, int H, int d, double scale,
                          const double *q, const double *k, const double *v,
                          const double *bias, const double *mask,
                          const double *dout, const int *sel, int nsel,
                          double *dbias, int planted)
{
    if (B <= 0 || N <= 0 || H <= 0 || d <= 0 || !q || !k || !v || !bias || !dout || !dbias)
        return ORC_ERR_ARGS;
    int st = check_rows_have_keys(B, N, mask);
    if (st) return st;
    int total = (nsel < 0) ? B * H * N : nsel;
    int err = 0;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < total; ++r) {
        int b, h, j;
        if (nsel < 0) { b = r / (H * N); h = (r / N) % H; j = r % N; }
        else { b = sel[3 * r]; h = sel[3 * r + 1]; j = sel[3 * r + 2]; }
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        double *acc = (double *)calloc((size_t)N, sizeof(double));
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
        if (!s || !p || !acc || !o) {
            free(s); free(p); free(acc); free(o);
            #pragma omp atomic write
            err = ORC_ERR_NOMEM;
            continue;
        }
        if (planted == 6) {
            /* wrong axis: sum over queries j of row i = j instead of over rows i */
            for (int jj = 0; jj < N; ++jj) {
                scores(B, N, H, d, scale, q, k, bias, mask, b, j, h, jj, s, 0);
                softmax_row(N, s, p);
                for (int c = 0; c < d; ++c) {
                    double a = 0.0;
                    for (int kk = 0; kk < N; ++kk) a += p[kk] * v[ix5(b, j, kk, h, c, N, H, d)];
                    o[c] = a;
                }
                double Dj = 0.0;
                for (int c = 0; c < d; ++c) Dj += dout[ix5(b, j, jj, h, c, N, H, d)] * o[c];
                for (int kk = 0; kk < N; ++kk) {
                    double dp = 0.0;
                    for (int c = 0; c < d; ++c)
                        dp += dout[ix5(b, j, jj, h, c, N, H, d)] * v[ix5(b, j, kk, h, c, N, H, d)];
                    acc[kk] += p[kk] * (dp - Dj);
                }
            }
        } else {
            for (int i = 0; i < N; ++i) {
                scores(B, N, H, d, scale, q, k, bias, mask, b, i, h, j, s, planted);
                softmax_row(N, s, p);
                for (int c = 0; c < d; ++c) {
                    double a = 0.0;
                    for (int kk = 0; kk < N; ++kk) a += p[kk] * v[ix5(b, i, kk, h, c, N, H, d)];
                    o[c] = a;
                }
                double Dj = 0.0;
                for (int c = 0; c < d; ++c)
                    Dj += ((planted == 4) ? 1.0 : dout[ix5(b, i, j, h, c, N, H, d)]) * o[c];
                for (int kk = 0; kk < N; ++kk) {
                    double dp = 0.0;
                    for (int c = 0; c < d; ++c)
                        dp += dout[ix5(b, i, j, h, c, N, H, d)] * v[ix5(b, i, kk, h, c, N, H, d)];
                    double ds = (planted == 5) ? p[kk] * (Dj - dp) : p[kk] * (dp - Dj);
                    acc[kk] += ds;
                }
            }
        }
        for (int kk = 0; kk < N; ++kk) dbias[ix_bias(b, h, j, kk, N, H)] = acc[kk];
        free(s); free(p); free(acc); free(o);
    }
    return err;
}

/*
 * One pair row (b,i) on its own, for crops too large to hold the whole pair
 * stack in FP64 on the host.  Row i of the starting-node definition reads only
 * that row's q, k, v, dout ([N,H,d] each), the batch's bias ([H,N,N]) and the
 * row's mask ([N], or NULL); it is the full definition above with B = 1 and
 * the row at i = 0, and runs the very same code (problem_probs, problem_ds, the
 * dq/dk/dv loops), so its results equal the whole-stack functions' row bit for
 * bit.  Writes out_row, dq_row, dk_row, dv_row ([N,H,d]) and lse_row ([H,N]);
 * dout_row and the gradient outputs may be NULL to run the forward only.
 */
int tri_attn_oracle_row(int N, int H, int d, double scale,
                        const double *q, const double *k, const double *v,
                        const double *bias, const double *mask_row, const double *dout,
                        double *out, double *lse_row, double *dq, double *dk, double *dv)
{
    if (N <= 0 || H <= 0 || d <= 0 || !q || !k || !v || !bias || !out || !lse_row)
        return ORC_ERR_ARGS;
    if (mask_row) {
        int any = 0;
        for (int kk = 0; kk < N; ++kk)
            if (mask_row[kk] > ORC_MASKED_AT) { any = 1; break; }
        if (!any) return ORC_ERR_FULLY_MASKED;
    }
    const int grads = dout && dq && dk && dv;
    int err = 0;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        double *P = problem_probs(1, N, H, d, scale, q, k, bias, mask_row, 0, 0, h, lse_row + (size_t)h * N, 0);
        double *ds = grads ? (double *)malloc(sizeof(double) * (size_t)N * N) : NULL;
        if (!P || (grads && !ds)) {
            free(P); free(ds);
            #pragma omp atomic write
            err = ORC_ERR_NOMEM;
            continue;
        }
        for (int j = 0; j < N; ++j)
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int kk = 0; kk < N; ++kk)
                    acc += P[(size_t)j * N + kk] * v[ix5(0, 0, kk, h, c, N, H, d)];
                out[ix5(0, 0, j, h, c, N, H, d)] = acc;
            }
        if (grads) {
            problem_ds(N, H, d, P, v, dout, 0, 0, h, ds, 0);
            for (int kk = 0; kk < N; ++kk)
                for (int c = 0; c < d; ++c) {
                    double av = 0.0, ak = 0.0;
                    for (int j = 0; j < N; ++j) {
                        av += P[(size_t)j * N + kk] * dout[ix5(0, 0, j, h, c, N, H, d)];
                        ak += ds[(size_t)j * N + kk] * q[ix5(0, 0, j, h, c, N, H, d)];
                    }
                    dv[ix5(0, 0, kk, h, c, N, H, d)] = av;
                    dk[ix5(0, 0, kk, h, c, N, H, d)] = scale * ak;
                }
            for (int j = 0; j < N; ++j)
                for (int c = 0; c < d; ++c) {
                    double aq = 0.0;
                    for (int kk = 0; kk < N; ++kk)
                        aq += ds[(size_t)j * N + kk] * k[ix5(0, 0, kk, h, c, N, H, d)];
                    dq[ix5(0, 0, j, h, c, N, H, d)] = scale * aq;
                }
        }
        free(P);
        free(ds);
    }
    return err;
}

/*
 * dbias accumulation one pair row at a time: adds row i's ds[b,i,j,h,:] for
 * one (h, j) to acc[N].  Called for i = 0, 1, ..., N-1 in turn, it performs the
 * same FP64 operations in the same order as tri_attn_oracle_dbias does for
 * that (b,h,j), so the two agree bit for bit.  Inputs are one row's q, k, v,
 * dout ([N,H,d]), the batch's bias ([H,N,N]) and the row's mask ([N] or NULL).
 */
int tri_attn_oracle_dbias_row_add(int N, int H, int d, double scale,
                                  const double *q, const double *k, const double *v,
                                  const double *bias, const double *mask_row, const double *dout,
                                  int h, int j, double *acc)
{
    if (N <= 0 || H <= 0 || d <= 0 || h < 0 || h >= H || j < 0 || j >= N || !q || !k || !v || !bias ||
        !dout || !acc)
        return ORC_ERR_ARGS;
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    if (!s || !p || !o) { free(s); free(p); free(o); return ORC_ERR_NOMEM; }
    scores(1, N, H, d, scale, q, k, bias, mask_row, 0, 0, h, j, s, 0);
    softmax_row(N, s, p);
    for (int c = 0; c < d; ++c) {
        double a = 0.0;
        for (int kk = 0; kk < N; ++kk) a += p[kk] * v[ix5(0, 0, kk, h, c, N, H, d)];
        o[c] = a;
    }
    double Dj = 0.0;
    for (int c = 0; c < d; ++c) Dj += dout[ix5(0, 0, j, h, c, N, H, d)] * o[c];
    for (int kk = 0; kk < N; ++kk) {
        double dp = 0.0;
        for (int c = 0; c < d; ++c)
            dp += dout[ix5(0, 0, j, h, c, N, H, d)] * v[ix5(0, 0, kk, h, c, N, H, d)];
        acc[kk] += p[kk] * (dp - Dj);
    }
    free(s); free(p); free(o);
    return ORC_OK;
}

/*
 * Row i's share of dbias for every (h, j): adds ds[b,i,j,h,:] into acc
 * ([H][N][N], the batch's dbias accumulator), with the operations of
 * tri_attn_oracle_dbias_row_add.  Called for i = 0, 1, ..., N-1 in turn it
 * reproduces tri_attn_oracle_dbias for the batch bit for bit; called for a
 * subset of rows it is that subset's part of the sum (what a row-sampled
 * timing of the whole backward has to include).
 */
int tri_attn_oracle_dbias_row_add_all(int N, int H, int d, double scale,
                                      const double *q, const double *k, const double *v,
                                      const double *bias, const double *mask_row, const double *dout,
                                      double *acc)
{
    if (N <= 0 || H <= 0 || d <= 0 || !acc) return ORC_ERR_ARGS;
    int err = 0;
    #pragma omp parallel for schedule(dynamic, 8) collapse(2)
    for (int h = 0; h < H; ++h)
        for (int j = 0; j < N; ++j) {
            int st = tri_attn_oracle_dbias_row_add(N, H, d, scale, q, k, v, bias, mask_row, dout, h, j,
                                                   acc + ((size_t)h * N + j) * (size_t)N);
            if (st) {
                #pragma omp atomic write
                err = st;
            }
        }
    return err;
}
