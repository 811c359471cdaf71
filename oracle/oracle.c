/*
 * Float64 CPU oracle for linear attention with the feature map phi(x) = elu(x) + 1.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this
 * file: only the tests, the smoke check and the CPU-baseline leg of the benchmark use it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (page "Efficient Transformers: Linear Attention and Flash Attention",
 * section "Linear attention: reordering the matmuls, not shrinking them", the
 * kernelised attention formula):
 *
 *     out_i = phi(q_i) . sum_j phi(k_j) v_j^T  /  phi(q_i) . sum_j phi(k_j)
 *
 * non-causal: j runs over all tokens; causal: j <= i, the diagonal included, as in the
 * same page's section "The recurrent view: attention as an RNN", where the state after
 * token t already holds token t and the output at t reads that state:
 *
 *     S_t = S_{t-1} + phi(k_t) v_t^T,   z_t = z_{t-1} + phi(k_t),
 *     out_t = phi(q_t) S_t / phi(q_t) . z_t.
 *
 * The oracle follows those two statements literally: the non-causal mode forms S and z
 * over all tokens in token order, then reads every row out; the causal mode runs the
 * token recurrence, one token at a time.  No chunking, no blocking, no reordering.
 *
 * Readings where the pages are silent:
 *   - elu has alpha = 1 (the page writes elu(x)+1 with no parameter);
 *   - no 1/sqrt(d) scale inside the method (the formula has none; inputs may be
 *     pre-scaled by the caller);
 *   - no epsilon in the denominator (phi > 0 keeps it positive, page's answer A4);
 *   - the feature dimension D equals d and the value dimension equals d.
 *
 * Layouts: q, k, v, out are row-major [B][H][n][d]; S is [..][D][d] with row r the
 * feature index and column c the value index; z is [..][D].
 *
 * PHI_IDENTITY selects phi(x) = x, which the page's worked example ("Worked example:
 * the reassociation trick, by hand") uses on non-negative inputs.  It exists only so
 * that example can pin this code; it is not part of the method.
 *
 * Compile-time ORACLE_PLANT=1..8 plants one deliberate mistake each.  Only the test
 * that shows the pins catch such mistakes builds those variants.
 *
 * The backward pass (gradients of a loss through the forward pass; the pages give no
 * formulas for it) is the chain rule through the forward's definition written as weights
 * w_ij = phi(q_i) . phi(k_j); see oracle_backward_f64.
 */
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_PLANT
#define ORACLE_PLANT 0
#endif

enum { PHI_ELU1 = 0, PHI_IDENTITY = 1 };

/* phi(x) = elu(x) + 1: x + 1 for x > 0 and exp(x) for x <= 0 (alpha = 1). */
double oracle_phi(double x, int phi_kind)
{
    if (phi_kind == PHI_IDENTITY) return x;
#if ORACLE_PLANT == 4
    return x > 0.0 ? x : exp(x); /* planted: dropped the +1 on the positive branch */
#else
    return x > 0.0 ? x + 1.0 : exp(x);
#endif
}

/* Rank-1 update of one head's state by one token: S += phi(k) v^T, z += phi(k).
 * k has dk entries (the feature dimension D), v has dv (the value dimension d); S is [dk][dv]. */
static void state_add_token(double *S, double *z, const double *k, const double *v,
                            int64_t dk, int64_t dv, int phi_kind)
{
    for (int64_t r = 0; r < dk; ++r) {
        double pk = oracle_phi(k[r], phi_kind);
        for (int64_t c = 0; c < dv; ++c) {
#if ORACLE_PLANT == 2
            S[c * dk + r] += pk * v[c]; /* planted: transposed state */
#else
            S[r * dv + c] += pk * v[c];
#endif
        }
        z[r] += pk;
    }
}

/* out = phi(q) S / (phi(q) . z) for one token and one head (q: dk entries, out: dv). */
static void readout_token(const double *S, const double *z, const double *q, double *out,
                          int64_t dk, int64_t dv, int phi_kind, double *pq_scratch)
{
    double den = 0.0;
    for (int64_t r = 0; r < dk; ++r) {
        pq_scratch[r] = oracle_phi(q[r], phi_kind);
#if ORACLE_PLANT != 3
        den += pq_scratch[r] * z[r];
#endif
    }
#if ORACLE_PLANT == 3
    den = 1.0; /* planted: normaliser dropped */
#endif
    for (int64_t c = 0; c < dv; ++c) {
        double num = 0.0;
        for (int64_t r = 0; r < dk; ++r) num += pq_scratch[r] * S[r * dv + c];
        out[c] = num / den;
    }
}

/* Forward pass over B*H independent heads; causal selects the token recurrence. */
void oracle_forward_f64(const double *q, const double *k, const double *v, double *out,
                        int64_t B, int64_t H, int64_t n, int64_t d, int causal,
                        int phi_kind)
{
    const int64_t heads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < heads; ++bh) {
        double *S = (double *)calloc((size_t)(d * d), sizeof(double));
        double *z = (double *)calloc((size_t)d, sizeof(double));
        double *pq = (double *)malloc((size_t)d * sizeof(double));
        const int64_t base = bh * n * d;
        if (!causal) {
            for (int64_t t = 0; t < n; ++t)
                state_add_token(S, z, k + base + t * d, v + base + t * d, d, d, phi_kind);
            for (int64_t t = 0; t < n; ++t)
                readout_token(S, z, q + base + t * d, out + base + t * d, d, d, phi_kind, pq);
        } else {
            for (int64_t t = 0; t < n; ++t) {
#if ORACLE_PLANT == 1
                /* planted: diagonal excluded (read before adding token t) */
                readout_token(S, z, q + base + t * d, out + base + t * d, d, d, phi_kind, pq);
                state_add_token(S, z, k + base + t * d, v + base + t * d, d, d, phi_kind);
#else
                state_add_token(S, z, k + base + t * d, v + base + t * d, d, d, phi_kind);
                readout_token(S, z, q + base + t * d, out + base + t * d, d, d, phi_kind, pq);
#endif
            }
        }
        free(S);
        free(z);
        free(pq);
    }
}

/* Forward pass on features of their own dimension: q, k [heads][n][dk] (taken through
 * phi_kind, normally the identity: caller-computed features such as FAVOR+), v and out
 * [heads][n][dv].  The same order as oracle_forward_f64: S = sum_j phi(k_j) v_j^T is dk x dv
 * and z = sum_j phi(k_j) has dk entries (page "Linear Attention > Memory Efficiency" writes
 * the state as D x d with D the feature dimension). */
void oracle_forward_dkv_f64(const double *q, const double *k, const double *v, double *out,
                            int64_t heads, int64_t n, int64_t dk, int64_t dv, int causal,
                            int phi_kind)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < heads; ++bh) {
        double *S = (double *)calloc((size_t)(dk * dv), sizeof(double));
        double *z = (double *)calloc((size_t)dk, sizeof(double));
        double *pq = (double *)malloc((size_t)dk * sizeof(double));
        const double *qh = q + bh * n * dk, *kh = k + bh * n * dk, *vh = v + bh * n * dv;
        double *oh = out + bh * n * dv;
        if (!causal) {
            for (int64_t t = 0; t < n; ++t)
                state_add_token(S, z, kh + t * dk, vh + t * dv, dk, dv, phi_kind);
            for (int64_t t = 0; t < n; ++t)
                readout_token(S, z, qh + t * dk, oh + t * dv, dk, dv, phi_kind, pq);
        } else {
            for (int64_t t = 0; t < n; ++t) {
                state_add_token(S, z, kh + t * dk, vh + t * dv, dk, dv, phi_kind);
                readout_token(S, z, qh + t * dk, oh + t * dv, dk, dv, phi_kind, pq);
            }
        }
        free(S);
        free(z);
        free(pq);
    }
}

/* Causal forward for selected rows only: runs the whole recurrence of each head but
 * writes only the rows listed in rows[0..nrows) (ascending) to out[bh][nrows][d].
 * Used for sampled checks at sizes where the full output would not fit in a test. */
void oracle_forward_rows_f64(const double *q, const double *k, const double *v, double *out,
                             int64_t heads, int64_t n, int64_t d, int causal,
                             const int64_t *rows, int64_t nrows, int phi_kind)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < heads; ++bh) {
        double *S = (double *)calloc((size_t)(d * d), sizeof(double));
        double *z = (double *)calloc((size_t)d, sizeof(double));
        double *pq = (double *)malloc((size_t)d * sizeof(double));
        const int64_t base = bh * n * d;
        if (!causal) {
            for (int64_t t = 0; t < n; ++t)
                state_add_token(S, z, k + base + t * d, v + base + t * d, d, d, phi_kind);
            for (int64_t s = 0; s < nrows; ++s)
                readout_token(S, z, q + base + rows[s] * d, out + (bh * nrows + s) * d, d, d,
                              phi_kind, pq);
        } else {
            int64_t s = 0;
            for (int64_t t = 0; t < n && s < nrows; ++t) {
                state_add_token(S, z, k + base + t * d, v + base + t * d, d, d, phi_kind);
                while (s < nrows && rows[s] == t) {
                    readout_token(S, z, q + base + t * d, out + (bh * nrows + s) * d, d, d,
                                  phi_kind, pq);
                    ++s;
                }
            }
        }
        free(S);
        free(z);
        free(pq);
    }
}

/* Final state of a causal pass: S = sum_j phi(k_j) v_j^T, z = sum_j phi(k_j), per head.
 * This is the state the recurrent view carries after the last token. */
void oracle_state_f64(const double *k, const double *v, double *S, double *z,
                      int64_t heads, int64_t n, int64_t d, int phi_kind)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < heads; ++bh) {
        double *Sh = S + bh * d * d;
        double *zh = z + bh * d;
        memset(Sh, 0, (size_t)(d * d) * sizeof(double));
        memset(zh, 0, (size_t)d * sizeof(double));
        for (int64_t t = 0; t < n; ++t)
            state_add_token(Sh, zh, k + (bh * n + t) * d, v + (bh * n + t) * d, d, d, phi_kind);
    }
}

/* One recurrent decode step for Bseq*H independent states, updated in place:
 * S += phi(k) v^T, z += phi(k), then out = phi(q) S / phi(q) . z with the updated state. */
void oracle_decode_step_f64(double *S, double *z, const double *q, const double *k,
                            const double *v, double *out, int64_t Bseq, int64_t H, int64_t d,
                            int phi_kind)
{
    const int64_t heads = Bseq * H;
#pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < heads; ++bh) {
        double *pq = (double *)malloc((size_t)d * sizeof(double));
#if ORACLE_PLANT == 5
        /* planted: output read from the state before the update */
        readout_token(S + bh * d * d, z + bh * d, q + bh * d, out + bh * d, d, d, phi_kind, pq);
        state_add_token(S + bh * d * d, z + bh * d, k + bh * d, v + bh * d, d, d, phi_kind);
#else
        state_add_token(S + bh * d * d, z + bh * d, k + bh * d, v + bh * d, d, d, phi_kind);
        readout_token(S + bh * d * d, z + bh * d, q + bh * d, out + bh * d, d, d, phi_kind, pq);
#endif
        free(pq);
    }
}

/* phi'(x): 1 above zero, exp(x) at or below zero (the derivative of elu + 1, alpha = 1;
 * both one-sided derivatives are 1 at zero). */
static double phi_deriv(double x, int phi_kind)
{
    if (phi_kind == PHI_IDENTITY) return 1.0;
#if ORACLE_PLANT == 7
    return 1.0; /* planted: the chain rule through phi dropped on the negative branch */
#else
    return x > 0.0 ? 1.0 : exp(x);
#endif
}

/*
 * Gradients of the loss L = sum_i g_i . out_i with respect to q, k and v, per head, for
 * the forward pass above (causal: j <= i; non-causal: all j).  The forward is written as
 *     w_ij = phi(q_i) . phi(k_j),   den_i = sum_j w_ij,   out_i = sum_j w_ij v_j / den_i,
 * and differentiated term by term:
 *     dL/dw_ij      = g_i . (v_j - out_i) / den_i
 *     dL/dv_j       = sum_i w_ij g_i / den_i
 *     dL/dphi(q_i)  = sum_j dL/dw_ij phi(k_j)
 *     dL/dphi(k_j)  = sum_i dL/dw_ij phi(q_i)
 *     dL/dq = dL/dphi(q) * phi'(q),   dL/dk = dL/dphi(k) * phi'(k).
 * Plain O(n^2 d) loops in float64; g, dq, dk, dv are [B][H][n][d] like q.
 */
void oracle_backward_f64(const double *q, const double *k, const double *v, const double *g,
                         double *dq, double *dk, double *dv, int64_t B, int64_t H, int64_t n,
                         int64_t d, int causal, int phi_kind)
{
    const int64_t heads = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < heads; ++bh) {
        const int64_t base = bh * n * d;
        double *pq = (double *)malloc((size_t)(n * d) * sizeof(double));
        double *pk = (double *)malloc((size_t)(n * d) * sizeof(double));
        double *den = (double *)malloc((size_t)n * sizeof(double));
        double *gout = (double *)malloc((size_t)n * sizeof(double)); /* g_i . out_i */
        double *out = (double *)malloc((size_t)d * sizeof(double));
        for (int64_t t = 0; t < n * d; ++t) {
            pq[t] = oracle_phi(q[base + t], phi_kind);
            pk[t] = oracle_phi(k[base + t], phi_kind);
        }
        /* forward quantities per query row */
        for (int64_t i = 0; i < n; ++i) {
            const int64_t jend = causal ? i + 1 : n;
            double s = 0.0;
            for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
            for (int64_t j = 0; j < jend; ++j) {
                double w = 0.0;
                for (int64_t r = 0; r < d; ++r) w += pq[i * d + r] * pk[j * d + r];
                s += w;
                for (int64_t c = 0; c < d; ++c) out[c] += w * v[base + j * d + c];
            }
            den[i] = s;
            double go = 0.0;
            for (int64_t c = 0; c < d; ++c) go += g[base + i * d + c] * out[c] / s;
            gout[i] = go;
        }
        for (int64_t t = 0; t < n * d; ++t) {
            dq[base + t] = 0.0;
            dk[base + t] = 0.0;
            dv[base + t] = 0.0;
        }
        /* every (i, j) pair of the sum: dL/dw_ij feeds phi(q_i) and phi(k_j); w_ij feeds v_j */
        for (int64_t i = 0; i < n; ++i) {
            const int64_t jend = causal ? i + 1 : n;
            for (int64_t j = 0; j < jend; ++j) {
                double w = 0.0, gv = 0.0;
                for (int64_t r = 0; r < d; ++r) w += pq[i * d + r] * pk[j * d + r];
                for (int64_t c = 0; c < d; ++c) gv += g[base + i * d + c] * v[base + j * d + c];
#if ORACLE_PLANT == 6
                const double dw = gv / den[i]; /* planted: the normaliser's term dropped */
#else
                const double dw = (gv - gout[i]) / den[i];
#endif
                for (int64_t r = 0; r < d; ++r) {
                    dq[base + i * d + r] += dw * pk[j * d + r];
                    dk[base + j * d + r] += dw * pq[i * d + r];
                }
                for (int64_t c = 0; c < d; ++c)
                    dv[base + j * d + c] += w * g[base + i * d + c] / den[i];
            }
        }
        for (int64_t t = 0; t < n * d; ++t) {
            dq[base + t] *= phi_deriv(q[base + t], phi_kind);
            dk[base + t] *= phi_deriv(k[base + t], phi_kind);
        }
        free(pq);
        free(pk);
        free(den);
        free(gout);
        free(out);
    }
}

/*
 * Positive random features of Performer's FAVOR+ (named on the page "Efficient Transformers:
 * Linear Attention and Flash Attention", section "Linear attention: reordering the matmuls,
 * not shrinking them", as random features whose dot products approximate the softmax
 * kernel exp(q . k); the page gives no formula, and this is the positive-feature form of
 * that method):
 *     phi(x)_i = exp(w_i . x - |x|^2 / 2) / sqrt(m),   i = 0 .. m-1,
 * for random rows w_i of W [m][d] (the caller draws them, typically N(0, I_d)), so that
 * E_w[phi(q) . phi(k)] = exp(q . k).  x: [rows][d]; out: [rows][m].
 */
void oracle_favor_features_f64(const double *x, const double *W, double *out, int64_t rows,
                               int64_t d, int64_t m)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < rows; ++t) {
        double sq = 0.0;
        for (int64_t r = 0; r < d; ++r) sq += x[t * d + r] * x[t * d + r];
        for (int64_t i = 0; i < m; ++i) {
            double dot = 0.0;
            for (int64_t r = 0; r < d; ++r) dot += W[i * d + r] * x[t * d + r];
#if ORACLE_PLANT == 8
            out[t * m + i] = exp(dot) / sqrt((double)m); /* planted: the -|x|^2/2 term dropped */
#else
            out[t * m + i] = exp(dot - 0.5 * sq) / sqrt((double)m);
#endif
        }
    }
}

int oracle_plant(void) { return ORACLE_PLANT; }

/* Threads the OpenMP loops above use from now on (timing only; results do not depend on it). */
void oracle_set_threads(int threads) {
#ifdef _OPENMP
  if (threads > 0) omp_set_num_threads(threads);
#else
  (void)threads;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
