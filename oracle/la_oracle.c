/*
 * la_oracle.c -- CPU fp64 oracle for gated linear attention (TEST INFRASTRUCTURE ONLY).
 *
 * This file is the checker, not the product.  Only tests/, __graft_entry__.smoke() and
 * bench.py's cpu_baseline / reference legs may load it.  It shares no code, header, table
 * or helper with the CUDA path.
 *
 * What it computes is the plain definition of gated linear attention (GLA), token by
 * token, in double precision, with no chunking and no segmentation:
 *
 *   S_{-1} = S0 (or 0)                                  state, d_k x d_v
 *   S_t    = diag(exp(log_g_t)) . S_{t-1} + k_t^T v_t   gated state update
 *   o_t    = q_t . S_t                                  inclusive read-out
 *   S_final = S_{L-1}
 *
 * Sources (the ZeCO pages):
 *  - ZeCO review, "key machinery": the state S in R^{dk x dv} is updated with a per-key-dim
 *    cumulative decay broadcast over d_v, written (gamma^T 1) (.) S; the same field states
 *    the linear-decomposition identity (global state = decay . incoming + local residual).
 *  - ZeCO review, "core discovery": the GLA recurrence updates a fixed dk x dv state, and
 *    ZeCO reproduces the single-device result exactly.
 *  - ZeCO review, supporting citations (Yang et al. 2024, GLA): the chunkwise recurrence
 *    being parallelised; its token-level form is the recurrence above.
 *  The pages do not say whether o_t reads S_t or S_{t-1}.  The inclusive form (token t
 *  enters the state before its own read-out) is the reading taken here and everywhere.
 *
 * The backward pass is the exact reverse-mode derivative of the recurrence above (ZeCO
 * review, "forward implications": the backward reuses the forward's global state).  With
 * dS_t the gradient of the loss with respect to S_t (accumulated from o_t and S_{t+1}):
 *
 *   dS_{L-1} = dS_final + q_{L-1}^T dO_{L-1};   dS_t = diag(a_{t+1}) dS_{t+1} + q_t^T dO_t
 *   dq_t = dO_t S_t^T          dk_t = (dS_t v_t^T)^T        dv_t = k_t dS_t
 *   dlog_g_t[i] = a_t[i] * sum_j S_{t-1}[i][j] dS_t[i][j]   dS0 = diag(a_0) dS_0
 *
 * The forward states needed by the reverse sweep are recomputed block by block from
 * checkpoints stored every LA_ORACLE_CKPT tokens.
 *
 * Layout: every sequence tensor is [B, H, L, d] row-major (d fastest); states are
 * [B, H, d_k, d_v] row-major.  Parallel over the B*H independent (b, h) pairs with OpenMP.
 */
#include <math.h>
#include <omp.h>
#include <stdlib.h>
#include <string.h>

#define LA_ORACLE_CKPT 64

/* Forward for one (b, h) pair.  S_seg (nullable): for p = 0 .. L/seg_len - 1, the state
 * entering token p*seg_len, i.e. S_{p*seg_len - 1} (S0 for p = 0). */
static void forward_one(const double *q, const double *k, const double *v, const double *g,
                        const double *S0, long L, long dk, long dv, long seg_len,
                        double *o, double *S_final, double *S_seg, double *S, double *a)
{
    if (S0) memcpy(S, S0, sizeof(double) * dk * dv);
    else memset(S, 0, sizeof(double) * dk * dv);
    for (long t = 0; t < L; ++t) {
        if (S_seg && seg_len > 0 && t % seg_len == 0)
            memcpy(S_seg + (t / seg_len) * dk * dv, S, sizeof(double) * dk * dv);
        const double *qt = q + t * dk, *kt = k + t * dk, *vt = v + t * dv, *gt = g + t * dk;
        for (long i = 0; i < dk; ++i) a[i] = exp(gt[i]);
        for (long i = 0; i < dk; ++i) {
            double *Si = S + i * dv;
            for (long j = 0; j < dv; ++j) Si[j] = a[i] * Si[j] + kt[i] * vt[j];
        }
        double *ot = o + t * dv;
        for (long j = 0; j < dv; ++j) ot[j] = 0.0;
        for (long i = 0; i < dk; ++i) {
            const double *Si = S + i * dv;
            for (long j = 0; j < dv; ++j) ot[j] += qt[i] * Si[j];
        }
    }
    if (S_final) memcpy(S_final, S, sizeof(double) * dk * dv);
}

void la_oracle_forward(const double *q, const double *k, const double *v, const double *log_g,
                       const double *S0, long B, long H, long L, long dk, long dv, long seg_len,
                       double *o, double *S_final, double *S_seg)
{
    const long BH = B * H;
    const long nseg = (S_seg && seg_len > 0) ? L / seg_len : 0;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * dk * dv);
        double *a = (double *)malloc(sizeof(double) * dk);
#pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < BH; ++bh) {
            forward_one(q + bh * L * dk, k + bh * L * dk, v + bh * L * dv, log_g + bh * L * dk,
                        S0 ? S0 + bh * dk * dv : NULL, L, dk, dv, seg_len, o + bh * L * dv,
                        S_final ? S_final + bh * dk * dv : NULL,
                        nseg ? S_seg + bh * nseg * dk * dv : NULL, S, a);
        }
        free(S);
        free(a);
    }
}

/* Backward for one (b, h) pair.  ckpt holds one state per block of LA_ORACLE_CKPT tokens,
 * blk holds the LA_ORACLE_CKPT + 1 states of the block being reversed, dS one state. */
static void backward_one(const double *q, const double *k, const double *v, const double *g,
                         const double *S0, const double *dO, const double *dS_final, long L,
                         long dk, long dv, double *dq, double *dk_, double *dv_, double *dg,
                         double *dS0, double *ckpt, double *blk, double *dS, double *a)
{
    const long DD = dk * dv;
    const long nblk = (L + LA_ORACLE_CKPT - 1) / LA_ORACLE_CKPT;
    /* Pass 1: the forward recurrence, keeping S_{b*CKPT - 1} for every block b. */
    double *S = blk; /* scratch, overwritten below */
    if (S0) memcpy(S, S0, sizeof(double) * DD);
    else memset(S, 0, sizeof(double) * DD);
    for (long t = 0; t < L; ++t) {
        if (t % LA_ORACLE_CKPT == 0) memcpy(ckpt + (t / LA_ORACLE_CKPT) * DD, S, sizeof(double) * DD);
        for (long i = 0; i < dk; ++i) {
            const double ai = exp(g[t * dk + i]);
            for (long j = 0; j < dv; ++j) S[i * dv + j] = ai * S[i * dv + j] + k[t * dk + i] * v[t * dv + j];
        }
    }
    /* Pass 2: reverse sweep, block by block; blk[r] = S_{t0 + r - 1} (blk[0] = checkpoint). */
    if (dS_final) memcpy(dS, dS_final, sizeof(double) * DD);
    else memset(dS, 0, sizeof(double) * DD);
    for (long b = nblk - 1; b >= 0; --b) {
        const long t0 = b * LA_ORACLE_CKPT;
        const long t1 = (t0 + LA_ORACLE_CKPT < L) ? t0 + LA_ORACLE_CKPT : L;
        memcpy(blk, ckpt + b * DD, sizeof(double) * DD);
        for (long t = t0; t < t1; ++t) {
            const double *Sp = blk + (t - t0) * DD;
            double *Sn = blk + (t - t0 + 1) * DD;
            for (long i = 0; i < dk; ++i) {
                const double ai = exp(g[t * dk + i]);
                for (long j = 0; j < dv; ++j) Sn[i * dv + j] = ai * Sp[i * dv + j] + k[t * dk + i] * v[t * dv + j];
            }
        }
        for (long t = t1 - 1; t >= t0; --t) {
            const double *St = blk + (t - t0 + 1) * DD;  /* S_t     */
            const double *Sm = blk + (t - t0) * DD;      /* S_{t-1} */
            const double *qt = q + t * dk, *kt = k + t * dk, *vt = v + t * dv, *dOt = dO + t * dv;
            for (long i = 0; i < dk; ++i) a[i] = exp(g[t * dk + i]);
            /* dS_t = (carried) + q_t^T dO_t */
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) dS[i * dv + j] += qt[i] * dOt[j];
            /* dq_t = dO_t S_t^T */
            for (long i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (long j = 0; j < dv; ++j) acc += dOt[j] * St[i * dv + j];
                dq[t * dk + i] = acc;
            }
            /* dk_t[i] = sum_j dS_t[i][j] v_t[j] */
            for (long i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (long j = 0; j < dv; ++j) acc += dS[i * dv + j] * vt[j];
                dk_[t * dk + i] = acc;
            }
            /* dv_t[j] = sum_i k_t[i] dS_t[i][j] */
            for (long j = 0; j < dv; ++j) dv_[t * dv + j] = 0.0;
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) dv_[t * dv + j] += kt[i] * dS[i * dv + j];
            /* dlog_g_t[i] = a_t[i] sum_j S_{t-1}[i][j] dS_t[i][j] */
            for (long i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (long j = 0; j < dv; ++j) acc += Sm[i * dv + j] * dS[i * dv + j];
                dg[t * dk + i] = a[i] * acc;
            }
            /* carry to t-1: dS <- diag(a_t) dS_t */
            for (long i = 0; i < dk; ++i)
                for (long j = 0; j < dv; ++j) dS[i * dv + j] *= a[i];
        }
    }
    if (dS0) memcpy(dS0, dS, sizeof(double) * DD);
}

void la_oracle_backward(const double *q, const double *k, const double *v, const double *log_g,
                        const double *S0, const double *dO, const double *dS_final, long B, long H,
                        long L, long dk, long dv, double *dq, double *dk_, double *dv_, double *dg,
                        double *dS0)
{
    const long BH = B * H;
    const long DD = dk * dv;
    const long nblk = (L + LA_ORACLE_CKPT - 1) / LA_ORACLE_CKPT;
#pragma omp parallel
    {
        double *ckpt = (double *)malloc(sizeof(double) * (nblk + 1) * DD);
        double *blk = (double *)malloc(sizeof(double) * (LA_ORACLE_CKPT + 1) * DD);
        double *dS = (double *)malloc(sizeof(double) * DD);
        double *a = (double *)malloc(sizeof(double) * dk);
#pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < BH; ++bh) {
            backward_one(q + bh * L * dk, k + bh * L * dk, v + bh * L * dv, log_g + bh * L * dk,
                         S0 ? S0 + bh * DD : NULL, dO + bh * L * dv,
                         dS_final ? dS_final + bh * DD : NULL, L, dk, dv, dq + bh * L * dk,
                         dk_ + bh * L * dk, dv_ + bh * L * dv, dg + bh * L * dk,
                         dS0 ? dS0 + bh * DD : NULL, ckpt, blk, dS, a);
        }
        free(ckpt);
        free(blk);
        free(dS);
        free(a);
    }
}

/* Number of OpenMP threads the two entry points above will use. */
int la_oracle_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
    return n;
}
