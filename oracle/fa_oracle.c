/*
 * fa_oracle.c -- float64 CPU oracle for exact scaled dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or helper with the CUDA
 * library; the two meet only at the seeded input arrays the tests hand to both.
 *
 * What it computes (plain definition, no tiling, no fusion, no reordering):
 *
 *   S = scale * Q K^T + mask                       "Attention is where tokens meet",
 *                                                  FlashAttention case-study slides
 *                                                  (nmj0.github.io), the SDPA formula
 *   m_i = max_j S_ij,  l_i = sum_j exp(S_ij - m_i),
 *   P_ij = exp(S_ij - m_i) / l_i                   same slides, "Problem: softmax needs
 *                                                  the whole row" (safe softmax)
 *   O_i = sum_j P_ij V_j,   LSE_i = m_i + ln l_i   same slides, "Online softmax: divide
 *                                                  once, at the end" (o_i / l_i form)
 *
 * Every row of S and P is materialised in full (the two-pass safe softmax), which
 * is exactly what the fused method avoids; here it is the point: the result is
 * the definition written out.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - mask = causal (bottom-right aligned: key j visible to query i iff
 *     j <= i + (Nk - Nq)) and/or an additive per-key bias [B, Nk] and/or a
 *     general additive mask M [B or 1, H or 1, Nq, Nk] (the "+ mask" of the
 *     SDPA formula in full), both added after scaling; -inf entries give
 *     probability 0;
 *   - a row with no visible key has O = 0 and LSE = -inf;
 *   - LSE is the natural log of sum_j exp(S_ij) over visible keys.
 *
 * Backward (the pages only say that scores are recomputed rather than stored;
 * the gradients below follow from differentiating the definition above with
 * loss L = sum(O * dO)):
 *   dV = P^T dO,  dP = dO V^T,  dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik),
 *   dQ = scale dS K,  dK = scale dS^T Q.  The mask/bias gets no gradient.
 *
 * Inputs are float64 arrays in [B, H, N, D] layout (D fastest); the caller
 * upcasts the same 16-bit-rounded values the GPU receives.  Work is split over
 * (b, h) pairs with OpenMP; nothing else is parallel or blocked.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

static int key_visible(long i, long j, long Nq, long Nk, int causal)
{
    if (!causal) return 1;
    return j <= i + (Nk - Nq);
}

/* The softmax row P_i of one query row (safe softmax over the materialised
 * S row).  Writes P_ij (normalised) into p_row[0..Nk) and returns LSE_i;
 * a row with no visible key gets P = 0 and LSE = -inf. */
static double softmax_row(const double *qi, const double *kh,
                          const double *bias_b, const double *mask_bh, long i,
                          long Nq, long Nk, long D, int causal, double scale,
                          double *p_row)
{
    double m = -INFINITY;
    for (long j = 0; j < Nk; ++j) {
        double s;
        if (!key_visible(i, j, Nq, Nk, causal)) {
            s = -INFINITY;
        } else {
            double dot = 0.0;
            for (long d = 0; d < D; ++d) dot += qi[d] * kh[j * D + d];
            s = scale * dot;
            if (bias_b) s += bias_b[j];
            if (mask_bh) s += mask_bh[i * Nk + j];
        }
        p_row[j] = s;
        if (s > m) m = s;
    }
    if (m == -INFINITY) {
        for (long j = 0; j < Nk; ++j) p_row[j] = 0.0;
        return -INFINITY;
    }
    double l = 0.0;
    for (long j = 0; j < Nk; ++j) {
        double e = (p_row[j] == -INFINITY) ? 0.0 : exp(p_row[j] - m);
        p_row[j] = e;
        l += e;
    }
    for (long j = 0; j < Nk; ++j) p_row[j] /= l;
    return m + log(l);
}

/* One query row: O_i = sum_j P_ij V_j and LSE_i. */
static void attn_row(const double *qi, const double *kh, const double *vh,
                     const double *bias_b, const double *mask_bh, long i, long Nq,
                     long Nk, long D, int causal, double scale, double *p_row,
                     double *o_i, double *lse_i)
{
    *lse_i = softmax_row(qi, kh, bias_b, mask_bh, i, Nq, Nk, D, causal, scale, p_row);
    for (long d = 0; d < D; ++d) o_i[d] = 0.0;
    for (long j = 0; j < Nk; ++j) {
        if (p_row[j] == 0.0) continue;
        for (long d = 0; d < D; ++d) o_i[d] += p_row[j] * vh[j * D + d];
    }
}

/*
 * Forward with a general additive mask.  mask == NULL means none; otherwise
 * entry (b, h, i, j) is mask[b * mask_bstride + h * mask_hstride + i * Nk + j]
 * (strides in elements; 0 broadcasts over that axis).  rows == NULL computes
 * every query row; otherwise the nrows listed row indices (each in [0, Nq)) of
 * every (b, h).  Output o is [B, H, nrows_eff, D] and lse [B, H, nrows_eff] in
 * float64.
 */
void oracle_fwd_mask(const double *q, const double *k, const double *v,
                     const double *key_bias, const double *mask, long mask_bstride,
                     long mask_hstride, int B, int H, int Nq, int Nk, int D,
                     int causal, double scale, const int *rows, int nrows,
                     double *o, double *lse)
{
    long nr = rows ? nrows : Nq;
    long BH = (long)B * H;
#pragma omp parallel
    {
        double *s_row = (double *)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
#pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < BH; ++bh) {
            long b = bh / H;
            const double *qh = q + bh * (long)Nq * D;
            const double *kh = k + bh * (long)Nk * D;
            const double *vh = v + bh * (long)Nk * D;
            const double *bias_b = key_bias ? key_bias + b * (long)Nk : NULL;
            const double *mask_bh = mask ? mask + b * mask_bstride + (bh % H) * mask_hstride : NULL;
            for (long r = 0; r < nr; ++r) {
                long i = rows ? rows[r] : r;
                attn_row(qh + i * D, kh, vh, bias_b, mask_bh, i, Nq, Nk, D, causal,
                         scale, s_row, o + (bh * nr + r) * D, lse + bh * nr + r);
            }
        }
        free(s_row);
    }
}

/* Forward without a general mask (causal and per-key bias only). */
void oracle_fwd(const double *q, const double *k, const double *v,
                const double *key_bias, int B, int H, int Nq, int Nk, int D,
                int causal, double scale, const int *rows, int nrows,
                double *o, double *lse)
{
    oracle_fwd_mask(q, k, v, key_bias, NULL, 0, 0, B, H, Nq, Nk, D, causal, scale,
                    rows, nrows, o, lse);
}

/*
 * Backward for a list of (b, h) pairs (bh_list[t] = b * H + h), full gradients,
 * with the general mask addressed as in oracle_fwd_mask (NULL = none).
 * Outputs dq [n_bh, Nq, D], dk and dv [n_bh, Nk, D] in float64.
 * Row by row: materialise P_i and dP_i, form dS_i, accumulate the three
 * gradients.  No stored O or LSE is used: both are recomputed from scratch.
 * q_rows == NULL processes every query row; otherwise only the n_q_rows listed
 * rows contribute (their dQ rows are exact, dK and dV hold only their share):
 * a bounded sample of the same work, used for CPU timing.
 */
void oracle_bwd_mask(const double *q, const double *k, const double *v,
                     const double *key_bias, const double *mask, long mask_bstride,
                     long mask_hstride, const double *dO, int B, int H, int Nq,
                     int Nk, int D, int causal, double scale, const int *bh_list,
                     int n_bh, const int *q_rows, int n_q_rows, double *dq,
                     double *dk, double *dv)
{
    (void)B;
#pragma omp parallel
    {
        double *p = (double *)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
        double *dp = (double *)malloc(sizeof(double) * (Nk > 0 ? Nk : 1));
#pragma omp for schedule(dynamic, 1)
        for (long t = 0; t < n_bh; ++t) {
            long bh = bh_list[t];
            long b = bh / H;
            const double *qh = q + bh * (long)Nq * D;
            const double *kh = k + bh * (long)Nk * D;
            const double *vh = v + bh * (long)Nk * D;
            const double *doh = dO + bh * (long)Nq * D;
            const double *bias_b = key_bias ? key_bias + b * (long)Nk : NULL;
            const double *mask_bh = mask ? mask + b * mask_bstride + (bh % H) * mask_hstride : NULL;
            double *dqh = dq + t * (long)Nq * D;
            double *dkh = dk + t * (long)Nk * D;
            double *dvh = dv + t * (long)Nk * D;
            memset(dqh, 0, sizeof(double) * Nq * D);
            memset(dkh, 0, sizeof(double) * Nk * D);
            memset(dvh, 0, sizeof(double) * Nk * D);
            long n_rows = q_rows ? n_q_rows : Nq;
            for (long r = 0; r < n_rows; ++r) {
                long i = q_rows ? q_rows[r] : r;
                /* P_i: the softmax row, rebuilt from scratch */
                double lse = softmax_row(qh + i * D, kh, bias_b, mask_bh, i, Nq, Nk,
                                         D, causal, scale, p);
                if (lse == -INFINITY) continue;   /* no visible key: no gradient */
                /* dP_ij = dO_i . V_j ;  Di = sum_j P_ij dP_ij */
                double Di = 0.0;
                for (long j = 0; j < Nk; ++j) {
                    double acc = 0.0;
                    for (long d = 0; d < D; ++d) acc += doh[i * D + d] * vh[j * D + d];
                    dp[j] = acc;
                    Di += p[j] * acc;
                }
                for (long j = 0; j < Nk; ++j) {
                    if (p[j] == 0.0) continue;
                    double ds = p[j] * (dp[j] - Di);
                    for (long d = 0; d < D; ++d) {
                        dqh[i * D + d] += scale * ds * kh[j * D + d];
                        dkh[j * D + d] += scale * ds * qh[i * D + d];
                        dvh[j * D + d] += p[j] * doh[i * D + d];
                    }
                }
            }
        }
        free(p);
        free(dp);
    }
}

/* Backward without a general mask (causal and per-key bias only). */
void oracle_bwd(const double *q, const double *k, const double *v,
                const double *key_bias, const double *dO, int B, int H, int Nq,
                int Nk, int D, int causal, double scale, const int *bh_list,
                int n_bh, const int *q_rows, int n_q_rows, double *dq, double *dk,
                double *dv)
{
    oracle_bwd_mask(q, k, v, key_bias, NULL, 0, 0, dO, B, H, Nq, Nk, D, causal,
                    scale, bh_list, n_bh, q_rows, n_q_rows, dq, dk, dv);
}

/* Thread control for timing runs (OpenMP over (b, h) pairs). */
#ifdef _OPENMP
#include <omp.h>
void oracle_set_threads(int n) { if (n > 0) omp_set_num_threads(n); }
int oracle_max_threads(void) { return omp_get_max_threads(); }
#else
void oracle_set_threads(int n) { (void)n; }
int oracle_max_threads(void) { return 1; }
#endif
