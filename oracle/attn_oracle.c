/*
 * attn_oracle.c -- fp64 CPU oracle for exact attention, forward and backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this
 * file; only the test-suite, the smoke check and the benchmark's CPU-baseline leg do.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes.  FlashAttention returns exactly the result of standard attention
 * (anthology note "NOTE-005: FlashAttention", Key results, Theorem 1: the algorithm
 * returns O = softmax(QK^T)V; "FlashAttention: The IO-Aware Algorithm That Rewrote GPU
 * Training Speed Records", section "Tiling: keeping computation inside SRAM": the output
 * is mathematically identical to standard attention).  So this oracle is the plain
 * definition of standard attention, written out in fp64, with the score matrix
 * materialised (promptingindex page, "Why attention is memory-bound, not
 * compute-bound": the op chain is QK^T, scaling, masking, softmax, then the product
 * with V).  No tiling, no online softmax, no recomputation: one row panel of the
 * score matrix is held in full (the whole N x N matrix when the panel covers every
 * row), every step is the textbook formula.
 *
 * Per (batch, head), inputs Q, K, V, dO are N x d row-major fp64 arrays:
 *   S_ij  = scale * <q_i, k_j>
 *   allowed(i, j) = (j < L) && (!causal || j <= i)            (masked scores are -inf)
 *   m_i   = max over allowed j of S_ij
 *   P_ij  = exp(S_ij - m_i) / sum_allowed exp(S_ij' - m_i),  0 where not allowed
 *   O_i   = sum_j P_ij v_j
 *   LSE_i = m_i + ln sum_allowed exp(S_ij - m_i)               (natural log)
 * Backward of the scalar loss sum(O * dO) (the chain rule through the same chain;
 * the pages state only that P is recomputed in the backward pass, NOTE-005 "Method"):
 *   dV_j  = sum_i P_ij dO_i
 *   dP_ij = <dO_i, v_j>
 *   D_i   = sum_j P_ij dP_ij
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_i dS_ij q_i
 * A row with no allowed key has O = 0, LSE = -inf, zero gradients.
 *
 * Block-sparse attention (promptingindex page, "Benchmark results": the same tiling
 * applied to a sparse pattern; NOTE-005, "Key components": the block-sparse extension)
 * restricts the allowed set further: with a block mask M of (ceil(N/bs))^2 bytes,
 *   allowed(i, j) &= M[i / bs][j / bs] != 0,
 * and is otherwise the same computation.  With M all ones it is dense attention.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* Optional block mask (one per (batch, head) call): NULL means dense. */
typedef struct {
    const unsigned char *m;
    long bs; /* block size */
    long nb; /* blocks per side */
} block_mask_t;

static int is_allowed(long i, long j, int causal, long L, const block_mask_t *bm)
{
    if (!(j < L && (!causal || j <= i))) return 0;
    if (bm && bm->m) return bm->m[(i / bm->bs) * bm->nb + (j / bm->bs)] != 0;
    return 1;
}

/* Rows of the panel processed together.  The score panel holds at most this many
 * doubles per matrix (two matrices are live: P and dS). */
static long panel_rows(long N, long R)
{
    const long cap = 1L << 26; /* 512 MiB of fp64 per matrix */
    long p = cap / (N > 0 ? N : 1);
    if (p < 1) p = 1;
    if (p > R) p = R;
    return p;
}

int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Exact attention for the query rows rows[0..R) of one (batch, head).
 *
 * q, k, v, dout : N x d fp64, row-major.  dout may be NULL (forward only).
 * L             : number of valid keys (key padding), 0 <= L <= N.
 * o             : R x d out; lse : R out (natural log).
 * dq            : R x d out or NULL.
 * dk, dv        : N x d, ACCUMULATED (+=) with the contributions of the given rows, or
 *                 NULL.  Over rows = 0..N-1 they are the full gradients.
 */
int oracle_attention_rows_masked(const double *q, const double *k, const double *v,
                                 const double *dout, long N, long d, double scale, int causal,
                                 long L, const unsigned char *block_mask, long block_size,
                                 const long *rows, long R, double *o, double *lse, double *dq,
                                 double *dk, double *dv)
{
    block_mask_t bmv;
    const block_mask_t *bm = NULL;
    if (block_mask) {
        if (block_size < 1) return ORACLE_ERR_ARG;
        bmv.m = block_mask;
        bmv.bs = block_size;
        bmv.nb = (N + block_size - 1) / block_size;
        bm = &bmv;
    }
    if (!q || !k || !v || !rows || !o || !lse || N < 1 || d < 1 || R < 0 || L < 0 || L > N)
        return ORACLE_ERR_ARG;
    if ((dq || dk || dv) && !dout) return ORACLE_ERR_ARG;
    for (long r = 0; r < R; ++r)
        if (rows[r] < 0 || rows[r] >= N) return ORACLE_ERR_ARG;
    if (R == 0) return ORACLE_OK;

    const long PR = panel_rows(N, R);
    double *P = (double *)malloc(sizeof(double) * PR * N);
    double *dS = dout ? (double *)malloc(sizeof(double) * PR * N) : NULL;
    if (!P || (dout && !dS)) {
        free(P);
        free(dS);
        return ORACLE_ERR_NOMEM;
    }

    for (long p0 = 0; p0 < R; p0 += PR) {
        const long pr = (R - p0 < PR) ? (R - p0) : PR;

#pragma omp parallel for schedule(dynamic, 1)
        for (long r = 0; r < pr; ++r) {
            const long i = rows[p0 + r];
            const double *qi = q + i * d;
            double *Srow = P + r * N;
            /* 1. scaled scores with the mask applied */
            double m = -INFINITY;
            for (long j = 0; j < N; ++j) {
                if (!is_allowed(i, j, causal, L, bm)) {
                    Srow[j] = -INFINITY;
                    continue;
                }
                const double *kj = k + j * d;
                double acc = 0.0;
                for (long c = 0; c < d; ++c) acc += qi[c] * kj[c];
                Srow[j] = scale * acc;
                if (Srow[j] > m) m = Srow[j];
            }
            double *oi = o + (p0 + r) * d;
            for (long c = 0; c < d; ++c) oi[c] = 0.0;
            if (m == -INFINITY) { /* no allowed key */
                lse[p0 + r] = -INFINITY;
                for (long j = 0; j < N; ++j) Srow[j] = 0.0;
                if (dout) {
                    for (long j = 0; j < N; ++j) dS[r * N + j] = 0.0;
                    if (dq)
                        for (long c = 0; c < d; ++c) dq[(p0 + r) * d + c] = 0.0;
                }
                continue;
            }
            /* 2. softmax: P = exp(S - m) / sum */
            double sum = 0.0;
            for (long j = 0; j < N; ++j) {
                double e = (Srow[j] == -INFINITY) ? 0.0 : exp(Srow[j] - m);
                Srow[j] = e;
                sum += e;
            }
            for (long j = 0; j < N; ++j) Srow[j] /= sum;
            lse[p0 + r] = m + log(sum);
            /* 3. O = P V */
            for (long j = 0; j < N; ++j) {
                const double pij = Srow[j];
                if (pij == 0.0) continue;
                const double *vj = v + j * d;
                for (long c = 0; c < d; ++c) oi[c] += pij * vj[c];
            }
            if (!dout) continue;
            /* 4. dP = dO V^T, D = rowsum(P * dP), dS = P * (dP - D), dQ = scale dS K */
            const double *doi = dout + i * d;
            double *dSrow = dS + r * N;
            double D = 0.0;
            for (long j = 0; j < N; ++j) {
                if (!is_allowed(i, j, causal, L, bm)) {
                    dSrow[j] = 0.0;
                    continue;
                }
                const double *vj = v + j * d;
                double acc = 0.0;
                for (long c = 0; c < d; ++c) acc += doi[c] * vj[c];
                dSrow[j] = acc; /* dP_ij for now */
                D += Srow[j] * acc;
            }
            for (long j = 0; j < N; ++j) dSrow[j] = Srow[j] * (dSrow[j] - D);
            if (dq) {
                double *dqi = dq + (p0 + r) * d;
                for (long c = 0; c < d; ++c) dqi[c] = 0.0;
                for (long j = 0; j < N; ++j) {
                    const double s = dSrow[j];
                    if (s == 0.0) continue;
                    const double *kj = k + j * d;
                    for (long c = 0; c < d; ++c) dqi[c] += s * kj[c];
                }
                for (long c = 0; c < d; ++c) dqi[c] *= scale;
            }
        }

        /* 5. dV += P^T dO and dK += scale dS^T Q over the rows of this panel */
        if (dout && (dk || dv)) {
#pragma omp parallel for schedule(static)
            for (long j = 0; j < N; ++j) {
                for (long r = 0; r < pr; ++r) {
                    const long i = rows[p0 + r];
                    if (dv) {
                        const double pij = P[r * N + j];
                        if (pij != 0.0) {
                            const double *doi = dout + i * d;
                            for (long c = 0; c < d; ++c) dv[j * d + c] += pij * doi[c];
                        }
                    }
                    if (dk) {
                        const double s = dS[r * N + j];
                        if (s != 0.0) {
                            const double *qi = q + i * d;
                            for (long c = 0; c < d; ++c) dk[j * d + c] += scale * s * qi[c];
                        }
                    }
                }
            }
        }
    }
    free(P);
    free(dS);
    return ORACLE_OK;
}

/* Dense entry point: oracle_attention_rows_masked without a block mask. */
int oracle_attention_rows(const double *q, const double *k, const double *v,
                          const double *dout, long N, long d, double scale, int causal,
                          long L, const long *rows, long R, double *o, double *lse,
                          double *dq, double *dk, double *dv)
{
    return oracle_attention_rows_masked(q, k, v, dout, N, d, scale, causal, L, NULL, 0, rows,
                                        R, o, lse, dq, dk, dv);
}
