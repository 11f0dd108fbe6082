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
 * Queries and keys may differ in number (the inference shape: a short block of Nq new
 * queries against Nk cached keys; stackzen.ai glossary entry "FlashAttention").  The
 * queries are then the last Nq positions of the key sequence, so the causal rule reads
 *   allowed(i, j) = (j < L) && (!causal || j <= i + Nk - Nq),
 * which is the rule above when Nq = Nk.
 *
 * Block-sparse attention (promptingindex page, "Benchmark results": the same tiling
 * applied to a sparse pattern; NOTE-005, "Key components": the block-sparse extension)
 * restricts the allowed set further: with a block mask M of (ceil(N/bs))^2 bytes,
 *   allowed(i, j) &= M[i / bs][j / bs] != 0,
 * and is otherwise the same computation.  With M all ones it is dense attention.
 *
 * Dropout (promptingindex page, "Why attention is memory-bound, not compute-bound": the
 * op chain is matmul, scale, mask, softmax, dropout, matmul) multiplies the normalised
 * probabilities by a random keep mask before the product with V:
 *   K_ij  = 1 if byte_ij >= t else 0,  r = 256 / (256 - t)   (drop probability t / 256)
 *   O_i   = sum_j P_ij K_ij r v_j,      LSE_i as without dropout
 * and the backward pass goes through the same chain:
 *   dV_j  = sum_i P_ij K_ij r dO_i
 *   dP_ij = K_ij r <dO_i, v_j>          (gradient with respect to P, before the mask)
 *   D_i   = sum_j P_ij dP_ij,  dS_ij = P_ij (dP_ij - D_i),  dQ, dK as above.
 * byte_ij is a counter-based random byte, so the backward pass regenerates the mask
 * instead of storing it: byte (j mod 16) of the 16 output bytes of Philox4x32-10
 * (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011)
 * with counter (floor(j / 16), i, bh, offset) and key (seed mod 2^32, seed / 2^32); byte
 * b of the output is bits 8 (b mod 4) .. 8 (b mod 4) + 7 of output word floor(b / 4).
 */
#include <math.h>
#include <stdint.h>
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

/* Optional dropout (NULL or threshold 0 means none). */
typedef struct {
    unsigned threshold; /* t in [0, 255]: a byte below t drops the element */
    unsigned long long seed;
    unsigned offset;
    unsigned bh; /* batch * heads + head of this call */
} oracle_dropout_t;

/* Philox4x32-10 as defined in the SC 2011 paper: ten rounds of the S-box
 *   (x0, x1, x2, x3) -> (hi(M1 x2) ^ x1 ^ k0, lo(M1 x2), hi(M0 x0) ^ x3 ^ k1, lo(M0 x0))
 * with M0 = 0xD2511F53, M1 = 0xCD9E8D57, the key bumped by the Weyl constants
 * (0x9E3779B9, 0xBB67AE85) between rounds. */
void oracle_philox4x32_10(const unsigned ctr[4], const unsigned key[2], unsigned out[4])
{
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        const uint64_t p0 = (uint64_t)0xD2511F53u * x0;
        const uint64_t p1 = (uint64_t)0xCD9E8D57u * x2;
        const uint32_t y0 = (uint32_t)(p1 >> 32) ^ x1 ^ k0;
        const uint32_t y1 = (uint32_t)p1;
        const uint32_t y2 = (uint32_t)(p0 >> 32) ^ x3 ^ k1;
        const uint32_t y3 = (uint32_t)p0;
        x0 = y0;
        x1 = y1;
        x2 = y2;
        x3 = y3;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    out[0] = x0;
    out[1] = x1;
    out[2] = x2;
    out[3] = x3;
}

/* The random byte of element (i, j) of head bh. */
unsigned oracle_dropout_byte(unsigned long long seed, unsigned offset, unsigned bh, long i, long j)
{
    const unsigned ctr[4] = {(unsigned)(j / 16), (unsigned)i, bh, offset};
    const unsigned key[2] = {(unsigned)(seed & 0xFFFFFFFFu), (unsigned)(seed >> 32)};
    unsigned out[4];
    oracle_philox4x32_10(ctr, key, out);
    const long b = j % 16;
    return (out[b / 4] >> (8 * (b % 4))) & 0xFFu;
}

/* Keep mask of query rows [0, Nq) against keys [0, Nk): keep[i * Nk + j] = 0 or 1. */
int oracle_dropout_keep(unsigned threshold, unsigned long long seed, unsigned offset, unsigned bh,
                        long Nq, long Nk, unsigned char *keep)
{
    if (!keep || Nq < 0 || Nk < 0 || threshold > 255) return 1;
    for (long i = 0; i < Nq; ++i)
        for (long j = 0; j < Nk; ++j)
            keep[i * Nk + j] = oracle_dropout_byte(seed, offset, bh, i, j) >= threshold;
    return 0;
}

static int is_allowed(long i, long j, int causal, long L, long off, const block_mask_t *bm)
{
    if (!(j < L && (!causal || j <= i + off))) return 0;
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

/* Sets the OpenMP thread count of later calls (for timing the oracle on fewer cores). */
void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Exact attention for the query rows rows[0..R) of one (batch, head).
 *
 * q, dout       : Nq x d fp64, row-major.  dout may be NULL (forward only).
 * k, v          : Nk x d fp64, row-major.
 * L             : number of valid keys (key padding), 0 <= L <= Nk.
 * o             : R x d out; lse : R out (natural log).
 * dq            : R x d out or NULL.
 * dk, dv        : Nk x d, ACCUMULATED (+=) with the contributions of the given rows, or
 *                 NULL.  Over rows = 0..Nq-1 they are the full gradients.
 * A block mask or dropout needs Nq = Nk.
 */
int oracle_attention_rows_qk(const double *q, const double *k, const double *v,
                             const double *dout, long Nq, long Nk, long d, double scale,
                             int causal, long L, const unsigned char *block_mask, long block_size,
                             const oracle_dropout_t *drop, const long *rows, long R, double *o,
                             double *lse, double *dq, double *dk, double *dv)
{
    const long N = Nk; /* keys per row of the score matrix */
    const long off = Nk - Nq;
    if (Nq < 1 || (Nq != Nk && (block_mask || (drop && drop->threshold > 0)))) return ORACLE_ERR_ARG;
    if (drop && drop->threshold > 255) return ORACLE_ERR_ARG;
    const int dropping = drop && drop->threshold > 0;
    const double keep_scale = dropping ? 256.0 / (256.0 - (double)drop->threshold) : 1.0;
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
        if (rows[r] < 0 || rows[r] >= Nq) return ORACLE_ERR_ARG;
    if (R == 0) return ORACLE_OK;

    const long PR = panel_rows(N, R);
    double *P = (double *)malloc(sizeof(double) * PR * N);
    double *dS = dout ? (double *)malloc(sizeof(double) * PR * N) : NULL;
    /* dropout factor K_ij r of every panel element (1 without dropout) */
    double *KR = dropping ? (double *)malloc(sizeof(double) * PR * N) : NULL;
    if (!P || (dout && !dS) || (dropping && !KR)) {
        free(P);
        free(dS);
        free(KR);
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
                if (!is_allowed(i, j, causal, L, off, bm)) {
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
                if (dropping)
                    for (long j = 0; j < N; ++j) KR[r * N + j] = 0.0;
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
            /* 3. dropout factors K_ij r */
            double *KRrow = dropping ? KR + r * N : NULL;
            if (dropping)
                for (long j = 0; j < N; ++j)
                    KRrow[j] = oracle_dropout_byte(drop->seed, drop->offset, drop->bh, i, j) >=
                                       drop->threshold
                                   ? keep_scale
                                   : 0.0;
            /* 4. O = (P o K r) V */
            for (long j = 0; j < N; ++j) {
                const double pij = dropping ? Srow[j] * KRrow[j] : Srow[j];
                if (pij == 0.0) continue;
                const double *vj = v + j * d;
                for (long c = 0; c < d; ++c) oi[c] += pij * vj[c];
            }
            if (!dout) continue;
            /* 5. dP = (dO V^T) o K r, D = rowsum(P * dP), dS = P * (dP - D), dQ = scale dS K */
            const double *doi = dout + i * d;
            double *dSrow = dS + r * N;
            double D = 0.0;
            for (long j = 0; j < N; ++j) {
                if (!is_allowed(i, j, causal, L, off, bm)) {
                    dSrow[j] = 0.0;
                    continue;
                }
                const double *vj = v + j * d;
                double acc = 0.0;
                for (long c = 0; c < d; ++c) acc += doi[c] * vj[c];
                if (dropping) acc *= KRrow[j];
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

        /* 6. dV += (P o K r)^T dO and dK += scale dS^T Q over the rows of this panel */
        if (dout && (dk || dv)) {
#pragma omp parallel for schedule(static)
            for (long j = 0; j < N; ++j) {
                for (long r = 0; r < pr; ++r) {
                    const long i = rows[p0 + r];
                    if (dv) {
                        const double pij = dropping ? P[r * N + j] * KR[r * N + j] : P[r * N + j];
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
    free(KR);
    return ORACLE_OK;
}

/* Nq = Nk = N. */
int oracle_attention_rows_ex(const double *q, const double *k, const double *v,
                             const double *dout, long N, long d, double scale, int causal, long L,
                             const unsigned char *block_mask, long block_size,
                             const oracle_dropout_t *drop, const long *rows, long R, double *o,
                             double *lse, double *dq, double *dk, double *dv)
{
    return oracle_attention_rows_qk(q, k, v, dout, N, N, d, scale, causal, L, block_mask,
                                    block_size, drop, rows, R, o, lse, dq, dk, dv);
}

/* oracle_attention_rows_ex without dropout. */
int oracle_attention_rows_masked(const double *q, const double *k, const double *v,
                                 const double *dout, long N, long d, double scale, int causal,
                                 long L, const unsigned char *block_mask, long block_size,
                                 const long *rows, long R, double *o, double *lse, double *dq,
                                 double *dk, double *dv)
{
    return oracle_attention_rows_ex(q, k, v, dout, N, d, scale, causal, L, block_mask, block_size,
                                    NULL, rows, R, o, lse, dq, dk, dv);
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
