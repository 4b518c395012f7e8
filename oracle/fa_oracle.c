/*
 * fa_oracle.c -- fp64 reference for the exact attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file: only the tests, the package smoke check and the CPU
 * baseline leg of the benchmark do.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * What it computes is the plain definition of attention that the pages
 * state as "standard attention" (Chapter 15 -- FlashAttention, section
 * "Standard vs Flash Attention", left column, steps 1-4):
 *
 *     S = scale * Q K^T          full rows of the score matrix, in fp64
 *     causal: s_ij = -inf for j > i
 *     P = softmax(S)             two passes over each row: max, then exp/sum
 *     O = P V
 *     lse_i = m_i + ln(sum_j exp(s_ij - m_i))     natural log
 *
 * The pages never write the scale, the causal mask or the log-sum-exp
 * output; those come from the workload definition and are applied in the
 * plainest way (scale multiplies Q K^T before softmax; the causal mask keeps
 * keys j <= i; lse is the natural log of the row's softmax denominator in
 * scaled units).  Exactness is what the method promises (Chapter 15 --
 * FlashAttention, "Key Takeaways: Online Softmax Enables It": exact results,
 * no approximation), so the oracle is the definition, not the tiled
 * algorithm.
 *
 * Memory: the score rows of one head are materialised in blocks of at most
 * ORACLE_ROW_BLOCK rows by N columns.  That bounds memory only; every row is
 * still the full, two-pass, non-online computation.
 *
 * Inputs are fp32 arrays holding the exact values the GPU reads (bf16 values
 * are exactly representable in fp32); every arithmetic step is in fp64.
 * Layout: q, k, v are contiguous [BH][N][d]; o is [BH][nrows][d] fp64 and
 * lse is [BH][nrows] fp64, one entry per requested row.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_ROW_BLOCK 64

int oracle_version(void) { return 1; }

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * One block of rows of one head.
 *   q_rows: the requested query rows (indices into [0, n)), count nr <= ORACLE_ROW_BLOCK
 *   s:      scratch of nr * n doubles (the materialised score rows)
 */
static void attention_row_block(const float* q, const float* k, const float* v,
                                int64_t n, int64_t d, double scale, int causal,
                                const int64_t* q_rows, int64_t nr, double* s,
                                double* o_out, double* lse_out) {
    /* Step 1: S = scale * Q K^T for the requested rows, masked. */
    for (int64_t r = 0; r < nr; ++r) {
        const int64_t i = q_rows[r];
        const float* qi = q + i * d;
        double* srow = s + r * n;
        for (int64_t j = 0; j < n; ++j) {
            if (causal && j > i) {
                srow[j] = -INFINITY;
                continue;
            }
            const float* kj = k + j * d;
            double dot = 0.0;
            for (int64_t t = 0; t < d; ++t) dot += (double)qi[t] * (double)kj[t];
            srow[j] = scale * dot;
        }
    }
    /* Steps 2-3: P = softmax(S), first pass the row max, second pass the sum. */
    for (int64_t r = 0; r < nr; ++r) {
        double* srow = s + r * n;
        double m = -INFINITY;
        for (int64_t j = 0; j < n; ++j)
            if (srow[j] > m) m = srow[j];
        double l = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            srow[j] = exp(srow[j] - m); /* exp(-inf) = 0 for masked keys */
            l += srow[j];
        }
        for (int64_t j = 0; j < n; ++j) srow[j] /= l; /* srow now holds P */
        lse_out[r] = m + log(l);
    }
    /* Step 4: O = P V, summed over the keys the mask allows. */
    for (int64_t r = 0; r < nr; ++r) {
        const double* prow = s + r * n;
        double* orow = o_out + r * d;
        const int64_t j_end = causal ? q_rows[r] + 1 : n;
        for (int64_t t = 0; t < d; ++t) orow[t] = 0.0;
        for (int64_t j = 0; j < j_end; ++j) {
            const double p = prow[j];
            const float* vj = v + j * d;
            for (int64_t t = 0; t < d; ++t) orow[t] += p * (double)vj[t];
        }
    }
}

/*
 * oracle_attention_fwd
 *   q, k, v:  [bh][n][d] fp32 (exact input values)
 *   rows:     [bh][nrows] int64 row indices per head (each in [0, n))
 *   o:        [bh][nrows][d] fp64 output
 *   lse:      [bh][nrows] fp64 output (natural log)
 * Returns 0 on success, -1 on bad arguments, -2 if scratch cannot be allocated.
 */
int oracle_attention_fwd(const float* q, const float* k, const float* v,
                         int64_t bh, int64_t n, int64_t d, double scale, int causal,
                         const int64_t* rows, int64_t nrows, double* o, double* lse) {
    if (!q || !k || !v || !rows || !o || !lse) return -1;
    if (bh <= 0 || n <= 0 || d <= 0 || nrows <= 0) return -1;
    for (int64_t x = 0; x < bh * nrows; ++x)
        if (rows[x] < 0 || rows[x] >= n) return -1;

    const int64_t nblocks = (nrows + ORACLE_ROW_BLOCK - 1) / ORACLE_ROW_BLOCK;
    int failed = 0;
#pragma omp parallel
    {
        double* s = NULL;
        int64_t s_rows = 0;
#pragma omp for schedule(dynamic, 1)
        for (int64_t task = 0; task < bh * nblocks; ++task) {
            const int64_t h = task / nblocks;
            const int64_t b0 = (task % nblocks) * ORACLE_ROW_BLOCK;
            const int64_t nr = (nrows - b0 < ORACLE_ROW_BLOCK) ? nrows - b0 : ORACLE_ROW_BLOCK;
            if (s_rows < nr) {
                free(s);
                s = (double*)malloc((size_t)(nr * n) * sizeof(double));
                s_rows = s ? nr : 0;
            }
            if (!s) {
#pragma omp atomic write
                failed = 1;
                continue;
            }
            const int64_t head = h * n * d;
            attention_row_block(q + head, k + head, v + head, n, d, scale, causal,
                                rows + h * nrows + b0, nr, s,
                                o + (h * nrows + b0) * d, lse + h * nrows + b0);
        }
        free(s);
    }
    return failed ? -2 : 0;
}

/*
 * oracle_attention_decode -- the same definition for new tokens attending
 * to a key/value cache ("FlashAttention: Tiled & Fused", card "KV Cache: Why
 * Generation Speeds Up": past K and V are cached and each new token computes
 * only its own).  nq new queries, nk cached keys (the new tokens' own keys
 * are the last nq of them).  Query i sits at sequence position
 * nk - nq + i; with causal it may use keys kj <= nk - nq + i, without it all
 * nk keys.  Each query's full score row is materialised and softmaxed in
 * two passes, as above.
 *   q:    [bh][nq][d] fp32         k, v: [bh][nk][d] fp32
 *   o:    [bh][nq][d] fp64         lse:  [bh][nq] fp64 (natural log)
 * Returns 0 on success, -1 on bad arguments, -2 if scratch cannot be allocated.
 */
int oracle_attention_decode(const float* q, const float* k, const float* v,
                            int64_t bh, int64_t nq, int64_t nk, int64_t d, double scale, int causal,
                            double* o, double* lse) {
    if (!q || !k || !v || !o || !lse) return -1;
    if (bh <= 0 || nq <= 0 || nk <= 0 || d <= 0) return -1;
    if (causal && nq > nk) return -1;
    int failed = 0;
#pragma omp parallel
    {
        double* w = (double*)malloc((size_t)nk * sizeof(double)); /* one score row */
        if (!w) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t task = 0; task < bh * nq; ++task) {
            if (!w) continue;
            const int64_t h = task / nq, qi = task % nq;
            const float* qrow = q + (h * nq + qi) * d;
            const float* kh = k + h * nk * d;
            const float* vh = v + h * nk * d;
            const int64_t last = causal ? nk - nq + qi : nk - 1; /* last key this query may use */
            /* scores of the allowed keys */
            for (int64_t kj = 0; kj <= last; ++kj) {
                double acc = 0.0;
                for (int64_t t = 0; t < d; ++t) acc += (double)qrow[t] * (double)kh[kj * d + t];
                w[kj] = acc * scale;
            }
            /* softmax: the max, then the exponentials and their sum */
            double mx = w[0];
            for (int64_t kj = 1; kj <= last; ++kj) mx = (w[kj] > mx) ? w[kj] : mx;
            double sum = 0.0;
            for (int64_t kj = 0; kj <= last; ++kj) {
                w[kj] = exp(w[kj] - mx);
                sum += w[kj];
            }
            /* O = P V with P = w / sum */
            double* orow = o + (h * nq + qi) * d;
            for (int64_t t = 0; t < d; ++t) {
                double acc = 0.0;
                for (int64_t kj = 0; kj <= last; ++kj) acc += w[kj] * (double)vh[kj * d + t];
                orow[t] = acc / sum;
            }
            lse[h * nq + qi] = mx + log(sum);
        }
        free(w);
    }
    return failed ? -2 : 0;
}

/*
 * oracle_attention_bwd -- gradients of the same attention with respect to
 * Q, K and V for an upstream gradient dO of the output.  The pages give the
 * forward only and name training as what the method enables ("FlashAttention:
 * Tiled & Fused", section "Enabling longer contexts in training and
 * inference"); the plain reading is the gradient of the exact function,
 * written out from its definition with every score matrix materialised:
 *
 *     P  = softmax(scale * Q K^T [causal])          (two passes per row)
 *     dV = P^T dO
 *     dP = dO V^T
 *     dS = P * (dP - rowsum(dO * O)),  O = P V       (softmax Jacobian)
 *     dQ = scale * dS K,   dK = scale * dS^T Q
 *
 *   q, k, v, dout: [bh][n][d] fp32        dq, dk, dv: [bh][n][d] fp64
 * Memory: three n x n fp64 matrices per head at a time.
 * Returns 0 on success, -1 on bad arguments, -2 if scratch cannot be allocated.
 */
int oracle_attention_bwd(const float* q, const float* k, const float* v, const float* dout,
                         int64_t bh, int64_t n, int64_t d, double scale, int causal,
                         double* dq, double* dk, double* dv) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return -1;
    if (bh <= 0 || n <= 0 || d <= 0) return -1;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t h = 0; h < bh; ++h) {
        double* pm = (double*)malloc((size_t)(n * n) * sizeof(double));   /* P */
        double* gm = (double*)malloc((size_t)(n * n) * sizeof(double));   /* dP, then dS */
        double* om = (double*)malloc((size_t)(n * d) * sizeof(double));   /* O */
        if (!pm || !gm || !om) {
#pragma omp atomic write
            failed = 1;
            free(pm);
            free(gm);
            free(om);
            continue;
        }
        const float* qh = q + h * n * d;
        const float* kh = k + h * n * d;
        const float* vh = v + h * n * d;
        const float* gh = dout + h * n * d;
        /* P, row by row */
        for (int64_t r = 0; r < n; ++r) {
            double* prow = pm + r * n;
            double mrow = -INFINITY;
            for (int64_t c = 0; c < n; ++c) {
                if (causal && c > r) {
                    prow[c] = -INFINITY;
                    continue;
                }
                double acc = 0.0;
                for (int64_t t = 0; t < d; ++t) acc += (double)qh[r * d + t] * (double)kh[c * d + t];
                prow[c] = scale * acc;
                if (prow[c] > mrow) mrow = prow[c];
            }
            double tot = 0.0;
            for (int64_t c = 0; c < n; ++c) {
                prow[c] = exp(prow[c] - mrow);
                tot += prow[c];
            }
            for (int64_t c = 0; c < n; ++c) prow[c] /= tot;
        }
        /* O = P V and dP = dO V^T */
        for (int64_t r = 0; r < n; ++r)
            for (int64_t t = 0; t < d; ++t) {
                double acc = 0.0;
                for (int64_t c = 0; c < n; ++c) acc += pm[r * n + c] * (double)vh[c * d + t];
                om[r * d + t] = acc;
            }
        for (int64_t r = 0; r < n; ++r)
            for (int64_t c = 0; c < n; ++c) {
                double acc = 0.0;
                for (int64_t t = 0; t < d; ++t) acc += (double)gh[r * d + t] * (double)vh[c * d + t];
                gm[r * n + c] = acc;
            }
        /* dS = P * (dP - rowsum(dO * O)) */
        for (int64_t r = 0; r < n; ++r) {
            double drow = 0.0;
            for (int64_t t = 0; t < d; ++t) drow += (double)gh[r * d + t] * om[r * d + t];
            for (int64_t c = 0; c < n; ++c) gm[r * n + c] = pm[r * n + c] * (gm[r * n + c] - drow);
        }
        /* dV = P^T dO, dK = scale dS^T Q, dQ = scale dS K */
        double* dvh = dv + h * n * d;
        double* dkh = dk + h * n * d;
        double* dqh = dq + h * n * d;
        for (int64_t c = 0; c < n; ++c)
            for (int64_t t = 0; t < d; ++t) {
                double av = 0.0, ak = 0.0;
                for (int64_t r = 0; r < n; ++r) {
                    av += pm[r * n + c] * (double)gh[r * d + t];
                    ak += gm[r * n + c] * (double)qh[r * d + t];
                }
                dvh[c * d + t] = av;
                dkh[c * d + t] = scale * ak;
            }
        for (int64_t r = 0; r < n; ++r)
            for (int64_t t = 0; t < d; ++t) {
                double aq = 0.0;
                for (int64_t c = 0; c < n; ++c) aq += gm[r * n + c] * (double)kh[c * d + t];
                dqh[r * d + t] = scale * aq;
            }
        free(pm);
        free(gm);
        free(om);
    }
    return failed ? -2 : 0;
}

/*
 * oracle_attention_bwd_rows -- the gradients of oracle_attention_bwd for
 * chosen rows only: dq for query rows qrows[h][0..nq) and dk, dv for key rows
 * krows[h][0..nk) of each head, for heads too long for the n x n matrices
 * (three fp64 8192 x 8192 matrices take 1.6 GB).  The same definition,
 * written element by element:
 *
 *     s_ij  = scale * q_i . k_j             (j <= i under the causal mask)
 *     lse_i = m_i + log sum_j exp(s_ij - m_i),  m_i = max_j s_ij   (two passes)
 *     P_ij  = exp(s_ij - lse_i),   O_i = sum_j P_ij v_j,   D_i = dO_i . O_i
 *     dP_ij = dO_i . v_j,          dS_ij = P_ij (dP_ij - D_i)
 *     dq_i  = scale sum_j dS_ij k_j
 *     dv_j  = sum_i P_ij dO_i,     dk_j  = scale sum_i dS_ij q_i
 *
 * Every key's gradients sum over all the queries that see it, so lse and D
 * come first for every row of the head (one pass over all scores); each
 * chosen row then costs O(n d).
 *   q, k, v, dout: [bh][n][d] fp32;  qrows [bh][nq], krows [bh][nk] int64
 *   dq [bh][nq][d], dk, dv [bh][nk][d] fp64
 * Returns 0 on success, -1 on bad arguments, -2 if scratch cannot be allocated.
 */
int oracle_attention_bwd_rows(const float* q, const float* k, const float* v, const float* dout,
                              int64_t bh, int64_t n, int64_t d, double scale, int causal,
                              const int64_t* qrows, int64_t nq, const int64_t* krows, int64_t nk,
                              double* dq, double* dk, double* dv) {
    if (!q || !k || !v || !dout || (nq > 0 && (!qrows || !dq)) || (nk > 0 && (!krows || !dk || !dv))) return -1;
    if (bh <= 0 || n <= 0 || d <= 0 || nq < 0 || nk < 0) return -1;
    for (int64_t i = 0; i < bh * nq; ++i)
        if (qrows[i] < 0 || qrows[i] >= n) return -1;
    for (int64_t i = 0; i < bh * nk; ++i)
        if (krows[i] < 0 || krows[i] >= n) return -1;
    double* lse = (double*)malloc((size_t)n * sizeof(double));
    double* dsum = (double*)malloc((size_t)n * sizeof(double));
    if (!lse || !dsum) {
        free(lse);
        free(dsum);
        return -2;
    }
    int failed = 0;
    for (int64_t h = 0; h < bh && !failed; ++h) {
        const float* qh = q + h * n * d;
        const float* kh = k + h * n * d;
        const float* vh = v + h * n * d;
        const float* gh = dout + h * n * d;
#pragma omp parallel
        {
            double* srow = (double*)malloc((size_t)n * sizeof(double));
            double* orow = (double*)malloc((size_t)d * sizeof(double));
            if (!srow || !orow) {
#pragma omp atomic write
                failed = 1;
            }
#pragma omp barrier
            if (!failed) {
                /* lse_i and D_i for every query row */
#pragma omp for schedule(dynamic, 16)
                for (int64_t i = 0; i < n; ++i) {
                    const int64_t jend = causal ? i + 1 : n;
                    double m = -INFINITY;
                    for (int64_t j = 0; j < jend; ++j) {
                        double acc = 0.0;
                        for (int64_t t = 0; t < d; ++t) acc += (double)qh[i * d + t] * (double)kh[j * d + t];
                        srow[j] = scale * acc;
                        m = srow[j] > m ? srow[j] : m;
                    }
                    double l = 0.0;
                    for (int64_t j = 0; j < jend; ++j) l += exp(srow[j] - m);
                    lse[i] = m + log(l);
                    for (int64_t t = 0; t < d; ++t) orow[t] = 0.0;
                    for (int64_t j = 0; j < jend; ++j) {
                        const double pij = exp(srow[j] - lse[i]);
                        for (int64_t t = 0; t < d; ++t) orow[t] += pij * (double)vh[j * d + t];
                    }
                    double acc = 0.0;
                    for (int64_t t = 0; t < d; ++t) acc += (double)gh[i * d + t] * orow[t];
                    dsum[i] = acc;
                }
                /* dq for the chosen query rows */
#pragma omp for schedule(dynamic, 1)
                for (int64_t r = 0; r < nq; ++r) {
                    const int64_t i = qrows[h * nq + r];
                    const int64_t jend = causal ? i + 1 : n;
                    double* out = dq + (h * nq + r) * d;
                    for (int64_t t = 0; t < d; ++t) out[t] = 0.0;
                    for (int64_t j = 0; j < jend; ++j) {
                        double s = 0.0, dp = 0.0;
                        for (int64_t t = 0; t < d; ++t) {
                            s += (double)qh[i * d + t] * (double)kh[j * d + t];
                            dp += (double)gh[i * d + t] * (double)vh[j * d + t];
                        }
                        const double pij = exp(scale * s - lse[i]);
                        const double dsij = pij * (dp - dsum[i]);
                        for (int64_t t = 0; t < d; ++t) out[t] += dsij * (double)kh[j * d + t];
                    }
                    for (int64_t t = 0; t < d; ++t) out[t] *= scale;
                }
                /* dk, dv for the chosen key rows */
#pragma omp for schedule(dynamic, 1)
                for (int64_t r = 0; r < nk; ++r) {
                    const int64_t j = krows[h * nk + r];
                    const int64_t ibeg = causal ? j : 0;
                    double* okv = dv + (h * nk + r) * d;
                    double* okk = dk + (h * nk + r) * d;
                    for (int64_t t = 0; t < d; ++t) okv[t] = okk[t] = 0.0;
                    for (int64_t i = ibeg; i < n; ++i) {
                        double s = 0.0, dp = 0.0;
                        for (int64_t t = 0; t < d; ++t) {
                            s += (double)qh[i * d + t] * (double)kh[j * d + t];
                            dp += (double)gh[i * d + t] * (double)vh[j * d + t];
                        }
                        const double pij = exp(scale * s - lse[i]);
                        const double dsij = pij * (dp - dsum[i]);
                        for (int64_t t = 0; t < d; ++t) {
                            okv[t] += pij * (double)gh[i * d + t];
                            okk[t] += dsij * (double)qh[i * d + t];
                        }
                    }
                    for (int64_t t = 0; t < d; ++t) okk[t] *= scale;
                }
            }
            free(srow);
            free(orow);
        }
    }
    free(lse);
    free(dsum);
    return failed ? -2 : 0;
}

/*
 * oracle_lse_merge -- combine attention results computed over disjoint key
 * sets into the result over their union.  Each part i gives, per query row,
 * o_i = sum_j exp(s_j - lse_i) v_j / 1 over its keys and lse_i = ln sum_j
 * exp(s_j) over its keys; the union's softmax is then
 *     lse = ln sum_i exp(lse_i),   o = sum_i exp(lse_i - lse) o_i
 * -- the same identity the online softmax applies tile by tile
 * ("FlashAttention, Playable", EP 04: rescale what was accumulated by the
 * change of the running max), applied to whole partial results.  A part
 * with lse_i = -inf (no key) contributes nothing.
 *   o_parts: [parts][rows][d] fp32     lse_parts: [parts][rows] fp32
 *   o: [rows][d] fp64                  lse: [rows] fp64
 */
int oracle_lse_merge(const float* o_parts, const float* lse_parts, int64_t parts, int64_t rows, int64_t d,
                     double* o, double* lse) {
    if (!o_parts || !lse_parts || !o || !lse || parts <= 0 || rows <= 0 || d <= 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        double big = -INFINITY;
        for (int64_t i = 0; i < parts; ++i) {
            const double x = (double)lse_parts[i * rows + r];
            if (x > big) big = x;
        }
        double tot = 0.0;
        for (int64_t t = 0; t < d; ++t) o[r * d + t] = 0.0;
        if (big == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        for (int64_t i = 0; i < parts; ++i) {
            const double w = exp((double)lse_parts[i * rows + r] - big);
            tot += w;
            for (int64_t t = 0; t < d; ++t) o[r * d + t] += w * (double)o_parts[(i * rows + r) * d + t];
        }
        for (int64_t t = 0; t < d; ++t) o[r * d + t] /= tot;
        lse[r] = big + log(tot);
    }
    return 0;
}
