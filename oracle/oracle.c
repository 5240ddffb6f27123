/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the Ulysses per-rank
 * attention path. TEST INFRASTRUCTURE ONLY: it is built and called by the
 * tests, by __graft_entry__.smoke() and by bench.py's CPU-baseline leg, and by
 * nothing on the product path. It shares no code, header or table with the
 * CUDA library.
 *
 * What it computes, and where the pages say so:
 *
 *  - seq_to_head / head_to_seq: the two all-to-all exchanges, written out as
 *    index formulas. Page "Hugging Face并行加速：10倍提升超长序列训练效率",
 *    section "Ulysses的工作原理", steps 序列分片 (GPU i owns tokens
 *    [i*n/P,(i+1)*n/P)), 全体间通信 (after the exchange each GPU holds the
 *    heads it is responsible for) and 全体间通信复原 (the second exchange
 *    restores sequence sharding). The same steps appear on the page
 *    "DeepSpeed Ulysses 详解", section "DeepSpeed-Ulysses 的核心机制", items 1, 3
 *    and 5 (after the first exchange a GPU holds the whole sequence for part of
 *    the heads).
 *  - doc_start: packed documents are masked through position ids (page
 *    "Ulysses verteilt Millionen-Token-Kontexte auf mehrere GPUs", section
 *    "Integration in den Hugging-Face-Stack"); a document starts at every i
 *    with position_ids[i] == 0, and always at i = 0.
 *  - attention forward: exact causal softmax attention per head (the
 *    "本地注意力计算" step; heads are independent, same section), restricted to
 *    keys of the query's own document, with grouped KV heads (query head h
 *    reads KV head h / (Hl/Hkvl)), in fp64 with max subtraction.
 *  - attention backward: the exact gradient of L = sum(dO * O) with respect
 *    to Q, K and V, by the chain rule through the softmax, in fp64.
 *
 * All bf16 inputs arrive as raw 16-bit patterns and are widened exactly.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_f64(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* relayouts                                                                 */
/* ------------------------------------------------------------------------ */

/* src: P rank buffers [P][N/P][Hx][d] (rank i holds tokens i*N/P ..).
 * dst: P head slices  [P][N][Hx/P][d] (rank r holds heads r*Hx/P ..).
 * dst[r][n][h][c] = src[n / (N/P)][n % (N/P)][r*Hx/P + h][c].             */
int oracle_seq_to_head(const uint16_t *src, uint16_t *dst, int64_t N, int P, int Hx, int d)
{
    if (P <= 0 || N % P != 0 || Hx % P != 0) return -1;
    const int64_t T = N / P;
    const int Hl = Hx / P;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int r = 0; r < P; ++r)
        for (int64_t n = 0; n < N; ++n) {
            const int64_t i = n / T, m = n % T;
            for (int h = 0; h < Hl; ++h)
                for (int c = 0; c < d; ++c)
                    dst[((r * N + n) * Hl + h) * (int64_t)d + c] =
                        src[((i * T + m) * Hx + (int64_t)r * Hl + h) * (int64_t)d + c];
        }
    return 0;
}

/* Inverse exchange: src [P][N][Hx/P][d] -> dst [P][N/P][Hx][d].
 * dst[p][m][r*Hx/P + h][c] = src[r][p*N/P + m][h][c].                      */
int oracle_head_to_seq(const uint16_t *src, uint16_t *dst, int64_t N, int P, int Hx, int d)
{
    if (P <= 0 || N % P != 0 || Hx % P != 0) return -1;
    const int64_t T = N / P;
    const int Hl = Hx / P;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int p = 0; p < P; ++p)
        for (int64_t m = 0; m < T; ++m)
            for (int r = 0; r < P; ++r)
                for (int h = 0; h < Hl; ++h)
                    for (int c = 0; c < d; ++c)
                        dst[((p * T + m) * Hx + (int64_t)r * Hl + h) * (int64_t)d + c] =
                            src[(((int64_t)r * N + p * T + m) * Hl + h) * (int64_t)d + c];
    return 0;
}

/* ------------------------------------------------------------------------ */
/* document starts                                                          */
/* ------------------------------------------------------------------------ */

/* doc_start[i] = the largest j <= i with pos[j] == 0, or 0 if there is none. */
void oracle_doc_start(const int32_t *pos, int64_t N, int32_t *doc_start)
{
    int64_t last = 0;
    for (int64_t i = 0; i < N; ++i) {
        if (pos[i] == 0) last = i;
        doc_start[i] = (int32_t)last;
    }
}

/* ------------------------------------------------------------------------ */
/* attention forward                                                         */
/* ------------------------------------------------------------------------ */

/* One row of one head: o[d] and the natural-log logsumexp of the scaled
 * logits over keys j in [lo, i]. s_j = scale * q_i . k_j.                   */
static void attn_row(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     int64_t i, int64_t lo, int h, int kvh, int Hl, int Hkvl, int d,
                     double scale, double *s_buf, double *o, double *lse)
{
    const uint16_t *qi = q + (i * Hl + h) * (int64_t)d;
    double m = -INFINITY;
    for (int64_t j = lo; j <= i; ++j) {
        const uint16_t *kj = k + (j * Hkvl + kvh) * (int64_t)d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += bf16_to_f64(qi[c]) * bf16_to_f64(kj[c]);
        acc *= scale;
        s_buf[j - lo] = acc;
        if (acc > m) m = acc;
    }
    double l = 0.0;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int64_t j = lo; j <= i; ++j) {
        const double e = exp(s_buf[j - lo] - m);
        l += e;
        const uint16_t *vj = v + (j * Hkvl + kvh) * (int64_t)d;
        for (int c = 0; c < d; ++c) o[c] += e * bf16_to_f64(vj[c]);
    }
    for (int c = 0; c < d; ++c) o[c] /= l;
    *lse = m + log(l);
}

/* Forward attention of one rank's head slice, on a list of rows.
 * q [N][Hl][d], k/v [N][Hkvl][d] (bf16 bits), pos [N].
 * rows[nrows] are query indices; o is [Hl][nrows][d], lse is [Hl][nrows].  */
int oracle_attn_fwd_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                         const int32_t *pos, int64_t N, int Hl, int Hkvl, int d,
                         double scale, const int64_t *rows, int64_t nrows,
                         double *o, double *lse)
{
    if (Hkvl <= 0 || Hl % Hkvl != 0) return -1;
    int32_t *ds = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
    if (!ds) return -2;
    oracle_doc_start(pos, N, ds);
    const int G = Hl / Hkvl;
    int err = 0;
    #pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        if (!s_buf) {
            #pragma omp atomic write
            err = -2;
        } else {
            #pragma omp for collapse(2) schedule(dynamic, 4)
            for (int h = 0; h < Hl; ++h)
                for (int64_t r = 0; r < nrows; ++r) {
                    const int64_t i = rows[r];
                    attn_row(q, k, v, i, ds[i], h, h / G, Hl, Hkvl, d, scale, s_buf,
                             o + (h * nrows + r) * (int64_t)d, lse + h * nrows + r);
                }
            free(s_buf);
        }
    }
    free(ds);
    return err;
}

/* ------------------------------------------------------------------------ */
/* attention backward                                                        */
/* ------------------------------------------------------------------------ */

/* Exact gradients of L = sum_{i,h,c} dO[i][h][c] * O[i][h][c] for one rank's
 * head slice. With P_ij = softmax_j(s_i.) and s_ij = scale * q_i . k_j:
 *   D_i   = sum_c dO_ic O_ic
 *   dP_ij = dO_i . v_j
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j  = scale * sum_{h in group} sum_i dS_ij q_i
 *   dV_j  = sum_{h in group} sum_i P_ij dO_i
 * Outputs are fp64: dq [N][Hl][d], dk and dv [N][Hkvl][d].
 * Optional o_out [N][Hl][d] and lse_out [Hl][N] receive the forward values.  */
int oracle_attn_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                    const uint16_t *dout, const int32_t *pos, int64_t N, int Hl,
                    int Hkvl, int d, double scale, double *dq, double *dk, double *dv,
                    double *o_out, double *lse_out)
{
    if (Hkvl <= 0 || Hl % Hkvl != 0) return -1;
    const int G = Hl / Hkvl;
    const size_t nz = (size_t)(N > 0 ? N : 1);
    int32_t *ds = (int32_t *)malloc(sizeof(int32_t) * nz);
    int64_t *de = (int64_t *)malloc(sizeof(int64_t) * nz);   /* one past the document's last row */
    double *O = (double *)malloc(sizeof(double) * nz * Hl * d);
    double *LSE = (double *)malloc(sizeof(double) * nz * Hl);
    double *D = (double *)malloc(sizeof(double) * nz * Hl);
    if (!ds || !de || !O || !LSE || !D) {
        free(ds); free(de); free(O); free(LSE); free(D);
        return -2;
    }
    oracle_doc_start(pos, N, ds);
    for (int64_t i = N - 1, end = N; i >= 0; --i) {
        de[i] = end;
        if (ds[i] == i) end = i;
    }
    int err = 0;

    /* Step 1: forward values and D_i. */
    #pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * nz);
        if (!s_buf) {
            #pragma omp atomic write
            err = -2;
        } else {
            #pragma omp for collapse(2) schedule(dynamic, 4)
            for (int h = 0; h < Hl; ++h)
                for (int64_t i = 0; i < N; ++i) {
                    double *oi = O + (i * Hl + h) * (int64_t)d;
                    attn_row(q, k, v, i, ds[i], h, h / G, Hl, Hkvl, d, scale, s_buf, oi,
                             LSE + (int64_t)h * N + i);
                    const uint16_t *gi = dout + (i * Hl + h) * (int64_t)d;
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c) acc += bf16_to_f64(gi[c]) * oi[c];
                    D[(int64_t)h * N + i] = acc;
                }
            free(s_buf);
        }
    }
    if (err) goto done;

    /* Step 2: dQ, row by row. */
    #pragma omp parallel for collapse(2) schedule(dynamic, 4)
    for (int h = 0; h < Hl; ++h)
        for (int64_t i = 0; i < N; ++i) {
            const int kvh = h / G;
            const uint16_t *qi = q + (i * Hl + h) * (int64_t)d;
            const uint16_t *gi = dout + (i * Hl + h) * (int64_t)d;
            double *dqi = dq + (i * Hl + h) * (int64_t)d;
            for (int c = 0; c < d; ++c) dqi[c] = 0.0;
            for (int64_t j = ds[i]; j <= i; ++j) {
                const uint16_t *kj = k + (j * Hkvl + kvh) * (int64_t)d;
                const uint16_t *vj = v + (j * Hkvl + kvh) * (int64_t)d;
                double s = 0.0, dp = 0.0;
                for (int c = 0; c < d; ++c) {
                    s += bf16_to_f64(qi[c]) * bf16_to_f64(kj[c]);
                    dp += bf16_to_f64(gi[c]) * bf16_to_f64(vj[c]);
                }
                const double p = exp(scale * s - LSE[(int64_t)h * N + i]);
                const double dsij = p * (dp - D[(int64_t)h * N + i]);
                for (int c = 0; c < d; ++c) dqi[c] += scale * dsij * bf16_to_f64(kj[c]);
            }
        }

    /* Step 3: dK and dV, key by key, summed over the query heads of the group. */
    #pragma omp parallel for collapse(2) schedule(dynamic, 4)
    for (int kvh = 0; kvh < Hkvl; ++kvh)
        for (int64_t j = 0; j < N; ++j) {
            const uint16_t *kj = k + (j * Hkvl + kvh) * (int64_t)d;
            const uint16_t *vj = v + (j * Hkvl + kvh) * (int64_t)d;
            double *dkj = dk + (j * Hkvl + kvh) * (int64_t)d;
            double *dvj = dv + (j * Hkvl + kvh) * (int64_t)d;
            for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
            for (int g = 0; g < G; ++g) {
                const int h = kvh * G + g;
                for (int64_t i = j; i < de[j]; ++i) {
                    const uint16_t *qi = q + (i * Hl + h) * (int64_t)d;
                    const uint16_t *gi = dout + (i * Hl + h) * (int64_t)d;
                    double s = 0.0, dp = 0.0;
                    for (int c = 0; c < d; ++c) {
                        s += bf16_to_f64(qi[c]) * bf16_to_f64(kj[c]);
                        dp += bf16_to_f64(gi[c]) * bf16_to_f64(vj[c]);
                    }
                    const double p = exp(scale * s - LSE[(int64_t)h * N + i]);
                    const double dsij = p * (dp - D[(int64_t)h * N + i]);
                    for (int c = 0; c < d; ++c) {
                        dvj[c] += p * bf16_to_f64(gi[c]);
                        dkj[c] += scale * dsij * bf16_to_f64(qi[c]);
                    }
                }
            }
        }

    if (o_out) memcpy(o_out, O, sizeof(double) * (size_t)N * Hl * d);
    if (lse_out) memcpy(lse_out, LSE, sizeof(double) * (size_t)N * Hl);
done:
    free(ds); free(de); free(O); free(LSE); free(D);
    return err;
}

/* ------------------------------------------------------------------------ */
/* attention backward on sampled rows and keys                              */
/* ------------------------------------------------------------------------ */

/* The same gradients as oracle_attn_bwd, evaluated only where asked: dQ for
 * the query rows rows[0..nrows) and dK, dV for the keys keys[0..nkeys). This
 * lets a long document's heaviest keys (its first ones, which every later
 * query of the document attends to) be checked without the whole backward.
 * Every query row whose values enter those results (the sampled rows, and
 * rows j .. end of document - 1 of every sampled key j) first gets its exact
 * forward values (LSE_i, and D_i = sum_c dO_ic O_ic); then
 *   dQ_i = scale * sum_{j in [doc_start(i), i]} dS_ij k_j
 *   dK_j = scale * sum_{h in group} sum_{i in [j, doc end)} dS_ij q_i
 *   dV_j = sum_{h in group} sum_{i in [j, doc end)} P_ij dO_i
 * with P_ij = exp(scale q_i.k_j - LSE_i) and dS_ij = P_ij (dO_i.v_j - D_i).
 * Outputs: dq [nrows][Hl][d], dk and dv [nkeys][Hkvl][d], fp64.            */
int oracle_attn_bwd_sampled(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            const uint16_t *dout, const int32_t *pos, int64_t N, int Hl,
                            int Hkvl, int d, double scale, const int64_t *rows, int64_t nrows,
                            const int64_t *keys, int64_t nkeys, double *dq, double *dk, double *dv)
{
    if (Hkvl <= 0 || Hl % Hkvl != 0) return -1;
    const int G = Hl / Hkvl;
    const size_t nz = (size_t)(N > 0 ? N : 1);
    int32_t *ds = (int32_t *)malloc(sizeof(int32_t) * nz);
    int64_t *de = (int64_t *)malloc(sizeof(int64_t) * nz);
    unsigned char *need = (unsigned char *)calloc(nz, 1);
    double *LSE = (double *)malloc(sizeof(double) * nz * Hl);
    double *D = (double *)malloc(sizeof(double) * nz * Hl);
    if (!ds || !de || !need || !LSE || !D) {
        free(ds); free(de); free(need); free(LSE); free(D);
        return -2;
    }
    oracle_doc_start(pos, N, ds);
    for (int64_t i = N - 1, end = N; i >= 0; --i) {
        de[i] = end;
        if (ds[i] == i) end = i;
    }
    for (int64_t r = 0; r < nrows; ++r) {
        if (rows[r] < 0 || rows[r] >= N) { free(ds); free(de); free(need); free(LSE); free(D); return -1; }
        need[rows[r]] = 1;
    }
    for (int64_t t = 0; t < nkeys; ++t) {
        if (keys[t] < 0 || keys[t] >= N) { free(ds); free(de); free(need); free(LSE); free(D); return -1; }
        for (int64_t i = keys[t]; i < de[keys[t]]; ++i) need[i] = 1;
    }
    int err = 0;

    /* Step 1: forward values and D_i of every row that is needed. */
    #pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * nz);
        double *oi = (double *)malloc(sizeof(double) * (size_t)d);
        if (!s_buf || !oi) {
            #pragma omp atomic write
            err = -2;
        } else {
            #pragma omp for collapse(2) schedule(dynamic, 4)
            for (int h = 0; h < Hl; ++h)
                for (int64_t i = 0; i < N; ++i) {
                    if (!need[i]) continue;
                    attn_row(q, k, v, i, ds[i], h, h / G, Hl, Hkvl, d, scale, s_buf, oi,
                             LSE + (int64_t)h * N + i);
                    const uint16_t *gi = dout + (i * Hl + h) * (int64_t)d;
                    double acc = 0.0;
                    for (int c = 0; c < d; ++c) acc += bf16_to_f64(gi[c]) * oi[c];
                    D[(int64_t)h * N + i] = acc;
                }
        }
        free(s_buf);
        free(oi);
    }
    if (err) goto done;

    /* Step 2: dQ of the sampled rows. */
    #pragma omp parallel for collapse(2) schedule(dynamic, 4)
    for (int h = 0; h < Hl; ++h)
        for (int64_t r = 0; r < nrows; ++r) {
            const int64_t i = rows[r];
            const int kvh = h / G;
            const uint16_t *qi = q + (i * Hl + h) * (int64_t)d;
            const uint16_t *gi = dout + (i * Hl + h) * (int64_t)d;
            double *dqi = dq + (r * Hl + h) * (int64_t)d;
            for (int c = 0; c < d; ++c) dqi[c] = 0.0;
            for (int64_t j = ds[i]; j <= i; ++j) {
                const uint16_t *kj = k + (j * Hkvl + kvh) * (int64_t)d;
                const uint16_t *vj = v + (j * Hkvl + kvh) * (int64_t)d;
                double s = 0.0, dp = 0.0;
                for (int c = 0; c < d; ++c) {
                    s += bf16_to_f64(qi[c]) * bf16_to_f64(kj[c]);
                    dp += bf16_to_f64(gi[c]) * bf16_to_f64(vj[c]);
                }
                const double p = exp(scale * s - LSE[(int64_t)h * N + i]);
                const double dsij = p * (dp - D[(int64_t)h * N + i]);
                for (int c = 0; c < d; ++c) dqi[c] += scale * dsij * bf16_to_f64(kj[c]);
            }
        }

    /* Step 3: dK and dV of the sampled keys, summed over the group's query heads. */
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int kvh = 0; kvh < Hkvl; ++kvh)
        for (int64_t t = 0; t < nkeys; ++t) {
            const int64_t j = keys[t];
            const uint16_t *kj = k + (j * Hkvl + kvh) * (int64_t)d;
            const uint16_t *vj = v + (j * Hkvl + kvh) * (int64_t)d;
            double *dkj = dk + (t * Hkvl + kvh) * (int64_t)d;
            double *dvj = dv + (t * Hkvl + kvh) * (int64_t)d;
            for (int c = 0; c < d; ++c) { dkj[c] = 0.0; dvj[c] = 0.0; }
            for (int g = 0; g < G; ++g) {
                const int h = kvh * G + g;
                for (int64_t i = j; i < de[j]; ++i) {
                    const uint16_t *qi = q + (i * Hl + h) * (int64_t)d;
                    const uint16_t *gi = dout + (i * Hl + h) * (int64_t)d;
                    double s = 0.0, dp = 0.0;
                    for (int c = 0; c < d; ++c) {
                        s += bf16_to_f64(qi[c]) * bf16_to_f64(kj[c]);
                        dp += bf16_to_f64(gi[c]) * bf16_to_f64(vj[c]);
                    }
                    const double p = exp(scale * s - LSE[(int64_t)h * N + i]);
                    const double dsij = p * (dp - D[(int64_t)h * N + i]);
                    for (int c = 0; c < d; ++c) {
                        dvj[c] += p * bf16_to_f64(gi[c]);
                        dkj[c] += scale * dsij * bf16_to_f64(qi[c]);
                    }
                }
            }
        }

done:
    free(ds); free(de); free(need); free(LSE); free(D);
    return err;
}

/* ------------------------------------------------------------------------ */
/* ring steps: attention over a key window, and the merge of partial results */
/* ------------------------------------------------------------------------ */

/* Ring attention (set against Ulysses on the page "Ulysses 序列並行：百萬 Token
 * 上下文訓練", section "競品分析", and on the page "Ulysses verteilt
 * Millionen-Token-Kontexte auf mehrere GPUs", section "Wann Ulysses sinnvoll
 * ist") passes the keys and values around the ranks chunk by chunk; each step
 * gives the attention of the local queries over one chunk of keys. That
 * partial result is the ordinary attention restricted to the keys of the
 * window [kv_lo, kv_hi): row i sees keys j in [max(doc_start(i), kv_lo),
 * min(i, kv_hi - 1)]. A row that sees no key gets o = 0 and lse = -inf.
 * rows[nrows] are query indices; o is [Hl][nrows][d], lse is [Hl][nrows].   */
int oracle_attn_fwd_window_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                const int32_t *pos, int64_t N, int Hl, int Hkvl, int d,
                                double scale, int64_t kv_lo, int64_t kv_hi,
                                const int64_t *rows, int64_t nrows, double *o, double *lse)
{
    if (Hkvl <= 0 || Hl % Hkvl != 0) return -1;
    int32_t *ds = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
    if (!ds) return -2;
    oracle_doc_start(pos, N, ds);
    const int G = Hl / Hkvl;
    int err = 0;
    #pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        if (!s_buf) {
            #pragma omp atomic write
            err = -2;
        } else {
            #pragma omp for collapse(2) schedule(dynamic, 4)
            for (int h = 0; h < Hl; ++h)
                for (int64_t r = 0; r < nrows; ++r) {
                    const int64_t i = rows[r];
                    const int64_t lo = ds[i] > kv_lo ? ds[i] : kv_lo;
                    const int64_t hi = i < kv_hi - 1 ? i : kv_hi - 1;
                    double *orow = o + (h * nrows + r) * (int64_t)d;
                    double *l_out = lse + h * nrows + r;
                    if (lo > hi) {
                        for (int c = 0; c < d; ++c) orow[c] = 0.0;
                        *l_out = -INFINITY;
                        continue;
                    }
                    const int kvh = h / G;
                    const uint16_t *qi = q + (i * Hl + h) * (int64_t)d;
                    double m = -INFINITY;
                    for (int64_t j = lo; j <= hi; ++j) {
                        const uint16_t *kj = k + (j * Hkvl + kvh) * (int64_t)d;
                        double acc = 0.0;
                        for (int c = 0; c < d; ++c) acc += bf16_to_f64(qi[c]) * bf16_to_f64(kj[c]);
                        acc *= scale;
                        s_buf[j - lo] = acc;
                        if (acc > m) m = acc;
                    }
                    double l = 0.0;
                    for (int c = 0; c < d; ++c) orow[c] = 0.0;
                    for (int64_t j = lo; j <= hi; ++j) {
                        const double e = exp(s_buf[j - lo] - m);
                        l += e;
                        const uint16_t *vj = v + (j * Hkvl + kvh) * (int64_t)d;
                        for (int c = 0; c < d; ++c) orow[c] += e * bf16_to_f64(vj[c]);
                    }
                    for (int c = 0; c < d; ++c) orow[c] /= l;
                    *l_out = m + log(l);
                }
            free(s_buf);
        }
    }
    free(ds);
    return err;
}

/* The merge of R partial results over disjoint key sets into the result over
 * their union: with L = log sum_s exp(lse_s), o = sum_s exp(lse_s - L) o_s and
 * lse = L (each partial o_s is already normalised by its own sum exp(lse_s)).
 * A partial with lse_s = -inf (no key) contributes nothing; if every one is
 * -inf, o = 0 and lse = -inf.
 * o_parts [R][M][Hl][d], lse_parts [R][Hl][M]; o [M][Hl][d], lse [Hl][M].  */
void oracle_merge(const double *o_parts, const double *lse_parts, int R, int64_t M, int Hl, int d,
                  double *o, double *lse)
{
    #pragma omp parallel for collapse(2) schedule(static)
    for (int h = 0; h < Hl; ++h)
        for (int64_t m = 0; m < M; ++m) {
            double mx = -INFINITY;
            for (int s = 0; s < R; ++s) {
                const double x = lse_parts[((int64_t)s * Hl + h) * M + m];
                if (x > mx) mx = x;
            }
            double *orow = o + (m * Hl + h) * (int64_t)d;
            for (int c = 0; c < d; ++c) orow[c] = 0.0;
            if (mx == -INFINITY) {
                lse[(int64_t)h * M + m] = -INFINITY;
                continue;
            }
            double sum = 0.0;
            for (int s = 0; s < R; ++s) sum += exp(lse_parts[((int64_t)s * Hl + h) * M + m] - mx);
            const double L = mx + log(sum);
            for (int s = 0; s < R; ++s) {
                const double w = exp(lse_parts[((int64_t)s * Hl + h) * M + m] - L);
                const double *op = o_parts + (((int64_t)s * M + m) * Hl + h) * (int64_t)d;
                for (int c = 0; c < d; ++c) orow[c] += w * op[c];
            }
            lse[(int64_t)h * M + m] = L;
        }
}

/* Host threads of the loops above (no arithmetic): a launcher that gives the
 * process one thread (torchrun does, for each rank) can hand rank 0 the whole
 * host back. */
void oracle_set_num_threads(int n)
{
    if (n > 0) omp_set_num_threads(n);
}

int oracle_max_threads(void) { return omp_get_max_threads(); }
