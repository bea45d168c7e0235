/*
 * attn_oracle.c -- plain, slow, fp64 CPU oracle for exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file: only the tests, the smoke check and the bench's CPU-baseline / reference arm do.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (source: the page "ms-swift集成FlashAttention 2/3，长文本训练更高效"
 * [ms-swift integrates FlashAttention 2/3, long-text training is more efficient],
 * section "为什么传统注意力这么'吃'显存" [why standard attention eats so much memory]):
 * the standard three-step attention -- scores S = Q K^T, a row softmax of S, then
 * O = P V -- with every score of a row materialised, exactly as that section describes
 * the native implementation.  The same page's section "FlashAttention 如何破局"
 * [how FlashAttention breaks the deadlock] states that the fused, tiled kernel keeps
 * exactly this result ("numerically consistent"), so this plain definition is the
 * thing the GPU path must reproduce up to rounding.
 *
 * Readings where the page is silent (the plainest one that fits the rest of the page):
 *   - scores carry a factor `scale` (1/sqrt(D) by default): s_ij = scale * q_i . k_j;
 *   - causal: key j is visible to query i iff j <= i, positions counted from the start
 *     of the query's own sequence; packed sequences never see each other;
 *   - grouped-query attention: query head h reads key/value head h / (Hq/Hkv)
 *     (contiguous groups);
 *   - LSE_i = ln sum_j exp(s_ij) (natural log of the scaled scores);
 *   - backward recomputes P from the row statistics (no stored S x S matrix), with
 *     dP = dO V^T, Delta_i = dO_i . O_i, dS = P o (dP - Delta), dQ = scale dS K,
 *     dK = scale dS^T Q, dV = P^T dO, and dK/dV summed over the query heads of a group.
 *
 * Layouts: tokens are numbered 0..T-1 (T = B*S dense, or the packed total);
 *   q, o, dO, dq : [T][Hq][D];   k, v, dk, dv : [T][Hkv][D];
 *   lse : dense [B][Hq][S], packed [Hq][T].
 * All arrays are fp64; bf16 inputs are widened exactly by the caller.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, Hq, Hkv, S, D, causal;
    double scale;
    const int32_t *cu; /* NULL: dense */
} prob_t;

static int64_t seq_start(const prob_t *p, int b) { return p->cu ? p->cu[b] : (int64_t)b * p->S; }
static int seq_len(const prob_t *p, int b) { return p->cu ? p->cu[b + 1] - p->cu[b] : p->S; }
static int64_t total_tokens(const prob_t *p) { return p->cu ? p->cu[p->B] : (int64_t)p->B * p->S; }

static int64_t lse_index(const prob_t *p, int b, int h, int i) {
    if (p->cu) return (int64_t)h * total_tokens(p) + seq_start(p, b) + i;
    return ((int64_t)b * p->Hq + h) * p->S + i;
}

static int check(const prob_t *p) {
    if (p->B < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->D <= 0 || p->S < 0) return 1;
    if (p->Hq % p->Hkv) return 1;
    if (p->cu) {
        if (p->cu[0] != 0) return 1;
        for (int b = 0; b < p->B; ++b)
            if (p->cu[b + 1] < p->cu[b]) return 1;
    }
    return 0;
}

static const double *row_q(const prob_t *p, const double *q, int64_t t, int h) {
    return q + (t * p->Hq + h) * (int64_t)p->D;
}
static const double *row_kv(const prob_t *p, const double *k, int64_t t, int g) {
    return k + (t * p->Hkv + g) * (int64_t)p->D;
}

/* Number of keys of the sequence visible to query i. */
static int visible(const prob_t *p, int L, int i) { return p->causal ? i + 1 : L; }

/*
 * One query row, forward: s_j, m, P_j, O_i, LSE_i (section "why standard attention
 * eats so much memory": scores, softmax, then P V).  `s` is scratch of length >= L.
 */
static void fwd_row(const prob_t *p, const double *q, const double *k, const double *v,
                    int b, int h, int i, double *s, double *o_row, double *lse_out) {
    const int L = seq_len(p, b);
    const int64_t t0 = seq_start(p, b);
    const int g = h / (p->Hq / p->Hkv);
    const int D = p->D;
    const int n = visible(p, L, i);
    const double *qi = row_q(p, q, t0 + i, h);
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) {
        const double *kj = row_kv(p, k, t0 + j, g);
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += qi[d] * kj[d];
        s[j] = p->scale * acc;
        if (s[j] > m) m = s[j];
    }
    double sum = 0.0;
    for (int j = 0; j < n; ++j) {
        s[j] = exp(s[j] - m);
        sum += s[j];
    }
    for (int d = 0; d < D; ++d) o_row[d] = 0.0;
    for (int j = 0; j < n; ++j) {
        const double pj = s[j] / sum;
        s[j] = pj;
        const double *vj = row_kv(p, v, t0 + j, g);
        for (int d = 0; d < D; ++d) o_row[d] += pj * vj[d];
    }
    *lse_out = m + log(sum);
}

/* Flattened (b, h, i) index space of all query rows. */
typedef struct { int b, h, i; } rowid_t;

static int64_t count_rows(const prob_t *p) {
    return total_tokens(p) * p->Hq;
}

static rowid_t row_at(const prob_t *p, int64_t r) {
    /* r enumerates (token t, head h) with h fastest; map t to (b, i). */
    rowid_t id;
    int64_t t = r / p->Hq;
    id.h = (int)(r % p->Hq);
    if (!p->cu) {
        id.b = (int)(t / p->S);
        id.i = (int)(t % p->S);
    } else {
        int lo = 0, hi = p->B - 1; /* last b with cu[b] <= t and non-empty */
        while (lo < hi) {
            int mid = (lo + hi + 1) / 2;
            if (p->cu[mid] <= t) lo = mid; else hi = mid - 1;
        }
        while (lo > 0 && p->cu[lo + 1] <= t) ++lo; /* not reached for t < T */
        id.b = lo;
        id.i = (int)(t - p->cu[lo]);
    }
    return id;
}

static int max_len(const prob_t *p) {
    int m = 0;
    for (int b = 0; b < p->B; ++b) if (seq_len(p, b) > m) m = seq_len(p, b);
    return m;
}

/* Forward over every query row.  o: [T][Hq][D]; lse as documented above. */
int oracle_attn_fwd(const double *q, const double *k, const double *v, double *o, double *lse,
                    int B, int Hq, int Hkv, int S, int D, int causal, double scale,
                    const int32_t *cu_seqlens) {
    prob_t p = {B, Hq, Hkv, S, D, causal, scale, cu_seqlens};
    if (check(&p)) return 1;
    const int64_t R = count_rows(&p);
    const int Lmax = max_len(&p);
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (Lmax > 0 ? Lmax : 1));
        if (!s) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < R; ++r) {
            if (!s) continue;
            rowid_t id = row_at(&p, r);
            const int64_t t = seq_start(&p, id.b) + id.i;
            double l;
            fwd_row(&p, q, k, v, id.b, id.h, id.i, s, o + (t * Hq + id.h) * (int64_t)D, &l);
            lse[lse_index(&p, id.b, id.h, id.i)] = l;
        }
        free(s);
    }
    return err;
}

/* Forward for a list of query rows (b, h, i): o_rows [n][D], lse_rows [n]. */
int oracle_attn_fwd_rows(const double *q, const double *k, const double *v,
                         int B, int Hq, int Hkv, int S, int D, int causal, double scale,
                         const int32_t *cu_seqlens, int n, const int32_t *rb, const int32_t *rh,
                         const int32_t *ri, double *o_rows, double *lse_rows) {
    prob_t p = {B, Hq, Hkv, S, D, causal, scale, cu_seqlens};
    if (check(&p)) return 1;
    for (int r = 0; r < n; ++r)
        if (rb[r] < 0 || rb[r] >= B || rh[r] < 0 || rh[r] >= Hq || ri[r] < 0 || ri[r] >= seq_len(&p, rb[r]))
            return 1;
    const int Lmax = max_len(&p);
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (Lmax > 0 ? Lmax : 1));
        if (!s) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < n; ++r) {
            if (!s) continue;
            fwd_row(&p, q, k, v, rb[r], rh[r], ri[r], s, o_rows + (int64_t)r * D, &lse_rows[r]);
        }
        free(s);
    }
    return err;
}

/*
 * Backward, row part for one query row: recomputes P_i (fwd_row), O_i, then
 * Delta_i = dO_i . O_i, dP_ij = dO_i . v_j, dS_ij = P_ij (dP_ij - Delta_i) and
 * dQ_i = scale sum_j dS_ij k_j.
 */
static void bwd_row_dq(const prob_t *p, const double *q, const double *k, const double *v,
                       const double *dout, int b, int h, int i, double *s, double *o_tmp,
                       double *dq_row, double *lse_out, double *delta_out) {
    const int L = seq_len(p, b);
    const int64_t t0 = seq_start(p, b);
    const int g = h / (p->Hq / p->Hkv);
    const int D = p->D;
    const int n = visible(p, L, i);
    double l;
    fwd_row(p, q, k, v, b, h, i, s, o_tmp, &l); /* s[j] now holds P_ij */
    const double *doi = row_q(p, dout, t0 + i, h);
    double delta = 0.0;
    for (int d = 0; d < D; ++d) delta += doi[d] * o_tmp[d];
    for (int d = 0; d < D; ++d) dq_row[d] = 0.0;
    for (int j = 0; j < n; ++j) {
        const double *vj = row_kv(p, v, t0 + j, g);
        double dp = 0.0;
        for (int d = 0; d < D; ++d) dp += doi[d] * vj[d];
        const double ds = s[j] * (dp - delta);
        const double *kj = row_kv(p, k, t0 + j, g);
        for (int d = 0; d < D; ++d) dq_row[d] += ds * kj[d];
    }
    for (int d = 0; d < D; ++d) dq_row[d] *= p->scale;
    *lse_out = l;
    *delta_out = delta;
}

/*
 * Backward, column part for key j of kv head g: sums over the group's query heads and
 * every query row that sees key j; P_ij = exp(s_ij - LSE_i) from the row pass.
 *   dV_j = sum P_ij dO_i,   dK_j = scale sum dS_ij q_i.
 * `lse_g`/`delta_g` hold the row statistics of the group's heads for this sequence,
 * indexed [hh][i] (hh = head within the group).
 */
static void bwd_col(const prob_t *p, const double *q, const double *k, const double *v,
                    const double *dout, int b, int g, int j, const double *lse_g,
                    const double *delta_g, double *dk_row, double *dv_row) {
    const int L = seq_len(p, b);
    const int64_t t0 = seq_start(p, b);
    const int G = p->Hq / p->Hkv;
    const int D = p->D;
    const double *kj = row_kv(p, k, t0 + j, g);
    const double *vj = row_kv(p, v, t0 + j, g);
    for (int d = 0; d < D; ++d) { dk_row[d] = 0.0; dv_row[d] = 0.0; }
    for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        for (int i = p->causal ? j : 0; i < L; ++i) {
            const double *qi = row_q(p, q, t0 + i, h);
            const double *doi = row_q(p, dout, t0 + i, h);
            double acc = 0.0, dp = 0.0;
            for (int d = 0; d < D; ++d) { acc += qi[d] * kj[d]; dp += doi[d] * vj[d]; }
            const double pij = exp(p->scale * acc - lse_g[(int64_t)hh * L + i]);
            const double ds = pij * (dp - delta_g[(int64_t)hh * L + i]);
            for (int d = 0; d < D; ++d) {
                dv_row[d] += pij * doi[d];
                dk_row[d] += ds * qi[d];
            }
        }
    }
    for (int d = 0; d < D; ++d) dk_row[d] *= p->scale;
}

/* Full backward.  dq [T][Hq][D], dk/dv [T][Hkv][D]. */
int oracle_attn_bwd(const double *q, const double *k, const double *v, const double *dout,
                    double *dq, double *dk, double *dv,
                    int B, int Hq, int Hkv, int S, int D, int causal, double scale,
                    const int32_t *cu_seqlens) {
    prob_t p = {B, Hq, Hkv, S, D, causal, scale, cu_seqlens};
    if (check(&p)) return 1;
    const int64_t T = total_tokens(&p);
    const int Lmax = max_len(&p);
    const int G = Hq / Hkv;
    double *lse = (double *)malloc(sizeof(double) * (T * Hq > 0 ? T * Hq : 1));
    double *delta = (double *)malloc(sizeof(double) * (T * Hq > 0 ? T * Hq : 1));
    if (!lse || !delta) { free(lse); free(delta); return 2; }
    int err = 0;
    /* Row pass: dQ, LSE and Delta, stored per (head, token) as [h][t]. */
    const int64_t R = count_rows(&p);
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (Lmax > 0 ? Lmax : 1));
        double *ot = (double *)malloc(sizeof(double) * D);
        if (!s || !ot) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < R; ++r) {
            if (!s || !ot) continue;
            rowid_t id = row_at(&p, r);
            const int64_t t = seq_start(&p, id.b) + id.i;
            bwd_row_dq(&p, q, k, v, dout, id.b, id.h, id.i, s, ot,
                       dq + (t * Hq + id.h) * (int64_t)D, &lse[(int64_t)id.h * T + t],
                       &delta[(int64_t)id.h * T + t]);
        }
        free(s);
        free(ot);
    }
    if (err) { free(lse); free(delta); return err; }
    /* Column pass: dK, dV per (b, g, j). */
    const int64_t C = T * Hkv;
#pragma omp parallel
    {
        double *lg = (double *)malloc(sizeof(double) * (size_t)G * (Lmax > 0 ? Lmax : 1));
        double *dg = (double *)malloc(sizeof(double) * (size_t)G * (Lmax > 0 ? Lmax : 1));
        if (!lg || !dg) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t c = 0; c < C; ++c) {
            if (!lg || !dg) continue;
            const int64_t t = c / Hkv;
            const int g = (int)(c % Hkv);
            /* map token t to (b, j) */
            prob_t pq = p;
            pq.Hq = 1; /* row_at with one head maps r=t */
            rowid_t id = row_at(&pq, t);
            const int L = seq_len(&p, id.b);
            const int64_t t0 = seq_start(&p, id.b);
            for (int hh = 0; hh < G; ++hh)
                for (int i = 0; i < L; ++i) {
                    lg[(int64_t)hh * L + i] = lse[(int64_t)(g * G + hh) * T + t0 + i];
                    dg[(int64_t)hh * L + i] = delta[(int64_t)(g * G + hh) * T + t0 + i];
                }
            bwd_col(&p, q, k, v, dout, id.b, g, id.i, lg, dg, dk + (t * Hkv + g) * (int64_t)D,
                    dv + (t * Hkv + g) * (int64_t)D);
        }
        free(lg);
        free(dg);
    }
    free(lse);
    free(delta);
    return err;
}

/* dQ for a list of query rows (b, h, i): dq_rows [n][D]; also the row's LSE and Delta. */
int oracle_attn_bwd_dq_rows(const double *q, const double *k, const double *v, const double *dout,
                            int B, int Hq, int Hkv, int S, int D, int causal, double scale,
                            const int32_t *cu_seqlens, int n, const int32_t *rb,
                            const int32_t *rh, const int32_t *ri, double *dq_rows,
                            double *lse_rows, double *delta_rows) {
    prob_t p = {B, Hq, Hkv, S, D, causal, scale, cu_seqlens};
    if (check(&p)) return 1;
    for (int r = 0; r < n; ++r)
        if (rb[r] < 0 || rb[r] >= B || rh[r] < 0 || rh[r] >= Hq || ri[r] < 0 || ri[r] >= seq_len(&p, rb[r]))
            return 1;
    const int Lmax = max_len(&p);
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (Lmax > 0 ? Lmax : 1));
        double *ot = (double *)malloc(sizeof(double) * D);
        if (!s || !ot) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < n; ++r) {
            if (!s || !ot) continue;
            bwd_row_dq(&p, q, k, v, dout, rb[r], rh[r], ri[r], s, ot, dq_rows + (int64_t)r * D,
                       &lse_rows[r], &delta_rows[r]);
        }
        free(s);
        free(ot);
    }
    return err;
}

/*
 * dK, dV for the keys j0 <= j < j1 of kv head g in sequence b: dk_rows/dv_rows [j1-j0][D].
 * Computes the row statistics only for the query rows that can see those keys
 * (i >= j0 when causal), so keys near the end of a long sequence are cheap.
 */
int oracle_attn_bwd_dkdv_range(const double *q, const double *k, const double *v,
                               const double *dout, int B, int Hq, int Hkv, int S, int D,
                               int causal, double scale, const int32_t *cu_seqlens, int b, int g,
                               int j0, int j1, double *dk_rows, double *dv_rows) {
    prob_t p = {B, Hq, Hkv, S, D, causal, scale, cu_seqlens};
    if (check(&p)) return 1;
    if (b < 0 || b >= B || g < 0 || g >= Hkv) return 1;
    const int L = seq_len(&p, b);
    if (j0 < 0 || j1 > L || j0 > j1) return 1;
    const int G = Hq / Hkv;
    const int i0 = causal ? j0 : 0;
    const int Lmax = L;
    double *lg = (double *)calloc((size_t)G * (L > 0 ? L : 1), sizeof(double));
    double *dg = (double *)calloc((size_t)G * (L > 0 ? L : 1), sizeof(double));
    if (!lg || !dg) { free(lg); free(dg); return 2; }
    int err = 0;
    const int nr = L - i0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (Lmax > 0 ? Lmax : 1));
        double *ot = (double *)malloc(sizeof(double) * D);
        double *dqt = (double *)malloc(sizeof(double) * D);
        if (!s || !ot || !dqt) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < (int64_t)G * nr; ++r) {
            if (!s || !ot || !dqt) continue;
            const int hh = (int)(r / nr);
            const int i = i0 + (int)(r % nr);
            bwd_row_dq(&p, q, k, v, dout, b, g * G + hh, i, s, ot, dqt, &lg[(int64_t)hh * L + i],
                       &dg[(int64_t)hh * L + i]);
        }
        free(s);
        free(ot);
        free(dqt);
    }
    if (!err) {
#pragma omp parallel for schedule(dynamic, 1)
        for (int j = j0; j < j1; ++j)
            bwd_col(&p, q, k, v, dout, b, g, j, lg, dg, dk_rows + (int64_t)(j - j0) * D,
                    dv_rows + (int64_t)(j - j0) * D);
    }
    free(lg);
    free(dg);
    return err;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Merge of partial attention results (page "ms-swift集成FlashAttention 2/3，长文本训练更高效", section
 * "单靠 FlashAttention 不够？那就加上序列并行", subsection "Ring-Attention": every device
 * accumulates partial attention over the key/value chunks that pass by).  A partial over a
 * key subset K_p is (O_p, LSE_p) with O_p the softmax-weighted mean over K_p and LSE_p the
 * log of its normaliser, so over the union of disjoint subsets
 *     LSE = ln sum_p exp(LSE_p),   O = sum_p exp(LSE_p - LSE) O_p.
 * Partials with LSE_p = -inf (no visible key) contribute nothing; if every partial is
 * -inf the result is O = 0, LSE = -inf.
 * o_parts: nparts arrays of [R][D]; lse_parts: nparts arrays of [R]; o: [R][D]; lse: [R].
 */
int oracle_merge_partials(int nparts, const double *const *o_parts, const double *const *lse_parts,
                          double *o, double *lse, int64_t R, int D) {
    if (nparts < 1 || R < 0 || D < 1) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        double m = -INFINITY;
        for (int p = 0; p < nparts; ++p)
            if (lse_parts[p][r] > m) m = lse_parts[p][r];
        for (int d = 0; d < D; ++d) o[r * D + d] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int p = 0; p < nparts; ++p) sum += exp(lse_parts[p][r] - m);
        const double L = m + log(sum);
        for (int p = 0; p < nparts; ++p) {
            const double w = exp(lse_parts[p][r] - L);
            for (int d = 0; d < D; ++d) o[r * D + d] += w * o_parts[p][r * D + d];
        }
        lse[r] = L;
    }
    return 0;
}

/*
 * Decode attention over a key/value cache (page "ms-swift长文本训练秘诀：Ulysses并行技术解析",
 * section 5 on deploying the fine-tuned model for 32K-context inference; the computation is
 * the standard attention of page "ms-swift集成FlashAttention 2/3，长文本训练更高效", section
 * "为什么传统注意力这么'吃'显存", for one new query token).  Sequence b has one query token
 * q[b] (all Hq heads) and cache_len[b] cached keys/values; the new token attends to every
 * cached key (it is the last position, so the causal mask hides nothing):
 *     s_j = scale * q_bh . k_bjg,  P = softmax_j(s),  o_bh = sum_j P_j v_bjg,
 *     lse_bh = ln sum_j exp(s_j),  g = h / (Hq/Hkv).
 * cache_len[b] = 0 gives o = 0 and lse = -inf (nothing to attend to).
 * Layouts: q, o [B][Hq][D]; k_cache, v_cache [B][Lmax][Hkv][D]; lse [B][Hq].
 */
int oracle_attn_decode(const double *q, const double *k_cache, const double *v_cache,
                       const int32_t *cache_len, double *o, double *lse, int B, int Hq, int Hkv,
                       int Lmax, int D, double scale) {
    if (B < 1 || Hq < 1 || Hkv < 1 || Lmax < 0 || D < 1 || Hq % Hkv) return 1;
    for (int b = 0; b < B; ++b)
        if (cache_len[b] < 0 || cache_len[b] > Lmax) return 1;
    const int G = Hq / Hkv;
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (Lmax > 0 ? Lmax : 1));
        if (!s) {
#pragma omp atomic write
            err = 2;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < (int64_t)B * Hq; ++r) {
            if (!s) continue;
            const int b = (int)(r / Hq), h = (int)(r % Hq), g = h / G;
            const int L = cache_len[b];
            const double *qi = q + r * D;
            double *orow = o + r * D;
            for (int d = 0; d < D; ++d) orow[d] = 0.0;
            if (L == 0) {
                lse[r] = -INFINITY;
                continue;
            }
            double m = -INFINITY;
            for (int j = 0; j < L; ++j) {
                const double *kj = k_cache + (((int64_t)b * Lmax + j) * Hkv + g) * D;
                double acc = 0.0;
                for (int d = 0; d < D; ++d) acc += qi[d] * kj[d];
                s[j] = scale * acc;
                if (s[j] > m) m = s[j];
            }
            double sum = 0.0;
            for (int j = 0; j < L; ++j) {
                s[j] = exp(s[j] - m);
                sum += s[j];
            }
            for (int j = 0; j < L; ++j) {
                const double pj = s[j] / sum;
                const double *vj = v_cache + (((int64_t)b * Lmax + j) * Hkv + g) * D;
                for (int d = 0; d < D; ++d) orow[d] += pj * vj[d];
            }
            lse[r] = m + log(sum);
        }
        free(s);
    }
    return err;
}

/*
 * Backward of one query/key block pair of a larger attention, given the FULL problem's row
 * statistics (page "ms-swift集成FlashAttention 2/3，长文本训练更高效", section "单靠
 * FlashAttention 不够？那就加上序列并行", subsection "Ring-Attention": with the sequence
 * split across devices, each device computes the part of the result its own queries and the
 * passing key/value block contribute).  With O and LSE of the whole row, the block's share
 * of the gradient is exactly:
 *     P_ij = exp(scale q_i . k_j - LSE_i),  Delta_i = dO_i . O_i,
 *     dS_ij = P_ij (dO_i . v_j - Delta_i),
 *     dQ_i += scale sum_j dS_ij k_j,  dK_j += scale sum_i dS_ij q_i,  dV_j += sum_i P_ij dO_i,
 * summed over the query heads of each kv head; summing the blocks gives the full gradient.
 * Dense batches: q, o, dout, dq [B*S][Hq][D]; k, v, dk, dv [B*S][Hkv][D]; lse [B][Hq][S].
 * causal masks key j for query i when j > i (positions within the block pair: the diagonal
 * block of a causal split).  Outputs are overwritten.
 */
int oracle_attn_bwd_given(const double *q, const double *k, const double *v, const double *o,
                          const double *lse, const double *dout, double *dq, double *dk, double *dv,
                          int B, int Hq, int Hkv, int S, int D, int causal, double scale) {
    if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || D < 1 || Hq % Hkv) return 1;
    const int G = Hq / Hkv;
    memset(dq, 0, sizeof(double) * (size_t)B * S * Hq * D);
    memset(dk, 0, sizeof(double) * (size_t)B * S * Hkv * D);
    memset(dv, 0, sizeof(double) * (size_t)B * S * Hkv * D);
    /* dQ: parallel over query rows */
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t r = 0; r < (int64_t)B * S * Hq; ++r) {
        const int64_t t = r / Hq;
        const int h = (int)(r % Hq), b = (int)(t / S), i = (int)(t % S), g = h / G;
        const double *qi = q + r * D, *oi = o + r * D, *doi = dout + r * D;
        double delta = 0.0;
        for (int d = 0; d < D; ++d) delta += doi[d] * oi[d];
        const double L = lse[((int64_t)b * Hq + h) * S + i];
        double *dqi = dq + r * D;
        const int n = causal ? i + 1 : S;
        for (int j = 0; j < n; ++j) {
            const double *kj = k + (((int64_t)b * S + j) * Hkv + g) * D;
            const double *vj = v + (((int64_t)b * S + j) * Hkv + g) * D;
            double s = 0.0, dp = 0.0;
            for (int d = 0; d < D; ++d) { s += qi[d] * kj[d]; dp += doi[d] * vj[d]; }
            const double p = exp(scale * s - L);
            const double ds = p * (dp - delta);
            for (int d = 0; d < D; ++d) dqi[d] += scale * ds * kj[d];
        }
    }
    /* dK, dV: parallel over key rows */
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t c = 0; c < (int64_t)B * S * Hkv; ++c) {
        const int64_t t = c / Hkv;
        const int g = (int)(c % Hkv), b = (int)(t / S), j = (int)(t % S);
        const double *kj = k + c * D, *vj = v + c * D;
        double *dkj = dk + c * D, *dvj = dv + c * D;
        for (int hh = 0; hh < G; ++hh) {
            const int h = g * G + hh;
            for (int i = causal ? j : 0; i < S; ++i) {
                const int64_t r = ((int64_t)b * S + i) * Hq + h;
                const double *qi = q + r * D, *oi = o + r * D, *doi = dout + r * D;
                double delta = 0.0, s = 0.0, dp = 0.0;
                for (int d = 0; d < D; ++d) {
                    delta += doi[d] * oi[d];
                    s += qi[d] * kj[d];
                    dp += doi[d] * vj[d];
                }
                const double p = exp(scale * s - lse[((int64_t)b * Hq + h) * S + i]);
                const double ds = p * (dp - delta);
                for (int d = 0; d < D; ++d) {
                    dkj[d] += scale * ds * qi[d];
                    dvj[d] += p * doi[d];
                }
            }
        }
    }
    return 0;
}
