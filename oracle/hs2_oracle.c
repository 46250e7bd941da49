/*
 * hs2_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 CPU statement of what HySparse2's token-level KV Reuse
 * computes.  Only the tests, the smoke check and the bench's CPU-baseline leg
 * may load this library; the product path never does.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * Source of the method: onedev.kr/papers/146 (HySparse2 summary),
 *   - "How it works": inside each hybrid block the sparse layers reuse the
 *     full-attention layer's KV cache and selection indices unchanged (KV Reuse).
 *   - "What differs": selection is per token (top-k over individual tokens of
 *     the full layer); the recent-token window is always selected first, then
 *     the highest-scoring tokens outside it; the full layers give the sparse
 *     layers their token selection from exact attention scores.
 *   - "How to use": one shared KV head (MQA), NoPE in full and sparse
 *     attention, 128 forced local tokens and 1,024 global tokens; FP8 KV cache
 *     (its efficiency figures are quoted "on an FP8 KV cache basis").
 * Readings where the page is silent (each is listed in the design notes):
 *   score(t,s) = sum over query heads of the softmax probability of key s;
 *   window = the W most recent positions t-W+1..t including t itself;
 *   global candidates are the positions before the window, 0..t-W;
 *   fewer than k candidates -> all of them; ties -> lower index first;
 *   scale = 1/sqrt(d) is passed in; no sink, softcap, bias or dropout;
 *   decode query position is T-1, the cache already holding its own K/V;
 *   an FP8 row is x = scale_row * e4m3(code), one fp32 scale per token.
 *
 * Every floating-point step runs in double from the exact values of the
 * stored bf16 / e4m3 inputs.  Parallelism (OpenMP) only splits independent
 * per-key or per-head work; sums over keys are serial, except the output sum
 * of a full-attention row, which adds 64 fixed key ranges in order so the
 * result does not depend on the thread count.
 *
 * Parity pins for each function live in tests/test_oracle_*.py: brute force
 * on tiny inputs, closed forms (all keys equal, L = 1), invariants (per-row
 * probability mass summed over heads = Hq, window inside the selection,
 * W+k >= t+1 makes the sparse layer equal full attention), library routines
 * (float64 scaled-dot-product attention, full sort, torch's e4m3 cast) and
 * planted-needle recovery.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define KV_BF16 0
#define KV_E4M3 1
#define O_CHUNKS 64

/* ---------------------------------------------------------------- formats */

/* bf16: the upper 16 bits of an IEEE-754 binary32 value. */
double hs2o_bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* e4m3 (OCP FP8, "fn" variant): 1 sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits; exponent field 0 is subnormal (value = m/8 * 2^-6);
 * S.1111.111 is NaN; there are no infinities; largest finite is 448. */
double hs2o_e4m3_value(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* A view of one KV tensor [rows, d] (bf16, or e4m3 codes with per-row fp32 scale). */
typedef struct {
    int dtype;
    const void* base;
    const float* scale;
    int d;
} kv_view;

static void load_row(const kv_view* v, int64_t row, double* out) {
    if (v->dtype == KV_BF16) {
        const uint16_t* p = (const uint16_t*)v->base + row * (int64_t)v->d;
        for (int i = 0; i < v->d; i++) out[i] = hs2o_bf16_value(p[i]);
    } else {
        const uint8_t* p = (const uint8_t*)v->base + row * (int64_t)v->d;
        double s = (double)v->scale[row];
        for (int i = 0; i < v->d; i++) out[i] = s * hs2o_e4m3_value(p[i]);
    }
}

/* ------------------------------------------------------ full attention row */

/*
 * Exact causal attention of one query position t over keys 0..t of one
 * sequence (MQA: every head reads the same K and V rows).
 *   l_h(s)   = scale * <q_h, k_s>
 *   lse_h    = log sum_s exp(l_h(s))          (max-shifted for range)
 *   P_h(s)   = exp(l_h(s) - lse_h)
 *   O_h      = sum_s P_h(s) v_s
 *   score(s) = sum_h P_h(s)
 * q: [Hq][d] doubles; K/V views are offset to the sequence's first row.
 * logit: work array [Hq][t+1]; score: [t+1].
 */
static void attend_row(int Hq, int d, double scale, const double* q, const kv_view* K,
                       const kv_view* V, int64_t t, double* lse, double* o, double* score,
                       double* logit) {
    int64_t n = t + 1;
#pragma omp parallel
    {
        double* row = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(static)
        for (int64_t s = 0; s < n; s++) {
            load_row(K, s, row);
            for (int h = 0; h < Hq; h++) {
                double acc = 0.0;
                for (int i = 0; i < d; i++) acc += q[h * d + i] * row[i];
                logit[h * n + s] = scale * acc;
            }
        }
        free(row);
    }
#pragma omp parallel for schedule(static)
    for (int h = 0; h < Hq; h++) {
        double m = -INFINITY;
        for (int64_t s = 0; s < n; s++)
            if (logit[h * n + s] > m) m = logit[h * n + s];
        double sum = 0.0;
        for (int64_t s = 0; s < n; s++) sum += exp(logit[h * n + s] - m);
        lse[h] = m + log(sum);
    }
    /* probabilities, head-summed score */
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < n; s++) {
        double acc = 0.0;
        for (int h = 0; h < Hq; h++) {
            double p = exp(logit[h * n + s] - lse[h]);
            logit[h * n + s] = p; /* logit now holds P_h(s) */
            acc += p;
        }
        score[s] = acc;
    }
    /* O_h = sum_s P_h(s) v_s: the keys are cut into O_CHUNKS fixed ranges
     * (independent of the thread count), each summed in ascending s, and the
     * range sums are added in ascending order. */
    double* part = (double*)calloc((size_t)O_CHUNKS * Hq * d, sizeof(double));
#pragma omp parallel
    {
        double* row = (double*)malloc(sizeof(double) * d);
#pragma omp for schedule(dynamic, 1)
        for (int c = 0; c < O_CHUNKS; c++) {
            double* acc = part + (size_t)c * Hq * d;
            int64_t s0 = n * c / O_CHUNKS, s1 = n * (c + 1) / O_CHUNKS;
            for (int64_t s = s0; s < s1; s++) {
                load_row(V, s, row);
                for (int h = 0; h < Hq; h++) {
                    double p = logit[h * n + s];
                    for (int i = 0; i < d; i++) acc[h * d + i] += p * row[i];
                }
            }
        }
        free(row);
    }
    memset(o, 0, sizeof(double) * Hq * d);
    for (int c = 0; c < O_CHUNKS; c++)
        for (int i = 0; i < Hq * d; i++) o[i] += part[(size_t)c * Hq * d + i];
    free(part);
}

/* ---------------------------------------------------------------- top-k  */

typedef struct {
    double score;
    int64_t s;
} cand;

/* order: higher score first; equal scores -> lower index first */
static int cand_cmp(const void* a, const void* b) {
    const cand* x = (const cand*)a;
    const cand* y = (const cand*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->s < y->s) ? -1 : (x->s > y->s);
}

/*
 * Selection of query position t: window {max(0,t-W+1)..t} in ascending
 * order, then the k best candidates among 0..t-W by (score desc, index asc),
 * or all candidates when there are at most k of them (ascending); the rest
 * of the W+k slots is -1.  sel_score gets the score of every selected slot
 * (NaN for padding); *sigma_k the k-th global score when a cut was made,
 * else -1.
 */
static void select_row(int64_t t, int W, int k, const double* score, int32_t* idx,
                       double* sel_score, double* sigma_k) {
    int S = W + k;
    int j = 0;
    int64_t w0 = t - W + 1;
    if (w0 < 0) w0 = 0;
    for (int64_t s = w0; s <= t; s++, j++) {
        idx[j] = (int32_t)s;
        sel_score[j] = score[s];
    }
    int64_t nc = t - W + 1; /* candidates 0..t-W */
    if (nc < 0) nc = 0;
    *sigma_k = -1.0;
    if (nc <= k) {
        for (int64_t s = 0; s < nc; s++, j++) {
            idx[j] = (int32_t)s;
            sel_score[j] = score[s];
        }
    } else {
        cand* c = (cand*)malloc(sizeof(cand) * nc);
        for (int64_t s = 0; s < nc; s++) {
            c[s].score = score[s];
            c[s].s = s;
        }
        qsort(c, (size_t)nc, sizeof(cand), cand_cmp);
        for (int i = 0; i < k; i++, j++) {
            idx[j] = (int32_t)c[i].s;
            sel_score[j] = c[i].score;
        }
        *sigma_k = c[k - 1].score;
        free(c);
    }
    for (; j < S; j++) {
        idx[j] = -1;
        sel_score[j] = NAN;
    }
}

static void load_query(const uint16_t* q, int Hq, int d, double* out) {
    for (int i = 0; i < Hq * d; i++) out[i] = hs2o_bf16_value(q[i]);
}

/* probe scores: for each requested index p (or -1), score[p] (NaN for -1 / out of range) */
static void probe_row(int64_t t, const double* score, int n_probe, const int32_t* probe,
                      double* out) {
    for (int i = 0; i < n_probe; i++) {
        int32_t p = probe[i];
        out[i] = (p >= 0 && p <= t) ? score[p] : NAN;
    }
}

/* ------------------------------------------------------------ public API */

/*
 * Full-attention layer with selection (prefill), evaluated on a list of
 * query rows.  q [B,L,Hq,d] bf16 bits; k, v [B,L,d] bf16 bits.
 * rows[r] = b*L + t.  Outputs per row r:
 *   o [r][Hq][d], lse [r][Hq], idx [r][W+k], sel_score [r][W+k], sigma_k [r],
 *   probe_score [r][n_probe] = score(t, probe_idx[r][i]) (optional, n_probe may be 0),
 *   score_row [r][L] = the whole score row (optional, NULL to skip; -1 beyond t).
 */
int hs2o_full_select(int B, int L, int Hq, int d, int W, int k, double scale,
                     const uint16_t* q, const uint16_t* kk, const uint16_t* v, int64_t n_rows,
                     const int64_t* rows, double* o, double* lse, int32_t* idx,
                     double* sel_score, double* sigma_k, int n_probe,
                     const int32_t* probe_idx, double* probe_score, double* score_row) {
    if (B <= 0 || L <= 0 || Hq <= 0 || d <= 0 || W < 1 || k < 0) return 1;
    int S = W + k;
    double* qd = (double*)malloc(sizeof(double) * Hq * d);
    double* score = (double*)malloc(sizeof(double) * L);
    double* logit = (double*)malloc(sizeof(double) * (size_t)Hq * L);
    for (int64_t r = 0; r < n_rows; r++) {
        int64_t b = rows[r] / L, t = rows[r] % L;
        if (b < 0 || b >= B) continue;
        kv_view K = {KV_BF16, (const uint16_t*)kk + b * (int64_t)L * d, NULL, d};
        kv_view V = {KV_BF16, (const uint16_t*)v + b * (int64_t)L * d, NULL, d};
        load_query(q + rows[r] * (int64_t)Hq * d, Hq, d, qd);
        attend_row(Hq, d, scale, qd, &K, &V, t, lse + r * Hq, o + r * Hq * d, score, logit);
        select_row(t, W, k, score, idx + r * S, sel_score + r * S, sigma_k + r);
        if (n_probe > 0 && probe_idx && probe_score)
            probe_row(t, score, n_probe, probe_idx + r * n_probe, probe_score + r * n_probe);
        if (score_row) {
            for (int64_t s = 0; s < L; s++) score_row[r * L + s] = (s <= t) ? score[s] : -1.0;
        }
    }
    free(qd);
    free(score);
    free(logit);
    return 0;
}

/*
 * Exact softmax attention of one query over a given index set (entries < 0
 * are ignored; an entry may not repeat).  Returns 0, or 2 if the set is empty.
 */
static int sparse_row(int Hq, int d, double scale, const double* q, const kv_view* K,
                      const kv_view* V, int S, const int32_t* sel, double* o, double* krow,
                      double* logit) {
    int n = 0;
    for (int j = 0; j < S; j++) {
        if (sel[j] < 0) continue;
        load_row(K, sel[j], krow);
        for (int h = 0; h < Hq; h++) {
            double acc = 0.0;
            for (int i = 0; i < d; i++) acc += q[h * d + i] * krow[i];
            logit[h * S + n] = scale * acc;
        }
        n++;
    }
    memset(o, 0, sizeof(double) * Hq * d);
    if (n == 0) return 2;
    for (int h = 0; h < Hq; h++) {
        double m = -INFINITY;
        for (int j = 0; j < n; j++)
            if (logit[h * S + j] > m) m = logit[h * S + j];
        double sum = 0.0;
        for (int j = 0; j < n; j++) sum += exp(logit[h * S + j] - m);
        for (int j = 0; j < n; j++) logit[h * S + j] = exp(logit[h * S + j] - m) / sum;
    }
    int jj = 0;
    for (int j = 0; j < S; j++) {
        if (sel[j] < 0) continue;
        load_row(V, sel[j], krow);
        for (int h = 0; h < Hq; h++) {
            double p = logit[h * S + jj];
            for (int i = 0; i < d; i++) o[h * d + i] += p * krow[i];
        }
        jj++;
    }
    return 0;
}

/*
 * Sparse layer (prefill): each query row attends to the K/V rows its index
 * set names, with its own queries; K/V are the full layer's cache, reused
 * unchanged.  q [B,L,Hq,d] bf16; k, v [B,L,d] (bf16, or e4m3 codes with
 * k_scale/v_scale [B,L]); idx [B*L][S].  Output o [r][Hq][d] for rows[r].
 */
int hs2o_sparse(int B, int L, int Hq, int d, double scale, const uint16_t* q, int kv_dtype,
                const void* kk, const void* v, const float* k_scale, const float* v_scale, int S,
                const int32_t* idx, int64_t n_rows, const int64_t* rows, double* o) {
    if (B <= 0 || L <= 0 || Hq <= 0 || d <= 0 || S <= 0) return 1;
    int rc = 0;
    size_t esz = kv_dtype == KV_BF16 ? 2 : 1;
#pragma omp parallel
    {
        double* qd = (double*)malloc(sizeof(double) * Hq * d);
        double* krow = (double*)malloc(sizeof(double) * d);
        double* logit = (double*)malloc(sizeof(double) * (size_t)Hq * S);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; r++) {
            int64_t b = rows[r] / L;
            int64_t off = b * (int64_t)L;
            kv_view K = {kv_dtype, (const char*)kk + off * d * esz, k_scale ? k_scale + off : NULL, d};
            kv_view V = {kv_dtype, (const char*)v + off * d * esz, v_scale ? v_scale + off : NULL, d};
            load_query(q + rows[r] * (int64_t)Hq * d, Hq, d, qd);
            int e = sparse_row(Hq, d, scale, qd, &K, &V, S, idx + rows[r] * S, o + r * Hq * d,
                               krow, logit);
            if (e) {
#pragma omp atomic write
                rc = e;
            }
        }
        free(qd);
        free(krow);
        free(logit);
    }
    return rc;
}

/*
 * Decode: one new query per sequence at position t = lengths[b]-1; the cache
 * rows 0..t already hold its own K/V.  Same definitions as the prefill row.
 * q [B,Hq,d] bf16; caches [B,Tmax,d] (bf16, or e4m3 with scales [B,Tmax]).
 * Outputs o [B][Hq][d], lse [B][Hq], idx/sel_score [B][W+k], sigma_k [B],
 * probe_score [B][n_probe] (optional).
 */
int hs2o_decode_select(int B, int Tmax, int Hq, int d, int W, int k, double scale,
                       const uint16_t* q, int kv_dtype, const void* kc, const void* vc,
                       const float* k_scale, const float* v_scale, const int32_t* lengths,
                       double* o, double* lse, int32_t* idx, double* sel_score, double* sigma_k,
                       int n_probe, const int32_t* probe_idx, double* probe_score) {
    if (B <= 0 || Tmax <= 0 || Hq <= 0 || d <= 0 || W < 1 || k < 0) return 1;
    int S = W + k;
    size_t esz = kv_dtype == KV_BF16 ? 2 : 1;
    double* qd = (double*)malloc(sizeof(double) * Hq * d);
    double* score = (double*)malloc(sizeof(double) * Tmax);
    double* logit = (double*)malloc(sizeof(double) * (size_t)Hq * Tmax);
    int rc = 0;
    for (int b = 0; b < B; b++) {
        int64_t T = lengths[b];
        if (T < 1 || T > Tmax) {
            rc = 1;
            continue;
        }
        int64_t off = (int64_t)b * Tmax;
        kv_view K = {kv_dtype, (const char*)kc + off * d * esz, k_scale ? k_scale + off : NULL, d};
        kv_view V = {kv_dtype, (const char*)vc + off * d * esz, v_scale ? v_scale + off : NULL, d};
        load_query(q + (int64_t)b * Hq * d, Hq, d, qd);
        attend_row(Hq, d, scale, qd, &K, &V, T - 1, lse + b * Hq, o + (int64_t)b * Hq * d, score,
                   logit);
        select_row(T - 1, W, k, score, idx + (int64_t)b * S, sel_score + (int64_t)b * S,
                   sigma_k + b);
        if (n_probe > 0 && probe_idx && probe_score)
            probe_row(T - 1, score, n_probe, probe_idx + (int64_t)b * n_probe,
                      probe_score + (int64_t)b * n_probe);
    }
    free(qd);
    free(score);
    free(logit);
    return rc;
}

/*
 * Decode sparse layer: sequence b's query attends to the cache rows idx[b]
 * names (entries < 0 ignored).  Output o [B][Hq][d].
 */
int hs2o_decode_sparse(int B, int Tmax, int Hq, int d, double scale, const uint16_t* q,
                       int kv_dtype, const void* kc, const void* vc, const float* k_scale,
                       const float* v_scale, int S, const int32_t* idx, double* o) {
    if (B <= 0 || Tmax <= 0 || Hq <= 0 || d <= 0 || S <= 0) return 1;
    int rc = 0;
    size_t esz = kv_dtype == KV_BF16 ? 2 : 1;
#pragma omp parallel
    {
        double* qd = (double*)malloc(sizeof(double) * Hq * d);
        double* krow = (double*)malloc(sizeof(double) * d);
        double* logit = (double*)malloc(sizeof(double) * (size_t)Hq * S);
#pragma omp for schedule(dynamic, 1)
        for (int b = 0; b < B; b++) {
            int64_t off = (int64_t)b * Tmax;
            kv_view K = {kv_dtype, (const char*)kc + off * d * esz, k_scale ? k_scale + off : NULL, d};
            kv_view V = {kv_dtype, (const char*)vc + off * d * esz, v_scale ? v_scale + off : NULL, d};
            load_query(q + (int64_t)b * Hq * d, Hq, d, qd);
            int e = sparse_row(Hq, d, scale, qd, &K, &V, S, idx + (int64_t)b * S,
                               o + (int64_t)b * Hq * d, krow, logit);
            if (e) {
#pragma omp atomic write
                rc = e;
            }
        }
        free(qd);
        free(krow);
        free(logit);
    }
    return rc;
}

int hs2o_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
