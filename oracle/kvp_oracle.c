/*
 * CPU oracle for prefill KV-cache token eviction by S1 * S2 scores.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load this
 * file: only the test-suite, the smoke check and the benchmark's CPU-baseline leg use
 * it. It shares no code with the CUDA library.
 *
 * It is the plain definition, written for a reader to check by eye, in double
 * precision, one (sequence, KV head) at a time (OpenMP over those independent units):
 *
 *   "Preserving Large Activations: The Key to KV Cache Pruning" (SlimKV), Section 3:
 *     Eq. 3  S1[j] = sum over the query heads g of the KV head's GQA group (Section 3.1,
 *                    "grouped-wise" scoring) and over the queries i of the observation
 *                    window of softmax_j(q_{g,i} . k_j / C)
 *     Eq. 4  S2[j] = max over the head dimension of |V[j, :]|
 *     Eq. 5  S[j]  = S1[j] * S2[j]
 *     Listing 1: hyperparameters window_size (w) and max_capacity_prompt (B).
 *   CurDKV rebuttal page (paperhub.cn/paper/klmc4fwPLd), "Clarification of the claims in
 *   Section 3.1": attention is softmax(Q K^T / C) V with C a constant of the dimension;
 *   read here as C = sqrt(d).
 *
 * Readings taken where the pages are silent:
 *   - window query i (0 <= i < w) sits at absolute position p_i = L - w + i and sees keys
 *     j <= p_i (causal prefill);
 *   - B counts every kept position, the w window positions included; the other B - w
 *     are the highest-S positions among j < L - w, ties going to the lower j;
 *   - kept positions are listed in ascending order;
 *   - query head hq belongs to KV head hq / G, G = Hq / Hkv.
 *
 * bf16 inputs arrive as their 16-bit patterns and are widened exactly to double.
 *
 * Selection policies (oracle_select_policy), for the variants the pages name around the
 * method: attention sinks (the CurDKV rebuttal page, "how our method processes the KV
 * cache", step 5: the first s tokens are always kept), the ablations that rank by S1 alone
 * or S2 alone (SlimKV page, the review of Section 4.6), and a pooling "kernel size" (same
 * review; read here as SnapKV's 1-D max pooling of S1 over the positions before the window,
 * the kernel centred on each position, positions past either end left out).
 *
 * CurDKV leverage scores (oracle_leverage), the CurDKV rebuttal page, "A clearer
 * description of Algorithm 1", steps 1-4, for one KV head's K and V (L x d each):
 *   project both rows with the caller's Gaussian G (d x r); a row's leverage score is its
 *   row norm after the projection; the key and value scores are combined and normalised.
 * Readings: the row norm is the squared Euclidean norm (leverage scores are squared row
 * norms); "combined" is the product lk_j * lv_j (as SlimKV combines S1 and S2); the
 * normalisation divides by the sum over the head's L positions (all zero if that is 0).
 *
 * Adaptive per-head budgets (oracle_select_adaptive), the AdaKV scheme the CurDKV
 * rebuttal page describes in "On the sensitivity of the safeguard parameter (alpha)"
 * (Tables 5-6): the heads of a layer share one budget, and alpha sets the share every head
 * keeps for itself. Readings: per sequence, each KV head keeps its w window positions
 * and a floor of f = floor(alpha (B - w)) of its own best candidates (score descending,
 * then position ascending); the other hkv (B - w - f) positions go to the best of all
 * heads' remaining candidates (score descending, then head, then position ascending). The
 * sequence keeps hkv B positions in all, as with a uniform budget.
 *
 * Parity pins (tests): sum_j S1 = G w; closed forms for identical keys and for a
 * single planted key; G = 1, w = 1 against a library softmax; brute force on tiny
 * inputs; selection against a library stable sort; gather against library indexing;
 * pooling against a library sliding maximum and a planted spike; leverage scores against
 * library row norms for an identity projection, a rank-one closed form, brute force on
 * tiny inputs and their invariants (sum 1, scale and permutation).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double widen_bf16(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/*
 * Scores of every position j in [0, L) of every (sequence b, KV head h).
 *   q      [batch, hq, w, d]   bf16 bits, the last w queries of the prefill
 *   k, v   [batch, hkv, L, d]  bf16 bits
 *   s1, s2, score [batch, hkv, L]  double (s1, s2 may be NULL)
 *   lse    [batch, hq, w] double, log-sum-exp of each window query's logits (may be NULL)
 * Returns 0, or -1 on a bad shape.
 */
int oracle_score(int batch, int hq, int hkv, int d, int L, int w,
                 const uint16_t* q, const uint16_t* k, const uint16_t* v,
                 double* s1_out, double* s2_out, double* score, double* lse_out) {
    if (batch < 1 || hkv < 1 || hq % hkv || d < 1 || w < 1 || w > L) return -1;
    const int G = hq / hkv;
    const double C = sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < batch * hkv; ++bh) {
        const int b = bh / hkv, h = bh % hkv;
        const uint16_t* kh = k + (size_t)bh * L * d;
        const uint16_t* vh = v + (size_t)bh * L * d;
        double* s1 = (double*)calloc((size_t)L, sizeof(double));
        double* logit = (double*)malloc((size_t)L * sizeof(double));
        double* qrow = (double*)malloc((size_t)d * sizeof(double));
        double* kd = (double*)malloc((size_t)L * d * sizeof(double));
        for (size_t e = 0; e < (size_t)L * d; ++e) kd[e] = widen_bf16(kh[e]);

        /* Eq. 3: one softmax row per (query head g of the group, window query i). */
        for (int g = 0; g < G; ++g) {
            const int head_q = h * G + g;
            for (int i = 0; i < w; ++i) {
                const uint16_t* qi = q + (((size_t)b * hq + head_q) * w + i) * d;
                for (int c = 0; c < d; ++c) qrow[c] = widen_bf16(qi[c]);
                const int p = L - w + i; /* causal: keys 0..p are visible */
                double mx = -INFINITY;
                for (int j = 0; j <= p; ++j) {
                    double dot = 0.0;
                    for (int c = 0; c < d; ++c) dot += qrow[c] * kd[(size_t)j * d + c];
                    logit[j] = dot / C;
                    if (logit[j] > mx) mx = logit[j];
                }
                double sum = 0.0;
                for (int j = 0; j <= p; ++j) sum += exp(logit[j] - mx);
                const double lse = mx + log(sum);
                if (lse_out) lse_out[((size_t)b * hq + head_q) * w + i] = lse;
                for (int j = 0; j <= p; ++j) s1[j] += exp(logit[j] - lse);
            }
        }
        /* Eq. 4 and Eq. 5. */
        for (int j = 0; j < L; ++j) {
            double m = 0.0;
            for (int c = 0; c < d; ++c) {
                double a = fabs(widen_bf16(vh[(size_t)j * d + c]));
                if (a > m) m = a;
            }
            const size_t o = (size_t)bh * L + j;
            if (s1_out) s1_out[o] = s1[j];
            if (s2_out) s2_out[o] = m;
            score[o] = s1[j] * m;
        }
        free(kd);
        free(qrow);
        free(logit);
        free(s1);
    }
    return 0;
}

typedef struct {
    double s;
    int32_t j;
} cand_t;

/* Higher score first; equal scores: lower position first. */
static int by_score_then_pos(const void* a, const void* b) {
    const cand_t* x = (const cand_t*)a;
    const cand_t* y = (const cand_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

/*
 * Kept positions of every (b, h) row: the w window positions [L-w, L) and the B - w
 * highest-scoring positions of [0, L-w), listed in ascending order.
 *   score [rows, L] double;  idx [rows, B] int32.
 * Returns 0, or -1 on a bad shape.
 */
int oracle_select(int rows, int L, int w, int B, const double* score, int32_t* idx) {
    if (rows < 0 || w < 1 || w > L || B < w || B > L) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
        const double* s = score + (size_t)r * L;
        const int n = L - w, kk = B - w;
        cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
        unsigned char* keep = (unsigned char*)calloc((size_t)L, 1);
        for (int j = 0; j < n; ++j) {
            c[j].s = s[j];
            c[j].j = j;
        }
        qsort(c, (size_t)n, sizeof(cand_t), by_score_then_pos);
        for (int t = 0; t < kk; ++t) keep[c[t].j] = 1;
        for (int j = n; j < L; ++j) keep[j] = 1;
        int32_t* out = idx + (size_t)r * B;
        int t = 0;
        for (int j = 0; j < L; ++j)
            if (keep[j]) out[t++] = j;
        free(keep);
        free(c);
    }
    return 0;
}

/*
 * Compaction: k_out[r, t, :] = k[r, idx[r, t], :] and the same for v, as a copy of the
 * 16-bit patterns.  k, v [rows, L, d];  idx [rows, B];  k_out, v_out [rows, B, d].
 * Returns 0, or -1 if an index lies outside [0, L).
 */
int oracle_compact(int rows, int L, int d, int B, const uint16_t* k, const uint16_t* v,
                   const int32_t* idx, uint16_t* k_out, uint16_t* v_out) {
    for (int r = 0; r < rows; ++r)
        for (int t = 0; t < B; ++t) {
            const int32_t j = idx[(size_t)r * B + t];
            if (j < 0 || j >= L) return -1;
            memcpy(k_out + ((size_t)r * B + t) * d, k + ((size_t)r * L + j) * d, sizeof(uint16_t) * d);
            memcpy(v_out + ((size_t)r * B + t) * d, v + ((size_t)r * L + j) * d, sizeof(uint16_t) * d);
        }
    return 0;
}

/*
 * Kept positions of every row under a selection policy.
 *   s1, s2 [rows, L] double: S1 and S2 (Eq. 3 and Eq. 4)
 *   sinks  s >= 0: positions [0, s) are always kept
 *   kernel k >= 1, odd: S1 is max-pooled over [j - k/2, j + k/2] within [0, L - w)
 *   mode   0: rank by pool(S1) * S2 (Eq. 5 with pooling); 1: by pool(S1); 2: by S2
 *   fp32_key  nonzero: the ranking key is formed in single precision with subnormal
 *             results flushed to zero (the arithmetic of the CUDA path), so that a
 *             selection made on that path's own S1 and S2 can be compared exactly
 *   idx    [rows, B] int32: [0, s), then the B - w - s highest keys among [s, L - w) (equal
 *          keys: lower position first), then the window [L - w, L); ascending
 *   key_out [rows, L] double (may be NULL): the ranking key of every position before the window
 * Returns 0, or -1 on a bad policy (s + w > B, s > L - w, k even or < 1, mode outside 0..2).
 */
int oracle_select_policy(int rows, int L, int w, int B, int sinks, int kernel, int mode,
                         int fp32_key, const double* s1, const double* s2, int32_t* idx,
                         double* key_out) {
    if (rows < 0 || w < 1 || w > L || B < w || B > L) return -1;
    if (sinks < 0 || sinks + w > B || sinks > L - w) return -1;
    if (kernel < 1 || kernel % 2 == 0 || mode < 0 || mode > 2) return -1;
    const int n = L - w, half = kernel / 2;
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
        const double* a = s1 + (size_t)r * L;
        const double* v = s2 + (size_t)r * L;
        double* key = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        for (int j = 0; j < n; ++j) {
            double pooled = a[j];
            for (int t = j - half; t <= j + half; ++t)
                if (t >= 0 && t < n && a[t] > pooled) pooled = a[t];
            double k;
            if (fp32_key) {
                const float pf = (float)pooled, vf = (float)v[j];
                float kf = mode == 0 ? pf * vf : mode == 1 ? pf : vf;
                if (kf != 0.f && fabsf(kf) < 1.17549435e-38f) kf = 0.f;   /* flush subnormals */
                k = (double)kf;
            } else {
                k = mode == 0 ? pooled * v[j] : mode == 1 ? pooled : v[j];
            }
            key[j] = k;
            if (key_out) key_out[(size_t)r * L + j] = k;
        }
        const int nc = n - sinks, kk = B - w - sinks;
        cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)(nc > 0 ? nc : 1));
        unsigned char* keep = (unsigned char*)calloc((size_t)L, 1);
        for (int j = 0; j < nc; ++j) {
            c[j].s = key[sinks + j];
            c[j].j = sinks + j;
        }
        qsort(c, (size_t)nc, sizeof(cand_t), by_score_then_pos);
        for (int j = 0; j < sinks; ++j) keep[j] = 1;
        for (int t = 0; t < kk; ++t) keep[c[t].j] = 1;
        for (int j = n; j < L; ++j) keep[j] = 1;
        int32_t* out = idx + (size_t)r * B;
        int t = 0;
        for (int j = 0; j < L; ++j)
            if (keep[j]) out[t++] = j;
        free(keep);
        free(c);
        free(key);
    }
    return 0;
}

/*
 * CurDKV leverage scores of every position of `rows` (sequence, KV head) rows.
 *   k, v   [rows][L][d] bf16 bits;  g [d][r] bf16 bits
 *   lk, lv [rows][L] squared norms of K_j G and V_j G (may be NULL)
 *   score  [rows][L] lk * lv / sum over the row's positions of lk * lv
 * Returns 0, or -1 on a bad size.
 */
int oracle_leverage(int rows, int L, int d, int r, const uint16_t* k, const uint16_t* v,
                    const uint16_t* g, double* lk, double* lv, double* score) {
    if (rows < 0 || L < 1 || d < 1 || r < 1) return -1;
    double* gd = (double*)malloc(sizeof(double) * (size_t)d * r);
    for (size_t t = 0; t < (size_t)d * r; ++t) gd[t] = widen_bf16(g[t]);
#pragma omp parallel for schedule(dynamic, 1)
    for (int row = 0; row < rows; ++row) {
        const uint16_t* K = k + (size_t)row * L * d;
        const uint16_t* V = v + (size_t)row * L * d;
        double* out = score + (size_t)row * L;
        double total = 0.0;
        for (int j = 0; j < L; ++j) {
            double nk = 0.0, nv = 0.0;
            for (int c = 0; c < r; ++c) {
                double pk = 0.0, pv = 0.0;               /* (K_j G)_c and (V_j G)_c */
                for (int t = 0; t < d; ++t) {
                    pk += widen_bf16(K[(size_t)j * d + t]) * gd[(size_t)t * r + c];
                    pv += widen_bf16(V[(size_t)j * d + t]) * gd[(size_t)t * r + c];
                }
                nk += pk * pk;
                nv += pv * pv;
            }
            if (lk) lk[(size_t)row * L + j] = nk;
            if (lv) lv[(size_t)row * L + j] = nv;
            out[j] = nk * nv;
            total += out[j];
        }
        for (int j = 0; j < L; ++j) out[j] = total > 0.0 ? out[j] / total : 0.0;
    }
    free(gd);
    return 0;
}

typedef struct {
    double s;
    int h, j;
} cand3_t;

static int by_score_head_pos(const void* a, const void* b) {
    const cand3_t* x = (const cand3_t*)a;
    const cand3_t* y = (const cand3_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    if (x->h != y->h) return x->h < y->h ? -1 : 1;
    return x->j < y->j ? -1 : (x->j > y->j);
}

/*
 * Adaptive budgets for `batch` sequences of `hkv` KV heads.
 *   score  [batch][hkv][L]
 *   counts [batch][hkv]      kept positions of each head (window included)
 *   idx    [batch][hkv * B]  each head's kept positions, ascending, heads one after another
 * Returns 0, or -1 on a bad size or alpha outside [0, 1].
 */
int oracle_select_adaptive(int batch, int hkv, int L, int w, int B, double alpha,
                           const double* score, int32_t* idx, int32_t* counts) {
    if (batch < 0 || hkv < 1 || w < 1 || w > L || B < w || B > L) return -1;
    if (!(alpha >= 0.0 && alpha <= 1.0)) return -1;
    const int n = L - w;
    const int f = (int)floor(alpha * (double)(B - w));
    const long long R = (long long)hkv * (B - w - f);
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < batch; ++b) {
        unsigned char* keep = (unsigned char*)calloc((size_t)hkv * L, 1);
        cand_t* c = (cand_t*)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
        cand3_t* pool = (cand3_t*)malloc(sizeof(cand3_t) * (size_t)hkv * (n > 0 ? n : 1));
        long long np = 0;
        for (int h = 0; h < hkv; ++h) {
            const double* row = score + ((size_t)b * hkv + h) * L;
            unsigned char* kr = keep + (size_t)h * L;
            for (int j = 0; j < n; ++j) {
                c[j].s = row[j];
                c[j].j = j;
            }
            qsort(c, (size_t)n, sizeof(cand_t), by_score_then_pos);
            for (int t = 0; t < f; ++t) kr[c[t].j] = 1;          /* the head's floor */
            for (int t = f; t < n; ++t) {                          /* the rest joins the pool */
                pool[np].s = c[t].s;
                pool[np].h = h;
                pool[np].j = c[t].j;
                ++np;
            }
            for (int j = n; j < L; ++j) kr[j] = 1;                 /* the window */
        }
        qsort(pool, (size_t)np, sizeof(cand3_t), by_score_head_pos);
        for (long long t = 0; t < R && t < np; ++t) keep[(size_t)pool[t].h * L + pool[t].j] = 1;
        int32_t* out = idx + (size_t)b * hkv * B;
        long long o = 0;
        for (int h = 0; h < hkv; ++h) {
            int cnt = 0;
            for (int j = 0; j < L; ++j)
                if (keep[(size_t)h * L + j]) {
                    out[o++] = j;
                    ++cnt;
                }
            counts[(size_t)b * hkv + h] = cnt;
        }
        free(pool);
        free(c);
        free(keep);
    }
    return 0;
}
