/*
 * fp64 CPU oracle for the cluster-attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code with the CUDA kernels.
 *
 * The method is stated on two model cards:
 *   [P1] "Hooshaai/distilbert-sst2-cluster-attention": Architecture Overview,
 *        the data-flow diagram, and "Mathematical Formulation & Derivation"
 *        section 1 (Batch-Wise Lloyd's K-Means Clustering);
 *   [P2] "Hooshaai/svd-sst2-roberta-cluster": section 2.1 (k-means with the
 *        expanded distance), section 3 (tensor execution trace) and section 4
 *        (complexity model).
 *
 * Every step below is the plain definition written out, one (batch, head) at
 * a time, in IEEE double arithmetic with sums taken in index order.  There is
 * no blocking, fusion or reordering.  Readings of points the cards leave open:
 *   - init index floor(k L / K) ([P1] section 1, [P2] section 2.1);
 *   - argmin ties go to the lowest cluster index;
 *   - an empty cluster becomes the zero vector (sum / max(1, count));
 *   - centroids are stored in fp32 between iterations when mu_f32 != 0: the
 *     card's module casts its centroids to float before measuring distances
 *     ([P2] section 5, the k-means routine), so the assignment decision is
 *     taken on fp32 centroids, measured exactly; mu_f32 == 0 keeps them fp64;
 *   - the window holds keys with |i - j| <= floor(W / 2), clipped to [0, L);
 *   - both attention branches scale logits by 1 / sqrt(d) ([P1] diagram: "/8"
 *     for d = 64).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

/* Variants of the module's own code ([P2] section 5), all off by default:
 *   window_module: band |i - j| <= W (the module's radius) and, when W == 0
 *                  or W >= L, no local branch at all (O = gathered);
 *   empty_keep:    an empty cluster keeps its previous centroid;
 *   init_stride:   starting centroid k is query k * max(1, L / K);
 *   soft_gather:   gathered_i = softmax(Q_i mu^T / sqrt(d)) V_cent;
 *   key_valid:     [B][L] bytes (1 = valid) or NULL; invalid keys take no
 *                  weight in either softmax and rows of invalid queries are
 *                  zero (the module fills -10000 and then zeroes them);
 *   H_kv:          number of key/value heads (0 = H); query head h reads key
 *                  and value head h / (H / H_kv). */
typedef struct {
    int window_module, empty_keep, init_stride, soft_gather;
    const uint8_t *key_valid;
    int H_kv;
} oracle_opts;

static const oracle_opts kDefaultOpts = {0, 0, 0, 0, NULL, 0};

/* Starting centroid k is query floor(k L / K) ([P1] section 1). */
static int64_t init_index(int64_t k, int64_t L, int64_t K) { return (k * L) / K; }

/* The module's stride: arange(0, L, max(1, L // K))[:K] (K <= L). */
static int64_t init_index_stride(int64_t k, int64_t L, int64_t K) {
    int64_t step = L / K;
    if (step < 1) step = 1;
    return k * step;
}

static double dot(const double *a, const double *b, int d) {
    double s = 0.0;
    for (int j = 0; j < d; ++j) s += a[j] * b[j];
    return s;
}

/* D_ik = |Q_i|^2 + |mu_k|^2 - 2 Q_i . mu_k  ([P2] section 2.1, expanded form). */
static double sq_distance(const double *q, const double *mu, int d) {
    return dot(q, q, d) + dot(mu, mu, d) - 2.0 * dot(q, mu, d);
}

/* c_i = argmin_k D_ik, the lowest k on ties ([P1] section 1). */
static int32_t assign_one(const double *q, const double *mu, int d, int K) {
    int32_t best = 0;
    double best_d = sq_distance(q, mu, d);
    for (int k = 1; k < K; ++k) {
        double dk = sq_distance(q, mu + (size_t)k * d, d);
        if (dk < best_d) {
            best_d = dk;
            best = k;
        }
    }
    return best;
}

/* mu_k = sum_{c_i = k} Q_i / max(1, count_k)  ([P1] section 1). */
static void update_centroids(const double *Q, const int32_t *c, int L, int d, int K,
                             int mu_f32, double *mu, double *sum, int64_t *cnt, int empty_keep) {
    memset(sum, 0, sizeof(double) * (size_t)K * d);
    memset(cnt, 0, sizeof(int64_t) * (size_t)K);
    for (int i = 0; i < L; ++i) {
        int k = c[i];
        cnt[k] += 1;
        for (int j = 0; j < d; ++j) sum[(size_t)k * d + j] += Q[(size_t)i * d + j];
    }
    for (int k = 0; k < K; ++k) {
        if (empty_keep && cnt[k] == 0) continue;
        double den = (double)(cnt[k] > 1 ? cnt[k] : 1);
        for (int j = 0; j < d; ++j) {
            double m = sum[(size_t)k * d + j] / den;
            mu[(size_t)k * d + j] = mu_f32 ? (double)(float)m : m;
        }
    }
}

/* Batch Lloyd's k-means on one head's queries Q[L][d].  Outputs c^(I) and
 * mu^(I); with iters == 0, c = 0 and mu = mu^(0).  hist (optional) receives
 * c^(t) for t = 1..iters as rows [iters][L]. */
static int kmeans_head(const double *Q, int L, int d, int K, int iters, int mu_f32,
                       int32_t *c, double *mu, int32_t *hist, const oracle_opts *op) {
    double *sum = (double *)malloc(sizeof(double) * (size_t)K * d);
    int64_t *cnt = (int64_t *)malloc(sizeof(int64_t) * (size_t)K);
    if (!sum || !cnt) {
        free(sum);
        free(cnt);
        return ORACLE_ENOMEM;
    }
    for (int k = 0; k < K; ++k) {
        const int64_t row = op->init_stride ? init_index_stride(k, L, K) : init_index(k, L, K);
        const double *src = Q + (size_t)row * d;
        for (int j = 0; j < d; ++j) mu[(size_t)k * d + j] = mu_f32 ? (double)(float)src[j] : src[j];
    }
    for (int i = 0; i < L; ++i) c[i] = 0;
    for (int t = 0; t < iters; ++t) {
        for (int i = 0; i < L; ++i) c[i] = assign_one(Q + (size_t)i * d, mu, d, K);
        if (hist) memcpy(hist + (size_t)t * L, c, sizeof(int32_t) * (size_t)L);
        update_centroids(Q, c, L, d, K, mu_f32, mu, sum, cnt, op->empty_keep);
    }
    free(sum);
    free(cnt);
    return ORACLE_OK;
}

/* Softmax over a list of logits, then the weighted sum of value rows:
 * out = sum_j p_j V[idx_j], p = softmax(z).  Max-subtracted for range only. */
static void softmax_combine(const double *z, int n, const double *V, int d, int first,
                            double *out, double *p) {
    double m = z[0];
    for (int j = 1; j < n; ++j)
        if (z[j] > m) m = z[j];
    double den = 0.0;
    for (int j = 0; j < n; ++j) {
        p[j] = exp(z[j] - m);
        den += p[j];
    }
    for (int t = 0; t < d; ++t) out[t] = 0.0;
    for (int j = 0; j < n; ++j) {
        const double *vr = V + (size_t)(first + j) * d;
        double w = p[j] / den;
        for (int t = 0; t < d; ++t) out[t] += w * vr[t];
    }
}

/* V_cent = softmax(mu K^T / sqrt(d)) V  ([P1] diagram "Centroid Cross-Attention";
 * [P2] section 3). */
static int centroid_attention_head(const double *mu, const double *Kh, const double *Vh,
                                   int L, int d, int K, const uint8_t *kv, double *vcent) {
    double *z = (double *)malloc(sizeof(double) * (size_t)L);
    double *p = (double *)malloc(sizeof(double) * (size_t)L);
    if (!z || !p) {
        free(z);
        free(p);
        return ORACLE_ENOMEM;
    }
    const double s = 1.0 / sqrt((double)d);
    int any_valid = 0;
    for (int j = 0; j < L; ++j) any_valid |= !kv || kv[j];
    for (int k = 0; k < K; ++k) {
        for (int j = 0; j < L; ++j) {
            z[j] = s * dot(mu + (size_t)k * d, Kh + (size_t)j * d, d);
            if (kv && any_valid && !kv[j]) z[j] = -INFINITY; /* no weight on padding keys */
            if (kv && !any_valid) z[j] = 0.0;                /* all padding: uniform weights */
        }
        softmax_combine(z, L, Vh, d, 0, vcent + (size_t)k * d, p);
    }
    free(z);
    free(p);
    return ORACLE_OK;
}

/* Local branch: o_i = softmax_{j in J_i}(Q_i . K_j / sqrt(d)) V, with
 * J_i = { j : |i - j| <= floor(W/2), 0 <= j < L }  ([P1] diagram
 * "Local Sliding-Window Branch"). */
static int window_attention_head(const double *Qh, const double *Kh, const double *Vh,
                                 int L, int d, int r, const uint8_t *kv, double *o) {
    const int64_t span = 2 * (int64_t)r + 1 < L ? 2 * (int64_t)r + 1 : L;
    double *z = (double *)malloc(sizeof(double) * (size_t)span);
    double *p = (double *)malloc(sizeof(double) * (size_t)span);
    if (!z || !p) {
        free(z);
        free(p);
        return ORACLE_ENOMEM;
    }
    const double s = 1.0 / sqrt((double)d);
    for (int i = 0; i < L; ++i) {
        int lo = i - r < 0 ? 0 : i - r;
        int hi = i + r > L - 1 ? L - 1 : i + r;
        int n = hi - lo + 1;
        int any_valid = 0;
        for (int j = 0; j < n; ++j) any_valid |= !kv || kv[lo + j];
        for (int j = 0; j < n; ++j) {
            z[j] = s * dot(Qh + (size_t)i * d, Kh + (size_t)(lo + j) * d, d);
            if (kv && any_valid && !kv[lo + j]) z[j] = -INFINITY;
            if (kv && !any_valid) z[j] = 0.0;
        }
        softmax_combine(z, n, Vh, d, lo, o + (size_t)i * d, p);
    }
    free(z);
    free(p);
    return ORACLE_OK;
}

/* O_i = (1 - alpha) V_cent[c_i] + alpha o_i  ([P1] Architecture Overview). */
static void blend_head(const double *g, const double *o, int L, int d, double alpha, int local,
                       const uint8_t *qv, double *out) {
    for (int i = 0; i < L; ++i)
        for (int t = 0; t < d; ++t) {
            double y = local ? (1.0 - alpha) * g[(size_t)i * d + t] + alpha * o[(size_t)i * d + t]
                             : g[(size_t)i * d + t];
            out[(size_t)i * d + t] = (qv && !qv[i]) ? 0.0 : y;
        }
}

/* Gathered global context: hard V_cent[c_i] ([P1] diagram "Centroid Context
 * Gathering"), or the module's soft assignment softmax(Q_i mu^T / sqrt(d))
 * V_cent ([P2] section 5). */
static int gather_head(const double *Q, const double *mu, const double *vcent, const int32_t *c,
                       int L, int d, int K, int soft, double *g) {
    if (!soft) {
        for (int i = 0; i < L; ++i)
            for (int t = 0; t < d; ++t) g[(size_t)i * d + t] = vcent[(size_t)c[i] * d + t];
        return ORACLE_OK;
    }
    double *z = (double *)malloc(sizeof(double) * (size_t)K);
    double *p = (double *)malloc(sizeof(double) * (size_t)K);
    if (!z || !p) {
        free(z);
        free(p);
        return ORACLE_ENOMEM;
    }
    const double s = 1.0 / sqrt((double)d);
    for (int i = 0; i < L; ++i) {
        for (int k = 0; k < K; ++k) z[k] = s * dot(Q + (size_t)i * d, mu + (size_t)k * d, d);
        softmax_combine(z, K, vcent, d, 0, g + (size_t)i * d, p);
    }
    free(z);
    free(p);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Whole forward over B*H heads, threads over heads.                          */

typedef struct {
    const double *q, *k, *v;
    int H, NH, L, d, K, iters, W, mu_f32;
    double alpha;
    double *out, *centroids;
    int32_t *assign, *hist;
    const int32_t *given_assign; /* non-NULL: skip k-means, use these c^(I) */
    oracle_opts op;
    int tid, nthreads;
    int status;
} fwd_job;

static void *fwd_worker(void *arg) {
    fwd_job *J = (fwd_job *)arg;
    const size_t hd = (size_t)J->L * J->d, kd = (size_t)J->K * J->d;
    double *vcent = (double *)malloc(sizeof(double) * kd);
    double *o = (double *)malloc(sizeof(double) * hd);
    double *gbuf = (double *)malloc(sizeof(double) * hd);
    double *sum = (double *)malloc(sizeof(double) * kd);
    int64_t *cnt = (int64_t *)malloc(sizeof(int64_t) * (size_t)J->K);
    int32_t *c_local = (int32_t *)malloc(sizeof(int32_t) * (size_t)J->L);
    double *mu_local = (double *)malloc(sizeof(double) * kd);
    if (!vcent || !o || !gbuf || !sum || !cnt || !c_local || !mu_local) {
        J->status = ORACLE_ENOMEM;
        goto done;
    }
    const int H_kv = J->op.H_kv > 0 ? J->op.H_kv : J->H;
    const int group = J->H / H_kv;
    for (int h = J->tid; h < J->NH; h += J->nthreads) {
        const int b = h / J->H, hq = h % J->H;
        const int64_t hkv = (int64_t)b * H_kv + hq / group;
        const double *Q = J->q + (size_t)h * hd;
        const double *Kh = J->k + (size_t)hkv * hd, *Vh = J->v + (size_t)hkv * hd;
        const uint8_t *kvalid = J->op.key_valid ? J->op.key_valid + (size_t)b * J->L : NULL;
        int32_t *c = J->assign ? J->assign + (size_t)h * J->L : c_local;
        double *mu = J->centroids ? J->centroids + (size_t)h * kd : mu_local;
        int st;
        if (J->given_assign) {
            /* mu^(I) from the given c^(I): init, then the update rule applied
             * (for empty_keep the previous centroids are not known here, so
             * this form is only used with empty_keep == 0). */
            memcpy(c, J->given_assign + (size_t)h * J->L, sizeof(int32_t) * (size_t)J->L);
            for (int k = 0; k < J->K; ++k) {
                const int64_t row = J->op.init_stride ? init_index_stride(k, J->L, J->K) : init_index(k, J->L, J->K);
                for (int j = 0; j < J->d; ++j) {
                    double x = Q[(size_t)row * J->d + j];
                    mu[(size_t)k * J->d + j] = J->mu_f32 ? (double)(float)x : x;
                }
            }
            if (J->iters > 0) update_centroids(Q, c, J->L, J->d, J->K, J->mu_f32, mu, sum, cnt, J->op.empty_keep);
        } else {
            int32_t *hist = J->hist ? J->hist + (size_t)h * J->iters * J->L : NULL;
            st = kmeans_head(Q, J->L, J->d, J->K, J->iters, J->mu_f32, c, mu, hist, &J->op);
            if (st) {
                J->status = st;
                goto done;
            }
        }
        st = centroid_attention_head(mu, Kh, Vh, J->L, J->d, J->K, kvalid, vcent);
        if (!st) st = gather_head(Q, mu, vcent, c, J->L, J->d, J->K, J->op.soft_gather, gbuf);
        int local = 1, r = J->W / 2;
        if (J->op.window_module) {
            r = J->W;
            local = J->W > 0 && J->W < J->L;
        }
        if (!st && local) st = window_attention_head(Q, Kh, Vh, J->L, J->d, r, kvalid, o);
        if (st) {
            J->status = st;
            goto done;
        }
        if (J->out) blend_head(gbuf, o, J->L, J->d, J->alpha, local, kvalid, J->out + (size_t)h * hd);
    }
done:
    free(vcent);
    free(o);
    free(gbuf);
    free(sum);
    free(cnt);
    free(c_local);
    free(mu_local);
    return NULL;
}

static int run_forward(const double *q, const double *k, const double *v, int B, int H, int L,
                       int d, int K, int iters, int W, double alpha, int mu_f32, double *out,
                       int32_t *assign, double *centroids, int32_t *hist,
                       const int32_t *given_assign, const oracle_opts *op, int nthreads) {
    if (!q || !k || !v || B < 1 || H < 1 || L < 1 || d < 1 || K < 1 || K > L || iters < 0 ||
        W < 0 || !(alpha >= 0.0 && alpha <= 1.0))
        return ORACLE_EINVAL;
    if (op->H_kv < 0 || (op->H_kv > 0 && H % op->H_kv != 0)) return ORACLE_EINVAL;
    int NH = B * H;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > NH) nthreads = NH;
    fwd_job *jobs = (fwd_job *)calloc((size_t)nthreads, sizeof(fwd_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) {
        free(jobs);
        free(th);
        return ORACLE_ENOMEM;
    }
    for (int t = 0; t < nthreads; ++t) {
        fwd_job J = {q, k, v, H, NH, L, d, K, iters, W, mu_f32, alpha, out, centroids,
                     assign, hist, given_assign, *op, t, nthreads, ORACLE_OK};
        jobs[t] = J;
    }
    int started = 0;
    for (int t = 1; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, fwd_worker, &jobs[t]) != 0) break;
        started = t;
    }
    fwd_worker(&jobs[0]);
    int status = ORACLE_OK;
    for (int t = 1; t <= started; ++t) pthread_join(th[t], NULL);
    for (int t = started + 1; t < nthreads; ++t) { /* threads that failed to start: run inline */
        fwd_worker(&jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        if (jobs[t].status) status = jobs[t].status;
    free(jobs);
    free(th);
    return status;
}

/* ------------------------------------------------------------------------ */
/* Exported entry points (all arrays row-major, float64 unless stated).      */

/* Full forward: q [B,H,L,d]; k, v [B,H,L,d] (or [B,H_kv,L,d] with the
 * extended form); out [B,H,L,d]; assign [B,H,L] int32 (may be NULL);
 * centroids [B,H,K,d] (may be NULL); hist [B,H,iters,L] (may be NULL). */
int oracle_forward(const double *q, const double *k, const double *v, int B, int H, int L, int d,
                   int K, int iters, int W, double alpha, int mu_f32, double *out,
                   int32_t *assign, double *centroids, int32_t *hist, int nthreads) {
    return run_forward(q, k, v, B, H, L, d, K, iters, W, alpha, mu_f32, out, assign, centroids,
                       hist, NULL, &kDefaultOpts, nthreads);
}

/* The forward with the module's variants (see oracle_opts).  key_valid is
 * [B][L] bytes or NULL; H_kv = 0 means H. */
int oracle_forward_ex(const double *q, const double *k, const double *v, int B, int H, int L,
                      int d, int K, int iters, int W, double alpha, int mu_f32,
                      int window_module, int empty_keep, int init_stride, int soft_gather,
                      const uint8_t *key_valid, int H_kv, double *out, int32_t *assign,
                      double *centroids, int32_t *hist, int nthreads) {
    oracle_opts op = {window_module, empty_keep, init_stride, soft_gather, key_valid, H_kv};
    return run_forward(q, k, v, B, H, L, d, K, iters, W, alpha, mu_f32, out, assign, centroids,
                       hist, NULL, &op, nthreads);
}

/* The forward evaluated at given final assignments c^(I) [B,H,L]: mu^(I) is the
 * update rule applied to them (mu^(0) when iters == 0), then centroid
 * attention, gather, window and blend. */
int oracle_forward_at(const double *q, const double *k, const double *v, int B, int H, int L,
                      int d, int K, int iters, int W, double alpha, int mu_f32,
                      const int32_t *given_assign, double *out, double *centroids, int nthreads) {
    if (!given_assign) return ORACLE_EINVAL;
    for (size_t i = 0; i < (size_t)B * H * L; ++i)
        if (given_assign[i] < 0 || given_assign[i] >= K) return ORACLE_EINVAL;
    return run_forward(q, k, v, B, H, L, d, K, iters, W, alpha, mu_f32, out, NULL, centroids,
                       NULL, given_assign, &kDefaultOpts, nthreads);
}

/* One head's k-means: q [L,d] -> c [L], mu [K,d], hist [iters,L] (optional). */
int oracle_kmeans(const double *q, int L, int d, int K, int iters, int mu_f32, int32_t *c,
                  double *mu, int32_t *hist) {
    if (!q || !c || !mu || L < 1 || d < 1 || K < 1 || K > L || iters < 0) return ORACLE_EINVAL;
    return kmeans_head(q, L, d, K, iters, mu_f32, c, mu, hist, &kDefaultOpts);
}

/* One head's update rule: given c [L], mu [K,d] = sum / max(1, count). */
int oracle_update(const double *q, const int32_t *c, int L, int d, int K, int mu_f32, double *mu) {
    if (!q || !c || !mu || L < 1 || d < 1 || K < 1) return ORACLE_EINVAL;
    for (int i = 0; i < L; ++i)
        if (c[i] < 0 || c[i] >= K) return ORACLE_EINVAL;
    double *sum = (double *)malloc(sizeof(double) * (size_t)K * d);
    int64_t *cnt = (int64_t *)malloc(sizeof(int64_t) * (size_t)K);
    if (!sum || !cnt) {
        free(sum);
        free(cnt);
        return ORACLE_ENOMEM;
    }
    update_centroids(q, c, L, d, K, mu_f32, mu, sum, cnt, 0);
    free(sum);
    free(cnt);
    return ORACLE_OK;
}

/* One head's distance matrix D [L,K] in the expanded form. */
int oracle_distances(const double *q, const double *mu, int L, int d, int K, double *D) {
    if (!q || !mu || !D || L < 1 || d < 1 || K < 1) return ORACLE_EINVAL;
    for (int i = 0; i < L; ++i)
        for (int k = 0; k < K; ++k)
            D[(size_t)i * K + k] = sq_distance(q + (size_t)i * d, mu + (size_t)k * d, d);
    return ORACLE_OK;
}

/* One head's centroid attention: mu [K,d], k, v [L,d] -> vcent [K,d]. */
int oracle_centroid_attention(const double *mu, const double *k, const double *v, int L, int d,
                              int K, double *vcent) {
    if (!mu || !k || !v || !vcent || L < 1 || d < 1 || K < 1) return ORACLE_EINVAL;
    return centroid_attention_head(mu, k, v, L, d, K, NULL, vcent);
}

/* One head's window attention: q, k, v [L,d] -> o [L,d] over |i-j| <= floor(W/2). */
int oracle_window_attention(const double *q, const double *k, const double *v, int L, int d,
                            int W, double *o) {
    if (!q || !k || !v || !o || L < 1 || d < 1 || W < 0) return ORACLE_EINVAL;
    return window_attention_head(q, k, v, L, d, W / 2, NULL, o);
}
