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

/* Starting centroid k is query floor(k L / K) ([P1] section 1). */
static int64_t init_index(int64_t k, int64_t L, int64_t K) { return (k * L) / K; }

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
                             int mu_f32, double *mu, double *sum, int64_t *cnt) {
    memset(sum, 0, sizeof(double) * (size_t)K * d);
    memset(cnt, 0, sizeof(int64_t) * (size_t)K);
    for (int i = 0; i < L; ++i) {
        int k = c[i];
        cnt[k] += 1;
        for (int j = 0; j < d; ++j) sum[(size_t)k * d + j] += Q[(size_t)i * d + j];
    }
    for (int k = 0; k < K; ++k) {
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
                       int32_t *c, double *mu, int32_t *hist) {
    double *sum = (double *)malloc(sizeof(double) * (size_t)K * d);
    int64_t *cnt = (int64_t *)malloc(sizeof(int64_t) * (size_t)K);
    if (!sum || !cnt) {
        free(sum);
        free(cnt);
        return ORACLE_ENOMEM;
    }
    for (int k = 0; k < K; ++k) {
        const double *src = Q + (size_t)init_index(k, L, K) * d;
        for (int j = 0; j < d; ++j) mu[(size_t)k * d + j] = mu_f32 ? (double)(float)src[j] : src[j];
    }
    for (int i = 0; i < L; ++i) c[i] = 0;
    for (int t = 0; t < iters; ++t) {
        for (int i = 0; i < L; ++i) c[i] = assign_one(Q + (size_t)i * d, mu, d, K);
        if (hist) memcpy(hist + (size_t)t * L, c, sizeof(int32_t) * (size_t)L);
        update_centroids(Q, c, L, d, K, mu_f32, mu, sum, cnt);
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
                                   int L, int d, int K, double *vcent) {
    double *z = (double *)malloc(sizeof(double) * (size_t)L);
    double *p = (double *)malloc(sizeof(double) * (size_t)L);
    if (!z || !p) {
        free(z);
        free(p);
        return ORACLE_ENOMEM;
    }
    const double s = 1.0 / sqrt((double)d);
    for (int k = 0; k < K; ++k) {
        for (int j = 0; j < L; ++j) z[j] = s * dot(mu + (size_t)k * d, Kh + (size_t)j * d, d);
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
                                 int L, int d, int W, double *o) {
    const int r = W / 2;
    double *z = (double *)malloc(sizeof(double) * (size_t)(2 * r + 1));
    double *p = (double *)malloc(sizeof(double) * (size_t)(2 * r + 1));
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
        for (int j = 0; j < n; ++j) z[j] = s * dot(Qh + (size_t)i * d, Kh + (size_t)(lo + j) * d, d);
        softmax_combine(z, n, Vh, d, lo, o + (size_t)i * d, p);
    }
    free(z);
    free(p);
    return ORACLE_OK;
}

/* O_i = (1 - alpha) V_cent[c_i] + alpha o_i  ([P1] Architecture Overview). */
static void blend_head(const double *vcent, const int32_t *c, const double *o, int L, int d,
                       double alpha, double *out) {
    for (int i = 0; i < L; ++i)
        for (int t = 0; t < d; ++t)
            out[(size_t)i * d + t] =
                (1.0 - alpha) * vcent[(size_t)c[i] * d + t] + alpha * o[(size_t)i * d + t];
}

/* ------------------------------------------------------------------------ */
/* Whole forward over B*H heads, threads over heads.                          */

typedef struct {
    const double *q, *k, *v;
    int NH, L, d, K, iters, W, mu_f32;
    double alpha;
    double *out, *centroids;
    int32_t *assign, *hist;
    const int32_t *given_assign; /* non-NULL: skip k-means, use these c^(I) */
    int tid, nthreads;
    int status;
} fwd_job;

static void *fwd_worker(void *arg) {
    fwd_job *J = (fwd_job *)arg;
    const size_t hd = (size_t)J->L * J->d, kd = (size_t)J->K * J->d;
    double *vcent = (double *)malloc(sizeof(double) * kd);
    double *o = (double *)malloc(sizeof(double) * hd);
    double *sum = (double *)malloc(sizeof(double) * kd);
    int64_t *cnt = (int64_t *)malloc(sizeof(int64_t) * (size_t)J->K);
    int32_t *c_local = (int32_t *)malloc(sizeof(int32_t) * (size_t)J->L);
    double *mu_local = (double *)malloc(sizeof(double) * kd);
    if (!vcent || !o || !sum || !cnt || !c_local || !mu_local) {
        J->status = ORACLE_ENOMEM;
        goto done;
    }
    for (int h = J->tid; h < J->NH; h += J->nthreads) {
        const double *Q = J->q + (size_t)h * hd, *Kh = J->k + (size_t)h * hd, *Vh = J->v + (size_t)h * hd;
        int32_t *c = J->assign ? J->assign + (size_t)h * J->L : c_local;
        double *mu = J->centroids ? J->centroids + (size_t)h * kd : mu_local;
        int st;
        if (J->given_assign) {
            memcpy(c, J->given_assign + (size_t)h * J->L, sizeof(int32_t) * (size_t)J->L);
            if (J->iters > 0) {
                update_centroids(Q, c, J->L, J->d, J->K, J->mu_f32, mu, sum, cnt);
            } else {
                for (int k = 0; k < J->K; ++k)
                    for (int j = 0; j < J->d; ++j) {
                        double x = Q[(size_t)init_index(k, J->L, J->K) * J->d + j];
                        mu[(size_t)k * J->d + j] = J->mu_f32 ? (double)(float)x : x;
                    }
            }
        } else {
            int32_t *hist = J->hist ? J->hist + (size_t)h * J->iters * J->L : NULL;
            st = kmeans_head(Q, J->L, J->d, J->K, J->iters, J->mu_f32, c, mu, hist);
            if (st) {
                J->status = st;
                goto done;
            }
        }
        st = centroid_attention_head(mu, Kh, Vh, J->L, J->d, J->K, vcent);
        if (!st) st = window_attention_head(Q, Kh, Vh, J->L, J->d, J->W, o);
        if (st) {
            J->status = st;
            goto done;
        }
        if (J->out) blend_head(vcent, c, o, J->L, J->d, J->alpha, J->out + (size_t)h * hd);
    }
done:
    free(vcent);
    free(o);
    free(sum);
    free(cnt);
    free(c_local);
    free(mu_local);
    return NULL;
}

static int run_forward(const double *q, const double *k, const double *v, int B, int H, int L,
                       int d, int K, int iters, int W, double alpha, int mu_f32, double *out,
                       int32_t *assign, double *centroids, int32_t *hist,
                       const int32_t *given_assign, int nthreads) {
    if (!q || !k || !v || B < 1 || H < 1 || L < 1 || d < 1 || K < 1 || K > L || iters < 0 ||
        W < 0 || !(alpha >= 0.0 && alpha <= 1.0))
        return ORACLE_EINVAL;
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
        fwd_job J = {q, k, v, NH, L, d, K, iters, W, mu_f32, alpha, out, centroids,
                     assign, hist, given_assign, t, nthreads, ORACLE_OK};
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

/* Full forward: q, k, v [B,H,L,d]; out [B,H,L,d]; assign [B,H,L] int32 (may be
 * NULL); centroids [B,H,K,d] (may be NULL); hist [B,H,iters,L] (may be NULL). */
int oracle_forward(const double *q, const double *k, const double *v, int B, int H, int L, int d,
                   int K, int iters, int W, double alpha, int mu_f32, double *out,
                   int32_t *assign, double *centroids, int32_t *hist, int nthreads) {
    return run_forward(q, k, v, B, H, L, d, K, iters, W, alpha, mu_f32, out, assign, centroids,
                       hist, NULL, nthreads);
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
                       NULL, given_assign, nthreads);
}

/* One head's k-means: q [L,d] -> c [L], mu [K,d], hist [iters,L] (optional). */
int oracle_kmeans(const double *q, int L, int d, int K, int iters, int mu_f32, int32_t *c,
                  double *mu, int32_t *hist) {
    if (!q || !c || !mu || L < 1 || d < 1 || K < 1 || K > L || iters < 0) return ORACLE_EINVAL;
    return kmeans_head(q, L, d, K, iters, mu_f32, c, mu, hist);
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
    update_centroids(q, c, L, d, K, mu_f32, mu, sum, cnt);
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
    return centroid_attention_head(mu, k, v, L, d, K, vcent);
}

/* One head's window attention: q, k, v [L,d] -> o [L,d]. */
int oracle_window_attention(const double *q, const double *k, const double *v, int L, int d,
                            int W, double *o) {
    if (!q || !k || !v || !o || L < 1 || d < 1 || W < 0) return ORACLE_EINVAL;
    return window_attention_head(q, k, v, L, d, W, o);
}
