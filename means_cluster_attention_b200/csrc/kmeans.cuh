// Batch Lloyd's k-means on the queries of every (batch, head).
//
// Model card "Hooshaai/distilbert-sst2-cluster-attention", Mathematical
// Formulation section 1, and "Hooshaai/svd-sst2-roberta-cluster" section 2.1:
// strided init mu_k = Q[floor(k L / K)], then per iteration
//   D_ik = |Q_i|^2 + |mu_k|^2 - 2 Q_i . mu_k,  c_i = argmin_k D_ik,
//   mu_k = sum_{c_i = k} Q_i / max(1, count_k).
//
// Exact decisions.  Centroids are fp32 (each the exact member sum over the
// count, computed in fp64 and rounded once).  The argmin over those fp32
// centroids is decided exactly:
//   * an fp32 pass computes s_k = |mu_k|^2 - 2 Q.mu_k with a rigorous error
//     bound e_k = 2^-16 (|Q| |mu_k| + |mu_k|^2).  Four 16-term FMA chains
//     give a dot-product error below 18 u |Q| |mu_k| (u = 2^-24), the fp32
//     |mu_k|^2 is within 65 u |mu_k|^2, and the final fma adds u |s_k|; the
//     total stays below 2^-16 (...) = 256 u (...) with a wide margin.
//   * the token is settled when exactly one k has s_k - e_k <= min_j (s_j +
//     e_j); otherwise every such candidate is re-measured in fp64 in the
//     expanded form with index-order sums and separately rounded products
//     and sums, and the lowest k with the smallest value wins.
// Member sums are taken in a fixed order, with no floating-point atomics:
// each CTA walks its token range in index order (thread j of a group of 64
// owns coordinate j of the clusters k = group (mod 4)) and writes its partial
// sums to its own slot; the update adds the CTA slots in CTA order.  The
// result is therefore bitwise reproducible for any input.  When a head fits
// one CTA (L <= 1024) the order is the oracle's index order, so the sums are
// bit-identical to it for any fp32 or bf16 input; across CTAs they equal it
// whenever the sums are exact in fp64, which holds for bf16 inputs whose
// non-zero magnitudes lie within 2^-27 .. 16 (L <= 32768), and otherwise
// differ by fp64 rounding only.
#pragma once

#include "common.cuh"

namespace ca {

constexpr float kFilterEps = 1.52587890625e-05f;  // 2^-16
constexpr int kAssignThreads = 256;

// mu^(0)_k = Q[floor(k L / K)] (or Q[k * max(1, L / K)], the module's
// stride, when init_stride), one block per head.
template <typename T>
__global__ void kmeans_init_kernel(const T *__restrict__ q, int L, int K, float *__restrict__ mu,
                                   int init_stride = 0) {
    const int64_t h = blockIdx.x;
    const T *qh = q + h * (int64_t)L * kD;
    float *muh = mu + h * (int64_t)K * kD;
    for (int idx = threadIdx.x; idx < K * kD; idx += blockDim.x) {
        const int k = idx / kD, j = idx % kD;
        const int64_t step = L / K > 1 ? L / K : 1;
        const int64_t row = init_stride ? (int64_t)k * step : ((int64_t)k * L) / K;
        muh[idx] = to_f32(qh[row * kD + j]);
    }
}

__device__ __forceinline__ float dot64_f32(const float (&x)[kD], const float *__restrict__ m) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    const float4 *m4 = reinterpret_cast<const float4 *>(m);
#pragma unroll
    for (int j = 0; j < kD / 4; ++j) {
        const float4 t = m4[j];
        a0 = fmaf(x[4 * j + 0], t.x, a0);
        a1 = fmaf(x[4 * j + 1], t.y, a1);
        a2 = fmaf(x[4 * j + 2], t.z, a2);
        a3 = fmaf(x[4 * j + 3], t.w, a3);
    }
    return (a0 + a1) + (a2 + a3);
}

// Index-order fp64 dot product with separately rounded products and sums.
__device__ __forceinline__ double dot64_f64_ordered(const float (&x)[kD], const float *__restrict__ m) {
    double a = 0.0;
#pragma unroll
    for (int j = 0; j < kD; ++j) a = __dadd_rn(a, __dmul_rn((double)x[j], (double)m[j]));
    return a;
}

// Shared-memory layout of the assignment kernel for K clusters.
struct AssignSmem {
    static __host__ __device__ size_t bytes(int K, int tokens_per_cta) {
        return (size_t)K * kD * sizeof(double)    // member sums
               + (size_t)K * kD * sizeof(float)   // centroids
               + (size_t)K * sizeof(double)       // |mu_k|^2 in fp64, index order
               + (size_t)K * 2 * sizeof(float)    // |mu_k|^2 and |mu_k| in fp32
               + (size_t)K * sizeof(int)          // member counts
               + (size_t)tokens_per_cta;          // the CTA's assignments
    }
};

// One Lloyd iteration's assignment step plus the per-CTA member sums.
// Grid (ceil(L / tokens_per_cta), heads).  Writes c_i to assign (and to hist
// when non-null) and the CTA's member sums / counts to its own slot of
// part_sum [heads][ctas][K][64] / part_cnt [heads][ctas][K].
template <typename T>
__global__ void __launch_bounds__(kAssignThreads)
    kmeans_assign_kernel(const T *__restrict__ q, int L, int K, int tokens_per_cta,
                         const float *__restrict__ mu, int32_t *__restrict__ assign,
                         int32_t *__restrict__ hist, int64_t hist_head_stride,
                         double *__restrict__ part_sum, int32_t *__restrict__ part_cnt) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    double *sum_s = reinterpret_cast<double *>(smem_raw);
    float *mu_s = reinterpret_cast<float *>(sum_s + (size_t)K * kD);
    double *mm64_s = reinterpret_cast<double *>(mu_s + (size_t)K * kD);
    float *mm32_s = reinterpret_cast<float *>(mm64_s + K);
    float *mun_s = mm32_s + K;
    int *cnt_s = reinterpret_cast<int *>(mun_s + K);
    uint8_t *c_s = reinterpret_cast<uint8_t *>(cnt_s + K);  // [tokens_per_cta]

    const int h = blockIdx.y;
    const int t0 = blockIdx.x * tokens_per_cta;
    const int t1 = min(L, t0 + tokens_per_cta);
    const T *qh = q + (int64_t)h * L * kD;
    const float *muh = mu + (int64_t)h * K * kD;

    for (int idx = threadIdx.x; idx < K * kD; idx += blockDim.x) {
        mu_s[idx] = muh[idx];
        sum_s[idx] = 0.0;
    }
    for (int k = threadIdx.x; k < K; k += blockDim.x) cnt_s[k] = 0;
    __syncthreads();
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
        const float *m = mu_s + (size_t)k * kD;
        float a = 0.f;
        double a64 = 0.0;
        for (int j = 0; j < kD; ++j) {
            a = fmaf(m[j], m[j], a);
            a64 = __dadd_rn(a64, __dmul_rn((double)m[j], (double)m[j]));
        }
        mm32_s[k] = a;
        mm64_s[k] = a64;
        mun_s[k] = sqrtf(a);
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    for (int base = t0 + warp * 32; base < t1; base += nwarps * 32) {
        const int i = base + lane;
        const bool valid = i < t1;
        int best = 0;
        if (valid) {
            float qf[kD];
            load_row64(qh + (int64_t)i * kD, qf);
            float qq = 0.f;
#pragma unroll
            for (int j = 0; j < kD; ++j) qq = fmaf(qf[j], qf[j], qq);
            const float qn = sqrtf(qq);
            float ub_min = INFINITY, lb_best = INFINITY, lb_other = INFINITY;
            for (int k = 0; k < K; ++k) {
                const float s = fmaf(-2.f, dot64_f32(qf, mu_s + (size_t)k * kD), mm32_s[k]);
                const float e = kFilterEps * fmaf(qn, mun_s[k], mm32_s[k]) + 1e-30f;
                const float ub = s + e, lb = s - e;
                if (ub < ub_min) {
                    lb_other = fminf(lb_other, lb_best);
                    ub_min = ub;
                    lb_best = lb;
                    best = k;
                } else {
                    lb_other = fminf(lb_other, lb);
                }
            }
            if (lb_other <= ub_min) {
                // Ambiguous: re-measure every candidate exactly.
                double qq64 = 0.0;
#pragma unroll
                for (int j = 0; j < kD; ++j) qq64 = __dadd_rn(qq64, __dmul_rn((double)qf[j], (double)qf[j]));
                int rbest = -1;
                double dbest = 0.0;
                for (int k = 0; k < K; ++k) {
                    const float s = fmaf(-2.f, dot64_f32(qf, mu_s + (size_t)k * kD), mm32_s[k]);
                    const float e = kFilterEps * fmaf(qn, mun_s[k], mm32_s[k]) + 1e-30f;
                    if (s - e > ub_min) continue;
                    const double qm = dot64_f64_ordered(qf, mu_s + (size_t)k * kD);
                    const double D = __dsub_rn(__dadd_rn(qq64, mm64_s[k]), __dmul_rn(2.0, qm));
                    if (rbest < 0 || D < dbest) {
                        dbest = D;
                        rbest = k;
                    }
                }
                if (rbest < 0) {
                    record_error(5, 1);
                    rbest = best;
                }
                best = rbest;
            }
            assign[(int64_t)h * L + i] = best;
            if (hist) hist[(int64_t)h * hist_head_stride + i] = best;
            c_s[i - t0] = (uint8_t)best;
            atomicAdd(&cnt_s[best], 1);
        }
    }
    __syncthreads();
    // Member sums in index order: thread (grp, j) adds coordinate j of every
    // token of a cluster k = grp (mod 4), so each sum has one owner and a
    // fixed order of additions.
    {
        const int grp = threadIdx.x >> 6, j = threadIdx.x & 63;
        for (int i = t0; i < t1; ++i) {
            const int c = CA_IDX(c_s[i - t0], 0, K, 76);
            if ((c & 3) == grp)
                sum_s[(size_t)c * kD + j] = __dadd_rn(sum_s[(size_t)c * kD + j], (double)to_f32(qh[(int64_t)i * kD + j]));
        }
    }
    __syncthreads();
    const int64_t slot = (int64_t)h * gridDim.x + blockIdx.x;
    for (int idx = threadIdx.x; idx < K * kD; idx += blockDim.x) part_sum[slot * K * kD + idx] = sum_s[idx];
    for (int k = threadIdx.x; k < K; k += blockDim.x) part_cnt[slot * K + k] = cnt_s[k];
}

// mu_k = fp32(sum_k / max(1, count_k)) (an empty cluster keeps its previous
// centroid when empty_keep), the CTA slots of the member sums added in CTA
// order.  One block per head.
__global__ void kmeans_update_kernel(int K, int n_cta, const double *__restrict__ part_sum,
                                     const int32_t *__restrict__ part_cnt, float *__restrict__ mu,
                                     float *__restrict__ cent_out, int empty_keep = 0) {
    const int64_t h = blockIdx.x;
    const double *ps = part_sum + h * n_cta * K * kD;
    const int32_t *pc = part_cnt + h * n_cta * K;
    float *m = mu + h * K * kD;
    for (int idx = threadIdx.x; idx < K * kD; idx += blockDim.x) {
        const int k = idx / kD;
        double s = 0.0;
        int c = 0;
        for (int b = 0; b < n_cta; ++b) {
            s = __dadd_rn(s, ps[(int64_t)b * K * kD + idx]);
            c += pc[(int64_t)b * K + k];
        }
        const double v = s / (double)(c > 1 ? c : 1);
        const float f = (empty_keep && c == 0) ? m[idx] : __double2float_rn(v);
        m[idx] = f;
        if (cent_out) cent_out[h * K * kD + idx] = f;
    }
}

}  // namespace ca
