// Centroid cross-attention and the fused gather + window attention + blend.
//
// Model card "Hooshaai/distilbert-sst2-cluster-attention", data-flow diagram:
//   V_cent = softmax(mu K^T / sqrt(d)) V                  (centroid branch)
//   V_gathered_i = V_cent[c_i]                            (gather)
//   O_local = LocalAttn(Q, K, V, W)                       (window branch)
//   O = (1 - alpha) V_gathered + alpha O_local            (convex fusion)
// The window holds keys with |i - j| <= floor(W / 2), clipped to [0, L).
#pragma once

#include "common.cuh"

namespace ca {

constexpr int kCaThreads = 256;
constexpr int kCaTile = 64;       // keys per shared-memory tile
constexpr int kCaChunk = 512;     // keys per CTA (one partial softmax state)
constexpr int kCaMaxPerWarp = kMaxK / (kCaThreads / 32);

__host__ __device__ inline size_t centroid_attn_smem_bytes(int K) {
    return (size_t)K * kD * sizeof(float) + (size_t)kCaTile * (kD + 1) * sizeof(float) +
           (size_t)kCaTile * kD * sizeof(float);
}

// Partial softmax state of every centroid over one chunk of keys.
// part layout [head][chunk][K][kD + 2]: kD accumulator values, then the
// running max m and the running denominator l.
template <typename T>
__global__ void __launch_bounds__(kCaThreads)
    centroid_attn_partial_kernel(const T *__restrict__ kmat, const T *__restrict__ vmat, int L,
                                 int K, float scale, const float *__restrict__ mu, int n_chunks,
                                 float *__restrict__ part, Variant var = Variant()) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *mu_s = reinterpret_cast<float *>(smem_raw);
    float *ks = mu_s + (size_t)K * kD;            // [kCaTile][kD + 1]
    float *vs = ks + (size_t)kCaTile * (kD + 1);  // [kCaTile][kD]

    const int h = blockIdx.y, chunk = blockIdx.x;
    const int j0 = chunk * kCaChunk, j1 = min(L, j0 + kCaChunk);
    const int64_t hkv = var.kv_head(h);
    const T *kh = kmat + hkv * L * kD;
    const T *vh = vmat + hkv * L * kD;
    // Key-padding mask: invalid keys take no weight; a row with no valid key
    // at all gives every key the same weight (the module's all -10000 row).
    const uint8_t *kvp = var.key_valid ? var.key_valid + var.batch(h) * L : nullptr;
    int any_valid = 1;
    if (kvp) {
        int mine = 0;
        for (int j = threadIdx.x; j < L; j += blockDim.x) mine |= kvp[j];
        any_valid = __syncthreads_or(mine);
    }
    for (int idx = threadIdx.x; idx < K * kD; idx += blockDim.x) mu_s[idx] = mu[(int64_t)h * K * kD + idx];

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float m_r[kCaMaxPerWarp], l_r[kCaMaxPerWarp], a0_r[kCaMaxPerWarp], a1_r[kCaMaxPerWarp];
#pragma unroll
    for (int c = 0; c < kCaMaxPerWarp; ++c) {
        m_r[c] = -INFINITY;
        l_r[c] = 0.f;
        a0_r[c] = 0.f;
        a1_r[c] = 0.f;
    }

    for (int tb = j0; tb < j1; tb += kCaTile) {
        const int nt = min(kCaTile, j1 - tb);
        __syncthreads();
        for (int idx = threadIdx.x; idx < kCaTile * kD; idx += blockDim.x) {
            const int r = idx / kD, t = idx % kD;
            float kv = 0.f, vv = 0.f;
            if (r < nt) {
                kv = to_f32(kh[(int64_t)(tb + r) * kD + t]);
                vv = to_f32(vh[(int64_t)(tb + r) * kD + t]);
            }
            ks[r * (kD + 1) + t] = kv;
            vs[r * kD + t] = vv;
        }
        __syncthreads();
#pragma unroll
        for (int c = 0; c < kCaMaxPerWarp; ++c) {
            const int k = warp + c * (kCaThreads / 32);
            if (k >= K) break;
            const float *mk = mu_s + (size_t)k * kD;
            float z0 = 0.f, z1 = 0.f;
#pragma unroll 16
            for (int t = 0; t < kD; ++t) {
                const float mt = mk[t];
                z0 = fmaf(mt, ks[lane * (kD + 1) + t], z0);
                z1 = fmaf(mt, ks[(lane + 32) * (kD + 1) + t], z1);
            }
            z0 = lane < nt ? z0 * scale : -INFINITY;
            z1 = lane + 32 < nt ? z1 * scale : -INFINITY;
            if (kvp) {
                if (lane < nt) z0 = any_valid ? (kvp[tb + lane] ? z0 : -INFINITY) : 0.f;
                if (lane + 32 < nt) z1 = any_valid ? (kvp[tb + lane + 32] ? z1 : -INFINITY) : 0.f;
            }
            const float tmax = warp_max(fmaxf(z0, z1));
            const float m_new = fmaxf(m_r[c], tmax);
            const float corr = expf(m_r[c] - m_new);
            const float p0 = expf(z0 - m_new), p1 = expf(z1 - m_new);
            l_r[c] = l_r[c] * corr + warp_sum(p0 + p1);
            float a0 = a0_r[c] * corr, a1 = a1_r[c] * corr;
            for (int jj = 0; jj < nt; ++jj) {
                const float p = __shfl_sync(0xffffffffu, jj < 32 ? p0 : p1, jj & 31);
                a0 = fmaf(p, vs[jj * kD + 2 * lane], a0);
                a1 = fmaf(p, vs[jj * kD + 2 * lane + 1], a1);
            }
            a0_r[c] = a0;
            a1_r[c] = a1;
            m_r[c] = m_new;
        }
    }
#pragma unroll
    for (int c = 0; c < kCaMaxPerWarp; ++c) {
        const int k = warp + c * (kCaThreads / 32);
        if (k >= K) break;
        float *p = part + (((int64_t)h * n_chunks + chunk) * K + k) * (kD + 2);
        p[2 * lane] = a0_r[c];
        p[2 * lane + 1] = a1_r[c];
        if (lane == 0) {
            p[kD] = m_r[c];
            p[kD + 1] = l_r[c];
        }
    }
}

// V_cent = combination of the chunk states in chunk order.  One block per head.
__global__ void centroid_attn_combine_kernel(int K, int n_chunks, const float *__restrict__ part,
                                             float *__restrict__ vcent) {
    const int64_t h = blockIdx.x;
    for (int idx = threadIdx.x; idx < K * kD; idx += blockDim.x) {
        const int k = idx / kD, t = idx % kD;
        float M = -INFINITY;
        for (int c = 0; c < n_chunks; ++c) M = fmaxf(M, part[((h * n_chunks + c) * K + k) * (kD + 2) + kD]);
        float lsum = 0.f, acc = 0.f;
        for (int c = 0; c < n_chunks; ++c) {
            const float *p = part + ((h * n_chunks + c) * K + k) * (kD + 2);
            const float w = expf(p[kD] - M);
            lsum = fmaf(p[kD + 1], w, lsum);
            acc = fmaf(p[t], w, acc);
        }
        vcent[(h * K + k) * kD + t] = acc / lsum;
    }
}

constexpr int kWinQ = 64;  // queries per CTA, four threads per query
constexpr int kWinThreads = kWinQ * 4;

__host__ __device__ inline size_t window_smem_bytes() {
    return (size_t)kCaTile * (kD + 1) * sizeof(float) + (size_t)kCaTile * kD * sizeof(float);
}

// o_i = softmax_{j in J_i}(s Q_i . K_j) V_j over the clipped window, then
// out_i = (1 - alpha) V_cent[c_i] + alpha o_i in the output type.
template <typename T>
__global__ void __launch_bounds__(kWinThreads)
    window_blend_kernel(const T *__restrict__ q, const T *__restrict__ kmat,
                        const T *__restrict__ vmat, int L, int K, int r, float scale, float alpha,
                        const float *__restrict__ vcent, const int32_t *__restrict__ assign,
                        T *__restrict__ out, Variant var = Variant()) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *ks = reinterpret_cast<float *>(smem_raw);  // [kCaTile][kD + 1]
    float *vs = ks + (size_t)kCaTile * (kD + 1);      // [kCaTile][kD]

    const int h = blockIdx.y, i0 = blockIdx.x * kWinQ;
    const int qi = i0 + threadIdx.x / 4, sub = threadIdx.x & 3;
    const unsigned gmask = 0xFu << (threadIdx.x & 28);
    const bool valid = qi < L;
    const int64_t hoff = (int64_t)h * L * kD;
    const int64_t kvoff = var.kv_head(h) * L * kD;
    const uint8_t *kvp = var.key_valid ? var.key_valid + var.batch(h) * L : nullptr;

    float qf[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) qf[t] = valid ? to_f32(q[hoff + (int64_t)qi * kD + 16 * sub + t]) : 0.f;
    const int lo_q = max(0, qi - r), hi_q = min(L - 1, qi + r);
    int band_any = 1;  // some valid key in this query's window
    if (kvp && valid) {
        band_any = 0;
        for (int j = lo_q; j <= hi_q && !band_any; ++j) band_any = kvp[j];
    }
    const int i_last = min(L - 1, i0 + kWinQ - 1);
    const int lo = max(0, i0 - r), hi = min(L - 1, i_last + r);

    float m = -INFINITY, l = 0.f, acc[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) acc[t] = 0.f;

    for (int tb = lo; tb <= hi && var.local; tb += kCaTile) {
        const int nt = min(kCaTile, hi - tb + 1);
        __syncthreads();
        for (int idx = threadIdx.x; idx < kCaTile * kD; idx += blockDim.x) {
            const int rr = idx / kD, t = idx % kD;
            float kv = 0.f, vv = 0.f;
            if (rr < nt) {
                kv = to_f32(kmat[kvoff + (int64_t)(tb + rr) * kD + t]);
                vv = to_f32(vmat[kvoff + (int64_t)(tb + rr) * kD + t]);
            }
            ks[rr * (kD + 1) + t] = kv;
            vs[rr * kD + t] = vv;
        }
        __syncthreads();
        if (valid) {
            const int jb = max(lo_q, tb), je = min(hi_q, tb + nt - 1);
            for (int j = jb; j <= je; ++j) {
                if (kvp && band_any && !kvp[j]) continue;
                const float *kr = ks + (j - tb) * (kD + 1) + 16 * sub;
                float part = 0.f;
#pragma unroll
                for (int t = 0; t < 16; ++t) part = fmaf(qf[t], kr[t], part);
                part += __shfl_xor_sync(gmask, part, 1);
                part += __shfl_xor_sync(gmask, part, 2);
                const float z = (kvp && !band_any) ? 0.f : part * scale;
                if (z > m) {
                    const float corr = expf(m - z);
                    l *= corr;
#pragma unroll
                    for (int t = 0; t < 16; ++t) acc[t] *= corr;
                    m = z;
                }
                const float p = expf(z - m);
                l += p;
                const float *vr = vs + (j - tb) * kD + 16 * sub;
#pragma unroll
                for (int t = 0; t < 16; ++t) acc[t] = fmaf(p, vr[t], acc[t]);
            }
        }
    }
    if (!valid) return;
    // gathered global context: hard V_cent[c_i], or the soft assignment
    float gv[16];
    if (!var.soft) {
        const int c = CA_IDX(assign[(int64_t)h * L + qi], 0, K, 75);
        const float *g = vcent + ((int64_t)h * K + c) * kD + 16 * sub;
#pragma unroll
        for (int t = 0; t < 16; ++t) gv[t] = g[t];
    } else {
        float gm = -INFINITY, gl = 0.f;
#pragma unroll
        for (int t = 0; t < 16; ++t) gv[t] = 0.f;
        for (int k = 0; k < K; ++k) {
            const float *mk = var.mu + ((int64_t)h * K + k) * kD + 16 * sub;
            float part = 0.f;
#pragma unroll
            for (int t = 0; t < 16; ++t) part = fmaf(qf[t], mk[t], part);
            part += __shfl_xor_sync(gmask, part, 1);
            part += __shfl_xor_sync(gmask, part, 2);
            const float z = part * scale;
            if (z > gm) {
                const float corr = expf(gm - z);
                gl *= corr;
#pragma unroll
                for (int t = 0; t < 16; ++t) gv[t] *= corr;
                gm = z;
            }
            const float p = expf(z - gm);
            gl += p;
            const float *vk = vcent + ((int64_t)h * K + k) * kD + 16 * sub;
#pragma unroll
            for (int t = 0; t < 16; ++t) gv[t] = fmaf(p, vk[t], gv[t]);
        }
        const float inv = 1.f / gl;
#pragma unroll
        for (int t = 0; t < 16; ++t) gv[t] *= inv;
    }
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    const bool zero_row = kvp && !kvp[qi];
    T *o = out + hoff + (int64_t)qi * kD + 16 * sub;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
        const float y = var.local ? (1.f - alpha) * gv[t] + alpha * (acc[t] * inv_l) : gv[t];
        o[t] = from_f32<T>(zero_row ? 0.f : y);
    }
}

}  // namespace ca
