// Fused cluster-attention forward: one CTA per (batch, head) for L <= 512,
// bf16 inputs.  Every step of the path runs inside this kernel:
//
//   Q (resident in shared memory, loaded once)
//     -> strided init, I Lloyd iterations (distances on tensor cores, exact
//        argmin, exact fp64 member sums)            [k-means]
//   K, V (streamed in 64-key tiles through a 2-stage cp.async ring)
//     -> V_cent = softmax(mu K^T / sqrt(d)) V        [centroid attention]
//   Q, K, V blocks of 128 queries (second read, from L2)
//     -> clipped window attention, gather V_cent[c_i], convex blend, store O.
//
// Model card "Hooshaai/distilbert-sst2-cluster-attention": Architecture
// Overview (two branches and the convex fusion) and Mathematical Formulation
// section 1 (k-means); "Hooshaai/svd-sst2-roberta-cluster" sections 2.1
// (expanded distance) and 3 (execution trace).
//
// Distances: s_k = |mu_k|^2 - 2 Q.mu_k on bf16 tensor cores with the fp32
// centroid split into two bf16 terms (mu = hi + lo + r, |r| <= 2^-18 |mu|).
// Products of bf16 values are exact in fp32; the accumulated error of the
// split dot product stays below 2^-16 (|Q| |mu_k| + |mu_k|^2) even for a
// tensor-core accumulator that truncates.  A token is settled when its two
// smallest s differ by more than 2E, E = 2^-13 (|Q| max|mu| + max|mu|^2)
// (eight times the bound); otherwise every centroid is re-measured in fp64
// (index-order expanded form, separately rounded products and sums) and the
// lowest k with the smallest distance wins.  Centroids that are bitwise
// copies of a lower-index centroid can never win (their distances are equal
// and the lower index takes the tie) and are excluded up front.
#pragma once

#include "common.cuh"
#include "mma.cuh"

namespace ca {
namespace fused {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxL = 512;
constexpr int kMaxK = 64;
constexpr int kMaxR = 16;
constexpr int kTile = 64;       // keys per centroid-attention tile
constexpr int kWinBlock = 128;  // queries per window block (8 warps x 16)
constexpr int kMaxNT = (16 + 2 * kMaxR + 14) / 8;  // key n-tiles per window m-tile
constexpr float kEps = 1.220703125e-04f;           // 2^-13
constexpr float kLog2e = 1.4426950408889634f;

struct Layout {
    int Lp, Kp, r, win_rows;
    uint32_t q_off, ring_off, mu_off, hi_off, lo_off, vc_off, mm_off, hash_off, c_off, list_off,
        misc_off, ml_off, total;

    __host__ __device__ static uint32_t up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

    __host__ __device__ Layout(int L, int K, int r_) {
        Lp = (int)up((uint32_t)L, 64);
        Kp = K <= 16 ? 16 : (K <= 32 ? 32 : 64);
        r = r_;
        win_rows = (int)up((uint32_t)(kWinBlock + 2 * r + 8), 8);
        const uint32_t q_bytes = (uint32_t)Lp * 128u;
        const uint32_t win_bytes = (uint32_t)kWinBlock * 128u + 2u * (uint32_t)win_rows * 128u;
        uint32_t o = 0;
        q_off = o;
        o += up(q_bytes > win_bytes ? q_bytes : win_bytes, 1024);
        ring_off = o;
        o += 2u * 2u * kTile * 128u;  // 2 stages x (K tile, V tile); also combine scratch
        mu_off = o;
        o += up((uint32_t)Kp * 65u * 4u, 128);
        hi_off = o;
        o += (uint32_t)Kp * 128u;
        lo_off = o;
        o += (uint32_t)Kp * 128u;
        vc_off = o;
        o += (uint32_t)Kp * 64u * 4u;
        mm_off = o;
        o += (uint32_t)Kp * 4u;
        hash_off = o;
        o += (uint32_t)Kp * 4u;
        c_off = o;
        o += up((uint32_t)Lp, 16);
        list_off = o;
        o += up((uint32_t)Lp * 2u, 16);
        misc_off = o;
        o += 64;
        ml_off = o;
        o += (uint32_t)kWarps * 16u * 2u * 4u;
        total = up(o, 128);
    }
};

struct Params {
    const __nv_bfloat16 *q, *k, *v;
    __nv_bfloat16 *out;
    int32_t *assign;   // [NH, L] or null
    float *cent;       // [NH, K, 64] or null
    int32_t *hist;     // [NH, iters, L] or null
    int L, K, iters, r;
    float alpha, scale;
};

// Row state for the running argmin: smallest value, its index, second value.
struct Best {
    float m1, m2;
    int k1;
};

__device__ __forceinline__ void best_push(Best &b, float s, int k) {
    if (s < b.m1) {
        b.m2 = b.m1;
        b.m1 = s;
        b.k1 = k;
    } else {
        b.m2 = fminf(b.m2, s);
    }
}

__device__ __forceinline__ Best best_merge(const Best &a, const Best &b) {
    Best r;
    const bool take_b = (b.m1 < a.m1) || (b.m1 == a.m1 && b.k1 < a.k1);
    r.m1 = take_b ? b.m1 : a.m1;
    r.k1 = take_b ? b.k1 : a.k1;
    r.m2 = fminf(fminf(a.m2, b.m2), take_b ? a.m1 : b.m1);
    return r;
}

__device__ __forceinline__ Best best_quad(Best b) {
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
        Best x;
        x.m1 = __shfl_xor_sync(0xffffffffu, b.m1, o);
        x.m2 = __shfl_xor_sync(0xffffffffu, b.m2, o);
        x.k1 = __shfl_xor_sync(0xffffffffu, b.k1, o);
        b = best_merge(b, x);
    }
    return b;
}

// Issue the cp.async copies of `rows` rows of a [*, 64] bf16 matrix starting
// at global row g0 into a swizzled 128-byte-row buffer; rows at or beyond
// `valid` are zero-filled.
__device__ __forceinline__ void load_rows(uint32_t dst, const __nv_bfloat16 *src, int g0, int rows, int valid) {
    for (int e = threadIdx.x; e < rows * 8; e += kThreads) {
        const int row = e >> 3, ch = e & 7;
        const int g = g0 + row;
        const bool ok = g >= 0 && g < valid;
        const __nv_bfloat16 *s = src + (size_t)(ok ? g : 0) * kD + ch * 8;
        cp_async16(dst + swz(row, ch), s, ok ? 16 : 0);
    }
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__global__ void __launch_bounds__(kThreads, 2) fused_forward_kernel(Params P) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const Layout lay(P.L, P.K, P.r);
    const int L = P.L, K = P.K, Lp = lay.Lp, Kp = lay.Kp;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t head = blockIdx.x;
    const __nv_bfloat16 *qh = P.q + head * (int64_t)L * kD;
    const __nv_bfloat16 *kh = P.k + head * (int64_t)L * kD;
    const __nv_bfloat16 *vh = P.v + head * (int64_t)L * kD;

    const uint32_t sbase = smem_u32(smem);
    const uint32_t q_s = sbase + lay.q_off, ring_s = sbase + lay.ring_off;
    const uint32_t hi_s = sbase + lay.hi_off, lo_s = sbase + lay.lo_off;
    float *mu = reinterpret_cast<float *>(smem + lay.mu_off);   // [Kp][65]
    float *vc = reinterpret_cast<float *>(smem + lay.vc_off);   // [Kp][64]
    float *mm = reinterpret_cast<float *>(smem + lay.mm_off);   // [Kp]
    uint32_t *hsh = reinterpret_cast<uint32_t *>(smem + lay.hash_off);
    uint8_t *cs = smem + lay.c_off;                             // [Lp]
    uint16_t *list = reinterpret_cast<uint16_t *>(smem + lay.list_off);
    int *misc = reinterpret_cast<int *>(smem + lay.misc_off);  // 0 refine count, 1 mm_max, 2 mun_max
    float *ml = reinterpret_cast<float *>(smem + lay.ml_off);

    // ---- prologue: Q, then the first two K/V tiles --------------------------
    load_rows(q_s, qh, 0, Lp, L);
    cp_async_commit();
    const int nT = Lp / kTile;
    for (int s = 0; s < 2; ++s) {
        if (s < nT) {
            load_rows(ring_s + s * 2 * kTile * 128, kh, s * kTile, kTile, L);
            load_rows(ring_s + s * 2 * kTile * 128 + kTile * 128, vh, s * kTile, kTile, L);
        }
        cp_async_commit();
    }
    for (int i = threadIdx.x; i < Lp; i += kThreads) cs[i] = i < L ? 0 : 0xFF;
    if (threadIdx.x == 0) misc[0] = 0;
    cp_async_wait<2>();
    __syncthreads();

    // |Q_i| for the rows this thread sees in the k-means epilogue.
    const int n_mt = Lp / 16;
    float qn[kMaxL / 16 / kWarps][2];
#pragma unroll
    for (int j = 0; j < kMaxL / 16 / kWarps; ++j) {
        const int mt = warp + j * kWarps;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float a = 0.f;
            if (mt < n_mt) {
                const int row = mt * 16 + g + 8 * h;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(smem + lay.q_off + swz(row, 2 * t + c));
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float x0 = bf16lo(ws[e]), x1 = bf16hi(ws[e]);
                        a = fmaf(x0, x0, fmaf(x1, x1, a));
                    }
                }
            }
            a += __shfl_xor_sync(0xffffffffu, a, 1);
            a += __shfl_xor_sync(0xffffffffu, a, 2);
            qn[j][h] = sqrtf(a);
        }
    }

    // ---- centroid finalisation: fp32 row -> hi/lo bf16, |mu|^2, hash -------
    // Called by one warp per centroid, lane holding coordinates 2*lane, 2*lane+1.
    auto finalize_row = [&](int kk, float x0, float x1) {
        mu[kk * 65 + 2 * lane] = x0;
        mu[kk * 65 + 2 * lane + 1] = x1;
        const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
        const __nv_bfloat16 l0 = __float2bfloat16_rn(x0 - __bfloat162float(h0));
        const __nv_bfloat16 l1 = __float2bfloat16_rn(x1 - __bfloat162float(h1));
        const uint32_t off = swz(kk, lane >> 2) + (lane & 3) * 4;
        __nv_bfloat162 hv, lv;
        hv.x = h0; hv.y = h1;
        lv.x = l0; lv.y = l1;
        *reinterpret_cast<__nv_bfloat162 *>(smem + lay.hi_off + off) = hv;
        *reinterpret_cast<__nv_bfloat162 *>(smem + lay.lo_off + off) = lv;
        float sq = fmaf(x0, x0, x1 * x1);
        uint32_t hv32 = (__float_as_uint(x0) * 0x9E3779B1u) ^ (__float_as_uint(x1) * 0x85EBCA77u + (uint32_t)lane * 0xC2B2AE3Du);
        for (int o = 16; o > 0; o >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, o);
            hv32 += __shfl_xor_sync(0xffffffffu, hv32, o);
        }
        if (lane == 0) {
            mm[kk] = sq;
            hsh[kk] = hv32;
        }
    };

    // After every centroid row is final: mark duplicates and padding with
    // +inf, and take max |mu|, max |mu|^2 over the live centroids.
    auto finalize_set = [&]() {
        __syncthreads();
        const int kk = threadIdx.x;
        bool dead = true;
        if (kk < Kp) {
            dead = kk >= K;
            for (int a = 0; a < kk && !dead; ++a) {
                if (hsh[a] != hsh[kk]) continue;
                bool same = true;
                for (int j = 0; j < kD && same; ++j)
                    same = __float_as_uint(mu[a * 65 + j]) == __float_as_uint(mu[kk * 65 + j]);
                dead = same;
            }
            if (!dead) {
                atomicMax(&misc[1], __float_as_int(mm[kk]));
                atomicMax(&misc[2], __float_as_int(sqrtf(mm[kk])));
            }
        }
        __syncthreads();
        if (kk < Kp && dead) mm[kk] = INFINITY;
        __syncthreads();
    };

    // ---- strided init: mu_k = Q[floor(k L / K)] -----------------------------
    if (threadIdx.x == 0) {
        misc[1] = 0;
        misc[2] = 0;
    }
    for (int kk = warp; kk < Kp; kk += kWarps) {
        float x0 = 0.f, x1 = 0.f;
        if (kk < K) {
            const int row = (int)(((int64_t)kk * L) / K);
            const uint32_t w = *reinterpret_cast<const uint32_t *>(smem + lay.q_off + swz(row, lane >> 2) + (lane & 3) * 4);
            x0 = bf16lo(w);
            x1 = bf16hi(w);
        }
        finalize_row(kk, x0, x1);
    }
    finalize_set();

    // ---- Lloyd iterations ----------------------------------------------------
    for (int it = 0; it < P.iters; ++it) {
        const float mm_max = __int_as_float(misc[1]), mun_max = __int_as_float(misc[2]);
        // assignment: tensor-core distances + certified argmin
#pragma unroll
        for (int j = 0; j < kMaxL / 16 / kWarps; ++j) {
            const int mt = warp + j * kWarps;
            if (mt >= n_mt) break;
            uint32_t a[4][4];
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int m = lane >> 3;
                const int row = mt * 16 + (lane & 7) + ((m & 1) ? 8 : 0);
                ldmatrix_x4(a[ks], q_s + swz(row, 2 * ks + (m >> 1)));
            }
            Best b0{INFINITY, INFINITY, 0}, b1{INFINITY, INFINITY, 0};
            for (int nt = 0; nt < Kp / 8; ++nt) {
                float ch[4] = {0.f, 0.f, 0.f, 0.f}, cl[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kp = 0; kp < 2; ++kp) {
                    uint32_t bh[4], bl[4];
                    const int row = nt * 8 + (lane & 7);
                    const int chunk = 4 * kp + (lane >> 3);
                    ldmatrix_x4(bh, hi_s + swz(row, chunk));
                    ldmatrix_x4(bl, lo_s + swz(row, chunk));
                    mma_16816(ch, a[2 * kp], bh[0], bh[1]);
                    mma_16816(ch, a[2 * kp + 1], bh[2], bh[3]);
                    mma_16816(cl, a[2 * kp], bl[0], bl[1]);
                    mma_16816(cl, a[2 * kp + 1], bl[2], bl[3]);
                }
                const int c0 = nt * 8 + 2 * t;
                const float m0 = mm[c0], m1 = mm[c0 + 1];
                best_push(b0, fmaf(-2.f, ch[0] + cl[0], m0), c0);
                best_push(b0, fmaf(-2.f, ch[1] + cl[1], m1), c0 + 1);
                best_push(b1, fmaf(-2.f, ch[2] + cl[2], m0), c0);
                best_push(b1, fmaf(-2.f, ch[3] + cl[3], m1), c0 + 1);
            }
            b0 = best_quad(b0);
            b1 = best_quad(b1);
            if (t == 0) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const Best &b = h ? b1 : b0;
                    const int row = mt * 16 + g + 8 * h;
                    if (row < L) {
                        const float E = kEps * fmaf(qn[j][h], mun_max, mm_max);
                        cs[row] = (uint8_t)b.k1;
                        if (b.m2 <= b.m1 + 2.f * E) list[atomicAdd(&misc[0], 1)] = (uint16_t)row;
                    }
                }
            }
        }
        __syncthreads();
        // exact re-measure of ambiguous tokens, one warp per token
        const int n_ref = misc[0];
        for (int e = warp; e < n_ref; e += kWarps) {
            const int row = list[e];
            double qq = 0.0;
            double qm[2] = {0.0, 0.0}, m2[2] = {0.0, 0.0};
            for (int j = 0; j < kD; ++j) {
                const uint16_t bits = *reinterpret_cast<const uint16_t *>(smem + lay.q_off + swz(row, j >> 3) + (j & 7) * 2);
                const double qj = (double)__uint_as_float((uint32_t)bits << 16);
                qq = __dadd_rn(qq, __dmul_rn(qj, qj));
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    const int kk = lane + 32 * s;
                    const double mj = kk < Kp ? (double)mu[kk * 65 + j] : 0.0;
                    qm[s] = __dadd_rn(qm[s], __dmul_rn(qj, mj));
                    m2[s] = __dadd_rn(m2[s], __dmul_rn(mj, mj));
                }
            }
            double bd = INFINITY;
            int bk = 0x7fffffff;
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const int kk = lane + 32 * s;
                if (kk < Kp && !(mm[kk] == INFINITY)) {
                    const double D = __dsub_rn(__dadd_rn(qq, m2[s]), __dmul_rn(2.0, qm[s]));
                    if (D < bd) {
                        bd = D;
                        bk = kk;
                    }
                }
            }
            for (int o = 16; o > 0; o >>= 1) {
                const double od = __shfl_xor_sync(0xffffffffu, bd, o);
                const int ok = __shfl_xor_sync(0xffffffffu, bk, o);
                if (od < bd || (od == bd && ok < bk)) {
                    bd = od;
                    bk = ok;
                }
            }
            if (lane == 0) {
                if (bk >= K) {
                    record_error(5, 2);
                    bk = 0;
                }
                cs[row] = (uint8_t)bk;
            }
        }
        __syncthreads();
        if (P.hist) {
            int32_t *hrow = P.hist + (head * P.iters + it) * (int64_t)L;
            for (int i = threadIdx.x; i < L; i += kThreads) hrow[i] = cs[i];
        }
        if (threadIdx.x == 0) {
            misc[0] = 0;
            misc[1] = 0;
            misc[2] = 0;
        }
        // update: exact fp64 member sums, one warp per cluster
        const bool last = it == P.iters - 1;
        for (int kk = warp; kk < Kp; kk += kWarps) {
            double s0[4] = {0.0, 0.0, 0.0, 0.0}, s1[4] = {0.0, 0.0, 0.0, 0.0};
            int cnt = 0;
            if (kk < K) {
                for (int base = 0; base < Lp; base += 32) {
                    uint32_t m = __ballot_sync(0xffffffffu, cs[base + lane] == kk);
                    cnt += __popc(m);
                    while (m) {
                        int rows[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            if (m) {
                                rows[u] = base + __ffs(m) - 1;
                                m &= m - 1;
                            } else {
                                rows[u] = -1;
                            }
                        }
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            if (rows[u] >= 0) {
                                const uint32_t w = *reinterpret_cast<const uint32_t *>(smem + lay.q_off + swz(rows[u], lane >> 2) + (lane & 3) * 4);
                                s0[u] += (double)bf16lo(w);
                                s1[u] += (double)bf16hi(w);
                            }
                        }
                    }
                }
            }
            const double den = (double)(cnt > 1 ? cnt : 1);
            const float x0 = __double2float_rn(((s0[0] + s0[1]) + (s0[2] + s0[3])) / den);
            const float x1 = __double2float_rn(((s1[0] + s1[1]) + (s1[2] + s1[3])) / den);
            finalize_row(kk, x0, x1);
            if (last && P.cent && kk < K) {
                float2 *dst = reinterpret_cast<float2 *>(P.cent + (head * K + kk) * kD);
                dst[lane] = make_float2(x0, x1);
            }
        }
        finalize_set();
    }
    if (P.iters == 0 && P.cent) {
        for (int e = threadIdx.x; e < K * kD; e += kThreads) P.cent[head * K * kD + e] = mu[(e / kD) * 65 + e % kD];
    }
    if (P.assign) {
        for (int i = threadIdx.x; i < L; i += kThreads) P.assign[head * L + i] = cs[i];
    }

    // ---- centroid attention over streamed K/V tiles --------------------------
    const int n_cm = Kp / 16;          // centroid m-tiles: 1, 2 or 4
    const int G = kWarps / n_cm;       // warps sharing one m-tile: 8, 4 or 2
    const int cm = warp / G, kb = warp % G;
    const int keys_w = kTile / G;      // keys per warp per tile: 8, 16 or 32
    const float csc = P.scale * kLog2e;
    uint32_t ahi[4][4], alo[4][4];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
        const int m = lane >> 3;
        const int row = cm * 16 + (lane & 7) + ((m & 1) ? 8 : 0);
        ldmatrix_x4(ahi[ks], hi_s + swz(row, 2 * ks + (m >> 1)));
        ldmatrix_x4(alo[ks], lo_s + swz(row, 2 * ks + (m >> 1)));
    }
    float o_acc[8][4];
#pragma unroll
    for (int d = 0; d < 8; ++d)
#pragma unroll
        for (int e = 0; e < 4; ++e) o_acc[d][e] = 0.f;
    float rm[2] = {-INFINITY, -INFINITY}, rl[2] = {0.f, 0.f};

    for (int tt = 0; tt < nT; ++tt) {
        cp_async_wait<1>();
        __syncthreads();
        const uint32_t kt = ring_s + (tt & 1) * 2 * kTile * 128;
        const uint32_t vt = kt + kTile * 128;
        float sacc[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[n][e] = 0.f;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            if (n * 8 >= keys_w) break;
            const int key0 = kb * keys_w + n * 8;
#pragma unroll
            for (int kp = 0; kp < 2; ++kp) {
                uint32_t bk[4];
                ldmatrix_x4(bk, kt + swz(key0 + (lane & 7), 4 * kp + (lane >> 3)));
                mma_16816(sacc[n], ahi[2 * kp], bk[0], bk[1]);
                mma_16816(sacc[n], ahi[2 * kp + 1], bk[2], bk[3]);
                mma_16816(sacc[n], alo[2 * kp], bk[0], bk[1]);
                mma_16816(sacc[n], alo[2 * kp + 1], bk[2], bk[3]);
            }
        }
        // online softmax over this warp's keys of the tile
        float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            if (n * 8 >= keys_w) break;
            const int key = tt * kTile + kb * keys_w + n * 8 + 2 * t;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (key + (e & 1) >= L) sacc[n][e] = -INFINITY;
            }
            tmax[0] = fmaxf(tmax[0], fmaxf(sacc[n][0], sacc[n][1]));
            tmax[1] = fmaxf(tmax[1], fmaxf(sacc[n][2], sacc[n][3]));
        }
        float corr[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 1));
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 2));
            const float mn = fmaxf(rm[h], tmax[h]);
            corr[h] = (mn == -INFINITY) ? 1.f : exp2f((rm[h] - mn) * csc);
            rm[h] = mn;
            rl[h] *= corr[h];
        }
#pragma unroll
        for (int d = 0; d < 8; ++d) {
            o_acc[d][0] *= corr[0];
            o_acc[d][1] *= corr[0];
            o_acc[d][2] *= corr[1];
            o_acc[d][3] *= corr[1];
        }
        uint32_t pa[4][2];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            if (n * 8 >= keys_w) break;
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float mh = rm[e >> 1];
                p[e] = (mh == -INFINITY) ? 0.f : exp2f((sacc[n][e] - mh) * csc);
            }
            rl[0] += p[0] + p[1];
            rl[1] += p[2] + p[3];
            pa[n][0] = pack_bf16(p[0], p[1]);
            pa[n][1] = pack_bf16(p[2], p[3]);
        }
        // O += P V
        if (keys_w == 8) {
            const int key0 = kb * keys_w;
#pragma unroll
            for (int dq = 0; dq < 2; ++dq) {
                uint32_t bv[4];
                ldmatrix_x4_trans(bv, vt + swz(key0 + (lane & 7), 4 * dq + (lane >> 3)));
#pragma unroll
                for (int u = 0; u < 4; ++u) mma_1688(o_acc[4 * dq + u], pa[0][0], pa[0][1], bv[u]);
            }
        } else {
#pragma unroll
            for (int n2 = 0; n2 < 2; ++n2) {
                if (n2 * 16 >= keys_w) break;
                const uint32_t a4[4] = {pa[2 * n2][0], pa[2 * n2][1], pa[2 * n2 + 1][0], pa[2 * n2 + 1][1]};
                const int key0 = kb * keys_w + n2 * 16;
#pragma unroll
                for (int dq = 0; dq < 4; ++dq) {
                    uint32_t bv[4];
                    const int m = lane >> 3;
                    ldmatrix_x4_trans(bv, vt + swz(key0 + (lane & 7) + ((m & 1) ? 8 : 0), 2 * dq + (m >> 1)));
                    mma_16816(o_acc[2 * dq], a4, bv[0], bv[1]);
                    mma_16816(o_acc[2 * dq + 1], a4, bv[2], bv[3]);
                }
            }
        }
        __syncthreads();
        if (tt + 2 < nT) {
            load_rows(kt, kh, (tt + 2) * kTile, kTile, L);
            load_rows(vt, vh, (tt + 2) * kTile, kTile, L);
        }
        cp_async_commit();
    }
    cp_async_wait<0>();
    // combine the G partial states of each centroid m-tile (ring reused)
    {
        float *part = reinterpret_cast<float *>(smem + lay.ring_off);  // [warp][16][64]
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            rl[h] += __shfl_xor_sync(0xffffffffu, rl[h], 1);
            rl[h] += __shfl_xor_sync(0xffffffffu, rl[h], 2);
        }
        __syncthreads();
#pragma unroll
        for (int d = 0; d < 8; ++d) {
            float *p0 = part + (warp * 16 + g) * 64 + 8 * d + 2 * t;
            float *p1 = part + (warp * 16 + g + 8) * 64 + 8 * d + 2 * t;
            p0[0] = o_acc[d][0];
            p0[1] = o_acc[d][1];
            p1[0] = o_acc[d][2];
            p1[1] = o_acc[d][3];
        }
        if (t == 0) {
            ml[(warp * 16 + g) * 2 + 0] = rm[0];
            ml[(warp * 16 + g) * 2 + 1] = rl[0];
            ml[(warp * 16 + g + 8) * 2 + 0] = rm[1];
            ml[(warp * 16 + g + 8) * 2 + 1] = rl[1];
        }
        __syncthreads();
        for (int e = threadIdx.x; e < Kp * kD; e += kThreads) {
            const int row = e / kD, col = e % kD;
            const int mt = row / 16, rr = row % 16;
            float M = -INFINITY;
            for (int w = mt * G; w < mt * G + G; ++w) M = fmaxf(M, ml[(w * 16 + rr) * 2]);
            float num = 0.f, den = 0.f;
            for (int w = mt * G; w < mt * G + G; ++w) {
                const float mw = ml[(w * 16 + rr) * 2];
                const float f = (mw == -INFINITY) ? 0.f : exp2f((mw - M) * csc);
                den = fmaf(ml[(w * 16 + rr) * 2 + 1], f, den);
                num = fmaf(part[(w * 16 + rr) * 64 + col], f, num);
            }
            vc[row * kD + col] = num / den;
        }
        __syncthreads();
    }

    // ---- window attention + gather + blend, 128 queries per block ------------
    const int r = P.r;
    const uint32_t qb_s = q_s, kw_s = q_s + kWinBlock * 128, vw_s = kw_s + lay.win_rows * 128;
    for (int qb = 0; qb < L; qb += kWinBlock) {
        const int ks0 = max(0, qb - r) & ~7;
        const int ke = min(L - 1, qb + kWinBlock - 1 + r);
        const int nrows = (ke - ks0 + 1 + 7) & ~7;
        load_rows(qb_s, qh, qb, kWinBlock, L);
        load_rows(kw_s, kh, ks0, nrows, ke + 1);
        load_rows(vw_s, vh, ks0, nrows, ke + 1);
        cp_async_commit();
        cp_async_wait<0>();
        __syncthreads();
        const int i0 = qb + warp * 16;
        if (i0 < L) {
            uint32_t a[4][4];
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int m = lane >> 3;
                const int row = warp * 16 + (lane & 7) + ((m & 1) ? 8 : 0);
                ldmatrix_x4(a[ks], qb_s + swz(row, 2 * ks + (m >> 1)));
            }
            const int kst = max(0, i0 - r) & ~7;
            const int kend = min(L - 1, i0 + 15 + r);
            const int nt = (kend - kst) / 8 + 1;
            const int lr0 = kst - ks0;  // local row of the first key
            float sacc[kMaxNT][4];
#pragma unroll
            for (int n = 0; n < kMaxNT; ++n) {
#pragma unroll
                for (int e = 0; e < 4; ++e) sacc[n][e] = 0.f;
                if (n < nt) {
#pragma unroll
                    for (int kp = 0; kp < 2; ++kp) {
                        uint32_t bk[4];
                        ldmatrix_x4(bk, kw_s + swz(lr0 + n * 8 + (lane & 7), 4 * kp + (lane >> 3)));
                        mma_16816(sacc[n], a[2 * kp], bk[0], bk[1]);
                        mma_16816(sacc[n], a[2 * kp + 1], bk[2], bk[3]);
                    }
                }
            }
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int n = 0; n < kMaxNT; ++n) {
                if (n < nt) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = i0 + g + 8 * (e >> 1);
                        const int jk = kst + n * 8 + 2 * t + (e & 1);
                        const bool ok = jk >= i - r && jk <= i + r && jk < L;
                        if (!ok) sacc[n][e] = -INFINITY;
                    }
                    mx[0] = fmaxf(mx[0], fmaxf(sacc[n][0], sacc[n][1]));
                    mx[1] = fmaxf(mx[1], fmaxf(sacc[n][2], sacc[n][3]));
                }
            }
            float sum[2] = {0.f, 0.f};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
            }
            uint32_t pa[kMaxNT][2];
#pragma unroll
            for (int n = 0; n < kMaxNT; ++n) {
                pa[n][0] = pa[n][1] = 0u;
                if (n < nt) {
                    float p[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float mh = mx[e >> 1];
                        p[e] = (mh == -INFINITY) ? 0.f : exp2f((sacc[n][e] - mh) * csc);
                    }
                    sum[0] += p[0] + p[1];
                    sum[1] += p[2] + p[3];
                    pa[n][0] = pack_bf16(p[0], p[1]);
                    pa[n][1] = pack_bf16(p[2], p[3]);
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                sum[h] += __shfl_xor_sync(0xffffffffu, sum[h], 1);
                sum[h] += __shfl_xor_sync(0xffffffffu, sum[h], 2);
            }
            float oacc[8][4];
#pragma unroll
            for (int d = 0; d < 8; ++d)
#pragma unroll
                for (int e = 0; e < 4; ++e) oacc[d][e] = 0.f;
#pragma unroll
            for (int n2 = 0; n2 < (kMaxNT + 1) / 2; ++n2) {
                if (2 * n2 + 1 < nt) {
                    const uint32_t a4[4] = {pa[2 * n2][0], pa[2 * n2][1], pa[2 * n2 + 1][0], pa[2 * n2 + 1][1]};
#pragma unroll
                    for (int dq = 0; dq < 4; ++dq) {
                        uint32_t bv[4];
                        const int m = lane >> 3;
                        ldmatrix_x4_trans(bv, vw_s + swz(lr0 + n2 * 16 + (lane & 7) + ((m & 1) ? 8 : 0), 2 * dq + (m >> 1)));
                        mma_16816(oacc[2 * dq], a4, bv[0], bv[1]);
                        mma_16816(oacc[2 * dq + 1], a4, bv[2], bv[3]);
                    }
                } else if (2 * n2 < nt) {
#pragma unroll
                    for (int dq = 0; dq < 2; ++dq) {
                        uint32_t bv[4];
                        ldmatrix_x4_trans(bv, vw_s + swz(lr0 + n2 * 16 + (lane & 7), 4 * dq + (lane >> 3)));
#pragma unroll
                        for (int u = 0; u < 4; ++u) mma_1688(oacc[4 * dq + u], pa[2 * n2][0], pa[2 * n2][1], bv[u]);
                    }
                }
            }
            // gather + blend, staged into this warp's own Q rows
            const float inv0 = sum[0] > 0.f ? 1.f / sum[0] : 0.f, inv1 = sum[1] > 0.f ? 1.f / sum[1] : 0.f;
            const int ia = i0 + g, ib = i0 + g + 8;
            const int ca = ia < L ? cs[ia] : 0, cb = ib < L ? cs[ib] : 0;
            const float al = P.alpha, be = 1.f - P.alpha;
#pragma unroll
            for (int d = 0; d < 8; ++d) {
                const int col = 8 * d + 2 * t;
                const float y0 = be * vc[ca * kD + col] + al * (oacc[d][0] * inv0);
                const float y1 = be * vc[ca * kD + col + 1] + al * (oacc[d][1] * inv0);
                const float y2 = be * vc[cb * kD + col] + al * (oacc[d][2] * inv1);
                const float y3 = be * vc[cb * kD + col + 1] + al * (oacc[d][3] * inv1);
                *reinterpret_cast<uint32_t *>(smem + lay.q_off + swz(warp * 16 + g, d) + 4 * t) = pack_bf16(y0, y1);
                *reinterpret_cast<uint32_t *>(smem + lay.q_off + swz(warp * 16 + g + 8, d) + 4 * t) = pack_bf16(y2, y3);
            }
            __syncwarp();
            __nv_bfloat16 *oh = P.out + head * (int64_t)L * kD;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int e = lane + 32 * u;
                const int rr = e >> 3, ch = e & 7;
                const int i = i0 + rr;
                if (i < L) {
                    const uint4 val = *reinterpret_cast<const uint4 *>(smem + lay.q_off + swz(warp * 16 + rr, ch));
                    *reinterpret_cast<uint4 *>(oh + (int64_t)i * kD + ch * 8) = val;
                }
            }
        }
        __syncthreads();
    }
}

}  // namespace fused
}  // namespace ca
