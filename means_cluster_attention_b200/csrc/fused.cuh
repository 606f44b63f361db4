// Fused cluster-attention forward: one CTA per (batch, head) for L <= 512,
// bf16 inputs.  Every step of the path runs inside this kernel:
//
//   Q (resident in shared memory, loaded once)
//     -> strided init, I Lloyd iterations: distances on tensor cores with an
//        exact argmin, exact fp64 member sums          [k-means]
//   K, V (64-key tiles, up to five in flight)
//     -> V_cent = softmax(mu K^T / sqrt(d)) V           [centroid attention]
//   K, V blocks of 128 queries + halo (second read, from L2, double buffered)
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
//
// Member sums (kmeans_tile.cuh): tokens are grouped by cluster with a
// counting sort and each warp walks a contiguous slice of the sorted tokens,
// two tokens per step, adding exact doubles in fp64; a later iteration in
// which few tokens change cluster only subtracts / adds those.  The sums are
// exact for any input whose non-zero magnitudes lie within 2^-27 .. 16, so
// the centroid mu_k = fp32(sum / max(1, count)) does not depend on the order
// of the adds.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "kmeans_tile.cuh"
#include "mma.cuh"

namespace ca {
namespace fused {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxL = 512;
constexpr int kMaxK = 64;
constexpr int kMaxR = 16;
constexpr int kTile = 64;       // keys per centroid-attention tile
constexpr int kSlots = 5;       // centroid-attention tiles in flight
constexpr int kWinBlock = 128;  // queries per window block (8 warps x 16)
constexpr int kMaxNT = (16 + 2 * kMaxR + 14) / 8;  // key n-tiles per window m-tile
constexpr int kVcStride = 72;   // floats per V_cent row (conflict-free float2 gathers)
constexpr float kEps = 1.220703125e-04f;           // 2^-13
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ inline uint32_t up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline uint32_t umax(uint32_t a, uint32_t b) { return a > b ? a : b; }

struct Layout {
    int Lp, Kp, r, nT, win_rows;
    uint32_t big_off, sums_off, mu64_off, mu_off, hi_off, lo_off, vc_off, mm_off, hash_off, dead_off, c_off,
        list_off, perm_off, sc_off, cprev_off, cnt_off, misc_off, ml_off, win_stage,
        total;

    __host__ __device__ Layout(int L, int K, int r_) {
        Lp = (int)up((uint32_t)L, 64);
        Kp = K <= 16 ? 16 : (K <= 32 ? 32 : 64);
        r = r_;
        nT = Lp / kTile;
        const uint32_t wr = up((uint32_t)(kWinBlock + 2 * r + 8), 8);
        win_rows = (int)(wr < (uint32_t)Lp + 8 ? wr : (uint32_t)Lp + 8);
        win_stage = 2u * (uint32_t)win_rows * 128u;
        const uint32_t q_bytes = (uint32_t)Lp * 128u;
        const uint32_t sums_bytes = (uint32_t)Kp * 64u * 8u;
        const uint32_t mu64_bytes = (uint32_t)Kp * 65u * 8u;  // fp64 centroid copy for the re-measure
        const uint32_t slots = (uint32_t)(nT < kSlots ? nT : kSlots);
        uint32_t big = umax(q_bytes + sums_bytes + mu64_bytes, slots * 2u * kTile * 128u);
        big = umax(big, 2u * win_stage);
        big = umax(big, (uint32_t)kWarps * 16u * 64u * 4u);  // centroid-phase combine scratch
        uint32_t o = 0;
        big_off = o;
        sums_off = q_bytes;
        mu64_off = q_bytes + sums_bytes;
        o += up(big, 1024);
        mu_off = o;
        o += up((uint32_t)Kp * 65u * 4u, 128);
        hi_off = o;
        o += (uint32_t)Kp * 128u;
        lo_off = o;
        o += (uint32_t)Kp * 128u;
        vc_off = o;
        o += (uint32_t)Kp * (uint32_t)kVcStride * 4u;
        mm_off = o;
        o += (uint32_t)Kp * 4u;
        hash_off = o;
        o += (uint32_t)Kp * 4u;
        cnt_off = o;
        o += (uint32_t)Kp * 4u;
        dead_off = o;
        o += up((uint32_t)Kp, 16);
        c_off = o;
        o += up((uint32_t)Lp, 16);
        sc_off = o;
        o += up((uint32_t)Lp, 16);
        cprev_off = o;
        o += up((uint32_t)Lp, 16);
        list_off = o;
        o += up((uint32_t)Lp * 2u, 16);
        perm_off = o;
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

// Running argmin of one row: smallest value, its index, second value.
struct Best {
    float m1, m2;
    int k1;
};

__device__ __forceinline__ void best_push(Best &b, float s, int k) {
    const bool lt = s < b.m1;
    b.m2 = fminf(b.m2, fmaxf(b.m1, s));
    b.k1 = lt ? k : b.k1;
    b.m1 = fminf(b.m1, s);
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

// cp.async copies of `rows` rows of a [*, 64] bf16 matrix starting at global
// row g0 into a swizzled 128-byte-row buffer; rows at or beyond `valid` are
// zero-filled.
__device__ __forceinline__ void load_rows(uint32_t dst, const __nv_bfloat16 *src, int g0, int rows, int valid) {
    for (int e = threadIdx.x; e < rows * 8; e += kThreads) {
        const int row = e >> 3, ch = e & 7;
        const int gr = g0 + row;
        const bool ok = gr >= 0 && gr < valid;
        const __nv_bfloat16 *s = src + (size_t)(ok ? gr : 0) * kD + ch * 8;
        cp_async16(dst + swz(row, ch), s, ok ? 16 : 0);
    }
}

// 2^x with the MUFU instruction (relative error about 2^-22; 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

using tile::bf16_to_f64;

__global__ void __launch_bounds__(kThreads, 2) fused_forward_kernel(Params P) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const Layout lay(P.L, P.K, P.r);
    const int L = P.L, K = P.K, Lp = lay.Lp, Kp = lay.Kp, nT = lay.nT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t head = blockIdx.x;
    const __nv_bfloat16 *qh = P.q + head * (int64_t)L * kD;
    const __nv_bfloat16 *kh = P.k + head * (int64_t)L * kD;
    const __nv_bfloat16 *vh = P.v + head * (int64_t)L * kD;

    const uint32_t sbase = smem_u32(smem);
    const uint32_t big_s = sbase + lay.big_off;  // Q during k-means, then K/V staging
    const uint32_t hi_s = sbase + lay.hi_off, lo_s = sbase + lay.lo_off;
    unsigned char *qbytes = smem + lay.big_off;
    float *mu = reinterpret_cast<float *>(smem + lay.mu_off);                     // [Kp][65]
    float *vc = reinterpret_cast<float *>(smem + lay.vc_off);  // [Kp][kVcStride], (1 - alpha) V_cent
    float *mm = reinterpret_cast<float *>(smem + lay.mm_off);                     // [Kp]
    uint32_t *hsh = reinterpret_cast<uint32_t *>(smem + lay.hash_off);
    int *cnt_s = reinterpret_cast<int *>(smem + lay.cnt_off);
    double *sums = reinterpret_cast<double *>(smem + lay.big_off + lay.sums_off);  // [Kp][64]
    double *mu64 = reinterpret_cast<double *>(smem + lay.big_off + lay.mu64_off);  // [Kp][65], exact copy of mu
    uint8_t *dead = smem + lay.dead_off;
    uint8_t *cs = smem + lay.c_off;                                              // [Lp]
    uint8_t *sc = smem + lay.sc_off;        // [Lp] cluster ids in sorted order
    uint8_t *cprev = smem + lay.cprev_off;  // [Lp] previous iteration's assignment
    uint16_t *list = reinterpret_cast<uint16_t *>(smem + lay.list_off);
    uint16_t *perm = reinterpret_cast<uint16_t *>(smem + lay.perm_off);  // [Lp] tokens in sorted order
    int *misc = reinterpret_cast<int *>(smem + lay.misc_off);  // 0 refine count, 1 max |mu|^2 bits, 3 movers
    float *ml = reinterpret_cast<float *>(smem + lay.ml_off);

    // ---- prologue: Q ------------------------------------------------------
    load_rows(big_s, qh, 0, Lp, L);
    cp_async_commit();
    for (int i = threadIdx.x; i < Lp; i += kThreads) cs[i] = i < L ? 0 : 0xFF;
    if (threadIdx.x == 0) misc[0] = misc[1] = 0;
    cp_async_wait<0>();
    __syncthreads();

    // |Q_i| for the rows this thread sees in the k-means epilogue.
    const int n_mt = Lp / 16;
    constexpr int kMtPerWarp = kMaxL / 16 / kWarps;  // 4
    float qn[kMtPerWarp][2];
#pragma unroll
    for (int j = 0; j < kMtPerWarp; ++j) {
        const int mt = warp + j * kWarps;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float a = 0.f;
            if (mt < n_mt) {
                const int row = mt * 16 + g + 8 * h;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const uint4 w = *reinterpret_cast<const uint4 *>(qbytes + swz(row, 2 * t + c));
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

    // One warp per centroid row: lane holds coordinates 2*lane, 2*lane+1.
    auto finalize_row = [&](int kk, float x0, float x1) {
        mu[kk * 65 + 2 * lane] = x0;
        mu[kk * 65 + 2 * lane + 1] = x1;
        mu64[kk * 65 + 2 * lane] = (double)x0;
        mu64[kk * 65 + 2 * lane + 1] = (double)x1;
        const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
        const __nv_bfloat16 l0 = __float2bfloat16_rn(x0 - __bfloat162float(h0));
        const __nv_bfloat16 l1 = __float2bfloat16_rn(x1 - __bfloat162float(h1));
        const uint32_t off = swz(kk, lane >> 2) + (lane & 3) * 4;
        __nv_bfloat162 hv, lv;
        hv.x = h0;
        hv.y = h1;
        lv.x = l0;
        lv.y = l1;
        *reinterpret_cast<__nv_bfloat162 *>(smem + lay.hi_off + off) = hv;
        *reinterpret_cast<__nv_bfloat162 *>(smem + lay.lo_off + off) = lv;
        float sq = fmaf(x0, x0, x1 * x1);
        uint32_t hv32 = (__float_as_uint(x0) * 0x9E3779B1u) ^ (__float_as_uint(x1) * 0x85EBCA77u + (uint32_t)lane * 0xC2B2AE3Du);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, o);
            hv32 += __shfl_xor_sync(0xffffffffu, hv32, o);
        }
        if (lane == 0) {
            // padding rows can never win; live rows feed max |mu|^2 (a
            // duplicate has its original's norm, so it cannot raise the max)
            mm[kk] = kk < K ? sq : INFINITY;
            hsh[kk] = hv32;
            dead[kk] = kk < K ? 0 : 1;
            if (kk < K) atomicMax(&misc[1], __float_as_int(sq));
        }
    };

    // After every centroid row is final: mark bitwise duplicates of a
    // lower-index centroid dead (|mu|^2 = +inf); write the iteration's
    // assignments to hrow when given.
    auto finalize_set = [&](int32_t *hrow) {
        __syncthreads();
        if (threadIdx.x == 0) misc[0] = misc[3] = 0;
        if (hrow)
            for (int i = threadIdx.x; i < L; i += kThreads) hrow[i] = cs[i];
        mark_copies(K, hsh, mu, 65, dead, mm, warp, kWarps, lane);
        __syncthreads();
    };

    // ---- strided init: mu_k = Q[floor(k L / K)] -------------------------------
    for (int kk = warp; kk < Kp; kk += kWarps) {
        float x0 = 0.f, x1 = 0.f;
        if (kk < K) {
            const int row = (int)(((int64_t)kk * L) / K);
            const uint32_t w = *reinterpret_cast<const uint32_t *>(qbytes + swz(row, lane >> 2) + (lane & 3) * 4);
            x0 = bf16lo(w);
            x1 = bf16hi(w);
        }
        finalize_row(kk, x0, x1);
    }
    finalize_set(nullptr);

    const int nch = Lp / 32;
    // ---- Lloyd iterations -----------------------------------------------------
    for (int it = 0; it < P.iters; ++it) {
        const float mm_max = __int_as_float(misc[1]), mun_max = sqrtf(mm_max);
        if (it == 0) {
            for (int i = threadIdx.x; i < Kp * kD; i += kThreads) sums[i] = 0.0;
            if (threadIdx.x < Kp) cnt_s[threadIdx.x] = 0;
        }
        // (1) assignment: tensor-core distances + certified argmin, two m-tiles at a time
#pragma unroll
        for (int jp = 0; jp < kMtPerWarp; jp += 2) {
            const int mt0 = warp + jp * kWarps, mt1 = mt0 + kWarps;
            if (mt0 >= n_mt) break;
            const bool two = mt1 < n_mt;
            uint32_t a0[4][4], a1[4][4];
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int m = lane >> 3;
                const int rr = (lane & 7) + ((m & 1) ? 8 : 0);
                ldmatrix_x4(a0[ks], big_s + swz(mt0 * 16 + rr, 2 * ks + (m >> 1)));
                if (two) ldmatrix_x4(a1[ks], big_s + swz(mt1 * 16 + rr, 2 * ks + (m >> 1)));
                else a1[ks][0] = a1[ks][1] = a1[ks][2] = a1[ks][3] = 0u;
            }
            Best b[2][2];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int h = 0; h < 2; ++h) b[u][h] = Best{INFINITY, INFINITY, 0};
            for (int nt = 0; nt < Kp / 8; ++nt) {
                uint32_t bh[2][4], bl[2][4];
#pragma unroll
                for (int kp = 0; kp < 2; ++kp) {
                    const int row = nt * 8 + (lane & 7);
                    const int chunk = 4 * kp + (lane >> 3);
                    ldmatrix_x4(bh[kp], hi_s + swz(row, chunk));
                    ldmatrix_x4(bl[kp], lo_s + swz(row, chunk));
                }
                float acc[2][2][4];
#pragma unroll
                for (int u = 0; u < 2; ++u)
#pragma unroll
                    for (int s = 0; s < 2; ++s)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[u][s][e] = 0.f;
#pragma unroll
                for (int kp = 0; kp < 2; ++kp) {
                    mma_16816(acc[0][0], a0[2 * kp], bh[kp][0], bh[kp][1]);
                    mma_16816(acc[0][1], a0[2 * kp], bl[kp][0], bl[kp][1]);
                    mma_16816(acc[1][0], a1[2 * kp], bh[kp][0], bh[kp][1]);
                    mma_16816(acc[1][1], a1[2 * kp], bl[kp][0], bl[kp][1]);
                    mma_16816(acc[0][0], a0[2 * kp + 1], bh[kp][2], bh[kp][3]);
                    mma_16816(acc[0][1], a0[2 * kp + 1], bl[kp][2], bl[kp][3]);
                    mma_16816(acc[1][0], a1[2 * kp + 1], bh[kp][2], bh[kp][3]);
                    mma_16816(acc[1][1], a1[2 * kp + 1], bl[kp][2], bl[kp][3]);
                }
                const int c0 = nt * 8 + 2 * t;
                const float m0 = mm[c0], m1 = mm[c0 + 1];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    best_push(b[u][0], fmaf(-2.f, acc[u][0][0] + acc[u][1][0], m0), c0);
                    best_push(b[u][0], fmaf(-2.f, acc[u][0][1] + acc[u][1][1], m1), c0 + 1);
                    best_push(b[u][1], fmaf(-2.f, acc[u][0][2] + acc[u][1][2], m0), c0);
                    best_push(b[u][1], fmaf(-2.f, acc[u][0][3] + acc[u][1][3], m1), c0 + 1);
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int mt = u ? mt1 : mt0;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const Best bb = best_quad(b[u][h]);
                    const int row = mt * 16 + g + 8 * h;
                    if (t == 0 && (u == 0 || two) && row < L) {
                        const float E = kEps * fmaf(qn[jp + u][h], mun_max, mm_max);
                        cs[row] = (uint8_t)bb.k1;
                        if (bb.m2 <= bb.m1 + 2.f * E) list[CA_IDX(atomicAdd(&misc[0], 1), 0, kMaxL, 70)] = (uint16_t)row;
                    }
                }
            }
        }
        __syncthreads();
        // (2) exact re-measure of ambiguous tokens, one warp per token
        const int n_ref = misc[0];
        if (threadIdx.x == 0) misc[1] = 0;
        // Lane k holds centroid k (and k + 32 when Kp = 64); the chains of
        // the second set are only run when that set exists.
        auto mu_at = [&](int k, int j) { return mu64[k * 65 + j]; };
        for (int e = warp; e < n_ref; e += kWarps) {
            const int row = CA_IDX(list[e], 0, L, 71);
            int bk = Kp > 32 ? tile::remeasure_token<true>(qbytes, row, Kp, dead, mu_at, lane)
                             : tile::remeasure_token<false>(qbytes, row, Kp, dead, mu_at, lane);
            if (bk >= K) {
                if (lane == 0) record_error(5, 2);
                bk = 0;
            }
            if (lane == 0) cs[row] = (uint8_t)bk;
        }
        __syncthreads();
        // (3) member sums.  Later iterations first list the tokens whose
        // cluster changed; when they are few, only they move between the
        // sums (exact fp64 subtract / add) and the counts.
        int n_mv = L;
        if (it > 0) {
            for (int ch = warp; ch < nch; ch += kWarps) {
                const int i = ch * 32 + lane;
                const bool mv = i < L && cs[i] != cprev[i];
                const unsigned bal = __ballot_sync(0xffffffffu, mv);
                int base = 0;
                if (lane == 0 && bal) base = atomicAdd(&misc[3], __popc(bal));
                base = __shfl_sync(0xffffffffu, base, 0);
                if (mv) list[base + __popc(bal & ((1u << lane) - 1u))] = (uint16_t)i;
            }
            __syncthreads();
            n_mv = misc[3];
        }
        if (n_mv <= (L >> 2)) {
            for (int e = warp; e < n_mv; e += kWarps) {
                const int row = CA_IDX(list[e], 0, L, 72);
                const int co = CA_IDX(cprev[row], 0, Kp, 73), cn = CA_IDX(cs[row], 0, Kp, 73);
                const uint32_t w = *reinterpret_cast<const uint32_t *>(qbytes + swz(row, lane >> 2) + (lane & 3) * 4);
                const double d0 = bf16_to_f64(w & 0xffffu), d1 = bf16_to_f64(w >> 16);
                atomicAdd(&sums[co * kD + 2 * lane], -d0);
                atomicAdd(&sums[co * kD + 2 * lane + 1], -d1);
                atomicAdd(&sums[cn * kD + 2 * lane], d0);
                atomicAdd(&sums[cn * kD + 2 * lane + 1], d1);
                if (lane == 0) {
                    atomicSub(&cnt_s[co], 1);
                    atomicAdd(&cnt_s[cn], 1);
                }
            }
        } else {
            if (it > 0) {
                for (int i = threadIdx.x; i < Kp * kD; i += kThreads) sums[i] = 0.0;
                if (threadIdx.x < Kp) cnt_s[threadIdx.x] = 0;
                __syncthreads();
            }
            // Counting sort by cluster, then exact fp64 member sums over a
            // contiguous eighth of the sorted tokens per warp.
            tile::counting_sort(cs, nch, Kp, cnt_s, perm, sc, warp, kWarps, lane);
            const int seg = (L + kWarps - 1) / kWarps;
            tile::member_sums(qbytes, sc, perm, warp * seg, min(L, (warp + 1) * seg), sums, lane);
        }
        __syncthreads();
        for (int i = threadIdx.x; i < Lp; i += kThreads) cprev[i] = cs[i];
        // (5) mu_k = fp32(sum_k / max(1, count_k)), one warp per centroid
        // (two rows per warp at a time, so their fp64 divisions overlap)
        const bool last = it == P.iters - 1;
        for (int kb2 = warp; kb2 < Kp; kb2 += 2 * kWarps) {
            float x[2][2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int kk = kb2 + h * kWarps;
                const int cnt = kk < K ? cnt_s[kk] : 0;
                const double den = (double)(cnt > 1 ? cnt : 1);
                x[h][0] = kk < K ? __double2float_rn(sums[kk * kD + 2 * lane] / den) : 0.f;
                x[h][1] = kk < K ? __double2float_rn(sums[kk * kD + 2 * lane + 1] / den) : 0.f;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int kk = kb2 + h * kWarps;
                if (kk < Kp) {
                    finalize_row(kk, x[h][0], x[h][1]);
                    if (last && P.cent && kk < K) {
                        float2 *dst = reinterpret_cast<float2 *>(P.cent + (head * K + kk) * kD);
                        dst[lane] = make_float2(x[h][0], x[h][1]);
                    }
                }
            }
        }
        finalize_set(P.hist ? P.hist + (head * P.iters + it) * (int64_t)L : nullptr);
    }
    if (P.iters == 0 && P.cent) {
        for (int e = threadIdx.x; e < K * kD; e += kThreads) P.cent[head * K * kD + e] = mu[(e / kD) * 65 + e % kD];
    }
    if (P.assign) {
        for (int i = threadIdx.x; i < L; i += kThreads) P.assign[head * L + i] = cs[i];
    }

    // ---- centroid attention over K/V tiles, up to kSlots in flight ------------
    const int n_cm = Kp / 16;          // centroid m-tiles: 1, 2 or 4
    const int G = kWarps / n_cm;       // warps sharing one m-tile: 8, 4 or 2
    const int cm = warp / G, kb = warp % G;
    const int keys_w = kTile / G;      // keys per warp per tile: 8, 16 or 32
    const float csc = P.scale * kLog2e;
    __syncthreads();  // Q is no longer read: the big region becomes K/V slots
    for (int s = 0; s < kSlots; ++s) {
        if (s < nT) {
            const uint32_t slot = big_s + s * 2 * kTile * 128;
            load_rows(slot, kh, s * kTile, kTile, L);
            load_rows(slot + kTile * 128, vh, s * kTile, kTile, L);
        }
        cp_async_commit();
    }
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

    // One group is committed per iteration (empty when there is nothing to
    // load), so tile tt's group is always the fifth newest at the wait.  The
    // slot of tile tt-1 is refilled right after the barrier that shows every
    // warp is done with it.
    for (int tt = 0; tt < nT; ++tt) {
        cp_async_wait<kSlots - 1>();
        __syncthreads();
        if (tt >= 1 && tt - 1 + kSlots < nT) {
            const uint32_t ks = big_s + ((tt - 1) % kSlots) * 2 * kTile * 128;
            load_rows(ks, kh, (tt - 1 + kSlots) * kTile, kTile, L);
            load_rows(ks + kTile * 128, vh, (tt - 1 + kSlots) * kTile, kTile, L);
        }
        cp_async_commit();
        const uint32_t kt = big_s + (tt % kSlots) * 2 * kTile * 128;
        const uint32_t vt = kt + kTile * 128;
        float sacc[4][4], slo[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[n][e] = slo[n][e] = 0.f;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            if (n * 8 >= keys_w) break;
            const int key0 = kb * keys_w + n * 8;
#pragma unroll
            for (int kp = 0; kp < 2; ++kp) {
                uint32_t bk[4];
                ldmatrix_x4(bk, kt + swz(key0 + (lane & 7), 4 * kp + (lane >> 3)));
                mma_16816(sacc[n], ahi[2 * kp], bk[0], bk[1]);
                mma_16816(slo[n], alo[2 * kp], bk[0], bk[1]);
                mma_16816(sacc[n], ahi[2 * kp + 1], bk[2], bk[3]);
                mma_16816(slo[n], alo[2 * kp + 1], bk[2], bk[3]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[n][e] += slo[n][e];
        }
        float tmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            if (n * 8 >= keys_w) break;
            const int key = tt * kTile + kb * keys_w + n * 8 + 2 * t;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (key + (e & 1) >= L) sacc[n][e] = -INFINITY;
            tmax[0] = fmaxf(tmax[0], fmaxf(sacc[n][0], sacc[n][1]));
            tmax[1] = fmaxf(tmax[1], fmaxf(sacc[n][2], sacc[n][3]));
        }
        float corr[2];
        bool grew = false;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 1));
            tmax[h] = fmaxf(tmax[h], __shfl_xor_sync(0xffffffffu, tmax[h], 2));
            const float mn = fmaxf(rm[h], tmax[h]);
            grew |= mn != rm[h];
            corr[h] = (mn == -INFINITY) ? 1.f : ex2((rm[h] - mn) * csc);
            rm[h] = mn;
            rl[h] *= corr[h];
        }
        if (__any_sync(0xffffffffu, grew)) {
#pragma unroll
            for (int d = 0; d < 8; ++d) {
                o_acc[d][0] *= corr[0];
                o_acc[d][1] *= corr[0];
                o_acc[d][2] *= corr[1];
                o_acc[d][3] *= corr[1];
            }
        }
        uint32_t pa[4][2];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            pa[n][0] = pa[n][1] = 0u;
            if (n * 8 >= keys_w) break;
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float mh = rm[e >> 1];
                p[e] = (mh == -INFINITY) ? 0.f : ex2((sacc[n][e] - mh) * csc);
            }
            rl[0] += p[0] + p[1];
            rl[1] += p[2] + p[3];
            pa[n][0] = pack_bf16(p[0], p[1]);
            pa[n][1] = pack_bf16(p[2], p[3]);
        }
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
    }
    cp_async_wait<0>();
    // combine the G partial states of each centroid m-tile (big region reused)
    {
        float *part = reinterpret_cast<float *>(smem + lay.big_off);  // [warp][16][64]
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
                const float f = (mw == -INFINITY) ? 0.f : ex2((mw - M) * csc);
                den = fmaf(ml[(w * 16 + rr) * 2 + 1], f, den);
                num = fmaf(part[(w * 16 + rr) * 64 + col], f, num);
            }
            vc[row * kVcStride + col] = (1.f - P.alpha) * (num / den);
        }
        __syncthreads();
    }

    // ---- window attention + gather + blend: blocks of 128 queries, K/V
    // double buffered, Q fragments straight from global memory (L2) ---------
    const int r = P.r;
    const int nblk = (L + kWinBlock - 1) / kWinBlock;
    auto issue_block = [&](int b) {
        if (b < nblk) {
            const int qb = b * kWinBlock;
            const int ks0 = max(0, qb - r) & ~7;
            const int ke = min(L - 1, qb + kWinBlock - 1 + r);
            const int nrows = (ke - ks0 + 1 + 7) & ~7;
            const uint32_t st = big_s + (b & 1) * lay.win_stage;
            load_rows(st, kh, ks0, nrows, ke + 1);
            load_rows(st + lay.win_rows * 128, vh, ks0, nrows, ke + 1);
        }
        cp_async_commit();
    };
    issue_block(0);
    __nv_bfloat16 *oh = P.out + head * (int64_t)L * kD;
    // Band mask of a warp's 16 x (8 kMaxNT) score tile as bits 4n+e: key
    // kst + 8n + 2t + (e&1) against query i0 + g + 8(e>>1).  A warp whose
    // whole band lies inside [0, L) sees the same pattern everywhere.
    auto band_bits = [&](int kst, int i0, bool check_L) {
        uint32_t m = 0u;
#pragma unroll
        for (int n = 0; n < kMaxNT; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int i = i0 + g + 8 * (e >> 1);
                const int jk = kst + n * 8 + 2 * t + (e & 1);
                const bool ok = jk >= i - r && jk <= i + r && (!check_L || jk < L);
                m |= (ok ? 1u : 0u) << (4 * n + e);
            }
        return m;
    };
    const uint32_t inner_bits = band_bits(-((r + 7) & ~7), 0, false);
    // Per-warp output staging (8 rows x 128 bytes, swizzled) in the centroid
    // region, which is dead once V_cent is formed.
    const uint32_t ost = sbase + lay.mu_off + warp * 1024;
    // Q fragments of this warp's 16 rows of a block, read from global memory
    // (L2); fetched one block ahead.
    uint32_t a[4][4];
    auto fetch_q = [&](int b) {
        const int i0b = b * kWinBlock + warp * 16;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int row = i0b + g + ((e & 1) ? 8 : 0);
                const int col = 16 * ks + 2 * t + ((e & 2) ? 8 : 0);
                a[ks][e] = (b < nblk && row < L) ? __ldg(reinterpret_cast<const unsigned int *>(qh + (int64_t)row * kD + col)) : 0u;
            }
        }
    };
    fetch_q(0);
    // Block b's stage is waited for, then the other stage (last read by
    // block b-1, which every warp has left at this barrier) takes block b+1.
    for (int b = 0; b < nblk; ++b) {
        const int qb = b * kWinBlock;
        const int ks0 = max(0, qb - r) & ~7;
        const int i0 = qb + warp * 16;
        cp_async_wait<0>();
        __syncthreads();
        issue_block(b + 1);
        const uint32_t kw_s = big_s + (b & 1) * lay.win_stage;
        const uint32_t vw_s = kw_s + lay.win_rows * 128;
        if (i0 < L) {
            const int kst = max(0, i0 - r) & ~7;
            const int kend = min(L - 1, i0 + 15 + r);
            const int nt = (kend - kst) / 8 + 1;
            const int lr0 = kst - ks0;
            const uint32_t mbits = (i0 >= r && i0 + 15 + r <= L - 1) ? inner_bits : band_bits(kst, i0, true);
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
                    for (int e = 0; e < 4; ++e)
                        if (!((mbits >> (4 * n + e)) & 1u)) sacc[n][e] = -INFINITY;
                    mx[0] = fmaxf(mx[0], fmaxf(sacc[n][0], sacc[n][1]));
                    mx[1] = fmaxf(mx[1], fmaxf(sacc[n][2], sacc[n][3]));
                }
            }
            float sum[2] = {0.f, 0.f}, mxc[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
                mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
                // rows past L have no key: every score is -inf and p = 0
                mxc[h] = (mx[h] == -INFINITY) ? 0.f : mx[h] * csc;
            }
            uint32_t pa[kMaxNT][2];
#pragma unroll
            for (int n = 0; n < kMaxNT; ++n) {
                pa[n][0] = pa[n][1] = 0u;
                if (n < nt) {
                    float p[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) p[e] = ex2(fmaf(sacc[n][e], csc, -mxc[e >> 1]));
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
            // gather + blend: O = (1 - alpha) V_cent[c_i] + alpha o_i, staged
            // eight rows at a time through shared memory (stmatrix) and
            // stored as whole 128-byte rows
            const float f0 = sum[0] > 0.f ? P.alpha / sum[0] : 0.f, f1 = sum[1] > 0.f ? P.alpha / sum[1] : 0.f;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int i = i0 + g + 8 * hh;
                const float f = hh ? f1 : f0;
                const float *vrow = vc + (i < L ? CA_IDX(cs[i], 0, K, 74) : 0) * kVcStride + 2 * t;
                uint32_t wv[8];
#pragma unroll
                for (int d = 0; d < 8; ++d) {
                    const float2 c2 = *reinterpret_cast<const float2 *>(vrow + 8 * d);
                    wv[d] = pack_bf16(fmaf(f, oacc[d][2 * hh], c2.x), fmaf(f, oacc[d][2 * hh + 1], c2.y));
                }
                const int sr = lane & 7, sd = lane >> 3;
                stmatrix_x4(ost + sr * 128 + ((sd ^ sr) << 4), wv[0], wv[1], wv[2], wv[3]);
                stmatrix_x4(ost + sr * 128 + (((sd + 4) ^ sr) << 4), wv[4], wv[5], wv[6], wv[7]);
                __syncwarp();
#pragma unroll
                for (int it2 = 0; it2 < 2; ++it2) {
                    const int rr = it2 * 4 + (lane >> 3), ch = lane & 7;
                    const int row = i0 + 8 * hh + rr;
                    uint4 val;
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                                 : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                                 : "r"(ost + rr * 128 + ((ch ^ rr) << 4))
                                 : "memory");
                    if (row < L) *reinterpret_cast<uint4 *>(oh + (int64_t)row * kD + ch * 8) = val;
                }
                __syncwarp();
            }
        }
        fetch_q(b + 1);
    }
    cp_async_wait<0>();
}

}  // namespace fused
}  // namespace ca
