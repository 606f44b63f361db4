// Tiled cluster-attention kernels for long sequences (bf16): a head is split
// over several CTAs.
//
//   tiled_update_kernel    (heads)         mu = strided init, or the update
//                                          mu_k = fp32(sum_k / max(1, count_k))
//                                          from the head's exact running sums;
//                                          also the bf16 hi/lo split, |mu|^2,
//                                          the centroids that are bitwise
//                                          copies of a lower-index one (they
//                                          can never win the argmin) and
//                                          max |mu|^2.
//   tiled_assign_kernel    (tiles, heads)  one Lloyd assignment for a tile of
//                                          512 queries: TMA-staged queries,
//                                          distances on tcgen05 (tensor-memory
//                                          accumulators), certified argmin,
//                                          exact fp64 re-measure of ambiguous
//                                          tokens, the tile's exact share of
//                                          the head's running member sums.
//   tiled_centroid_tc_kernel (chunks, heads) partial softmax state of every
//                                          centroid over a chunk of 512 to
//                                          2048 keys on tcgen05 (M = 64 tiles
//                                          at two lane offsets);
//   tiled_combine_kernel   (K, heads)      combines the chunk states into
//                                          V_cent.
//   tiled_window_tc_kernel (blocks, heads) clipped window attention for 128
//                                          queries on tcgen05 (radius <= 64),
//                                          gather V_cent[c_i], blend;
//   tiled_window_kernel    (blocks, heads) the same on mma.sync for radii up
//                                          to 128.
//
// Consecutive kernels are chained with programmatic dependent launch: each
// lets its successor start early, and the successor touches only the
// forward's inputs (q, k, v) and its own shared / tensor memory before
// waiting for its predecessor (pdl_wait).
//
// Model card "Hooshaai/distilbert-sst2-cluster-attention", Architecture
// Overview and Mathematical Formulation section 1; "Hooshaai/svd-sst2-
// roberta-cluster" sections 2.1 and 3.
#pragma once

#include <cuda.h>

#include "fused.cuh"
#include "kmeans_tile.cuh"
#include "umma.cuh"

namespace ca {
namespace tiled {

using fused::bf16hi;
using fused::bf16lo;
using fused::ex2;
using tile::bf16_to_f64;
using fused::kEps;
using fused::kLog2e;
using fused::load_rows;
using fused::up;

constexpr int kThreads = 256;
constexpr int kWarps = 8;
constexpr int kTileQ = 512;   // queries per assignment tile
constexpr int kDirectMovers = 16;  // up to this many movers per tile skip the sort
constexpr int kMaxChunk = 2048;  // most keys per centroid-attention CTA (a multiple of 256)
constexpr int kWinQ = 128;    // queries per window CTA
constexpr int kMaxR = 128;    // largest window radius floor(W/2)
constexpr int kNTChunk = 6;   // key n-tiles per online-softmax step in the window

__host__ __device__ inline int kpad(int K) { return K <= 16 ? 16 : (K <= 32 ? 32 : 64); }

// ---------------------------------------------------------------------------
// Centroid set of one head: mu^(0) or the update from the running sums.
struct UpdateParams {
    const __nv_bfloat16 *q;
    double *sum;             // [NH][Kp][64] exact running member sums (coordinate j at 16 (j mod 4) + j / 4)
    int *cnt;                // [NH][Kp] running member counts
    float *mu;               // [NH][Kp][64]
    __nv_bfloat16 *hi, *lo;  // [NH][Kp][64]
    float *mm;               // [NH][Kp] |mu_k|^2
    uint8_t *dead;           // [NH][Kp] 1 for centroids that can never win
    float *mstat;            // [NH][2] max over k < K of |mu_k|^2, and its square root
    float *cent_out;         // [NH][K][64] or null
    int L, K, Kp, init;
    int init_stride;         // 1: mu_k = Q[k max(1, L / K)] (the module's stride) instead of Q[floor(k L / K)]
    int empty_keep;          // 1: an empty cluster keeps its previous centroid instead of becoming zero
    const uint8_t *key_valid;  // [B][L] key-padding mask or null
    uint8_t *any_valid;        // [NH] written in init mode: 1 when the head has a valid key
    int H;                     // query heads per batch row
};

// grid (NH), 1024 threads.  mu_k = Q[floor(k L / K)] (init; the running sums
// and counts are cleared for the first assignment) or fp32(sum_k /
// max(1, count_k)); padding rows k >= K are zero.  Also the bf16 hi/lo
// split, |mu_k|^2, the dead marks (a bitwise copy of a lower-index centroid
// has the same distances and loses every tie; padding rows never win) and
// max |mu_k|^2 for the assignment's error bound.
constexpr int kUpdThreads = 1024;
__global__ void __launch_bounds__(kUpdThreads) tiled_update_kernel(UpdateParams P) {
    __shared__ float mus[64][kD + 1];
    __shared__ uint32_t hs[64];
    __shared__ float ms[64];
    __shared__ uint8_t ds[64];
    __shared__ int ns[64];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int K = P.K, Kp = P.Kp;
    const int64_t head = blockIdx.x, hb = head * Kp;
    pdl_launch();
    pdl_wait();
    if (tid < Kp) ns[tid] = P.init ? 0 : P.cnt[hb + tid];
    // thread (k0, j) takes coordinate j of centroids k0, k0 + 16, ...: every
    // load is issued before the first is used
    constexpr int kPer = 64 * kD / kUpdThreads, kRows = kUpdThreads / kD, kUw = kUpdThreads / 32;
    const int j = tid & (kD - 1), k0 = tid >> 6;
    double sv[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int k = k0 + kRows * u;
        sv[u] = 0.0;
        if (k < K) {
            if (P.init) {
                const int64_t row = P.init_stride ? (int64_t)k * max(1, P.L / K) : ((int64_t)k * P.L) / K;
                sv[u] = (double)__bfloat162float(P.q[(head * P.L + row) * kD + j]);
            } else {
                sv[u] = P.sum[(hb + k) * kD + (j & 3) * 16 + (j >> 2)];
            }
        }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
        const int k = k0 + kRows * u;
        if (k >= Kp) break;
        const int64_t o = (hb + k) * kD + j;
        float x = 0.f;
        if (k < K) {
            const int n = ns[k];
            if (P.init)
                x = (float)sv[u];
            else if (n == 0 && P.empty_keep)  // the previous centroid is read only in this mode
                x = P.mu[o];
            else
                x = __double2float_rn(sv[u] / (double)(n > 1 ? n : 1));
        }
        if (P.init) P.sum[o] = 0.0;
        mus[k][j] = x;
        P.mu[o] = x;
        const __nv_bfloat16 h = __float2bfloat16_rn(x);
        P.hi[o] = h;
        P.lo[o] = __float2bfloat16_rn(x - __bfloat162float(h));
        if (P.cent_out && k < K) P.cent_out[(head * K + k) * kD + j] = x;
    }
    if (P.init && tid < Kp) P.cnt[hb + tid] = 0;
    if (P.init && P.key_valid) {
        const uint8_t *kv = P.key_valid + (head / P.H) * P.L;
        int mine = 0;
        for (int jj = tid; jj < P.L; jj += kUpdThreads) mine |= kv[jj];
        mine = __syncthreads_or(mine);
        if (tid == 0) P.any_valid[head] = mine ? 1 : 0;
    }
    __syncthreads();
    for (int k = warp; k < Kp; k += kUw) {
        const float x0 = mus[k][2 * lane], x1 = mus[k][2 * lane + 1];
        float sq = fmaf(x0, x0, x1 * x1);
        uint32_t hv = __float_as_uint(x0) * (0x9E3779B1u + 4u * (uint32_t)lane) +
                      __float_as_uint(x1) * (0x85EBCA77u + 4u * (uint32_t)lane) + (uint32_t)lane * 0xC2B2AE3Du;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
            hv += __shfl_xor_sync(0xffffffffu, hv, off);
        }
        if (lane == 0) {
            ms[k] = sq;
            hs[k] = hv;
            ds[k] = k >= K ? 1 : 0;
            P.mm[hb + k] = sq;
        }
    }
    __syncthreads();
    if (warp == kUw - 1) {
        float mx = 0.f;
        for (int k2 = lane; k2 < K; k2 += 32) mx = fmaxf(mx, ms[k2]);
        mx = warp_max(mx);
        if (lane == 0) {
            P.mstat[head * 2 + 0] = mx;
            P.mstat[head * 2 + 1] = sqrtf(mx);
        }
    }
    __syncthreads();
    mark_copies(K, hs, &mus[0][0], kD + 1, ds, ms, warp, kUw, lane);
    __syncthreads();
    if (tid < Kp) P.dead[hb + tid] = ds[tid];
}

// Floats per chunk state of the centroid attention: 64 accumulator values,
// the running max (natural-log units), the running denominator, and padding
// to a 16-byte multiple.
constexpr int kPartLd = kD + 4;

// Centroid-attention combine for the tiled path: grid (K, NH), 64 threads.
// Thread c takes chunk c of a group of 64 (all its loads in flight at once);
// the group's states are rescaled to the group max and summed column by
// column through shared memory, in chunk order.
__global__ void __launch_bounds__(64) tiled_combine_kernel(int K, int n_chunks, const float *__restrict__ part,
                                                            float *__restrict__ vcent) {
    __shared__ float rows[64][65];
    __shared__ float red_m[2], red_l[2];
    const int k = blockIdx.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int64_t h = blockIdx.y;
    pdl_launch();
    pdl_wait();
    float M = -INFINITY, lsum = 0.f, acc = 0.f;
    for (int c0 = 0; c0 < n_chunks; c0 += 64) {
        const int c = c0 + t;
        const bool ok = c < n_chunks;
        const float *p = part + ((h * n_chunks + (ok ? c : 0)) * K + k) * kPartLd;
        float4 r[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) r[u] = ok ? reinterpret_cast<const float4 *>(p)[u] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float2 ml = ok ? *reinterpret_cast<const float2 *>(p + kD) : make_float2(-INFINITY, 0.f);
        const float gm = warp_max(ml.x);
        if (lane == 0) red_m[w] = gm;
        __syncthreads();
        const float Mn = fmaxf(M, fmaxf(red_m[0], red_m[1]));
        const float f_old = (M == -INFINITY) ? 0.f : expf(M - Mn);
        const float wc = (ml.x == -INFINITY) ? 0.f : expf(ml.x - Mn);
        const float gl = warp_sum(wc * ml.y);
        if (lane == 0) red_l[w] = gl;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            rows[t][4 * u + 0] = wc * r[u].x;
            rows[t][4 * u + 1] = wc * r[u].y;
            rows[t][4 * u + 2] = wc * r[u].z;
            rows[t][4 * u + 3] = wc * r[u].w;
        }
        __syncthreads();
        float col = 0.f;
        for (int cc = 0; cc < 64; ++cc) col += rows[cc][t];
        acc = fmaf(acc, f_old, col);
        lsum = fmaf(lsum, f_old, red_l[0] + red_l[1]);
        M = Mn;
        __syncthreads();
    }
    vcent[(h * K + k) * kD + t] = acc / lsum;
}

// ---------------------------------------------------------------------------
// One Lloyd assignment for a tile of up to 512 queries.
//
// Q tile: two TMA loads of 256 rows (128-byte swizzle) into shared memory.
// Distances: one thread issues tcgen05.mma for each 128-token block,
// D = Q [128 x 64] . (hi + lo)^T [64 x Kp] - |mu|^2 / 2 accumulated in fp32
// in tensor memory (4 k-steps with hi, then 4 with lo, then one whose A is a
// column of ones and whose B holds -|mu_k|^2 / 2 split into three bf16 terms,
// -inf for centroids that can never win), so s_k = |mu_k|^2 - 2 D_k needs no
// arithmetic: s_k <= m1 + 2E is D_k >= max_k D_k - E.
// Epilogue: every thread owns one token row of a block (tcgen05.ld), takes
// the maximum of D and the set of k with D_k >= max D - E; a single member
// is the certified argmin, several send the token to the exact fp64
// re-measure.  Sums: the tile's tokens (first
// iteration) or its movers (later ones, signed) are sorted by cluster and
// added run by run to the head's running sums with fp64 reductions.
//
// Error bound: the split leaves |mu - hi - lo| <= 2^-18 |mu| per coordinate
// (2^-17 |Q| |mu| in s); the products are exact and even an accumulator that
// truncates every one of the 131 additions stays within 131 * 2^-23
// (1 + 2^-8) (|Q| |mu| + |mu|^2 / 2) of the exact value (2^-14.97 (...) in
// s); the fp32 |mu_k|^2 and its three-term split add under 2^-20 |mu_k|^2.
// So |s_k error| <= 2^-14.6 (|Q| |mu_k| + |mu_k|^2), and E = 2^-13 (|Q|
// max|mu| + max|mu|^2) covers it threefold.
struct AssignLayout {
    int Kp;
    uint32_t q_off, r_off, mu_off, ones_off, mb_off, dead_off, cnt_off, c_off, cprev_off, list_off,
        lmask_off, ent_off, misc_off, bar_off, total;
    __host__ __device__ AssignLayout(int K) {
        Kp = kpad(K);
        uint32_t o = 0;
        q_off = o;  // 512 rows x 128 bytes, 1024-aligned (TMA / MMA swizzle)
        o += (uint32_t)kTileQ * 128u;
        // The MMA's B operand [hi; lo] (2 Kp rows of 128 bytes, 1024-aligned)
        // beside the fp32 centroids (rows padded to 68 floats: 16-byte
        // copies) for the exact decisions.
        r_off = o;
        mu_off = o + 2u * (uint32_t)Kp * 128u;
        o += up(2u * (uint32_t)Kp * 128u + (uint32_t)Kp * 68u * 4u, 16);
        // The |mu|^2 step's operands, K-major without swizzle (8-row x 16-byte
        // core matrices): A = 8 rows [1 1 1 0 ...] read for all 128 rows, B =
        // the Kp rows [h m l 0 ...] of -|mu_k|^2 / 2 = h + m + l.
        ones_off = o;
        o += 256u;
        mb_off = o;
        o += (uint32_t)Kp / 8u * 256u;
        dead_off = o;
        o += up((uint32_t)Kp, 16);
        cnt_off = o;
        o += (uint32_t)Kp * 4u;
        c_off = o;
        o += (uint32_t)kTileQ;
        cprev_off = o;
        o += (uint32_t)kTileQ;
        list_off = o;
        o += (uint32_t)kTileQ * 2u;
        lmask_off = o;  // candidate bits of each listed token (two words)
        o += (uint32_t)kTileQ * 8u;
        ent_off = o;  // packed sum entries sorted by cluster (runs padded to even length)
        o += (uint32_t)(kTileQ + 64) * 4u;
        misc_off = o;
        o += 64;
        bar_off = o;  // five mbarriers (queries, the products of each 128-row block) and the tensor-memory address
        o += 64;
        total = up(o, 128) + 1024;  // + slack to align the base to 1024 bytes
    }
};

struct AssignParams {
    const __nv_bfloat16 *q;
    const float *mu;
    const __nv_bfloat16 *hi, *lo;
    const float *mm;     // [NH][Kp] |mu_k|^2
    const uint8_t *dead; // [NH][Kp] 1 for centroids that can never win
    const float *mstat;  // [NH][2]
    float *qnorm;        // [NH][L] |Q_i| (written by the first iteration, read later)
    int32_t *assign;     // [NH][L]
    int32_t *hist;       // [NH][iters][L] or null (already offset by the iteration)
    int64_t hist_stride; // iters * L
    double *sum;         // [NH][Kp][64] exact running member sums (red.global.add; coordinate j at 16 (j mod 4) + j / 4)
    int *cnt;            // [NH][Kp] running member counts
    int L, K;
    int first;           // 1: first Lloyd iteration (the sums are clear); 0: they hold the previous assignment's
};

template <int KP>
__global__ void __launch_bounds__(kThreads, 2) tiled_assign_kernel(const __grid_constant__ CUtensorMap tmq,
                                                                    AssignParams P) {
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const AssignLayout lay(P.K);
    const int K = P.K;
    constexpr int Kp = KP;
    constexpr uint32_t kCols = 4u * KP;  // four 128-token accumulators of KP columns
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tile = blockIdx.x;
    const int64_t head = blockIdx.y;
    const int t0 = tile * kTileQ;
    const int Lt = min(kTileQ, P.L - t0);  // tokens in this tile
    const int nblk = (Lt + 127) / 128;

    const uint32_t sbase = smem_u32(smem);
    const uint32_t q_s = sbase + lay.q_off, b_s = sbase + lay.r_off;
    const uint32_t bar_tma = sbase + lay.bar_off, bar_mma = bar_tma + 8;  // bar_mma + 8 m: block m
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + lay.bar_off + 48);
    unsigned char *qbytes = smem + lay.q_off;
    float *mu = reinterpret_cast<float *>(smem + lay.mu_off);        // [Kp][68]
    int *cnt_s = reinterpret_cast<int *>(smem + lay.cnt_off);
    uint8_t *dead = smem + lay.dead_off;
    uint8_t *cs = smem + lay.c_off;
    uint8_t *cprev = smem + lay.cprev_off;
    uint16_t *list = reinterpret_cast<uint16_t *>(smem + lay.list_off);
    uint32_t *lmask = reinterpret_cast<uint32_t *>(smem + lay.lmask_off);
    uint32_t *ent = reinterpret_cast<uint32_t *>(smem + lay.ent_off);
    int *misc = reinterpret_cast<int *>(smem + lay.misc_off);
    constexpr int mu_ld = 68;

    pdl_launch();
    // The query tile is an input of the forward: its load starts before the
    // previous kernel (the centroid update) has finished.
    if (threadIdx.x == 0) {
        umma::mbar_init(bar_tma, 1);
#pragma unroll
        for (int m = 0; m < 4; ++m) umma::mbar_init(bar_mma + 8u * m, 1);
        umma::mbar_init_fence();
        const int nbox = Lt > 256 ? 2 : 1;
        umma::mbar_expect_tx(bar_tma, (uint32_t)nbox * 256u * 128u);
        umma::tma_load_3d(q_s, &tmq, 0, t0, (int)head, bar_tma);
        if (nbox == 2) umma::tma_load_3d(q_s + 256u * 128u, &tmq, 0, t0 + 256, (int)head, bar_tma);
    }
    pdl_wait();
    __syncwarp();
    if (warp == 0) umma::tmem_alloc(smem_u32(tslot), kCols);

    // Staging, all of it asynchronous or issued before it is waited for:
    // [hi; lo] in the swizzled K-major layout of the MMA, and the fp32
    // centroids for the re-measure.
    const int64_t cb = head * Kp;
    for (int e = threadIdx.x; e < Kp * 8; e += kThreads) {
        const int kk = e >> 3, ch = e & 7;
        cp_async16(b_s + swz(kk, ch), P.hi + (cb + kk) * kD + ch * 8, 16);
        cp_async16(b_s + (uint32_t)Kp * 128u + swz(kk, ch), P.lo + (cb + kk) * kD + ch * 8, 16);
    }
    for (int e = threadIdx.x; e < Kp * (kD / 4); e += kThreads)
        cp_async16(smem_u32(mu + (e >> 4) * mu_ld + (e & 15) * 4), P.mu + cb * kD + e * 4, 16);
    cp_async_commit();
    float qn_g[2] = {0.f, 0.f};
    const int wg = warp >> 2, q4 = warp & 3;
    if (!P.first) {
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
            const int row = (2 * wg + mi) * 128 + q4 * 32 + lane;
            if (row < Lt) qn_g[mi] = P.qnorm[head * P.L + t0 + row];
        }
        int pv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = threadIdx.x + u * kThreads;
            pv[u] = i < Lt ? P.assign[head * P.L + t0 + i] : 0;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) cprev[threadIdx.x + u * kThreads] = (uint8_t)pv[u];
    }
    for (int kk = threadIdx.x; kk < Kp; kk += kThreads) {
        const uint8_t dd = P.dead[cb + kk];
        dead[kk] = dd;
        cnt_s[kk] = 0;
        // -|mu_k|^2 / 2 as three bf16 terms (-inf: this centroid never wins)
        uint32_t w0 = 0xFF80u, w1 = 0u;  // bf16 -inf, then zeros
        if (!dd) {
            const float v = -0.5f * P.mm[cb + kk];
            const __nv_bfloat16 h = __float2bfloat16_rn(v);
            const float r1 = v - __bfloat162float(h);
            const __nv_bfloat16 m = __float2bfloat16_rn(r1);
            const __nv_bfloat16 l = __float2bfloat16_rn(r1 - __bfloat162float(m));
            w0 = (uint32_t)__bfloat16_as_ushort(h) | ((uint32_t)__bfloat16_as_ushort(m) << 16);
            w1 = (uint32_t)__bfloat16_as_ushort(l);
        }
        *reinterpret_cast<uint4 *>(smem + lay.mb_off + (kk >> 3) * 256 + (kk & 7) * 16) = make_uint4(w0, w1, 0u, 0u);
        *reinterpret_cast<uint4 *>(smem + lay.mb_off + (kk >> 3) * 256 + 128 + (kk & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    if (threadIdx.x < 16) {  // 8 rows [1 1 1 0 0 0 0 0 | 0 ... 0]
        const uint4 w = threadIdx.x < 8 ? make_uint4(0x3F803F80u, 0x3F80u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4 *>(smem + lay.ones_off + threadIdx.x * 16) = w;
    }
    for (int i = threadIdx.x; i < kTileQ; i += kThreads) cs[i] = i < Lt ? 0 : 0xFF;
    if (threadIdx.x == 0) {
        misc[0] = 0;
        misc[3] = 0;
    }
    const float mm_max = P.mstat[head * 2 + 0], mun_max = P.mstat[head * 2 + 1];
    cp_async_wait<0>();
    umma::fence_proxy_async_smem();
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t taddr = *tslot;

    // Q tile in shared memory (every thread observes the TMA completion
    // before reading it), then the distance MMAs.
    const bool q_ok = __syncthreads_and(umma::mbar_wait(bar_tma, 0));
    if (threadIdx.x == 0) {
        if (q_ok) {
            // each 128-row block commits to its own barrier; blocks 0 and 2
            // (the first of each warpgroup) go first
            constexpr uint32_t idesc = umma::idesc_bf16_f32(128, KP);
            for (int mo = 0; mo < 4; ++mo) {
                const int m = (mo >> 1) | ((mo & 1) << 1);  // 0, 2, 1, 3
                if (m >= nblk) continue;
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma::mma_bf16(taddr + (uint32_t)(m * KP),
                                       umma::desc_sw128(q_s + (uint32_t)m * 16384u + (uint32_t)ks * 32u),
                                       umma::desc_sw128(b_s + (uint32_t)part * (uint32_t)Kp * 128u + (uint32_t)ks * 32u),
                                       idesc, part > 0 || ks > 0);
                umma::mma_bf16(taddr + (uint32_t)(m * KP), umma::desc_kmajor_plain(sbase + lay.ones_off, 128u, 0u),
                               umma::desc_kmajor_plain(sbase + lay.mb_off, 128u, 256u), idesc, true);
                umma::mma_commit(bar_mma + 8u * (uint32_t)m);
            }
        } else {
            record_error(4, 30);
        }
    }
    // |Q_i| of this thread's rows: computed in the first iteration from the
    // tile in shared memory (and stored), read back in later ones.
    float qn[2] = {qn_g[0], qn_g[1]};
    if (P.first) {
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
            const int row = (2 * wg + mi) * 128 + q4 * 32 + lane;
            if (row < Lt) {
                float a = 0.f;
                if (q_ok) {
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(qbytes + swz(row, c));
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float x0 = bf16lo(ws[e]), x1 = bf16hi(ws[e]);
                            a = fmaf(x0, x0, fmaf(x1, x1, a));
                        }
                    }
                }
                qn[mi] = sqrtf(a);
                P.qnorm[head * P.L + t0 + row] = qn[mi];
            }
        }
    }
    if (q_ok) {
#pragma unroll
        for (int mi = 0; mi < 2; ++mi) {
            const int m = 2 * wg + mi;
            if (m >= nblk) break;  // uniform across the warp
            // this block's products (the warp waits as one)
            if (!__all_sync(0xffffffffu, umma::mbar_wait(bar_mma + 8u * (uint32_t)m, 0))) {
                if (lane == 0) record_error(4, 31);
                break;
            }
            umma::tc_fence_after();
            const int row = m * 128 + q4 * 32 + lane;
            float sv[KP];
            const uint32_t ta = taddr + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(m * KP);
#pragma unroll
            for (int c = 0; c < KP; c += 16) {
                float v16[16];
                umma::tmem_ld16(ta + (uint32_t)c, v16);
#pragma unroll
                for (int i = 0; i < 16; ++i) sv[c + i] = v16[i];
            }
            umma::tmem_ld_wait();
            if (row < Lt) {
                // sv[k] = D_k = Q.mu_k - |mu_k|^2 / 2 = -s_k / 2
                float m1a = -INFINITY, m1b = -INFINITY;
#pragma unroll
                for (int k2 = 0; k2 < KP / 2; ++k2) {
                    m1a = fmaxf(m1a, sv[2 * k2]);
                    m1b = fmaxf(m1b, sv[2 * k2 + 1]);
                }
                const float dmax = fmaxf(m1a, m1b);
                const float E = kEps * fmaf(qn[mi], mun_max, mm_max);
                const float thr = dmax - E;  // s_k <= m1 + 2E
                uint32_t bits[(KP + 31) / 32];
#pragma unroll
                for (int w2 = 0; w2 < (KP + 31) / 32; ++w2) bits[w2] = 0u;
#pragma unroll
                for (int k = 0; k < KP; ++k) bits[k >> 5] |= (sv[k] >= thr ? 1u : 0u) << (k & 31);
                int c = -1, n = 0;
#pragma unroll
                for (int w2 = (KP + 31) / 32 - 1; w2 >= 0; --w2) {
                    n += __popc(bits[w2]);
                    if (bits[w2]) c = w2 * 32 + __ffs(bits[w2]) - 1;
                }
                cs[row] = (uint8_t)(c < 0 ? 0 : c);
                if (n != 1) {
                    // ambiguous: the candidates for the exact decision are
                    // every k with s_k <= m1 + 3E, so any other centroid is
                    // worse than the fp32 winner by at least E in exact
                    // arithmetic
                    const float thr3 = dmax - 1.5f * E;
                    uint32_t b3[(KP + 31) / 32];
#pragma unroll
                    for (int w2 = 0; w2 < (KP + 31) / 32; ++w2) b3[w2] = 0u;
#pragma unroll
                    for (int k = 0; k < KP; ++k) b3[k >> 5] |= (sv[k] >= thr3 ? 1u : 0u) << (k & 31);
                    const int e = CA_IDX(atomicAdd(&misc[0], 1), 0, kTileQ, 63);
                    list[e] = (uint16_t)row;
#pragma unroll
                    for (int w2 = 0; w2 < (KP + 31) / 32; ++w2) lmask[e * 2 + w2] = b3[w2];
                }
            }
        }
    }
    umma::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        umma::tc_fence_after();
        umma::tmem_dealloc(taddr, kCols);
    }
    // exact re-measure of ambiguous tokens, one warp per token
    const int n_ref = misc[0];
    for (int e = warp; e < n_ref; e += kWarps) {
        const int row = CA_IDX(list[e], 0, Lt, 64);
        auto mu_at = [&](int k, int j) { return (double)mu[k * mu_ld + j]; };
        bool certain;
        int bk = tile::decide_candidates(qbytes, row, lmask[2 * e], KP > 32 ? lmask[2 * e + 1] : 0u, dead, mu_at, lane,
                                         certain);
        if (!certain) bk = tile::remeasure_token<(KP > 32)>(qbytes, row, Kp, dead, mu_at, lane);
        if (lane == 0) {
            if (bk >= K) {
                record_error(5, 3);
                bk = 0;
            }
            cs[row] = (uint8_t)bk;
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < Lt; i += kThreads) {
        P.assign[head * P.L + t0 + i] = cs[i];
        if (P.hist) P.hist[head * P.hist_stride + t0 + i] = cs[i];
    }
    // The tile's share of the head's running sums and counts: in the first
    // iteration every token is added; later, every token whose cluster
    // changed is subtracted from its old cluster and added to its new one.
    double *gsum = P.sum + cb * kD;
    int *gcnt = P.cnt + cb;
    if (P.first) {
        tile::counting_sort_even([&](int i) { return (int)cs[i]; }, [](int i) { return (uint32_t)i; }, kTileQ / 32, Kp,
                                 cnt_s, ent, &misc[4], warp, kWarps, lane);
        const int n2 = misc[4], seg = ((n2 >> 1) + kWarps - 1) / kWarps * 2;
        tile::run_sums_red(qbytes, ent, warp * seg, min(n2, (warp + 1) * seg), gsum, gcnt, lane);
        return;
    }
    for (int ch = warp; ch < kTileQ / 32; ch += kWarps) {
        const int i = ch * 32 + lane;
        const bool mv = i < Lt && cs[i] != cprev[i];
        const unsigned bal = __ballot_sync(0xffffffffu, mv);
        int base = 0;
        if (lane == 0 && bal) base = atomicAdd(&misc[3], __popc(bal));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (mv) list[base + __popc(bal & ((1u << lane) - 1u))] = (uint16_t)i;
    }
    __syncthreads();
    const int n_mv = misc[3];
    if (n_mv <= kDirectMovers) {
        // few movers: each warp subtracts its movers' rows from their old
        // clusters and adds them to their new ones directly (lane l:
        // coordinates 2l and 2l + 1); the sums are exact, so this changes
        // no bit of them
        for (int e = warp; e < n_mv; e += kWarps) {
            const int row = CA_IDX((int)list[e], 0, Lt, 79);
            const int cn = CA_IDX((int)cs[row], 0, Kp, 80), co = CA_IDX((int)cprev[row], 0, Kp, 81);
            const uint32_t w = *reinterpret_cast<const uint32_t *>(qbytes + swz(row, lane >> 2) + (lane & 3) * 4);
            const double x0 = (double)bf16lo(w), x1 = (double)bf16hi(w);
            const int j0 = 2 * lane, j1 = 2 * lane + 1;
            const int o0 = (j0 & 3) * 16 + (j0 >> 2), o1 = (j1 & 3) * 16 + (j1 >> 2);
            atomicAdd(gsum + cn * kD + o0, x0);
            atomicAdd(gsum + cn * kD + o1, x1);
            atomicAdd(gsum + co * kD + o0, -x0);
            atomicAdd(gsum + co * kD + o1, -x1);
            if (lane == 0) {
                atomicAdd(gcnt + cn, 1);
                atomicAdd(gcnt + co, -1);
            }
        }
        return;
    }
    // batches of up to 256 movers: entry e < m adds mover b + e to its new
    // cluster, entry m + e subtracts it from its old one
    for (int b = 0; b < n_mv; b += kTileQ / 2) {
        const int m = min(kTileQ / 2, n_mv - b);
        for (int kk = threadIdx.x; kk < Kp; kk += kThreads) cnt_s[kk] = 0;
        __syncthreads();
        auto row_of = [&](int e) { return CA_IDX((int)list[b + (e < m ? e : e - m)], 0, Lt, 65); };
        auto cl = [&](int e) {
            if (e >= 2 * m) return 0xFF;
            const int row = row_of(e);
            return CA_IDX((int)(e < m ? cs[row] : cprev[row]), 0, Kp, 66);
        };
        auto info = [&](int e) { return (uint32_t)row_of(e) | (e < m ? 0u : tile::kEntNeg); };
        tile::counting_sort_even(cl, info, kTileQ / 32, Kp, cnt_s, ent, &misc[4], warp, kWarps, lane);
        const int n2 = misc[4], seg = ((n2 >> 1) + kWarps - 1) / kWarps * 2;
        tile::run_sums_red(qbytes, ent, warp * seg, min(n2, (warp + 1) * seg), gsum, gcnt, lane);
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Centroid attention over a chunk of up to kMaxChunk keys on tcgen05: the
// chunk's softmax state of every centroid (sum of exp-weighted V rows, max
// in natural-log units, denominator) in the layout tiled_combine_kernel reads.
//
// The chunk goes in steps of 256 keys.  S = mu K^T runs as M = 64
// tcgen05.mma tiles (rows = centroids) at tensor-memory lane offsets 0 and
// 16, so the two tiles together fill all 128 lanes: tile o takes keys
// [128 o, 128 o + 128) of the step.  Within a tile, G = 64 / KP groups of
// rows each see their own 2 KP keys: the A operand of group g is a 64-row
// window into a zero-padded copy of the centroids that holds them at rows
// [g KP, (g + 1) KP) and zeros elsewhere, and the G products accumulate into
// one [64 x 2 KP] tile.  Each row's softmax weights go to shared memory at
// its own keys (block-diagonal P, zeros elsewhere), so one P V product per
// tile gives every row the weighted sum over its own keys.  Two threads
// (warpgroups) share a row: KP scores each.  Every thread folds its row's
// step results into a running state; the rows of one centroid (tiles and
// groups) are merged at the end.  K / V of the next step are loaded by TMA
// while this one computes.
struct CentroidTcLayout {
    uint32_t z_off, k_off, v_off, p_off, red_off, km_off, bar_off, total;
    __host__ __device__ CentroidTcLayout(int Kp, bool mask) {
        uint32_t o = 0;
        z_off = o;  // (128 - Kp) rows of 128 bytes: zeros, the centroids at rows [64 - Kp, 64), zeros
        o += up((uint32_t)(128 - Kp) * 128u, 1024);
        k_off = o;  // 256 keys x 128 bytes
        o += 256u * 128u;
        v_off = o;
        o += 256u * 128u;
        p_off = o;  // P of tile o: 64 rows x 128 keys (two 64-key slabs of 8 KB), o = 0, 1
        o += 2u * 16384u;
        red_off = o;  // [2][128] half-row maxima, then [2][128] half-row sums
        o += 2u * 2u * 128u * 4u;
        km_off = o;  // key mask of the chunk, one bit per key (masked calls)
        o += mask ? (uint32_t)kMaxChunk / 8u : 0u;
        bar_off = o;  // four mbarriers, the tensor-memory address
        o += 48;
        total = up(o, 128) + 1024;  // + slack to align the base to 1024 bytes
    }
};

struct CentroidTcParams {
    const __nv_bfloat16 *hi;  // [NH][Kp][64] centroids rounded to bf16
    float *part;              // [NH][n_chunks][K][kPartLd]
    int L, K, n_chunks;
    int chunk_keys;           // keys per CTA: a multiple of 256, at most kMaxChunk
    int H, H_kv;              // query head h reads key/value head kv_head(h) of the [B H_kv] tensors
    float scale;
    const uint8_t *key_valid;  // [B][L] key-padding mask or null: invalid keys take no weight
    const uint8_t *any_valid;  // [NH]: 0 when the head has no valid key (every key then weighs the same)
};

// Key/value head of query head h when H query heads share H_kv key/value
// heads per batch row (H_kv divides H).
__host__ __device__ __forceinline__ int kv_head(int64_t h, int H, int H_kv) {
    if (H_kv == H) return (int)h;  // no grouping (B H < 2^16)
    const int hh = (int)h;
    return (hh / H) * H_kv + (hh % H) / (H / H_kv);
}

template <int KP, bool MASK>
__global__ void __launch_bounds__(256, 2) tiled_centroid_tc_kernel(const __grid_constant__ CUtensorMap tmk,
                                                                     const __grid_constant__ CUtensorMap tmv,
                                                                     CentroidTcParams P) {
    constexpr int G = 64 / KP;      // row groups per M = 64 tile
    constexpr int N = 2 * KP;       // keys per group (S columns)
    constexpr uint32_t kOCol = 128; // O columns [128, 192)
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const CentroidTcLayout lay(KP, MASK);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q = warp & 3, wg = warp >> 2;
    const int L = P.L, K = P.K;
    const int chunk = blockIdx.x;
    const int64_t head = blockIdx.y;
    const int kvh = kv_head(head, P.H, P.H_kv);
    const int c0 = chunk * P.chunk_keys;
    const int nsteps = min(P.chunk_keys / 256, (L - c0 + 255) / 256);
    const uint32_t sb = smem_u32(smem);
    const uint32_t z_s = sb + lay.z_off, k_s = sb + lay.k_off, v_s = sb + lay.v_off, p_s = sb + lay.p_off;
    const uint32_t bar_k = sb + lay.bar_off, bar_v = bar_k + 8, bar_s = bar_k + 16, bar_o = bar_k + 24;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + lay.bar_off + 32);
    float *red = reinterpret_cast<float *>(smem + lay.red_off);

    pdl_launch();
    if (tid == 0) {
        umma::mbar_init(bar_k, 1);
        umma::mbar_init(bar_v, 1);
        umma::mbar_init(bar_s, 1);
        umma::mbar_init(bar_o, 1);
        umma::mbar_init_fence();
        umma::mbar_expect_tx(bar_k, 256u * 128u);
        umma::tma_load_3d(k_s, &tmk, 0, c0, kvh, bar_k);
        umma::mbar_expect_tx(bar_v, 256u * 128u);
        umma::tma_load_3d(v_s, &tmv, 0, c0, kvh, bar_v);
    }
    uint8_t *kmask = smem + lay.km_off;  // bit (c & 7) of byte c / 8: key c0 + c is valid
    if constexpr (MASK) {
        const uint8_t *kv = P.key_valid + (head / P.H) * L;
        for (int b = tid; b < P.chunk_keys / 8; b += 256) {
            uint32_t bits = 0u;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c = c0 + 8 * b + j;
                bits |= (c < L && kv[c] != 0) ? 1u << j : 0u;
            }
            kmask[b] = (uint8_t)bits;
        }
    }
    // P starts as zeros (each row later writes only its own keys)
    for (int e = tid; e < 2 * 16384 / 16; e += 256)
        asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(p_s + (uint32_t)e * 16u), "r"(0u) : "memory");
    pdl_wait();  // the centroids come from the previous kernel
    __syncwarp();
    if (warp == 0) umma::tmem_alloc(smem_u32(tslot), 256u);
    {
        const __nv_bfloat16 *hh = P.hi + head * KP * kD;
        for (int e = tid; e < (128 - KP) * 8; e += 256) {
            const int row = e >> 3, ch = e & 7, kk = row - (64 - KP);
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (kk >= 0 && kk < KP) w = *reinterpret_cast<const uint4 *>(hh + kk * kD + ch * 8);
            *reinterpret_cast<uint4 *>(smem + lay.z_off + swz(row, ch)) = w;
        }
    }
    umma::fence_proxy_async_smem();
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t taddr = *tslot;

    // This thread: tensor-memory lane tl = 32 q + lane holds row r of tile o.
    const int tl = 32 * q + lane, o = lane >> 4, r = 16 * q + (lane & 15);
    const int g = r / KP, kc = r % KP;  // row group, centroid
    const int blk = o * G + g;          // key block of the row within a step
    const float csc = P.scale * fused::kLog2e;
    const uint32_t trow = taddr + ((uint32_t)(32 * q) << 16);
    float m_run = -INFINITY, l_run = 0.f, acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    bool ok = true;
    int k_issued = 1, v_issued = 1;  // loads issued (completions waited so far: s for K, s for V)
    for (int s = 0; s < nsteps; ++s) {
        const uint32_t par = (uint32_t)s & 1u;
        ok = __syncthreads_and(ok && umma::mbar_wait(bar_k, par));
        if (!ok) break;
        if (tid == 0) {
            constexpr uint32_t idesc = umma::idesc_bf16_f32(64, N);
#pragma unroll
            for (int oo = 0; oo < 2; ++oo)
#pragma unroll
                for (int gg = 0; gg < G; ++gg) {
                    const uint32_t a0 = z_s + (uint32_t)((64 - KP) - gg * KP) * 128u;
                    const uint32_t b0 = k_s + (uint32_t)((oo * G + gg) * N) * 128u;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        umma::mma_bf16(taddr + ((uint32_t)(16 * oo) << 16), umma::desc_sw128(a0 + (uint32_t)ks * 32u),
                                       umma::desc_sw128(b0 + (uint32_t)ks * 32u), idesc, gg > 0 || ks > 0);
                }
            umma::mma_commit(bar_s);
        }
        ok = __syncthreads_and(umma::mbar_wait(bar_s, par));
        if (!ok) break;
        umma::tc_fence_after();
        // this thread's KP scores: columns [wg KP, wg KP + KP) of its row
        float v[KP];
#pragma unroll
        for (int pc = 0; pc < KP / 16; ++pc) {
            float t16[16];
            umma::tmem_ld16(trow + (uint32_t)(wg * KP + 16 * pc), t16);
#pragma unroll
            for (int t = 0; t < 16; ++t) v[16 * pc + t] = t16[t];
        }
        umma::tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < KP; ++t) asm volatile("" : "+f"(v[t]));
        const int key0 = c0 + 256 * s + blk * N + wg * KP;  // key of v[0]
        if constexpr (MASK) {
            // an invalid key takes no weight; a head without a valid key
            // weighs every key the same
            const bool any = P.any_valid[head] != 0;
            // this thread's KP keys start at a multiple of KP within the
            // chunk: their bits are whole bytes of the mask
            const uint8_t *mrow = kmask + ((key0 - c0) >> 3);
#pragma unroll
            for (int t = 0; t < KP; ++t)
                if (key0 + t < L) v[t] = any ? (((mrow[t >> 3] >> (t & 7)) & 1u) ? v[t] : -INFINITY) : 0.f;
        }
        if (c0 + 256 * (s + 1) > L) {  // keys past L (zero rows of the load) do not exist
#pragma unroll
            for (int t = 0; t < KP; ++t)
                if (key0 + t >= L) v[t] = -INFINITY;
        }
        float m = -INFINITY;
#pragma unroll
        for (int t = 0; t < KP; ++t) m = fmaxf(m, v[t]);
        red[wg * 128 + tl] = m;
        __syncthreads();
        m = fmaxf(red[tl], red[128 + tl]);
        const float mc = (m == -INFINITY) ? 0.f : m * csc;
        float l = 0.f;
        {
            const uint32_t prow = p_s + (uint32_t)o * 16384u;
            const int kb = g * N + wg * KP;  // first key column of this thread in the tile's P
#pragma unroll
            for (int c8 = 0; c8 < KP / 8; ++c8) {
                uint32_t pk[4];
#pragma unroll
                for (int t = 0; t < 8; t += 2) {
                    const float p0 = fused::ex2(fmaf(v[8 * c8 + t], csc, -mc));
                    const float p1 = fused::ex2(fmaf(v[8 * c8 + t + 1], csc, -mc));
                    l += p0 + p1;
                    pk[t >> 1] = pack_bf16(p0, p1);
                }
                const int col = kb + 8 * c8;
                asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(prow + (uint32_t)(col >> 6) * 8192u +
                                                                              swz(r, (col & 63) >> 3)),
                             "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3])
                             : "memory");
            }
        }
        red[256 + wg * 128 + tl] = l;
        umma::fence_proxy_async_smem();
        umma::tc_fence_before();
        __syncthreads();
        umma::tc_fence_after();
        if (tid == 0) {
            // K of the next step into the buffer the S product has finished reading
            if (s + 1 < nsteps) {
                umma::mbar_expect_tx(bar_k, 256u * 128u);
                umma::tma_load_3d(k_s, &tmk, 0, c0 + 256 * (s + 1), kvh, bar_k);
                ++k_issued;
            }
            if (umma::mbar_wait(bar_v, par)) {
                constexpr uint32_t idesc = umma::idesc_bf16_f32_bmn(64, 64);
#pragma unroll
                for (int oo = 0; oo < 2; ++oo)
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        umma::mma_bf16(taddr + ((uint32_t)(16 * oo) << 16) + kOCol,
                                       umma::desc_sw128(p_s + (uint32_t)oo * 16384u + (uint32_t)(ks >> 2) * 8192u +
                                                        (uint32_t)(ks & 3) * 32u),
                                       umma::desc_sw128(v_s + (uint32_t)(oo * 128 + ks * 16) * 128u), idesc, ks > 0);
                umma::mma_commit(bar_o);
            } else {
                record_error(4, 45);
            }
        }
        l = red[256 + tl] + red[384 + tl];
        ok = __syncthreads_and(umma::mbar_wait(bar_o, par));
        if (!ok) break;
        umma::tc_fence_after();
        float ov[32];
        umma::tmem_ld32(trow + kOCol + (uint32_t)(32 * wg), ov);
        umma::tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 32; ++t) asm volatile("" : "+f"(ov[t]));
        if (m != -INFINITY) {
            const float M = fmaxf(m_run, m);
            const float a = (m_run == -INFINITY) ? 0.f : fused::ex2((m_run - M) * csc);
            const float b = fused::ex2((m - M) * csc);
#pragma unroll
            for (int t = 0; t < 32; ++t) acc[t] = fmaf(acc[t], a, ov[t] * b);
            l_run = fmaf(l_run, a, l * b);
            m_run = M;
        }
        umma::tc_fence_before();
        __syncthreads();
        umma::tc_fence_after();
        if (tid == 0 && s + 1 < nsteps) {
            // V of the next step into the buffer the P V product has finished reading
            umma::mbar_expect_tx(bar_v, 256u * 128u);
            umma::tma_load_3d(v_s, &tmv, 0, c0 + 256 * (s + 1), kvh, bar_v);
            ++v_issued;
        }
    }
    if (!ok && tid == 0) {
        record_error(4, 44);
        // no load may still be writing this block's shared memory when it
        // exits: wait (bounded) for the last K and V loads issued
        umma::mbar_wait(bar_k, (uint32_t)(k_issued - 1) & 1u);
        umma::mbar_wait(bar_v, (uint32_t)(v_issued - 1) & 1u);
    }
    // Merge the rows of one centroid: the two tiles (lanes l and l ^ 16),
    // then the G row groups (quadrants) through shared memory.
    auto merge = [&](float m2, float l2, const float *a2) {
        const float M = fmaxf(m_run, m2);
        if (M == -INFINITY) return;
        const float fa = (m_run == -INFINITY) ? 0.f : fused::ex2((m_run - M) * csc);
        const float fb = (m2 == -INFINITY) ? 0.f : fused::ex2((m2 - M) * csc);
#pragma unroll
        for (int t = 0; t < 32; ++t) acc[t] = fmaf(acc[t], fa, a2[t] * fb);
        l_run = fmaf(l_run, fa, l2 * fb);
        m_run = M;
    };
    {
        float a2[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) a2[t] = __shfl_xor_sync(0xffffffffu, acc[t], 16);
        const float m2 = __shfl_xor_sync(0xffffffffu, m_run, 16), l2 = __shfl_xor_sync(0xffffffffu, l_run, 16);
        merge(m2, l2, a2);
    }
    if constexpr (G > 1) {
        // rows of group g > 0 hand their state to group 0 through the (dead) P buffer
        float *xs = reinterpret_cast<float *>(smem + lay.p_off);  // [G][wg][KP][34]
        __syncthreads();
        if (g > 0 && o == 0) {
            float *dst = xs + (((g * 2 + wg) * KP) + kc) * 34;
#pragma unroll
            for (int t = 0; t < 32; ++t) dst[t] = acc[t];
            dst[32] = m_run;
            dst[33] = l_run;
        }
        __syncthreads();
        if (g == 0 && o == 0) {
#pragma unroll 1
            for (int g2 = 1; g2 < G; ++g2) {
                const float *src = xs + (((g2 * 2 + wg) * KP) + kc) * 34;
                float a2[32];
#pragma unroll
                for (int t = 0; t < 32; ++t) a2[t] = src[t];
                merge(src[32], src[33], a2);
            }
        }
    }
    if (ok && g == 0 && o == 0 && kc < K) {
        float *dst = P.part + ((head * P.n_chunks + chunk) * K + kc) * kPartLd;
#pragma unroll
        for (int t = 0; t < 32; t += 4)
            *reinterpret_cast<float4 *>(dst + 32 * wg + t) = make_float4(acc[t], acc[t + 1], acc[t + 2], acc[t + 3]);
        if (wg == 0) {
            dst[kD] = m_run * P.scale;
            dst[kD + 1] = l_run;
        }
    }
    umma::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        umma::tc_fence_after();
        umma::tmem_dealloc(taddr, 256u);
    }
}

// ---------------------------------------------------------------------------
// Window attention + gather + blend for 128 queries; any radius <= kMaxR.
struct WindowLayout {
    int rows, Kp;
    uint32_t k_off, v_off, vc_off, c_off, st_off, total;
    __host__ __device__ WindowLayout(int K, int r) {
        Kp = kpad(K);
        rows = (int)up((uint32_t)(kWinQ + 2 * r + 8), 8);
        uint32_t o = 0;
        k_off = o;
        o += (uint32_t)rows * 128u;
        v_off = o;
        o += (uint32_t)rows * 128u;
        vc_off = o;  // (1 - alpha) V_cent, rows of fused::kVcStride floats
        o += (uint32_t)K * (uint32_t)fused::kVcStride * 4u;
        c_off = o;
        o += (uint32_t)kWinQ * 4u;
        st_off = o;  // per-warp output staging, 8 rows x 128 bytes
        o += (uint32_t)kWarps * 1024u;
        total = up(o, 128);
    }
};

struct WindowParams {
    const __nv_bfloat16 *q, *k, *v;  // k, v: [B H_kv][L][64]
    const float *vcent;     // [NH][K][64]
    const int32_t *assign;  // [NH][L]
    __nv_bfloat16 *out;
    int L, K, r;
    int H, H_kv;            // query head h reads key/value head kv_head(h)
    float alpha, scale;
    const uint8_t *key_valid;  // [B][L] key-padding mask or null (tensor-core kernel only)
    const __nv_bfloat16 *hi;   // [NH][Kp][64] final centroids rounded to bf16 (soft gather)
    int Kp;
};

__global__ void __launch_bounds__(kThreads, 2) tiled_window_kernel(WindowParams P) {
    extern __shared__ __align__(1024) unsigned char smem[];
    const WindowLayout lay(P.K, P.r);
    const int L = P.L, K = P.K, r = P.r;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int64_t head = blockIdx.y;
    const int qb = blockIdx.x * kWinQ;
    const __nv_bfloat16 *qh = P.q + head * (int64_t)L * kD;
    const int64_t kvh = kv_head(head, P.H, P.H_kv);
    const __nv_bfloat16 *kh = P.k + kvh * (int64_t)L * kD;
    const __nv_bfloat16 *vh = P.v + kvh * (int64_t)L * kD;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t kw_s = sbase + lay.k_off, vw_s = sbase + lay.v_off;
    float *vc = reinterpret_cast<float *>(smem + lay.vc_off);
    int *cblk = reinterpret_cast<int *>(smem + lay.c_off);

    const int ks0 = max(0, qb - r) & ~7;
    const int ke = min(L - 1, qb + kWinQ - 1 + r);
    const int nrows = (ke - ks0 + 1 + 7) & ~7;
    pdl_launch();
    load_rows(kw_s, kh, ks0, nrows, ke + 1);
    load_rows(vw_s, vh, ks0, nrows, ke + 1);
    cp_async_commit();
    pdl_wait();  // V_cent and the assignments come from earlier kernels
    const float *vch = P.vcent + head * (int64_t)K * kD;
    const float be = 1.f - P.alpha;
    for (int e = threadIdx.x; e < K * kD / 4; e += kThreads) {
        float4 x = reinterpret_cast<const float4 *>(vch)[e];
        x.x *= be;
        x.y *= be;
        x.z *= be;
        x.w *= be;
        *reinterpret_cast<float4 *>(vc + (e >> 4) * fused::kVcStride + (e & 15) * 4) = x;
    }
    for (int i = threadIdx.x; i < kWinQ; i += kThreads)
        cblk[i] = (qb + i < L) ? CA_IDX(P.assign[head * L + qb + i], 0, K, 68) : 0;
    const int i0 = qb + warp * 16;
    uint32_t a[4][4];
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int row = i0 + g + ((e & 1) ? 8 : 0);
            const int col = 16 * ks + 2 * t + ((e & 2) ? 8 : 0);
            a[ks][e] = row < L ? __ldg(reinterpret_cast<const unsigned int *>(qh + (int64_t)row * kD + col)) : 0u;
        }
    }
    cp_async_wait<0>();
    __syncthreads();
    if (i0 >= L) return;
    const float csc = P.scale * kLog2e;
    const int kst = max(0, i0 - r) & ~7;
    const int kend = min(L - 1, i0 + 15 + r);
    const int nt = (kend - kst) / 8 + 1;
    const int lr0 = kst - ks0;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float oacc[8][4];
#pragma unroll
    for (int d = 0; d < 8; ++d)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[d][e] = 0.f;
    for (int c0 = 0; c0 < nt; c0 += kNTChunk) {
        const int cn = min(kNTChunk, nt - c0);
        float sacc[kNTChunk][4];
#pragma unroll
        for (int n = 0; n < kNTChunk; ++n) {
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[n][e] = 0.f;
            if (n < cn) {
#pragma unroll
                for (int kp = 0; kp < 2; ++kp) {
                    uint32_t bk[4];
                    ldmatrix_x4(bk, kw_s + swz(lr0 + (c0 + n) * 8 + (lane & 7), 4 * kp + (lane >> 3)));
                    mma_16816(sacc[n], a[2 * kp], bk[0], bk[1]);
                    mma_16816(sacc[n], a[2 * kp + 1], bk[2], bk[3]);
                }
            }
        }
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n = 0; n < kNTChunk; ++n) {
            if (n < cn) {
                // keys j0..j0+7 against rows i0..i0+15: only a tile that is not
                // inside every row's band (and inside [0, L)) needs the mask
                const int j0 = kst + (c0 + n) * 8;
                if (!(j0 >= i0 + 15 - r && j0 + 7 <= i0 + r && j0 + 7 < L)) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = i0 + g + 8 * (e >> 1);
                        const int jk = j0 + 2 * t + (e & 1);
                        const bool ok = jk >= i - r && jk <= i + r && jk < L;
                        if (!ok) sacc[n][e] = -INFINITY;
                    }
                }
                mx[0] = fmaxf(mx[0], fmaxf(sacc[n][0], sacc[n][1]));
                mx[1] = fmaxf(mx[1], fmaxf(sacc[n][2], sacc[n][3]));
            }
        }
        float corr[2], mhc[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
            const float mn = fmaxf(m_run[h], mx[h]);
            corr[h] = (mn == -INFINITY) ? 1.f : ex2((m_run[h] - mn) * csc);
            m_run[h] = mn;
            l_run[h] *= corr[h];
            // a row with no key yet: every score is -inf and p = 0
            mhc[h] = (mn == -INFINITY) ? 0.f : mn * csc;
        }
#pragma unroll
        for (int d = 0; d < 8; ++d) {
            oacc[d][0] *= corr[0];
            oacc[d][1] *= corr[0];
            oacc[d][2] *= corr[1];
            oacc[d][3] *= corr[1];
        }
        uint32_t pa[kNTChunk][2];
#pragma unroll
        for (int n = 0; n < kNTChunk; ++n) {
            pa[n][0] = pa[n][1] = 0u;
            if (n < cn) {
                float p[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) p[e] = ex2(fmaf(sacc[n][e], csc, -mhc[e >> 1]));
                l_run[0] += p[0] + p[1];
                l_run[1] += p[2] + p[3];
                pa[n][0] = pack_bf16(p[0], p[1]);
                pa[n][1] = pack_bf16(p[2], p[3]);
            }
        }
#pragma unroll
        for (int n2 = 0; n2 < kNTChunk / 2; ++n2) {
            if (2 * n2 + 1 < cn) {
                const uint32_t a4[4] = {pa[2 * n2][0], pa[2 * n2][1], pa[2 * n2 + 1][0], pa[2 * n2 + 1][1]};
#pragma unroll
                for (int dq = 0; dq < 4; ++dq) {
                    uint32_t bv[4];
                    const int m = lane >> 3;
                    ldmatrix_x4_trans(bv, vw_s + swz(lr0 + (c0 + 2 * n2) * 8 + (lane & 7) + ((m & 1) ? 8 : 0), 2 * dq + (m >> 1)));
                    mma_16816(oacc[2 * dq], a4, bv[0], bv[1]);
                    mma_16816(oacc[2 * dq + 1], a4, bv[2], bv[3]);
                }
            } else if (2 * n2 < cn) {
#pragma unroll
                for (int dq = 0; dq < 2; ++dq) {
                    uint32_t bv[4];
                    ldmatrix_x4_trans(bv, vw_s + swz(lr0 + (c0 + 2 * n2) * 8 + (lane & 7), 4 * dq + (lane >> 3)));
#pragma unroll
                    for (int u = 0; u < 4; ++u) mma_1688(oacc[4 * dq + u], pa[2 * n2][0], pa[2 * n2][1], bv[u]);
                }
            }
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
    }
    // gather + blend: O = (1 - alpha) V_cent[c_i] + alpha o_i, staged eight
    // rows at a time through shared memory (stmatrix) and stored as whole
    // 128-byte rows
    const float f0 = l_run[0] > 0.f ? P.alpha / l_run[0] : 0.f, f1 = l_run[1] > 0.f ? P.alpha / l_run[1] : 0.f;
    __nv_bfloat16 *oh = P.out + head * (int64_t)L * kD;
    const uint32_t ost = sbase + lay.st_off + warp * 1024;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int i = i0 + g + 8 * hh;
        const float f = hh ? f1 : f0;
        const float *vrow = vc + (i < L ? cblk[i - qb] : 0) * fused::kVcStride + 2 * t;
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

// ---------------------------------------------------------------------------
// Window attention + gather + blend for 128 queries on tcgen05, radius
// r <= RP (RP = 32 or 64).  Keys of the CTA's window: [q0 - RP, q0 + 127 +
// RP], NK = 128 + 2 RP of them, TMA-loaded with the query block (rows outside
// [0, L) arrive as zeros and are masked).
//
//   S = Q K^T           one thread issues 4 MMAs (M = 128, N = NK, K = 64),
//                       fp32 scores in tensor memory;
//   softmax             query row i is tensor-memory lane i; the 32 + 2 RP
//                       columns of its warp quarter are split between two
//                       threads (one per warpgroup) and read twice (row
//                       max, then exp2), with the partial maxima and sums
//                       exchanged through shared memory; keys outside
//                       |i - j| <= r or [0, L) get weight 0, and chunks
//                       inside every row's band skip the mask; P is
//                       rounded to bf16 into shared memory
//                       (over the dead Q and K tiles, K-major, 128-byte
//                       swizzled blocks of 64 keys);
//   O = P V             NK / 16 MMAs (M = 128, N = 64), V read N-major as
//                       loaded, accumulated over the first 64 columns of S;
//   epilogue            O = (1 - alpha) V_cent[c_i] + (alpha / l_i) o_i,
//                       rounded once to bf16, one 128-byte row per thread.
struct WindowTcLayout {
    int NK;
    uint32_t qk_off, v_off, red_off, km_off, mu_off, vc_off, p2_off, red2_off, bar_off, total;
    __host__ __device__ WindowTcLayout(int RP, bool mask, bool soft) {
        NK = 128 + 2 * RP;
        qk_off = 0;  // Q (16 KB) then K (NK rows); afterwards P (NK / 64 blocks of 16 KB)
        const uint32_t qk = 16384u + (uint32_t)NK * 128u, pb = (uint32_t)NK / 64u * 16384u;
        v_off = up(qk > pb ? qk : pb, 1024);
        red_off = v_off + (uint32_t)NK * 128u;  // [4][128] floats: partial row maxima and sums
        km_off = red_off + 4u * 128u * 4u;      // key mask of the window, then [2][128] row flags (masked calls)
        uint32_t o = km_off + (mask ? up((uint32_t)NK + 256u, 16) : 0u);
        // soft gather: the centroids (B of S2 = Q mu^T), V_cent in bf16 (B of
        // G = P2 V_cent, N-major), the weights P2, and their row maxima / sums
        mu_off = vc_off = p2_off = red2_off = o;
        if (soft) {
            mu_off = up(o, 1024);
            vc_off = mu_off + 64u * 128u;
            p2_off = vc_off + 64u * 128u;
            red2_off = p2_off + 128u * 128u;
            o = red2_off + 4u * 128u * 4u;
        }
        bar_off = o;
        total = up(bar_off + 32u, 128) + 1024;  // + slack to align the base to 1024 bytes
    }
};

template <int RP, bool MASK, bool SOFT>
__global__ void __launch_bounds__(256, 2) tiled_window_tc_kernel(const __grid_constant__ CUtensorMap tmq,
                                                                  const __grid_constant__ CUtensorMap tmk,
                                                                  const __grid_constant__ CUtensorMap tmv,
                                                                  const __grid_constant__ CUtensorMap tmo,
                                                                  WindowParams P) {
    constexpr int NK = 128 + 2 * RP;
    constexpr int NC = RP / 16 + 1;    // 32-column chunks of one warp quarter's window
    // soft gather: S2 = Q mu^T in tensor-memory columns [NK, NK + 64), which
    // exist only for the radius-32 window
    static_assert(!SOFT || NK + 64 <= 256, "the soft gather needs the radius-32 window");
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const WindowTcLayout lay(RP, MASK, SOFT);
    const int tid = threadIdx.x, warp = tid >> 5, wg = warp >> 2, q4 = warp & 3;
    const int L = P.L, K = P.K, r = P.r;
    const int64_t head = blockIdx.y;
    const int q0 = blockIdx.x * 128;
    const int kb0 = q0 - RP;  // key of window column 0
    const uint32_t sb = smem_u32(smem);
    const uint32_t q_s = sb + lay.qk_off, k_s = q_s + 16384u, v_s = sb + lay.v_off, p_s = q_s;
    const uint32_t bar_ld = sb + lay.bar_off, bar_s = bar_ld + 8, bar_o = bar_ld + 16;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + lay.bar_off + 24);
    float *red = reinterpret_cast<float *>(smem + lay.red_off);  // [2][128] partial max, then [2][128] partial sums

    pdl_launch();
    if (tid == 0) {
        umma::mbar_init(bar_ld, 1);
        umma::mbar_init(bar_s, 1);
        umma::mbar_init(bar_o, 1);
        umma::mbar_init_fence();
        umma::mbar_expect_tx(bar_ld, (uint32_t)(128 + 2 * NK) * 128u);
        umma::tma_load_3d(q_s, &tmq, 0, q0, (int)head, bar_ld);
        const int kvh = kv_head(head, P.H, P.H_kv);
        umma::tma_load_3d(k_s, &tmk, 0, kb0, kvh, bar_ld);
        umma::tma_load_3d(v_s, &tmv, 0, kb0, kvh, bar_ld);
    }
    uint8_t *kmask = smem + lay.km_off, *rowflag = kmask + NK;
    if constexpr (MASK) {  // the window's key mask (an input: before the wait)
        const uint8_t *kv = P.key_valid + (head / P.H) * L;
        for (int c = tid; c < NK; c += 256) kmask[c] = (kb0 + c >= 0 && kb0 + c < L) ? kv[kb0 + c] : 0;
    }
    pdl_wait();  // V_cent and the assignments come from earlier kernels
    __syncwarp();
    if (warp == 0) umma::tmem_alloc(smem_u32(tslot), 256u);
    // Thread (wg, q4, lane) serves query row i = 32 q4 + lane: warpgroup wg
    // reads its share of the row's score columns and writes half of its
    // output row.
    const int i = 32 * q4 + (tid & 31), qi = q0 + i;
    const int ci = (qi < L && !SOFT) ? CA_IDX(P.assign[head * L + qi], 0, K, 67) : 0;
    if constexpr (SOFT) {
        // centroids (rows >= K zero) and V_cent rounded to bf16, as 128-byte
        // swizzled rows for the two soft-gather products
        for (int e = tid; e < 64 * 8; e += 256) {
            const int kk = e >> 3, ch = e & 7;
            uint4 wm = make_uint4(0u, 0u, 0u, 0u), wv = wm;
            if (kk < K) {
                wm = *reinterpret_cast<const uint4 *>(P.hi + (head * P.Kp + kk) * kD + ch * 8);
                const float4 *src = reinterpret_cast<const float4 *>(P.vcent + (head * K + kk) * kD + ch * 8);
                const float4 a = src[0], b = src[1];
                wv = make_uint4(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w), pack_bf16(b.x, b.y), pack_bf16(b.z, b.w));
            }
            *reinterpret_cast<uint4 *>(smem + lay.mu_off + swz(kk, ch)) = wm;
            *reinterpret_cast<uint4 *>(smem + lay.vc_off + swz(kk, ch)) = wv;
        }
        umma::fence_proxy_async_smem();
    }
    const float4 *vrow = reinterpret_cast<const float4 *>(P.vcent + (head * K + ci) * kD) + 8 * wg;
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    const uint32_t taddr = *tslot;

    const bool ld_ok = __syncthreads_and(umma::mbar_wait(bar_ld, 0));
    if (tid == 0) {
        if (ld_ok) {
            constexpr uint32_t idesc = umma::idesc_bf16_f32(128, NK);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma::mma_bf16(taddr, umma::desc_sw128(q_s + (uint32_t)ks * 32u), umma::desc_sw128(k_s + (uint32_t)ks * 32u),
                               idesc, ks > 0);
            if constexpr (SOFT) {
                constexpr uint32_t idesc2 = umma::idesc_bf16_f32(128, 64);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma::mma_bf16(taddr + (uint32_t)NK, umma::desc_sw128(q_s + (uint32_t)ks * 32u),
                                   umma::desc_sw128(sb + lay.mu_off + (uint32_t)ks * 32u), idesc2, ks > 0);
            }
            umma::mma_commit(bar_s);
        } else {
            record_error(4, 40);
        }
    }
    const bool s_ok = __syncthreads_and(ld_ok && umma::mbar_wait(bar_s, 0));
    if (!s_ok && ld_ok && tid == 0) record_error(4, 41);
    umma::tc_fence_after();

    // Row i's keys: window columns [lo, hi] (inclusive).  The rows of warp
    // quarter q4 lie in columns [32 q4, 32 q4 + 32 NC); warpgroup wg takes
    // the half [32 q4 + HALF wg, + HALF) and reads it from tensor memory
    // once (16-column pieces, one wait); a piece inside [lo, hi] needs no
    // mask.
    constexpr int HALF = 16 * NC;         // 80 (RP = 64) or 48 (RP = 32) columns per thread
    constexpr int NP = HALF / 16;         // 16-column pieces per thread
    const float csc = P.scale * fused::kLog2e;
    const int lo = max(i + RP - r, RP - q0), hi = min(i + RP + r, L - 1 - kb0);
    const int cw = 32 * q4, cb0 = cw + HALF * wg;
    const uint32_t trow = taddr + ((uint32_t)(32 * q4) << 16);
    float v[HALF];
    float m = -INFINITY;
    if (s_ok) {
#pragma unroll
        for (int pc = 0; pc < NP; ++pc) {
            float t16[16];
            umma::tmem_ld16(trow + (uint32_t)(cb0 + 16 * pc), t16);
#pragma unroll
            for (int t = 0; t < 16; ++t) v[16 * pc + t] = t16[t];
        }
        umma::tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < HALF; ++t) asm volatile("" : "+f"(v[t]));  // used only after the wait
        // Scores outside [lo, hi] become -inf (their weight ex2(-inf) is
        // +0).  A piece inside the band of every row of the warp (a
        // warp-uniform test) needs no mask, so no branch diverges.
        const int lo_w = __reduce_max_sync(0xffffffffu, lo), hi_w = __reduce_min_sync(0xffffffffu, hi);
#pragma unroll
        for (int pc = 0; pc < NP; ++pc) {
            const int cb = cb0 + 16 * pc;
            if (!(cb >= lo_w && cb + 15 <= hi_w)) {
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    if ((unsigned)(cb + t - lo) > (unsigned)(hi - lo)) v[16 * pc + t] = -INFINITY;
            }
        }
        if constexpr (MASK) {
            // Invalid keys take no weight; a row whose window holds no valid
            // key weighs its window's keys the same (scores 0).
            int mine = 0;
#pragma unroll
            for (int t = 0; t < HALF; ++t) mine |= (v[t] != -INFINITY && kmask[cb0 + t]) ? 1 : 0;
            rowflag[wg * 128 + i] = (uint8_t)mine;
        }
    }
    if constexpr (MASK) {
        __syncthreads();
        const bool any = (rowflag[i] | rowflag[128 + i]) != 0;
        if (s_ok) {
#pragma unroll
            for (int t = 0; t < HALF; ++t)
                if (v[t] != -INFINITY) v[t] = any ? (kmask[cb0 + t] ? v[t] : -INFINITY) : 0.f;
        }
    }
    if (s_ok) {
#pragma unroll
        for (int t = 0; t < HALF; ++t) m = fmaxf(m, v[t]);
    }
    float *red2 = reinterpret_cast<float *>(smem + lay.red2_off);  // soft gather: [2][128] maxima, then sums
    if constexpr (SOFT) {
        // this thread's 32 centroid scores of the row (centroids 32 wg ..)
        float m2 = -INFINITY;
        if (s_ok) {
            float s2[32];
            umma::tmem_ld32(trow + (uint32_t)(NK + 32 * wg), s2);
            umma::tmem_ld_wait();
#pragma unroll
            for (int t = 0; t < 32; ++t) asm volatile("" : "+f"(s2[t]));
#pragma unroll
            for (int t = 0; t < 32; ++t) m2 = fmaxf(m2, 32 * wg + t < K ? s2[t] : -INFINITY);
        }
        red2[wg * 128 + i] = m2;
    }
    red[wg * 128 + i] = m;
    __syncthreads();
    m = fmaxf(red[i], red[128 + i]);
    const float mc = (m == -INFINITY) ? 0.f : m * csc;
    float l = 0.f;
    auto p_chunk = [&](int c8) -> uint32_t {  // byte address of 8-key chunk c8 of row i
        return p_s + (uint32_t)(c8 >> 3) * 16384u + swz(i, c8 & 7);
    };
    if (s_ok) {
        // zeros outside the warp quarter's columns (warpgroup 0 before them,
        // warpgroup 1 after them)
        const int z0 = wg == 0 ? 0 : (cw + 32 * NC) / 8, z1 = wg == 0 ? cw / 8 : NK / 8;
        for (int c8 = z0; c8 < z1; ++c8)
            asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(p_chunk(c8)), "r"(0u) : "memory");
#pragma unroll
        for (int pc = 0; pc < NP; ++pc) {
            const int cb = cb0 + 16 * pc;
            uint32_t pk[8];
#pragma unroll
            for (int t = 0; t < 16; t += 2) {
                const float p0 = fused::ex2(fmaf(v[16 * pc + t], csc, -mc));
                const float p1 = fused::ex2(fmaf(v[16 * pc + t + 1], csc, -mc));
                l += p0 + p1;
                pk[t >> 1] = pack_bf16(p0, p1);
            }
#pragma unroll
            for (int q = 0; q < 2; ++q)
                asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(p_chunk(cb / 8 + q)), "r"(pk[4 * q]),
                             "r"(pk[4 * q + 1]), "r"(pk[4 * q + 2]), "r"(pk[4 * q + 3])
                             : "memory");
        }
    }
    if constexpr (SOFT) {
        const float m2 = fmaxf(red2[i], red2[128 + i]), mc2 = m2 * csc;
        float l2 = 0.f;
        if (s_ok) {
            float s2[32];
            umma::tmem_ld32(trow + (uint32_t)(NK + 32 * wg), s2);
            umma::tmem_ld_wait();
#pragma unroll
            for (int t = 0; t < 32; ++t) asm volatile("" : "+f"(s2[t]));
            uint32_t pk[16];
#pragma unroll
            for (int t = 0; t < 32; t += 2) {
                const float p0 = 32 * wg + t < K ? fused::ex2(fmaf(s2[t], csc, -mc2)) : 0.f;
                const float p1 = 32 * wg + t + 1 < K ? fused::ex2(fmaf(s2[t + 1], csc, -mc2)) : 0.f;
                l2 += p0 + p1;
                pk[t >> 1] = pack_bf16(p0, p1);
            }
            const uint32_t p2_s = sb + lay.p2_off;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(p2_s + swz(i, 4 * wg + q)), "r"(pk[4 * q]),
                             "r"(pk[4 * q + 1]), "r"(pk[4 * q + 2]), "r"(pk[4 * q + 3])
                             : "memory");
        }
        red2[256 + wg * 128 + i] = l2;
    }
    red[256 + wg * 128 + i] = l;
    umma::fence_proxy_async_smem();
    umma::tc_fence_before();
    __syncthreads();
    umma::tc_fence_after();
    if (tid == 0 && s_ok) {
        constexpr uint32_t idesc = umma::idesc_bf16_f32_bmn(128, 64);
#pragma unroll
        for (int ks = 0; ks < NK / 16; ++ks)
            umma::mma_bf16(taddr, umma::desc_sw128(p_s + (uint32_t)(ks >> 2) * 16384u + (uint32_t)(ks & 3) * 32u),
                           umma::desc_sw128(v_s + (uint32_t)ks * 2048u), idesc, ks > 0);
        if constexpr (SOFT) {
            // G = P2 V_cent into columns [64, 128) (their scores were read)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma::mma_bf16(taddr + 64u, umma::desc_sw128(sb + lay.p2_off + (uint32_t)ks * 32u),
                               umma::desc_sw128(sb + lay.vc_off + (uint32_t)ks * 2048u), idesc, ks > 0);
        }
        umma::mma_commit(bar_o);
    }
    // this thread's half of the token's V_cent row
    float4 g[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) g[u] = SOFT ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldg(vrow + u);
    l = red[256 + i] + red[384 + i];
    const bool o_ok = __syncthreads_and(s_ok && umma::mbar_wait(bar_o, 0));
    if (!o_ok && s_ok && tid == 0) record_error(4, 42);
    umma::tc_fence_after();
    if (o_ok) {
        float be = 1.f - P.alpha;
        const float f = l > 0.f ? P.alpha / l : 0.f;
        float o[32];
        umma::tmem_ld32(trow + (uint32_t)(32 * wg), o);
        if constexpr (SOFT) {
            // the soft gather G / l2 takes the place of V_cent[c_i]
            float gs[32];
            umma::tmem_ld32(trow + (uint32_t)(64 + 32 * wg), gs);
            umma::tmem_ld_wait();
#pragma unroll
            for (int t = 0; t < 32; ++t) asm volatile("" : "+f"(gs[t]));
#pragma unroll
            for (int u = 0; u < 8; ++u) g[u] = make_float4(gs[4 * u], gs[4 * u + 1], gs[4 * u + 2], gs[4 * u + 3]);
            const float l2 = red2[256 + i] + red2[384 + i];
            be = l2 > 0.f ? be / l2 : 0.f;
        }
        umma::tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 32; ++t) asm volatile("" : "+f"(o[t]));
        uint32_t w[16];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            w[2 * u] = pack_bf16(fmaf(f, o[4 * u + 0], be * g[u].x), fmaf(f, o[4 * u + 1], be * g[u].y));
            w[2 * u + 1] = pack_bf16(fmaf(f, o[4 * u + 2], be * g[u].z), fmaf(f, o[4 * u + 3], be * g[u].w));
        }
        if (MASK && qi < L && !P.key_valid[(head / P.H) * L + qi]) {  // an invalid query's row is zero
#pragma unroll
            for (int u = 0; u < 16; ++u) w[u] = 0u;
        }
        // the output tile, 128-byte swizzled over the dead P block 0, then
        // one TMA store (rows past L are clipped)
#pragma unroll
        for (int q = 0; q < 4; ++q)
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(p_s + swz(i, 4 * wg + q)), "r"(w[4 * q]),
                         "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                         : "memory");
    }
    umma::fence_proxy_async_smem();
    umma::tc_fence_before();
    __syncthreads();
    if (tid == 0 && o_ok) {
        umma::tma_store_3d(&tmo, 0, q0, (int)head, p_s);
        umma::tma_store_commit();
    }
    if (warp == 0) {
        umma::tc_fence_after();
        umma::tmem_dealloc(taddr, 256u);
    }
    if (tid == 0 && o_ok) umma::tma_store_wait_read();  // shared memory stays live until read
}

}  // namespace tiled
}  // namespace ca
