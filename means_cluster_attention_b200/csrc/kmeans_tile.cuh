// Tile-level pieces of the exact Lloyd step shared by the fused (one CTA per
// head) and the tiled (512-query tiles) bf16 kernels: the exact fp64
// re-measure of an ambiguous token, the counting sort of a tile's tokens by
// cluster, and the exact fp64 member sums over the sorted tokens.
//
// Model card "Hooshaai/distilbert-sst2-cluster-attention", Mathematical
// Formulation section 1 (c_i = argmin_k D_ik, mu_k = sum / max(1, count));
// "Hooshaai/svd-sst2-roberta-cluster" section 2.1 (the expanded distance).
//
// The query tile lives in shared memory as 128-byte rows of 64 bf16 values,
// swizzled in 16-byte chunks (swz in mma.cuh).
#pragma once

#include "common.cuh"
#include "mma.cuh"

namespace ca {
namespace tile {

// Largest number of query rows a tile holds in shared memory (both kernels).
constexpr int kMaxTileRows = 512;

// Exact fp64 value of a bf16 bit pattern (low 16 bits of b) built with
// integer operations: the 8-bit exponent is rebiased (+896) into the 11-bit
// field and the 7 fraction bits become the top fraction bits.  Zero and
// subnormal inputs take the (exact) conversion path.  Inputs are finite.
__device__ __forceinline__ double bf16_to_f64(uint32_t b) {
    if ((b & 0x7F80u) == 0u) return (double)__uint_as_float(b << 16);
    const uint32_t hi = ((b & 0x8000u) << 16) | (((b & 0x7FFFu) << 13) + 0x38000000u);
    return __hiloint2double((int)hi, 0);
}

// Exact fp64 re-measure of one token against every centroid, in the
// oracle's operation order: D_k = (|Q|^2 + |mu_k|^2) - 2 Q.mu_k with
// index-order sums.  Every product (bf16 x bf16, bf16 x fp32, fp32 x fp32)
// is exact in fp64, so one fused multiply-add rounds exactly as a rounded
// product followed by a rounded sum.  Lane k holds centroid k (and k + 32
// when TWO); mu(k, j) returns coordinate j of centroid k as a double.  The
// lowest k with the smallest D among the live (not dead) centroids is
// returned on every lane.
template <bool TWO, typename MuAt>
__device__ __forceinline__ int remeasure_token(const unsigned char *qbytes, int row, int Kp, const uint8_t *dead,
                                               MuAt mu, int lane) {
    double qq = 0.0, qm0 = 0.0, qm1 = 0.0, m20 = 0.0, m21 = 0.0;
    const int k0 = lane, k1 = lane + 32;
    const bool v0 = k0 < Kp, v1 = TWO && k1 < Kp;
#pragma unroll 2
    for (int jb = 0; jb < kD; jb += 8) {
        const uint4 w = *reinterpret_cast<const uint4 *>(qbytes + swz(row, jb >> 3));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        double qj[8], mj0[8], mj1[8];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
            qj[2 * e2] = bf16_to_f64(ws[e2] & 0xffffu);
            qj[2 * e2 + 1] = bf16_to_f64(ws[e2] >> 16);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            mj0[u] = v0 ? mu(k0, jb + u) : 0.0;
            if constexpr (TWO) mj1[u] = v1 ? mu(k1, jb + u) : 0.0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            qq = __fma_rn(qj[u], qj[u], qq);
            qm0 = __fma_rn(qj[u], mj0[u], qm0);
            m20 = __fma_rn(mj0[u], mj0[u], m20);
            if constexpr (TWO) {
                qm1 = __fma_rn(qj[u], mj1[u], qm1);
                m21 = __fma_rn(mj1[u], mj1[u], m21);
            }
        }
    }
    double bd = INFINITY;
    int bk = 0x7fffffff;
    if (v0 && !dead[k0]) {
        bd = __dsub_rn(__dadd_rn(qq, m20), __dmul_rn(2.0, qm0));
        bk = k0;
    }
    if (v1 && !dead[k1]) {
        const double D = __dsub_rn(__dadd_rn(qq, m21), __dmul_rn(2.0, qm1));
        if (D < bd) {
            bd = D;
            bk = k1;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double od = __shfl_xor_sync(0xffffffffu, bd, o);
        const int ok = __shfl_xor_sync(0xffffffffu, bk, o);
        if (od < bd || (od == bd && ok < bk)) {
            bd = od;
            bk = ok;
        }
    }
    return bk;
}

// Fast exact decision among a token's candidate centroids (bit k of the
// 64-bit set cand1:cand0, lowest first).  Each distance D_k = (|Q|^2 + |mu_k|^2) - 2 Q.mu_k is
// formed in fp64 with warp-tree sums (lane l holds coordinates 2l, 2l+1;
// every product is exact).  Whatever the order of its sums, a computed D_k
// lies within 2^-45 (|Q|^2 + |mu_k|^2) of the exact value: 64 summands
// give at most 64 u of the sum of magnitudes per dot product (u = 2^-53),
// |Q.mu| <= (|Q|^2 + |mu|^2) / 2, and two more roundings add u each, so
// 67 u (|Q| + |mu|)^2 <= 2^-45 (|Q|^2 + |mu|^2); E_k takes twice that
// (2^-44) to cover the roundings of the gap tests themselves.  The
// index-order distances of the re-measure (and of the fp64 oracle) obey the
// same bound, so when min over k != b of (D_k - 2 E_k) exceeds D_b + 2 E_b
// the lowest-k argmin
// b of the tree distances is the argmin of the index-order ones, with no
// tie.  Returns b and sets certain; when certain is false the caller takes
// the index-order re-measure.  The result is the same on every lane.
template <typename MuAt>
__device__ __forceinline__ int decide_candidates(const unsigned char *qbytes, int row, uint32_t cand0, uint32_t cand1,
                                                 const uint8_t *dead, MuAt mu, int lane, bool &certain) {
    const uint32_t w = *reinterpret_cast<const uint32_t *>(qbytes + swz(row, lane >> 2) + (lane & 3) * 4);
    const double q0 = bf16_to_f64(w & 0xffffu), q1 = bf16_to_f64(w >> 16);
    auto tree = [](double x) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        return x;
    };
    const double qq = tree(__fma_rn(q0, q0, q1 * q1));
    double bd = INFINITY, be = 0.0, chall = INFINITY;
    int bk = -1;
#pragma unroll
    for (int wi = 0; wi < 2; ++wi) {
        uint32_t bits = wi ? cand1 : cand0;
        while (bits) {
            const int k = wi * 32 + __ffs(bits) - 1;
            bits &= bits - 1u;
            if (dead[k]) continue;
            const double m0 = mu(k, 2 * lane), m1 = mu(k, 2 * lane + 1);
            const double qm = tree(__fma_rn(q0, m0, q1 * m1));
            const double mm = tree(__fma_rn(m0, m0, m1 * m1));
            const double D = __dsub_rn(__dadd_rn(qq, mm), __dmul_rn(2.0, qm));
            const double E = ldexp(qq + mm, -44);  // twice the bound: room for the roundings of the gap tests
            if (D < bd) {
                if (bk >= 0) chall = fmin(chall, bd - 2.0 * be);
                bd = D;
                be = E;
                bk = k;
            } else {
                chall = fmin(chall, D - 2.0 * E);
            }
        }
    }
    certain = bk >= 0 && chall > bd + 2.0 * be;
    return bk;
}

// Counting sort of up to 32 * (number of chunks) tokens by cluster: cs[i] is
// token i's cluster (0xFF for no token), cnt[] (Kp <= 64 entries, zero on
// entry) receives the counts; perm[] and sc[] receive the tokens and their
// clusters in cluster order.  Peers of one cluster in a 32-token chunk take
// their offsets with one atomic on the count; every warp then scans the
// counts itself.  Each warp handles chunks warp and warp + nwarps (two per
// warp: up to 64 * nwarps tokens).  Contains __syncthreads.
__device__ __forceinline__ void counting_sort(const uint8_t *cs, int n_chunks, int Kp, int *cnt, uint16_t *perm,
                                              uint8_t *sc, int warp, int nwarps, int lane) {
    int my_c[2], my_off[2];
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
        const int ch = warp + s2 * nwarps;
        my_c[s2] = 0xFF;
        my_off[s2] = 0;
        if (ch < n_chunks) {
            const int c = cs[ch * 32 + lane];
            const unsigned peers = __match_any_sync(0xffffffffu, c);
            const int leader = __ffs(peers) - 1;
            int off = 0;
            if (c != 0xFF && lane == leader) off = atomicAdd(&cnt[c], __popc(peers));
            off = __shfl_sync(0xffffffffu, off, leader);
            my_c[s2] = c;
            my_off[s2] = off + __popc(peers & ((1u << lane) - 1u));
        }
    }
    __syncthreads();
    const int c0 = lane < Kp ? cnt[lane] : 0, c1 = lane + 32 < Kp ? cnt[lane + 32] : 0;
    int s0 = c0, s1 = c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x0 = __shfl_up_sync(0xffffffffu, s0, o), x1 = __shfl_up_sync(0xffffffffu, s1, o);
        if (lane >= o) {
            s0 += x0;
            s1 += x1;
        }
    }
    const int b0 = s0 - c0, b1 = __shfl_sync(0xffffffffu, s0, 31) + s1 - c1;
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
        const int c = my_c[s2];
        const int x0 = __shfl_sync(0xffffffffu, b0, c & 31), x1 = __shfl_sync(0xffffffffu, b1, c & 31);
        if (c != 0xFF) {
            const int pos = CA_IDX((c < 32 ? x0 : x1) + my_off[s2], 0, n_chunks * 32, 60);
            perm[pos] = (uint16_t)((warp + s2 * nwarps) * 32 + lane);
            sc[pos] = (uint8_t)c;
        }
    }
    __syncthreads();
}

// Exact fp64 member sums over sorted positions [p, p1): the warp walks them
// run by run (one cluster per run).  Each step takes four tokens, two per
// half-warp, lane l holding coordinates 4 (l mod 16) .. +3 of its token
// (one 8-byte load); bf16 -> fp32 is a bit shift and fp32 -> fp64 exact, so
// every addition adds an exact value; eight independent chains per lane.  A
// run's sum goes into sums[c][64] with fp64 shared-memory atomics; as the
// sums of bf16 values with non-zero magnitudes in 2^-27 .. 16 are exact, the
// order of the additions changes no bit.
__device__ __forceinline__ void member_sums(const unsigned char *qbytes, const uint8_t *sc, const uint16_t *perm, int p,
                                            int p1, double *sums, int lane) {
    const int h = lane >> 4, l16 = lane & 15;
    const uint32_t lane_off = (uint32_t)(l16 & 1) * 8u;
    const int chunk = l16 >> 1;
    while (p < p1) {
        const int c = CA_IDX(sc[p], 0, 64, 61);
        double a[4] = {0.0, 0.0, 0.0, 0.0}, b[4] = {0.0, 0.0, 0.0, 0.0};
        for (;;) {
            const int qq = p + lane;
            const unsigned same = __ballot_sync(0xffffffffu, qq < p1 && sc[qq] == c);
            const int n = __ffs(~same) ? __ffs(~same) - 1 : 32;
            const int rowl = (lane < n) ? CA_IDX(perm[p + lane], 0, kMaxTileRows, 62) : 0;
            for (int j = 0; j < n; j += 4) {
                const int r0 = __shfl_sync(0xffffffffu, rowl, (j + h) & 31);
                const int r1 = __shfl_sync(0xffffffffu, rowl, (j + 2 + h) & 31);
                uint2 w0 = make_uint2(0u, 0u), w1 = make_uint2(0u, 0u);
                if (j + h < n) w0 = *reinterpret_cast<const uint2 *>(qbytes + swz(r0, chunk) + lane_off);
                if (j + 2 + h < n) w1 = *reinterpret_cast<const uint2 *>(qbytes + swz(r1, chunk) + lane_off);
                // a missing token is the word 0 and adds +0
                a[0] += (double)__uint_as_float(w0.x << 16);
                a[1] += (double)__uint_as_float(w0.x & 0xffff0000u);
                a[2] += (double)__uint_as_float(w0.y << 16);
                a[3] += (double)__uint_as_float(w0.y & 0xffff0000u);
                b[0] += (double)__uint_as_float(w1.x << 16);
                b[1] += (double)__uint_as_float(w1.x & 0xffff0000u);
                b[2] += (double)__uint_as_float(w1.y << 16);
                b[3] += (double)__uint_as_float(w1.y & 0xffff0000u);
            }
            p += n;
            if (n < 32) break;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a[i] += b[i];
            a[i] += __shfl_xor_sync(0xffffffffu, a[i], 16);
        }
        if (h == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) atomicAdd(&sums[c * kD + 4 * l16 + i], a[i]);
        }
    }
}

// Packed sum entry: query row in bits 0..9, cluster in bits 16..21, bit 30
// for a padding entry (adds nothing), bit 31 for a subtracted row.
constexpr uint32_t kEntPad = 0x40000000u, kEntNeg = 0x80000000u;

// Counting sort of up to 32 * n_chunks entries by cluster into packed
// entries ent[], every cluster's run padded with one padding entry to even
// length (so the two halves of a warp always meet the same cluster).  cl(i)
// is entry i's cluster (0xFF for none) and info(i) its row and sign bits;
// cnt[] (Kp <= 64 entries) must be zero on entry.  *n_out receives the
// padded length.  Each warp handles chunks warp and warp + nwarps.
// Contains __syncthreads.
template <typename Cl, typename Info>
__device__ __forceinline__ void counting_sort_even(Cl cl, Info info, int n_chunks, int Kp, int *cnt, uint32_t *ent,
                                                   int *n_out, int warp, int nwarps, int lane) {
    int my_c[2], my_off[2];
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
        const int ch = warp + s2 * nwarps;
        my_c[s2] = 0xFF;
        my_off[s2] = 0;
        if (ch < n_chunks) {
            const int c = cl(ch * 32 + lane);
            const unsigned peers = __match_any_sync(0xffffffffu, c);
            const int leader = __ffs(peers) - 1;
            int off = 0;
            if (c != 0xFF && lane == leader) off = atomicAdd(&cnt[c], __popc(peers));
            off = __shfl_sync(0xffffffffu, off, leader);
            my_c[s2] = c;
            my_off[s2] = off + __popc(peers & ((1u << lane) - 1u));
        }
    }
    __syncthreads();
    const int c0 = lane < Kp ? cnt[lane] : 0, c1 = lane + 32 < Kp ? cnt[lane + 32] : 0;
    const int e0 = (c0 + 1) & ~1, e1 = (c1 + 1) & ~1;
    int s0 = e0, s1 = e1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x0 = __shfl_up_sync(0xffffffffu, s0, o), x1 = __shfl_up_sync(0xffffffffu, s1, o);
        if (lane >= o) {
            s0 += x0;
            s1 += x1;
        }
    }
    const int tot0 = __shfl_sync(0xffffffffu, s0, 31);
    const int b0 = s0 - e0, b1 = tot0 + s1 - e1;
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
        const int c = my_c[s2];
        const int x0 = __shfl_sync(0xffffffffu, b0, c & 31), x1 = __shfl_sync(0xffffffffu, b1, c & 31);
        if (c != 0xFF) {
            const int i = (warp + s2 * nwarps) * 32 + lane;
            const int pos = CA_IDX((c < 32 ? x0 : x1) + my_off[s2], 0, n_chunks * 32 + 64, 60);
            ent[pos] = info(i) | ((uint32_t)c << 16);
        }
    }
    const int total = tot0 + __shfl_sync(0xffffffffu, s1, 31);
    if (warp == 0) {
        if (c0 & 1) ent[CA_IDX(b0 + c0, 0, n_chunks * 32 + 64, 60)] = kEntPad | ((uint32_t)lane << 16);
        if (c1 & 1) ent[CA_IDX(b1 + c1, 0, n_chunks * 32 + 64, 60)] = kEntPad | ((uint32_t)(lane + 32) << 16);
        if (lane == 0) *n_out = total;
    }
    __syncthreads();
}

// Exact fp64 sums of signed query rows over the packed sorted entries
// [p, p1) (p, p1 even) into a head's running sums gsum and counts gcnt in
// global memory.  Each step takes two entries, one per half-warp, lane l
// holding coordinates 4 (l mod 16) .. +3 (one 8-byte load); both entries
// belong to the same cluster, so the walk never diverges.  A subtracted
// row has the sign bits of its bf16 values flipped (exact).  When the
// cluster changes, the run's sum goes out with two fp64 reductions
// (red.global.add.f64) per lane: coordinate 4 l16 + i is kept at position
// 16 i + l16 of its row of gsum, so each reduction instruction covers two
// whole 128-byte lines; the run's signed count goes out with one integer
// reduction.  When every partial state of the running sums is a multiple of
// the smallest ulp among the added values and below 2^53 of those ulps,
// every addition is exact and their order changes no bit.
__device__ __forceinline__ void run_sums_red(const unsigned char *qbytes, const uint32_t *ent, int p, int p1,
                                             double *gsum, int *gcnt, int lane) {
    if (p >= p1) return;
    const int h = lane >> 4, l16 = lane & 15;
    const uint32_t lane_off = (uint32_t)(l16 & 1) * 8u;
    const int chunk = l16 >> 1;
    double a[4] = {0.0, 0.0, 0.0, 0.0}, b[4] = {0.0, 0.0, 0.0, 0.0};
    int cnt = 0;
    int c_cur = (int)((ent[p] >> 16) & 63u);
    auto flush = [&](int c) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            a[i] += b[i];
            a[i] += __shfl_xor_sync(0xffffffffu, a[i], 16);
        }
        double *row = gsum + c * kD;
        atomicAdd(&row[32 * h + l16], h ? a[2] : a[0]);
        atomicAdd(&row[32 * h + 16 + l16], h ? a[3] : a[1]);
        const int t = cnt + __shfl_xor_sync(0xffffffffu, cnt, 16);
        if (lane == 0 && t != 0) atomicAdd(&gcnt[c], t);
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = b[i] = 0.0;
        cnt = 0;
    };
    auto fetch = [&](uint32_t e) {
        uint2 w = make_uint2(0u, 0u);
        if (!(e & kEntPad)) {
            w = *reinterpret_cast<const uint2 *>(qbytes + swz(CA_IDX((int)(e & 0x3FFu), 0, kMaxTileRows, 78), chunk) +
                                                 lane_off);
            const uint32_t f = (uint32_t)((int)e >> 31) & 0x80008000u;
            w.x ^= f;
            w.y ^= f;
        }
        return w;
    };
    auto delta = [](uint32_t e) { return (e & kEntPad) ? 0 : ((e & kEntNeg) ? -1 : 1); };
    for (; p < p1; p += 4) {
        const bool two = p + 2 < p1;  // uniform
        const uint32_t e0 = ent[p + h];
        const uint32_t e1 = two ? ent[p + 2 + h] : kEntPad | (e0 & (63u << 16));
        const uint2 w0 = fetch(e0), w1 = fetch(e1);
        const int c0 = (int)((e0 >> 16) & 63u), c1 = (int)((e1 >> 16) & 63u);
        if (c0 != c_cur) {
            flush(c_cur);
            c_cur = c0;
        }
        a[0] += (double)__uint_as_float(w0.x << 16);
        a[1] += (double)__uint_as_float(w0.x & 0xffff0000u);
        a[2] += (double)__uint_as_float(w0.y << 16);
        a[3] += (double)__uint_as_float(w0.y & 0xffff0000u);
        cnt += delta(e0);
        if (c1 != c_cur) {
            flush(c_cur);
            c_cur = c1;
        }
        b[0] += (double)__uint_as_float(w1.x << 16);
        b[1] += (double)__uint_as_float(w1.x & 0xffff0000u);
        b[2] += (double)__uint_as_float(w1.y << 16);
        b[3] += (double)__uint_as_float(w1.y & 0xffff0000u);
        cnt += delta(e1);
    }
    flush(c_cur);
}

}  // namespace tile
}  // namespace ca
