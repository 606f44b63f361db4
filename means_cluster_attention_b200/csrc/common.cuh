// Shared device helpers for the cluster-attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ca {

// Head dimension handled by this build.
constexpr int kD = 64;
// Largest cluster count accepted at the boundary.
constexpr int kMaxK = 128;

// First device-side error recorded by any kernel of the library (0 = none).
// Codes match ca_status; the host reads and clears it in ca_sync_status.
__device__ int g_dev_error;
__device__ int g_dev_error_where;

// Options of the general path for the variants of the card's module:
// grouped key/value heads, key-padding masks, no local branch, soft gather.
// The defaults leave the forward unchanged.
struct Variant {
    int H = 1, H_kv = 1;                  // query / key-value heads per batch row
    const uint8_t *key_valid = nullptr;   // [B][L], 1 = valid key (and query)
    int local = 1;                        // 0: no local branch, O = gathered
    int soft = 0;                         // 1: soft gather softmax(Q mu^T s) V_cent
    const float *mu = nullptr;            // [NH][K][64] final centroids (soft gather)
    __host__ __device__ int64_t kv_head(int64_t h) const {
        return (h / H) * H_kv + (h % H) / (H / H_kv);
    }
    __host__ __device__ int64_t batch(int64_t h) const { return h / H; }
};

// Programmatic dependent launch.  pdl_launch lets the next kernel of the
// stream be scheduled before this one completes; pdl_wait blocks until the
// previous kernel of the stream has completed and its writes are visible
// (no-ops when the launch did not ask for it).  A kernel touches nothing its
// predecessor writes, and writes nothing its predecessor reads, before
// pdl_wait: only the forward's inputs and its own shared memory.
__device__ __forceinline__ void pdl_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void record_error(int code, int where) {
    if (atomicCAS(&g_dev_error, 0, code) == 0) g_dev_error_where = where;
}

// Bounds-checked build (compiled with -DCA_CHECKED): CA_IDX(v, lo, hi, site)
// checks a computed index at a point where it addresses memory; an index
// outside [lo, hi) records CA_ERR_DEVICE with the site and is replaced by lo,
// so nothing is accessed out of bounds and nothing faults.  In the normal
// build CA_IDX is the index itself.
#ifdef CA_CHECKED
__device__ __forceinline__ int ca_checked_index(int v, int lo, int hi, int site) {
    if (v < lo || v >= hi) {
        record_error(5, site);
        return lo;
    }
    return v;
}
#define CA_IDX(v, lo, hi, site) ca_checked_index((v), (lo), (hi), (site))
#else
#define CA_IDX(v, lo, hi, site) (v)
#endif

// Records code the way a kernel that detected a problem does (site 99), for
// testing the host's error reporting without a fault.
__global__ void debug_record_error_kernel(int code) { record_error(code, 99); }

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Load one 64-element row (16-byte aligned) into fp32 registers.
__device__ __forceinline__ void load_row64(const float *__restrict__ p, float (&r)[kD]) {
    const float4 *p4 = reinterpret_cast<const float4 *>(p);
#pragma unroll
    for (int i = 0; i < kD / 4; ++i) {
        float4 t = __ldg(p4 + i);
        r[4 * i + 0] = t.x;
        r[4 * i + 1] = t.y;
        r[4 * i + 2] = t.z;
        r[4 * i + 3] = t.w;
    }
}

__device__ __forceinline__ void load_row64(const __nv_bfloat16 *__restrict__ p, float (&r)[kD]) {
    const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int i = 0; i < kD / 8; ++i) {
        uint4 t = __ldg(p4 + i);
        const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            r[8 * i + 2 * e + 0] = __uint_as_float(w[e] << 16);
            r[8 * i + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
        }
    }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Marks every centroid kk < K that is a bitwise copy of a lower-index
// centroid dead (dead[kk] = 1, mm[kk] = +inf): such a centroid can never win
// an argmin whose ties go to the lowest index.  One warp per centroid: the
// lanes compare the hashes of 32 lower indices at once, then each hash match,
// lowest first, row against row (two coordinates per lane) until one is equal.
// mu rows are mu_ld floats apart; the caller initialises dead and mm.
__device__ inline void mark_copies(int K, const uint32_t *hsh, const float *mu, int mu_ld, uint8_t *dead, float *mm,
                                   int warp, int nwarps, int lane) {
    for (int kk = warp; kk < K; kk += nwarps) {
        const uint32_t hk = hsh[kk];
        const uint32_t x0 = __float_as_uint(mu[kk * mu_ld + 2 * lane]);
        const uint32_t x1 = __float_as_uint(mu[kk * mu_ld + 2 * lane + 1]);
        bool found = false;
        for (int a0 = 0; a0 < kk && !found; a0 += 32) {
            const int a = a0 + lane;
            unsigned cand = __ballot_sync(0xffffffffu, a < kk && hsh[a] == hk);
            while (cand && !found) {
                const int b = a0 + __ffs(cand) - 1;
                cand &= cand - 1u;
                const bool eq = __float_as_uint(mu[b * mu_ld + 2 * lane]) == x0 &&
                                __float_as_uint(mu[b * mu_ld + 2 * lane + 1]) == x1;
                found = __all_sync(0xffffffffu, eq);
            }
        }
        if (found && lane == 0) {
            dead[kk] = 1;
            mm[kk] = INFINITY;
        }
    }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

}  // namespace ca
