// libclusterattn host layer: argument validation, stream-ordered scratch,
// kernel launches.  The C ABI is declared in include/clusterattn.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <string>
#include <utility>

#include "clusterattn.h"
#include "common.cuh"
#include "kmeans.cuh"
#include "attention.cuh"
#include "fused.cuh"
#include "tiled.cuh"
#include "profile.cuh"

namespace {

thread_local std::string g_last_error;

ca_status fail(ca_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

ca_status cuda_fail(cudaError_t e, const char *what) {
    return fail(CA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

#define CA_CUDA(call)                                          \
    do {                                                       \
        cudaError_t e_ = (call);                               \
        if (e_ != cudaSuccess) return cuda_fail(e_, #call);    \
    } while (0)

// NVTX range around one forward (header-only NVTX: free unless a profiler
// that records ranges is attached).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

struct Problem {
    int B, H, L, d, K, iters, W;
    float alpha;
    int64_t heads() const { return (int64_t)B * H; }
};

ca_status validate(const void *q, const void *k, const void *v, const void *out, const Problem &p) {
    if (!q || !k || !v || !out) return fail(CA_ERR_INVALID_ARG, "q, k, v and out must be non-null");
    if (p.B < 1 || p.H < 1 || p.L < 1)
        return fail(CA_ERR_INVALID_ARG, "B, H, L must be >= 1 (got %d, %d, %d)", p.B, p.H, p.L);
    if (p.d < 1) return fail(CA_ERR_INVALID_ARG, "d must be >= 1 (got %d)", p.d);
    if (p.d != ca::kD) return fail(CA_ERR_UNSUPPORTED, "only d == 64 is supported (got %d)", p.d);
    if (p.K < 1 || p.K > p.L)
        return fail(CA_ERR_INVALID_ARG, "K must satisfy 1 <= K <= L (got K=%d, L=%d)", p.K, p.L);
    if (p.K > ca::kMaxK) return fail(CA_ERR_UNSUPPORTED, "K must be <= %d (got %d)", ca::kMaxK, p.K);
    if (p.iters < 0) return fail(CA_ERR_INVALID_ARG, "iters must be >= 0 (got %d)", p.iters);
    if (p.W < 0) return fail(CA_ERR_INVALID_ARG, "W must be >= 0 (got %d)", p.W);
    if (!std::isfinite(p.alpha) || p.alpha < 0.f || p.alpha > 1.f)
        return fail(CA_ERR_INVALID_ARG, "alpha must be finite and in [0, 1]");
    if (p.heads() > 65535) return fail(CA_ERR_UNSUPPORTED, "B*H must be <= 65535 (got %lld)", (long long)p.heads());
    const int64_t elems = p.heads() * (int64_t)p.L * p.d;
    if (elems >= (int64_t(1) << 31)) return fail(CA_ERR_INVALID_ARG, "B*H*L*d must be < 2^31");
    const uintptr_t a = (uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)out;
    if (a & 15u) return fail(CA_ERR_INVALID_ARG, "q, k, v and out must be 16-byte aligned");
    return CA_OK;
}

// One stream-ordered memory pool per device, owned by the library.  Its
// release threshold is set to the maximum so that memory freed at the end of
// a call stays mapped for the next one (no OS round trip per call).
cudaError_t library_pool(cudaMemPool_t *out) {
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> g(mu);
    if (!pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p = nullptr;
        e = cudaMemPoolCreate(&p, &props);
        if (e != cudaSuccess) return e;
        uint64_t thr = ~0ull;
        e = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &thr);
        if (e != cudaSuccess) return e;
        pools[dev] = p;
    }
    *out = pools[dev];
    return cudaSuccess;
}

// Stream-ordered scratch from the library pool, released on the same stream
// when the object dies.
struct Scratch {
    cudaStream_t st;
    void *ptrs[16] = {};
    int n = 0;
    explicit Scratch(cudaStream_t s) : st(s) {}
    ~Scratch() {
        for (int i = 0; i < n; ++i) cudaFreeAsync(ptrs[i], st);
    }
    cudaError_t get(void **p, size_t bytes) {
        cudaMemPool_t pool;
        cudaError_t e = library_pool(&pool);
        if (e != cudaSuccess) return e;
        e = cudaMallocFromPoolAsync(p, bytes, pool, st);
        if (e == cudaSuccess) ptrs[n++] = *p;
        return e;
    }
};

// Every kernel that takes dynamic shared memory may use up to 227 KB of it.
// The attribute is per device and per function; it is set once per device,
// under a lock, before the first launch there.
static std::atomic<int> g_sm_count[64];  // multiprocessors of each device (set with the attributes)

ca_status ensure_kernel_attributes() {
    using namespace ca;
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    CA_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return fail(CA_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> g(mu);
    if (done[dev]) return CA_OK;
    const int big = 227 * 1024;
    CA_CUDA(cudaFuncSetAttribute(fused::fused_forward_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_assign_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_assign_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_assign_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_centroid_tc_kernel<16, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_centroid_tc_kernel<32, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_centroid_tc_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_centroid_tc_kernel<16, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_centroid_tc_kernel<32, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_centroid_tc_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_window_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_window_tc_kernel<32, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_window_tc_kernel<64, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_window_tc_kernel<32, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_window_tc_kernel<64, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_window_tc_kernel<32, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(tiled::tiled_window_tc_kernel<32, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(kmeans_assign_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(kmeans_assign_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(centroid_attn_partial_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(centroid_attn_partial_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(window_blend_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    CA_CUDA(cudaFuncSetAttribute(window_blend_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, big));
    int n_sm = 0;
    CA_CUDA(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
    g_sm_count[dev].store(n_sm);
    done[dev] = true;
    return CA_OK;
}

// Multiprocessors of the current device (ensure_kernel_attributes ran).
int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    const int n = g_sm_count[dev].load();
    return n > 0 ? n : 148;
}

// The fused one-CTA-per-head kernel handles bf16 heads with L <= 512,
// K <= 64 and a window radius floor(W/2) <= 16.
bool fused_eligible(int dtype, const Problem &p) {
    return dtype == 1 && p.L <= ca::fused::kMaxL && p.K <= ca::fused::kMaxK && p.W / 2 <= ca::fused::kMaxR;
}

ca_status run_fused(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v, const Problem &p,
                    __nv_bfloat16 *out, int32_t *assign_out, float *cent_out, int32_t *hist, cudaStream_t st) {
    using namespace ca;
    const fused::Layout lay(p.L, p.K, p.W / 2);
    fused::Params P;
    P.q = q;
    P.k = k;
    P.v = v;
    P.out = out;
    P.assign = assign_out;
    P.cent = cent_out;
    P.hist = hist;
    P.L = p.L;
    P.K = p.K;
    P.iters = p.iters;
    P.r = p.W / 2;
    P.alpha = p.alpha;
    P.scale = 1.0f / sqrtf((float)p.d);
    const double bytes = 4.0 * (double)p.heads() * p.L * kD * sizeof(__nv_bfloat16);
    {
        Launch pl("fused_forward", st, bytes);
        fused::fused_forward_kernel<<<(unsigned)p.heads(), fused::kThreads, lay.total, st>>>(P);
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    return CA_OK;
}

// TMA tensor map of a [NH, L, 64] bf16 tensor read in boxes of box_rows
// (<= 256) rows of one head, 128-byte swizzled (the layout the tcgen05 operand descriptors
// read).  Rows past L (inside a box) are filled with zeros by the TMA unit.
// The driver's encoder is looked up once through the runtime.
ca_status encode_rows_map(CUtensorMap *map, const void *base, int64_t NH, int L, int box_rows = 256) {
    static std::mutex mu;
    static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
    {
        std::lock_guard<std::mutex> g(mu);
        if (!encode) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
            cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
            if (e != cudaSuccess) return cuda_fail(e, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
            if (!fn || q != cudaDriverEntryPointSuccess)
                return fail(CA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
            encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
    }
    const cuuint64_t dims[3] = {(cuuint64_t)ca::kD, (cuuint64_t)L, (cuuint64_t)NH};
    const cuuint64_t strides[2] = {(cuuint64_t)ca::kD * 2u, (cuuint64_t)L * ca::kD * 2u};
    const cuuint32_t box[3] = {(cuuint32_t)ca::kD, (cuuint32_t)box_rows, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return CA_OK;
}

// Launches a kernel that may start before the previous kernel on the stream
// completes (programmatic dependent launch); the kernel itself waits for
// its predecessor (pdl_wait) before touching anything the predecessor
// writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The tiled bf16 path serves the heads the fused kernel does not take, for
// K <= 64 and a window radius floor(W/2) <= 128.
bool tiled_eligible(int dtype, const Problem &p) {
    return dtype == 1 && p.K <= 64 && p.W / 2 <= ca::tiled::kMaxR;
}

// The module's variants the tiled path runs (the defaults give the forward
// of the pages' formulas): window radius r (floor(W / 2), or W with
// window_mode), no local branch (O = gathered), the module's stride init,
// empty clusters keeping their centroid, grouped key/value heads.
struct TiledVariant {
    int r = 0, local = 1, init_stride = 0, empty_keep = 0, H_kv = 0;
    const uint8_t *key_valid = nullptr;  // [B][L] key-padding mask (radius <= 64 or no local branch)
    int soft = 0;                        // soft gather (radius <= 32 or no local branch)
    static TiledVariant plain(const Problem &p) {
        TiledVariant tv;
        tv.r = p.W / 2;
        tv.H_kv = p.H;
        return tv;
    }
};

ca_status run_tiled(const __nv_bfloat16 *q, const __nv_bfloat16 *k, const __nv_bfloat16 *v, const Problem &p,
                    __nv_bfloat16 *out, int32_t *assign_out, float *cent_out, int32_t *hist, cudaStream_t st,
                    const TiledVariant &tv) {
    using namespace ca;
    const int64_t NH = p.heads(), NH_kv = (int64_t)p.B * tv.H_kv;
    const int L = p.L, K = p.K, Kp = tiled::kpad(K);
    // Keys per centroid-attention CTA: long chunks (fewer partial states to
    // combine, each CTA's set-up spread over more steps) as long as the grid
    // still gives every multiprocessor a CTA.
    int chunk_keys = tiled::kMaxChunk;
    while (chunk_keys > 512 && NH * ((L + chunk_keys - 1) / chunk_keys) < sm_count()) chunk_keys /= 2;
    const int n_chunks = (L + chunk_keys - 1) / chunk_keys;
    const float scale = 1.0f / sqrtf((float)p.d);
    Scratch s(st);
    float *mu = nullptr, *mm = nullptr, *cpart = nullptr, *vcent = nullptr;
    __nv_bfloat16 *hi = nullptr, *lo = nullptr;
    double *rsum = nullptr;
    int *rcnt = nullptr;
    uint8_t *dead = nullptr, *any_valid = nullptr;
    float *mstat = nullptr, *qnorm = nullptr;
    int32_t *assign = assign_out;
    CA_CUDA(s.get((void **)&mu, sizeof(float) * NH * Kp * kD));
    CA_CUDA(s.get((void **)&mstat, sizeof(float) * NH * 2));
    CA_CUDA(s.get((void **)&dead, sizeof(uint8_t) * NH * Kp));
    if (tv.key_valid) CA_CUDA(s.get((void **)&any_valid, sizeof(uint8_t) * NH));
    CA_CUDA(s.get((void **)&qnorm, sizeof(float) * NH * L));
    CA_CUDA(s.get((void **)&hi, sizeof(__nv_bfloat16) * NH * Kp * kD));
    CA_CUDA(s.get((void **)&lo, sizeof(__nv_bfloat16) * NH * Kp * kD));
    CA_CUDA(s.get((void **)&mm, sizeof(float) * NH * Kp));
    CA_CUDA(s.get((void **)&rsum, sizeof(double) * NH * Kp * kD));
    CA_CUDA(s.get((void **)&rcnt, sizeof(int) * NH * Kp));
    CA_CUDA(s.get((void **)&cpart, sizeof(float) * NH * n_chunks * K * tiled::kPartLd));
    CA_CUDA(s.get((void **)&vcent, sizeof(float) * NH * K * kD));
    if (!assign) CA_CUDA(s.get((void **)&assign, sizeof(int32_t) * NH * L));
    CUtensorMap qmap;
    {
        ca_status ms = encode_rows_map(&qmap, q, NH, L);
        if (ms != CA_OK) return ms;
    }

    const double head_bytes = (double)NH * L * kD * sizeof(__nv_bfloat16);

    tiled::UpdateParams up{};
    up.q = q;
    up.sum = rsum;
    up.cnt = rcnt;
    up.mu = mu;
    up.hi = hi;
    up.lo = lo;
    up.mm = mm;
    up.dead = dead;
    up.mstat = mstat;
    up.L = L;
    up.K = K;
    up.Kp = Kp;
    up.init = 1;
    up.init_stride = tv.init_stride;
    up.empty_keep = tv.empty_keep;
    up.key_valid = tv.key_valid;
    up.any_valid = any_valid;
    up.H = p.H;
    up.cent_out = p.iters == 0 ? cent_out : nullptr;
    {
        Launch pl("tiled_init", st, 0.0);
        tiled::tiled_update_kernel<<<(unsigned)NH, tiled::kUpdThreads, 0, st>>>(up);
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    if (p.iters == 0) CA_CUDA(cudaMemsetAsync(assign, 0, sizeof(int32_t) * NH * L, st));

    const tiled::AssignLayout alay(K);
    tiled::AssignParams ap{};
    ap.q = q;
    ap.mu = mu;
    ap.hi = hi;
    ap.lo = lo;
    ap.mm = mm;
    ap.dead = dead;
    ap.mstat = mstat;
    ap.qnorm = qnorm;
    ap.assign = assign;
    ap.hist_stride = (int64_t)p.iters * L;
    ap.sum = rsum;
    ap.cnt = rcnt;
    ap.L = L;
    ap.K = K;
    up.init = 0;
    const dim3 agrid((L + tiled::kTileQ - 1) / tiled::kTileQ, (unsigned)NH);
    for (int t = 0; t < p.iters; ++t) {
        ap.hist = hist ? hist + (int64_t)t * L : nullptr;
        ap.first = t == 0;
        {
            Launch pl("tiled_assign", st, head_bytes);
            auto kern = Kp == 16 ? tiled::tiled_assign_kernel<16>
                                 : (Kp == 32 ? tiled::tiled_assign_kernel<32> : tiled::tiled_assign_kernel<64>);
            CA_CUDA(launch_pdl(kern, agrid, dim3(tiled::kThreads), alay.total, st, qmap, ap));
            pl.after();
        }
        CA_CUDA(cudaGetLastError());
        up.cent_out = t == p.iters - 1 ? cent_out : nullptr;
        {
            Launch pl("tiled_update", st, 0.0);
            CA_CUDA(launch_pdl(tiled::tiled_update_kernel, dim3((unsigned)NH), dim3(tiled::kUpdThreads), 0, st, up));
            pl.after();
        }
        CA_CUDA(cudaGetLastError());
    }

    {
        CUtensorMap kmap256, vmap256;
        ca_status ms = encode_rows_map(&kmap256, k, NH_kv, L, 256);
        if (ms == CA_OK) ms = encode_rows_map(&vmap256, v, NH_kv, L, 256);
        if (ms != CA_OK) return ms;
        tiled::CentroidTcParams cp{};
        cp.hi = hi;
        cp.part = cpart;
        cp.L = L;
        cp.K = K;
        cp.n_chunks = n_chunks;
        cp.chunk_keys = chunk_keys;
        cp.H = p.H;
        cp.H_kv = tv.H_kv;
        cp.scale = scale;
        cp.key_valid = tv.key_valid;
        cp.any_valid = any_valid;
        const tiled::CentroidTcLayout clay(Kp, tv.key_valid != nullptr);
        const bool msk = tv.key_valid != nullptr;
        auto kern = Kp == 16 ? (msk ? tiled::tiled_centroid_tc_kernel<16, true> : tiled::tiled_centroid_tc_kernel<16, false>)
                    : Kp == 32 ? (msk ? tiled::tiled_centroid_tc_kernel<32, true> : tiled::tiled_centroid_tc_kernel<32, false>)
                               : (msk ? tiled::tiled_centroid_tc_kernel<64, true> : tiled::tiled_centroid_tc_kernel<64, false>);
        Launch pl("tiled_centroid", st, 2.0 * head_bytes);
        CA_CUDA(launch_pdl(kern, dim3(n_chunks, (unsigned)NH), dim3(256), clay.total, st, kmap256, vmap256, cp));
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    {
        Launch pl("tiled_combine", st, 0.0);
        CA_CUDA(launch_pdl(tiled::tiled_combine_kernel, dim3(K, (unsigned)NH), dim3(64), 0, st, K, n_chunks,
                           (const float *)cpart, vcent));
        pl.after();
    }
    CA_CUDA(cudaGetLastError());

    tiled::WindowParams wp{};
    wp.q = q;
    wp.k = k;
    wp.v = v;
    wp.vcent = vcent;
    wp.assign = assign;
    wp.out = out;
    wp.L = L;
    wp.K = K;
    // without the local branch the epilogue blends with alpha = 0: O is the
    // gathered row exactly, and the window is the smallest one
    wp.r = tv.local ? tv.r : 0;
    wp.alpha = tv.local ? p.alpha : 0.f;
    wp.H = p.H;
    wp.H_kv = tv.H_kv;
    wp.scale = scale;
    wp.key_valid = tv.key_valid;
    wp.hi = hi;
    wp.Kp = Kp;
    if (wp.r <= 64) {
        // tensor-core window kernel: the key window [q0 - RP, q0 + 127 + RP]
        const int RP = wp.r <= 32 ? 32 : 64;
        const tiled::WindowTcLayout tlay(RP, tv.key_valid != nullptr, tv.soft != 0);
        CUtensorMap kmap, vmap, q128, o128;
        ca_status ms = encode_rows_map(&q128, q, NH, L, 128);
        if (ms == CA_OK) ms = encode_rows_map(&kmap, k, NH_kv, L, tlay.NK);
        if (ms == CA_OK) ms = encode_rows_map(&vmap, v, NH_kv, L, tlay.NK);
        if (ms == CA_OK) ms = encode_rows_map(&o128, out, NH, L, 128);
        if (ms != CA_OK) return ms;
        Launch pl("tiled_window", st, 4.0 * head_bytes);
        const bool msk = tv.key_valid != nullptr;
        auto wkern = tv.soft ? (msk ? tiled::tiled_window_tc_kernel<32, true, true> : tiled::tiled_window_tc_kernel<32, false, true>)
                     : RP == 32 ? (msk ? tiled::tiled_window_tc_kernel<32, true, false> : tiled::tiled_window_tc_kernel<32, false, false>)
                                : (msk ? tiled::tiled_window_tc_kernel<64, true, false> : tiled::tiled_window_tc_kernel<64, false, false>);
        CA_CUDA(launch_pdl(wkern,
                           dim3((L + 127) / 128, (unsigned)NH), dim3(256), tlay.total, st, q128, kmap, vmap, o128, wp));
        pl.after();
    } else {
        const tiled::WindowLayout wlay(K, wp.r);
        Launch pl("tiled_window", st, 4.0 * head_bytes);
        CA_CUDA(launch_pdl(tiled::tiled_window_kernel, dim3((L + tiled::kWinQ - 1) / tiled::kWinQ, (unsigned)NH),
                           dim3(tiled::kThreads), wlay.total, st, wp));
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    return CA_OK;
}

// Options of the module's variants for the general path (defaults: none).
struct ExOpts {
    int init_stride = 0, empty_keep = 0, r = -1;  // r < 0: floor(W / 2)
    ca::Variant var;
};

template <typename T>
ca_status run_forward(const T *q, const T *k, const T *v, const Problem &p, T *out,
                      int32_t *assign_out, float *cent_out, int32_t *hist, cudaStream_t st,
                      const ExOpts *ex = nullptr) {
    using namespace ca;
    const ExOpts dflt;
    const ExOpts &xo = ex ? *ex : dflt;
    const int64_t NH = p.heads();
    const int L = p.L, K = p.K;
    const float scale = 1.0f / sqrtf((float)p.d);

    Scratch s(st);
    float *mu = nullptr, *vcent = nullptr, *part = nullptr;
    double *sums = nullptr;
    int32_t *counts = nullptr, *assign = assign_out;
    const int n_chunks = (L + kCaChunk - 1) / kCaChunk;
    const int tokens_per_cta = 1024;
    const int n_cta = (L + tokens_per_cta - 1) / tokens_per_cta;
    CA_CUDA(s.get((void **)&mu, sizeof(float) * NH * K * kD));
    CA_CUDA(s.get((void **)&vcent, sizeof(float) * NH * K * kD));
    CA_CUDA(s.get((void **)&part, sizeof(float) * NH * n_chunks * K * (kD + 2)));
    CA_CUDA(s.get((void **)&sums, sizeof(double) * NH * n_cta * K * kD));
    CA_CUDA(s.get((void **)&counts, sizeof(int32_t) * NH * n_cta * K));
    if (!assign) CA_CUDA(s.get((void **)&assign, sizeof(int32_t) * NH * L));

    const double esz = (double)sizeof(T);
    const double head_bytes = (double)NH * L * kD * esz;  // one read of Q (or K, V, O)

    // 1. strided init (and c = 0 for iters == 0)
    {
        Launch pl("kmeans_init", st, 0.0);
        kmeans_init_kernel<T><<<(unsigned)NH, 256, 0, st>>>(q, L, K, mu, xo.init_stride);
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    if (p.iters == 0) {
        CA_CUDA(cudaMemsetAsync(assign, 0, sizeof(int32_t) * NH * L, st));
        if (cent_out) CA_CUDA(cudaMemcpyAsync(cent_out, mu, sizeof(float) * NH * K * kD, cudaMemcpyDeviceToDevice, st));
    }

    // 2. Lloyd iterations (every CTA writes all K rows of its partial-sum slot)
    const size_t asmem = AssignSmem::bytes(K, tokens_per_cta);
    const dim3 agrid(n_cta, (unsigned)NH);
    for (int t = 0; t < p.iters; ++t) {
        int32_t *hist_t = hist ? hist + (int64_t)t * L : nullptr;
        {
            Launch pl("kmeans_assign", st, head_bytes);
            kmeans_assign_kernel<T><<<agrid, kAssignThreads, asmem, st>>>(
                q, L, K, tokens_per_cta, mu, assign, hist_t, (int64_t)p.iters * L, sums, counts);
            pl.after();
        }
        CA_CUDA(cudaGetLastError());
        {
            Launch pl("kmeans_update", st, 0.0);
            kmeans_update_kernel<<<(unsigned)NH, 256, 0, st>>>(K, n_cta, sums, counts, mu,
                                                                t == p.iters - 1 ? cent_out : nullptr,
                                                                xo.empty_keep);
            pl.after();
        }
        CA_CUDA(cudaGetLastError());
    }

    // 3. centroid attention
    const size_t csmem = centroid_attn_smem_bytes(K);
    {
        Launch pl("centroid_attn", st, 2.0 * head_bytes);
        centroid_attn_partial_kernel<T><<<dim3(n_chunks, (unsigned)NH), kCaThreads, csmem, st>>>(
            k, v, L, K, scale, mu, n_chunks, part, xo.var);
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    {
        Launch pl("centroid_combine", st, 0.0);
        centroid_attn_combine_kernel<<<(unsigned)NH, 256, 0, st>>>(K, n_chunks, part, vcent);
        pl.after();
    }
    CA_CUDA(cudaGetLastError());

    // 4-6. gather + window attention + blend
    const size_t wsmem = window_smem_bytes();
    {
        Launch pl("window_blend", st, 4.0 * head_bytes);
        Variant wv = xo.var;
        wv.mu = mu;
        window_blend_kernel<T><<<dim3((L + kWinQ - 1) / kWinQ, (unsigned)NH), kWinThreads, wsmem, st>>>(
            q, k, v, L, K, xo.r >= 0 ? xo.r : p.W / 2, scale, p.alpha, vcent, assign, out, wv);
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    return CA_OK;
}

ca_status dispatch(const void *q, const void *k, const void *v, int dtype, const Problem &p,
                   void *out, int32_t *assign_out, float *cent_out, int32_t *hist, void *stream) {
    ca_status s = validate(q, k, v, out, p);
    if (s != CA_OK) return s;
    if (dtype != 0 && dtype != 1) return fail(CA_ERR_INVALID_ARG, "dtype must be 0 (fp32) or 1 (bf16), got %d", dtype);
    if (((uintptr_t)cent_out & 15u) || ((uintptr_t)assign_out & 3u) || ((uintptr_t)hist & 3u))
        return fail(CA_ERR_INVALID_ARG, "centroids_out must be 16-byte aligned, assign buffers 4-byte aligned");
    s = ensure_kernel_attributes();
    if (s != CA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    if (fused_eligible(dtype, p)) {
        NvtxRange range("ca_forward fused");
        return run_fused((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, p,
                         (__nv_bfloat16 *)out, assign_out, cent_out, hist, st);
    }
    if (tiled_eligible(dtype, p)) {
        NvtxRange range("ca_forward tiled");
        return run_tiled((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, p,
                         (__nv_bfloat16 *)out, assign_out, cent_out, hist, st, TiledVariant::plain(p));
    }
    NvtxRange range("ca_forward general");
    if (dtype == 0)
        return run_forward<float>((const float *)q, (const float *)k, (const float *)v, p, (float *)out,
                                  assign_out, cent_out, hist, st);
    if (dtype == 1)
        return run_forward<__nv_bfloat16>((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                          (const __nv_bfloat16 *)v, p, (__nv_bfloat16 *)out,
                                          assign_out, cent_out, hist, st);
    return fail(CA_ERR_INVALID_ARG, "dtype must be 0 (fp32) or 1 (bf16), got %d", dtype);
}

}  // namespace

extern "C" {

ca_status ca_forward(const float *q, const float *k, const float *v, int B, int H, int L, int d,
                     int K, int iters, int W, float alpha, float *out, int32_t *assign_out,
                     float *centroids_out, void *stream) {
    Problem p{B, H, L, d, K, iters, W, alpha};
    return dispatch(q, k, v, 0, p, out, assign_out, centroids_out, nullptr, stream);
}

ca_status ca_forward_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int H,
                          int L, int d, int K, int iters, int W, float alpha, uint16_t *out,
                          int32_t *assign_out, float *centroids_out, void *stream) {
    Problem p{B, H, L, d, K, iters, W, alpha};
    return dispatch(q, k, v, 1, p, out, assign_out, centroids_out, nullptr, stream);
}

ca_status ca_forward_trace(const void *q, const void *k, const void *v, int dtype, int B, int H,
                           int L, int d, int K, int iters, int W, float alpha, void *out,
                           int32_t *assign_out, float *centroids_out, int32_t *assign_hist,
                           void *stream) {
    Problem p{B, H, L, d, K, iters, W, alpha};
    return dispatch(q, k, v, dtype, p, out, assign_out, centroids_out, assign_hist, stream);
}

ca_status ca_forward_ex(const void *q, const void *k, const void *v, int dtype, int B, int H,
                        int L, int d, int K, int iters, int W, float alpha, const ca_options *opt,
                        void *out, int32_t *assign_out, float *centroids_out, int32_t *assign_hist,
                        void *stream) {
    Problem p{B, H, L, d, K, iters, W, alpha};
    if (!opt) return dispatch(q, k, v, dtype, p, out, assign_out, centroids_out, assign_hist, stream);
    const ca_options &o = *opt;
    if ((o.window_mode | o.empty_mode | o.init_mode | o.gather_mode) & ~1)
        return fail(CA_ERR_INVALID_ARG, "window_mode, empty_mode, init_mode and gather_mode must be 0 or 1");
    const int H_kv = o.H_kv == 0 ? H : o.H_kv;
    if (H_kv < 1 || H < 1 || H % H_kv != 0)
        return fail(CA_ERR_INVALID_ARG, "H_kv must divide H (got H=%d, H_kv=%d)", H, o.H_kv);
    const bool plain = !o.window_mode && !o.empty_mode && !o.init_mode && !o.gather_mode && !o.key_valid && H_kv == H;
    if (plain) return dispatch(q, k, v, dtype, p, out, assign_out, centroids_out, assign_hist, stream);
    ca_status s = validate(q, k, v, out, p);
    if (s != CA_OK) return s;
    if (((uintptr_t)centroids_out & 15u) || ((uintptr_t)assign_out & 3u) || ((uintptr_t)assign_hist & 3u))
        return fail(CA_ERR_INVALID_ARG, "centroids_out must be 16-byte aligned, assign buffers 4-byte aligned");
    ExOpts ex;
    ex.init_stride = o.init_mode;
    ex.empty_keep = o.empty_mode;
    ex.r = o.window_mode ? W : W / 2;
    ex.var.H = H;
    ex.var.H_kv = H_kv;
    ex.var.key_valid = o.key_valid;
    ex.var.local = o.window_mode ? (W > 0 && W < L) : 1;
    ex.var.soft = o.gather_mode;
    if (dtype != 0 && dtype != 1) return fail(CA_ERR_INVALID_ARG, "dtype must be 0 (fp32) or 1 (bf16), got %d", dtype);
    s = ensure_kernel_attributes();
    if (s != CA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    // bf16 with grouped key/value heads, the radius window, the stride init,
    // kept empty centroids, key masks (window radius <= 64 then) or the soft
    // gather (radius <= 32): the tiled kernels
    // masks: the tensor-core window kernel; the soft gather: its radius-32 form
    const int r_max = o.gather_mode ? 32 : (o.key_valid ? 64 : ca::tiled::kMaxR);
    if (dtype == 1 && K <= 64 && (!ex.var.local || ex.r <= r_max)) {
        TiledVariant tv;
        tv.key_valid = o.key_valid;
        tv.soft = o.gather_mode;
        tv.r = ex.r;
        tv.local = ex.var.local;
        tv.init_stride = ex.init_stride;
        tv.empty_keep = ex.empty_keep;
        tv.H_kv = H_kv;
        NvtxRange range("ca_forward_ex tiled");
        return run_tiled((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, p,
                         (__nv_bfloat16 *)out, assign_out, centroids_out, assign_hist, st, tv);
    }
    if (dtype == 0)
        return run_forward<float>((const float *)q, (const float *)k, (const float *)v, p, (float *)out,
                                  assign_out, centroids_out, assign_hist, st, &ex);
    if (dtype == 1)
        return run_forward<__nv_bfloat16>((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                          (const __nv_bfloat16 *)v, p, (__nv_bfloat16 *)out, assign_out,
                                          centroids_out, assign_hist, st, &ex);
    return fail(CA_ERR_INVALID_ARG, "dtype must be 0 (fp32) or 1 (bf16), got %d", dtype);
}

// Two library-owned streams per device for the host-buffer entry point: one
// runs the kernels, one copies results back, so that with several chunks the
// copies in, the kernels and the copies out of different chunks overlap.
cudaError_t host_streams(cudaStream_t *comp, cudaStream_t *back) {
    static std::mutex mu;
    static cudaStream_t streams[64][2] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> g(mu);
    for (int i = 0; i < 2; ++i) {
        if (!streams[dev][i]) {
            e = cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking);
            if (e != cudaSuccess) return e;
        }
    }
    *comp = streams[dev][0];
    *back = streams[dev][1];
    return cudaSuccess;
}

ca_status ca_forward_host(const void *q, const void *k, const void *v, int dtype, int B, int H,
                          int L, int d, int K, int iters, int W, float alpha, void *out,
                          int32_t *assign_out, float *centroids_out, void *stream) {
    Problem p{B, H, L, d, K, iters, W, alpha};
    if (!q || !k || !v || !out) return fail(CA_ERR_INVALID_ARG, "q, k, v and out must be non-null");
    if (dtype != 0 && dtype != 1) return fail(CA_ERR_INVALID_ARG, "dtype must be 0 or 1");
    ca_status s = validate((const void *)16, (const void *)16, (const void *)16, (void *)16, p);
    if (s != CA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t esz = dtype == 0 ? 4 : 2;
    const int64_t NH = p.heads();
    const size_t head_elems = (size_t)p.L * p.d;
    const size_t n = (size_t)NH * head_elems;
    // Heads are independent: a large problem runs as up to eight chunks of
    // whole heads, each copied in, computed and copied back in turn.
    const int n_chunks = (NH >= 2 && n * esz * 4 >= (size_t(32) << 20)) ? (int)(NH < 8 ? NH : 8) : 1;
    cudaStream_t s_comp = st, s_back = st;
    if (n_chunks > 1) CA_CUDA(host_streams(&s_comp, &s_back));
    cudaEvent_t ev[2 * 8 + 2] = {};
    const int n_ev = n_chunks > 1 ? 2 * n_chunks + 2 : 0;
    for (int i = 0; i < n_ev; ++i) CA_CUDA(cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming));
    struct Events {
        cudaEvent_t *ev;
        int n;
        ~Events() {
            for (int i = 0; i < n; ++i) cudaEventDestroy(ev[i]);
        }
    } ev_guard{ev, n_ev};
    void *dq = nullptr, *dk = nullptr, *dv = nullptr, *dout = nullptr, *dcent = nullptr;
    int32_t *dassign = nullptr;
    // A failure part-way stops queueing work but still lets the streams
    // drain: copies already queued into or out of the caller's host buffers
    // must be finished before this call returns, error or not.
    ca_status status = CA_OK;
#define CA_STEP(call)                                                          \
    {                                                                          \
        cudaError_t e_ = (call);                                               \
        if (e_ != cudaSuccess) {                                               \
            status = cuda_fail(e_, #call);                                     \
            break;                                                             \
        }                                                                      \
    }
    {
        Scratch sc(st);
        // Before the scratch is released on st (or on an early exit), st
        // waits for everything queued on the other two streams.
        struct Join {
            cudaStream_t st, a, b;
            cudaEvent_t ea, eb;
            bool on;
            ~Join() {
                if (!on) return;
                cudaEventRecord(ea, a);
                cudaEventRecord(eb, b);
                cudaStreamWaitEvent(st, ea, 0);
                cudaStreamWaitEvent(st, eb, 0);
            }
        } join{st, s_comp, s_back, n_ev ? ev[n_ev - 2] : nullptr, n_ev ? ev[n_ev - 1] : nullptr, n_chunks > 1};
        do {
            CA_STEP(sc.get(&dq, n * esz));
            CA_STEP(sc.get(&dk, n * esz));
            CA_STEP(sc.get(&dv, n * esz));
            CA_STEP(sc.get(&dout, n * esz));
            if (assign_out) CA_STEP(sc.get((void **)&dassign, sizeof(int32_t) * NH * p.L));
            if (centroids_out) CA_STEP(sc.get(&dcent, sizeof(float) * NH * p.K * p.d));
        } while (0);
        for (int c = 0; status == CA_OK && c < n_chunks; ++c) {
            const int64_t h0 = c * NH / n_chunks, h1 = (c + 1) * NH / n_chunks;
            const size_t off = (size_t)h0 * head_elems * esz, bytes = (size_t)(h1 - h0) * head_elems * esz;
            CA_STEP(cudaMemcpyAsync((char *)dq + off, (const char *)q + off, bytes, cudaMemcpyHostToDevice, st));
            CA_STEP(cudaMemcpyAsync((char *)dk + off, (const char *)k + off, bytes, cudaMemcpyHostToDevice, st));
            CA_STEP(cudaMemcpyAsync((char *)dv + off, (const char *)v + off, bytes, cudaMemcpyHostToDevice, st));
            if (n_chunks > 1) {
                CA_STEP(cudaEventRecord(ev[2 * c], st));
                CA_STEP(cudaStreamWaitEvent(s_comp, ev[2 * c], 0));
            }
            const Problem pc{1, (int)(h1 - h0), p.L, p.d, p.K, p.iters, p.W, p.alpha};
            int32_t *da = dassign ? dassign + h0 * p.L : nullptr;
            float *dc = dcent ? (float *)dcent + h0 * p.K * p.d : nullptr;
            s = dispatch((char *)dq + off, (char *)dk + off, (char *)dv + off, dtype, pc, (char *)dout + off, da, dc,
                         nullptr, s_comp);
            if (s != CA_OK) {
                status = s;
                break;
            }
            if (n_chunks > 1) {
                CA_STEP(cudaEventRecord(ev[2 * c + 1], s_comp));
                CA_STEP(cudaStreamWaitEvent(s_back, ev[2 * c + 1], 0));
            }
            CA_STEP(cudaMemcpyAsync((char *)out + off, (char *)dout + off, bytes, cudaMemcpyDeviceToHost, s_back));
            if (assign_out)
                CA_STEP(cudaMemcpyAsync(assign_out + h0 * p.L, da, sizeof(int32_t) * (h1 - h0) * p.L,
                                        cudaMemcpyDeviceToHost, s_back));
            if (centroids_out)
                CA_STEP(cudaMemcpyAsync(centroids_out + h0 * p.K * p.d, dc, sizeof(float) * (h1 - h0) * p.K * p.d,
                                        cudaMemcpyDeviceToHost, s_back));
        }
    }
#undef CA_STEP
    const std::string detail = status == CA_OK ? std::string() : g_last_error;
    cudaError_t e = cudaStreamSynchronize(st);
    if (status != CA_OK) {
        g_last_error = detail;
        return status;
    }
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    return CA_OK;
}

ca_status ca_debug_record_error(int code, void *stream) {
    if (code != CA_ERR_TIMEOUT && code != CA_ERR_DEVICE)
        return fail(CA_ERR_INVALID_ARG, "code must be CA_ERR_TIMEOUT or CA_ERR_DEVICE (got %d)", code);
    {
        ca::Launch pl("debug_record_error", (cudaStream_t)stream, 0.0);
        ca::debug_record_error_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(code);
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    return CA_OK;
}

ca_status ca_sync_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int code = 0, where = 0;
    e = cudaMemcpyFromSymbol(&code, ca::g_dev_error, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyFromSymbol");
    if (code != 0) {
        cudaMemcpyFromSymbol(&where, ca::g_dev_error_where, sizeof(int));
        const int zero = 0;
        cudaMemcpyToSymbol(ca::g_dev_error, &zero, sizeof(int));
        return fail((ca_status)code, "device-side error %d recorded at site %d", code, where);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pending CUDA error");
    return CA_OK;
}

const char *ca_status_string(ca_status s) {
    switch (s) {
        case CA_OK: return "CA_OK";
        case CA_ERR_INVALID_ARG: return "CA_ERR_INVALID_ARG: an argument is out of range";
        case CA_ERR_UNSUPPORTED: return "CA_ERR_UNSUPPORTED: valid request not handled by this build";
        case CA_ERR_CUDA: return "CA_ERR_CUDA: a CUDA call or launch failed";
        case CA_ERR_TIMEOUT: return "CA_ERR_TIMEOUT: a bounded device-side wait ran out";
        case CA_ERR_DEVICE: return "CA_ERR_DEVICE: a kernel recorded an internal consistency failure";
    }
    return "unknown ca_status";
}

const char *ca_last_error(void) { return g_last_error.c_str(); }

const char *ca_version(void) { return "libclusterattn 0.1 (sm_100a)"; }

ca_status ca_profile_start(const char *kernel_name) {
    ca::ProfileState &p = ca::profile();
    std::lock_guard<std::mutex> g(p.mu);
    if (p.active) return fail(CA_ERR_INVALID_ARG, "profiling already started");
    p.selected = kernel_name ? kernel_name : "";
    p.pairs.clear();
    p.active = true;
    return CA_OK;
}

ca_status ca_profile_stop(ca_kernel_stat *stat) {
    ca::ProfileState &p = ca::profile();
    std::lock_guard<std::mutex> g(p.mu);
    if (!p.active) return fail(CA_ERR_INVALID_ARG, "profiling not started");
    p.active = false;
    ca_kernel_stat r{0, 0.0, 0.0};
    ca_status status = CA_OK;
    for (auto &pr : p.pairs) {
        float ms = 0.f;
        cudaError_t e = cudaEventSynchronize(pr.b);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, pr.a, pr.b);
        if (e != cudaSuccess && status == CA_OK) status = cuda_fail(e, "cudaEventElapsedTime");
        r.launches += 1;
        r.total_ms += ms;
        r.algorithmic_bytes += pr.bytes;
        p.pool.push_back(pr.a);
        p.pool.push_back(pr.b);
    }
    p.pairs.clear();
    if (stat) *stat = r;
    return status;
}

long long ca_launch_count(void) { return ca::profile().launches.load(); }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free entry point.
//
// Some callers cannot let a library allocate device memory: runtimes that
// reserve the whole GPU for their own allocator up front (a new driver
// allocation would fail, or fragment memory they manage), and serving loops
// with hard latency budgets where an allocation call on the hot path is not
// acceptable.  ca_forward_noalloc serves them: it runs the multi-kernel path
// with its working memory taken from one fixed array that lives in this file.
//
//   - The array holds kNoAllocScratchBytes (16 MiB).  It is part of the
//     library's device image, so every GPU that loads the library holds it
//     until the process exits.
//   - Host code cannot use the array's name as a device address.  The first
//     call on each device looks up the real address with
//     cudaGetSymbolAddress, with that device current, and caches it; make
//     that first call before any stream capture.
//   - Every call shares the array and it keeps the previous call's contents:
//     the running sums and counts are cleared on each call before use.  Calls
//     that overlap on the GPU (two streams, or two threads) race on it.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

ca_status noalloc_scratch_address(unsigned char **out) {
    static std::mutex mu;
    static unsigned char *addr[64] = {};
    int dev = 0;
    CA_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return fail(CA_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> g(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(g_noalloc_scratch)");
        addr[dev] = static_cast<unsigned char *>(p);
    }
    *out = addr[dev];
    return CA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <typename T>
ca_status run_forward_noalloc(const T *q, const T *k, const T *v, const Problem &p, T *out,
                              int32_t *assign_out, float *cent_out, cudaStream_t st) {
    using namespace ca;
    const int64_t NH = p.heads();
    const int L = p.L, K = p.K;
    const float scale = 1.0f / sqrtf((float)p.d);
    const int n_chunks = (L + kCaChunk - 1) / kCaChunk;
    const int tokens_per_cta = 1024;
    const int n_cta = (L + tokens_per_cta - 1) / tokens_per_cta;

    // Carve the working buffers out of the fixed array.
    const size_t b_mu = align256(sizeof(float) * NH * K * kD);
    const size_t b_vc = b_mu;
    const size_t b_part = align256(sizeof(float) * NH * n_chunks * K * (kD + 2));
    const size_t b_sums = align256(sizeof(double) * NH * n_cta * K * kD);
    const size_t b_cnt = align256(sizeof(int32_t) * NH * n_cta * K);
    const size_t b_asg = assign_out ? 0 : align256(sizeof(int32_t) * NH * L);
    const size_t need = b_mu + b_vc + b_part + b_sums + b_cnt + b_asg;
    if (need > kNoAllocScratchBytes)
        return fail(CA_ERR_INVALID_ARG,
                    "problem needs %zu bytes of working memory; the allocation-free entry point holds %zu",
                    need, kNoAllocScratchBytes);
    unsigned char *base = nullptr;
    ca_status s = noalloc_scratch_address(&base);
    if (s != CA_OK) return s;
    float *mu = reinterpret_cast<float *>(base);
    float *vcent = reinterpret_cast<float *>(base + b_mu);
    float *part = reinterpret_cast<float *>(base + b_mu + b_vc);
    double *sums = reinterpret_cast<double *>(base + b_mu + b_vc + b_part);
    int32_t *counts = reinterpret_cast<int32_t *>(base + b_mu + b_vc + b_part + b_sums);
    int32_t *assign = assign_out ? assign_out
                                 : reinterpret_cast<int32_t *>(base + b_mu + b_vc + b_part + b_sums + b_cnt);
    const double head_bytes = (double)NH * L * kD * sizeof(T);

    {
        Launch pl("kmeans_init", st, 0.0);
        kmeans_init_kernel<T><<<(unsigned)NH, 256, 0, st>>>(q, L, K, mu);
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    if (p.iters == 0) {
        CA_CUDA(cudaMemsetAsync(assign, 0, sizeof(int32_t) * NH * L, st));
        if (cent_out) CA_CUDA(cudaMemcpyAsync(cent_out, mu, sizeof(float) * NH * K * kD, cudaMemcpyDeviceToDevice, st));
    }
    // The array keeps the last call's contents; nothing in it needs clearing:
    // every assignment launch writes all K rows of every partial-sum slot
    // before the update reads them.
    const size_t asmem = AssignSmem::bytes(K, tokens_per_cta);
    const dim3 agrid(n_cta, (unsigned)NH);
    for (int t = 0; t < p.iters; ++t) {
        {
            Launch pl("kmeans_assign", st, head_bytes);
            kmeans_assign_kernel<T><<<agrid, kAssignThreads, asmem, st>>>(
                q, L, K, tokens_per_cta, mu, assign, nullptr, (int64_t)p.iters * L, sums, counts);
            pl.after();
        }
        CA_CUDA(cudaGetLastError());
        {
            Launch pl("kmeans_update", st, 0.0);
            kmeans_update_kernel<<<(unsigned)NH, 256, 0, st>>>(K, n_cta, sums, counts, mu,
                                                                t == p.iters - 1 ? cent_out : nullptr);
            pl.after();
        }
        CA_CUDA(cudaGetLastError());
    }
    const size_t csmem = centroid_attn_smem_bytes(K);
    {
        Launch pl("centroid_attn", st, 2.0 * head_bytes);
        centroid_attn_partial_kernel<T><<<dim3(n_chunks, (unsigned)NH), kCaThreads, csmem, st>>>(
            k, v, L, K, scale, mu, n_chunks, part);
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    {
        Launch pl("centroid_combine", st, 0.0);
        centroid_attn_combine_kernel<<<(unsigned)NH, 256, 0, st>>>(K, n_chunks, part, vcent);
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    const size_t wsmem = window_smem_bytes();
    {
        Launch pl("window_blend", st, 4.0 * head_bytes);
        window_blend_kernel<T><<<dim3((L + kWinQ - 1) / kWinQ, (unsigned)NH), kWinThreads, wsmem, st>>>(
            q, k, v, L, K, p.W / 2, scale, p.alpha, vcent, assign, out);
        pl.after();
    }
    CA_CUDA(cudaGetLastError());
    return CA_OK;
}

}  // namespace

extern "C" ca_status ca_forward_noalloc(const void *q, const void *k, const void *v, int dtype, int B,
                                        int H, int L, int d, int K, int iters, int W, float alpha,
                                        void *out, int32_t *assign_out, float *centroids_out,
                                        void *stream) {
    Problem p{B, H, L, d, K, iters, W, alpha};
    ca_status s = validate(q, k, v, out, p);
    if (s != CA_OK) return s;
    if (((uintptr_t)centroids_out & 15u) || ((uintptr_t)assign_out & 3u))
        return fail(CA_ERR_INVALID_ARG, "centroids_out must be 16-byte aligned, assign_out 4-byte aligned");
    if (dtype != 0 && dtype != 1) return fail(CA_ERR_INVALID_ARG, "dtype must be 0 (fp32) or 1 (bf16), got %d", dtype);
    s = ensure_kernel_attributes();
    if (s != CA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    if (dtype == 0)
        return run_forward_noalloc<float>((const float *)q, (const float *)k, (const float *)v, p, (float *)out,
                                          assign_out, centroids_out, st);
    if (dtype == 1)
        return run_forward_noalloc<__nv_bfloat16>((const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k,
                                                  (const __nv_bfloat16 *)v, p, (__nv_bfloat16 *)out,
                                                  assign_out, centroids_out, st);
    return fail(CA_ERR_INVALID_ARG, "dtype must be 0 (fp32) or 1 (bf16), got %d", dtype);
}
