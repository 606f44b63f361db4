/*
 * libclusterattn: cluster-attention forward pass for NVIDIA B200 (sm_100a).
 *
 * The operation (model card "Hooshaai/distilbert-sst2-cluster-attention",
 * Architecture Overview and Mathematical Formulation section 1; model card
 * "Hooshaai/svd-sst2-roberta-cluster", sections 2.1 and 3), per (batch b,
 * head h), with Q, K, V the [L, d] slices of that head and s = 1 / sqrt(d):
 *
 *   1. strided init   mu_k = Q[floor(k L / K)],                k = 0..K-1
 *   2. for t = 1..iters (batch Lloyd's k-means on the queries):
 *        D_ik = |Q_i|^2 + |mu_k|^2 - 2 Q_i . mu_k
 *        c_i  = argmin_k D_ik                     (ties: lowest k)
 *        mu_k = sum_{c_i = k} Q_i / max(1, count_k) (empty cluster: zero)
 *      with iters == 0: c_i = 0 and mu stays at init;
 *   3. centroid attention  V_cent = softmax(mu K^T s) V            [K, d]
 *   4. gather             g_i = V_cent[c_i]
 *   5. window attention   o_i = softmax_{j : |i-j| <= floor(W/2), 0 <= j < L}
 *                                 (s Q_i . K_j) V_j
 *   6. convex fusion      O_i = (1 - alpha) g_i + alpha o_i.
 *
 * Precision.  Arithmetic is fp32 with fp32 accumulation; O is rounded once to
 * the input type.  Centroids are kept in fp32 (the cards' module measures
 * distances on centroids cast to float): each is the exact member sum divided
 * by the count in fp64 and rounded once to fp32.  The argmin is decided on
 * those fp32 centroids exactly: an fp32 pass with a rigorous error bound
 * settles almost every token, and the few whose two best candidates lie
 * within that bound are re-measured in fp64, in the expanded form above with
 * index-order sums.  On the bf16 paths the contractions run on tensor cores
 * with bf16 operands and fp32 accumulation: the distance pass splits each
 * fp32 centroid into two bf16 terms; the centroid-attention scores use the
 * centroids split in two terms (one CTA per head) or rounded once to bf16
 * (long sequences); the attention weights are rounded to bf16 for the P V
 * products.
 *
 * Execution.  On sm_100a the long-sequence bf16 path stages query, key and
 * value tiles with TMA (tensor maps over the caller's q, k, v) and issues its
 * distance and window-attention contractions as tcgen05.mma with tensor-
 * memory accumulators; its kernels are chained with programmatic dependent
 * launch (a kernel may start before its predecessor on the stream ends and
 * waits for it before reading its results; the first kernel of a call waits
 * for all earlier work on the stream).
 *
 * Conventions for every entry point below:
 *   - Tensors are dense, row-major [B, H, L, d] (d fastest), as produced by
 *     the cards' projection + view(B, L, H, d).transpose(1, 2); assign_out is
 *     [B, H, L] int32, centroids_out [B, H, K, d] fp32.
 *   - Pointers are DEVICE pointers owned by the caller (ca_forward_host takes
 *     HOST pointers instead), 16-byte aligned;
 *     out must not overlap q, k or v.  The library keeps no pointer after a
 *     call returns.
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Device entry points are asynchronous on that stream; their
 *     scratch memory comes from cudaMallocAsync / cudaFreeAsync on it.
 *   - assign_out and centroids_out may be NULL (not written).
 *   - Validation happens on the host before any launch and returns a status;
 *     nothing is launched on a non-OK status.  Launch failures return
 *     CA_ERR_CUDA.  Device-side problems are reported by ca_sync_status.
 *   - Supported: d == 64; 1 <= K <= min(L, 128); iters >= 0; W >= 0;
 *     0 <= alpha <= 1 (finite); B, H, L >= 1; B*H <= 65535; B*H*L*d < 2^31.
 *     Inputs must be finite.
 *   - Results are deterministic: the same inputs give bitwise-identical
 *     outputs on the same GPU, within this envelope.  The general path
 *     (every fp32 call; bf16 calls with K > 64 or floor(W/2) > 128) runs
 *     every floating-point reduction in a fixed order (the member sums of
 *     the centroid update in index order within each 1024-token block, the
 *     blocks in order), so any finite input is reproducible.  The bf16
 *     fused and tiled kernels add the member sums with fp64 atomics whose
 *     order varies, but the sums are exact (hence order-free) whenever every
 *     non-zero magnitude in Q is at least 2^-26 and, for each coordinate,
 *     the magnitudes of one head's queries add up to less than 2^19 (for
 *     instance |Q| < 16 with L <= 32768); outside that envelope the last
 *     bit of a centroid may vary between runs.
 */
#ifndef CLUSTERATTN_H_
#define CLUSTERATTN_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CA_OK = 0,
    CA_ERR_INVALID_ARG = 1, /* a size, pointer or scalar argument is out of range   */
    CA_ERR_UNSUPPORTED = 2, /* a valid request this build does not handle (e.g. d)  */
    CA_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed          */
    CA_ERR_TIMEOUT = 4,     /* a bounded device-side wait ran out                   */
    CA_ERR_DEVICE = 5       /* a kernel recorded an internal consistency failure    */
} ca_status;

/* fp32 Q, K, V and out.  Steps 1-6 above for all B*H heads. */
ca_status ca_forward(const float *q, const float *k, const float *v, int B, int H, int L, int d,
                     int K, int iters, int W, float alpha, float *out, int32_t *assign_out,
                     float *centroids_out, void *stream);

/* bf16 Q, K, V and out, as raw uint16 bit patterns; centroids_out stays fp32. */
ca_status ca_forward_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int H,
                          int L, int d, int K, int iters, int W, float alpha, uint16_t *out,
                          int32_t *assign_out, float *centroids_out, void *stream);

/* As ca_forward / ca_forward_bf16 (dtype 0 = fp32, 1 = bf16), and also writes
 * the assignment of every iteration to assign_hist [B, H, iters, L] int32
 * (device pointer, may be NULL).  Used to check each Lloyd step on its own. */
ca_status ca_forward_trace(const void *q, const void *k, const void *v, int dtype, int B, int H,
                           int L, int d, int K, int iters, int W, float alpha, void *out,
                           int32_t *assign_out, float *centroids_out, int32_t *assign_hist,
                           void *stream);

/* Variants of the card's own module ("Hooshaai/svd-sst2-roberta-cluster",
 * section 5), selected per call; all zero / NULL gives the forward above:
 *   window_mode  0: window |i-j| <= floor(W/2) (default);
 *                1: the module's radius |i-j| <= W, and no local branch at
 *                   all (O = gathered) when W == 0 or W >= L;
 *   empty_mode   0: an empty cluster becomes the zero vector (default);
 *                1: an empty cluster keeps its previous centroid;
 *   init_mode    0: mu_k = Q[floor(k L / K)] (default);
 *                1: mu_k = Q[k * max(1, L / K)] (the module's stride);
 *   gather_mode  0: hard gather V_cent[c_i] (default);
 *                1: soft assignment softmax(Q_i mu^T / sqrt(d)) V_cent;
 *   key_valid    [B, L] device bytes (1 = valid) or NULL: invalid keys take
 *                no weight in either softmax (a row with no valid key weighs
 *                every key equally, as the module's all -10000 row does) and
 *                output rows of invalid queries are zero; k-means still
 *                clusters every query, as the module does;
 *   H_kv         key/value heads (0 means H); k and v are [B, H_kv, L, d]
 *                and query head h reads key/value head h / (H / H_kv).
 * Unknown mode values or an H_kv that does not divide H return
 * CA_ERR_INVALID_ARG. */
typedef struct {
    int window_mode;
    int empty_mode;
    int init_mode;
    int gather_mode;
    const uint8_t *key_valid;
    int H_kv;
} ca_options;

/* ca_forward_trace with the variants of ca_options (opt may be NULL).  Calls
 * whose options are all defaults take the same kernels as ca_forward_trace.
 * bf16 calls with K <= 64 (grouped key/value heads, the radius window with
 * radius <= 128 or no local branch, the stride init, kept empty centroids,
 * key_valid with a window radius <= 64, the soft gather with a window radius
 * <= 32, or no local branch with either; alone or together) run the tiled
 * tensor-core kernels; every other option runs the general multi-kernel
 * path. */
ca_status ca_forward_ex(const void *q, const void *k, const void *v, int dtype, int B, int H,
                        int L, int d, int K, int iters, int W, float alpha, const ca_options *opt,
                        void *out, int32_t *assign_out, float *centroids_out, int32_t *assign_hist,
                        void *stream);

/* End-to-end form for callers holding HOST buffers (dtype 0 = fp32 with float
 * arrays, 1 = bf16 with uint16 arrays): copies q, k, v to the device, runs the
 * forward, copies out (and assign_out / centroids_out when non-NULL) back and
 * returns once everything has completed.  Problems of at least 32 MB (q, k, v
 * and out together) run as up to eight chunks of whole heads: copies in on
 * stream, kernels and copies back on two library-owned streams of the current
 * device, ordered with events, so that the chunks' transfers and kernels
 * overlap; results are identical to a single pass because heads are
 * independent.  Host buffers should be pinned for full copy bandwidth and for
 * the overlap; pageable buffers work but copy slower.  Device buffers are
 * stream-ordered allocations released before return. */
ca_status ca_forward_host(const void *q, const void *k, const void *v, int dtype, int B, int H,
                          int L, int d, int K, int iters, int W, float alpha, void *out,
                          int32_t *assign_out, float *centroids_out, void *stream);

/* Allocation-free form of ca_forward_trace (without the trace; dtype 0 =
 * fp32, 1 = bf16).  The model cards have no counterpart: this exists for
 * callers that cannot let a library allocate device memory, such as runtimes
 * that reserve the GPU for their own allocator up front, or serving loops
 * that allow no allocation call on their hot path.  The caller passes inputs
 * and outputs as usual; all other working memory comes from one fixed 16 MiB
 * device array inside the library (held on every GPU that loads the library,
 * until the process exits).  Problems whose working memory exceeds 16 MiB
 * are rejected with CA_ERR_INVALID_ARG and a message giving the size needed
 * (for example B*H = 384 heads of L = 128 with K = 16 fit; the working
 * memory grows with B*H*K and, when assign_out is NULL, with B*H*L).  The
 * call makes no cudaMalloc, cudaMallocAsync or cudaFree call.  Its first call
 * on each device looks up the array's device address (the device must be
 * current); make that first call before any stream capture.  Every call
 * reuses the same array, so calls that overlap on the GPU (on two streams,
 * or from two threads) race with each other; serialize them. */
ca_status ca_forward_noalloc(const void *q, const void *k, const void *v, int dtype, int B, int H,
                             int L, int d, int K, int iters, int W, float alpha, void *out,
                             int32_t *assign_out, float *centroids_out, void *stream);

/* Synchronizes stream, then reports (and clears) the first device-side error
 * recorded by a kernel of this library on the current device, or a pending
 * CUDA error.  CA_OK when nothing went wrong.  The device-side error word is
 * one per device, shared by every stream and thread using the library there:
 * a kernel on another stream can set it, and a caller that reads it clears
 * it for everyone; callers that need per-stream attribution must serialize
 * their work and their status checks. */
ca_status ca_sync_status(void *stream);

/* Test hook: launches one single-thread kernel on stream that records code
 * (CA_ERR_TIMEOUT or CA_ERR_DEVICE) in the device-side error word exactly as
 * a kernel that detected a problem would, without faulting; the next
 * ca_sync_status then returns that code once.  Any other code returns
 * CA_ERR_INVALID_ARG and launches nothing.  Not part of the forward pass. */
ca_status ca_debug_record_error(int code, void *stream);

/* Static description of a status code. */
const char *ca_status_string(ca_status s);

/* Thread-local detail of the last non-OK status returned on this thread. */
const char *ca_last_error(void);

/* Library version string. */
const char *ca_version(void);

/* Measurement support.  Every kernel launch of the library is counted
 * (ca_launch_count, process-wide, monotonic).  Between ca_profile_start and
 * ca_profile_stop, each launch of the kernel named kernel_name (NULL or ""
 * selects none) is bracketed by two CUDA events recorded on its launching
 * stream.  ca_profile_stop waits for those events and fills *stat with the
 * number of timed launches, their summed duration and their summed
 * algorithmic HBM bytes (one read of every input and one write of every
 * output the kernel must touch).  Kernel names: the fused one-CTA-per-head
 * kernel (bf16, L <= 512, K <= 64, floor(W/2) <= 16) is "fused_forward";
 * the tiled bf16 path (K <= 64, floor(W/2) <= 128) launches "tiled_init",
 * then per Lloyd iteration "tiled_assign" and "tiled_update", then
 * "tiled_centroid", "tiled_combine" and
 * "tiled_window"; every other case runs the general path "kmeans_init",
 * "kmeans_assign", "kmeans_update", "centroid_attn", "centroid_combine" and
 * "window_blend". */
typedef struct {
    long long launches;
    double total_ms;
    double algorithmic_bytes;
} ca_kernel_stat;

ca_status ca_profile_start(const char *kernel_name);
ca_status ca_profile_stop(ca_kernel_stat *stat);
long long ca_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* CLUSTERATTN_H_ */
